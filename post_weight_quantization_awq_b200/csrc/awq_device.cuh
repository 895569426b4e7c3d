// Device-side building blocks shared by the AWQ kernels: the fp32 group
// quantiser, the device status word, and thin inline-PTX wrappers for the
// sm_100a features the scored GEMM uses (mbarrier, TMA, tcgen05/TMEM).
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace awq {

// ---------------------------------------------------------------------------
// Device status word (first bytes of every workspace).
// ---------------------------------------------------------------------------
enum : uint32_t {
  kDevOk = 0,
  kDevTimeout = 1u << 0,    // a bounded wait ran out
  kDevNonFinite = 1u << 1,  // a score was NaN or infinite
  kDevBadIndex = 1u << 2,   // a clip index passed to the packing was >= n_clip
  kDevOutOfBounds = 1u << 3,  // a debug index check failed (debug library only)
};

struct DevStatus {
  uint32_t flags;      // kDev* bits, OR-ed by kernels
  uint32_t where;      // code of the first wait that ran out (debug aid)
  int32_t kscale;      // power-of-two exponent applied to the candidate errors
  uint32_t wmax_bits;  // bit pattern of max |W| (a non-negative float)
  uint32_t mse_done;   // blocks of the MSE reduction that have finished
};

__device__ __forceinline__ void dev_fail(DevStatus *st, uint32_t flag, uint32_t where) {
  if (st) {
    atomicOr(&st->flags, flag);
    atomicCAS(&st->where, 0u, where);
  }
}

// ---------------------------------------------------------------------------
// Debug index checks.  In the debug library (compiled with -DAWQ_DEBUG_BOUNDS:
// `python -m post_weight_quantization_awq_b200.build --debug-bounds` writes
// libawq_debug.so) AWQ_IN_BOUNDS(cond, site) guards a global access whose
// index the kernel derives from its grid: a failed check records
// kDevOutOfBounds and the first site's code in this translation unit's bounds
// word and yields false, so the access is skipped; awq_bounds_status() reads
// and clears the words of every unit.  In the release library the macro is
// the constant true.
// ---------------------------------------------------------------------------
#ifdef AWQ_DEBUG_BOUNDS
namespace {
__device__ DevStatus g_bounds_status;  // one per translation unit
__device__ __forceinline__ bool in_bounds(bool ok, uint32_t site) {
  if (!ok) dev_fail(&g_bounds_status, kDevOutOfBounds, site);
  return ok;
}
}  // namespace
#define AWQ_IN_BOUNDS(cond, site) ::awq::in_bounds((cond), (site))
// host reader of this unit's bounds word (read, then clear)
#define AWQ_BOUNDS_READER(fn)                                                        \
  cudaError_t fn(DevStatus *h) {                                                     \
    cudaError_t e = cudaMemcpyFromSymbol(h, g_bounds_status, sizeof(DevStatus));     \
    if (e != cudaSuccess) return e;                                                  \
    const DevStatus zero = {};                                                       \
    return cudaMemcpyToSymbol(g_bounds_status, &zero, sizeof(DevStatus));            \
  }
#else
#define AWQ_IN_BOUNDS(cond, site) true
#define AWQ_BOUNDS_READER(fn)
#endif

// ---------------------------------------------------------------------------
// Group quantiser ("05 — AWQ" §5/§9: groups of g input channels, asymmetric
// min/max with a zero point).  Every step is fp32, correctly rounded, with
// round-half-to-even; the explicit _rn intrinsics keep the compiler from
// contracting any of them into an FMA.
// ---------------------------------------------------------------------------
struct GroupQ {
  float delta;    // step
  float zero;     // zero point (integer valued)
  float qmax;     // 2^b - 1
  float rcp;      // approximate 1/delta: only proposes codes, never decides them
  float half_lo;  // delta * (0.5 - 2^-16): remainders below it prove a code exact
};

__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// rne(RN32(x / delta)) without a division on the common path.  k = rne of
// the approximate quotient x * rcp; the remainder x - k*delta comes from one
// FMA (a single rounding).  If |remainder| < delta (0.5 - 2^-16) and |k| < 64,
// then |x/delta - k| < 0.5 - 2^-16 + 2^-22, and the fp32 rounding of x/delta
// moves it by at most 2^-24 * 64.5 < 2^-17, so RN32(x/delta) is strictly within
// 0.5 of k and rounds to k -- however k was proposed.  Otherwise the correctly
// rounded quotient decides.
__device__ __forceinline__ float round_quotient(float x, float delta, float rcp, float half_lo) {
  const float k = rintf(__fmul_rn(x, rcp));
  const float rem = fmaf(-k, delta, x);
  if (fabsf(rem) < half_lo && fabsf(k) < 64.0f) return k;
  return rintf(__fdiv_rn(x, delta));
}

// Range of one group after the optional clip ratio r32 (1 = no clip).
// Asymmetric (zero point): delta = max(mx - mn, 1e-5) / (2^b - 1) and
// z = clamp(rne(-mn / delta), 0, 2^b - 1).  Symmetric (sym, no zero point):
// delta = max(|mx|, |mn|, 1e-5) / (2^(b-1) - 1) and z = 2^(b-1), so codes
// are centred on z in the same unsigned range [0, 2^b - 1].
// `guard` is the floor on the range (1e-5; 1e-5 2^k when every value of the
// group carries an exact factor 2^k, which leaves codes and zero points
// unchanged and scales delta by exactly 2^k).
__device__ __forceinline__ GroupQ group_params(float mx, float mn, float r32, float qmax, bool sym,
                                               float guard = 1e-5f) {
  if (r32 != 1.0f) {
    mx = __fmul_rn(r32, mx);
    mn = __fmul_rn(r32, mn);
  }
  // one division for both kinds: range and divisor are chosen, not branched
  GroupQ g;
  g.qmax = qmax;
  const float range = sym ? fmaxf(fabsf(mx), fabsf(mn)) : __fsub_rn(mx, mn);
  const float divisor = sym ? 0.5f * (qmax - 1.0f) : qmax;  // 2^(b-1) - 1 or 2^b - 1, exact
  g.delta = __fdiv_rn(fmaxf(range, guard), divisor);
  g.rcp = rcp_approx(g.delta);
  g.half_lo = __fmul_rn(g.delta, 0.4999847412109375f /* 0.5 - 2^-16 */);
  if (sym) {
    g.zero = 0.5f * (qmax + 1.0f);  // 2^(b-1), exact
  } else {
    const float z = round_quotient(-mn, g.delta, g.rcp, g.half_lo);
    g.zero = fminf(fmaxf(z, 0.0f), qmax);
  }
  return g;
}

__device__ __forceinline__ float round_quotient(float wt, const GroupQ &g) {
  return round_quotient(wt, g.delta, g.rcp, g.half_lo);
}

// rne(y) for |y| < 2^22 with two fp32 additions (FMA pipe): y + 1.5 2^23 lies
// in (2^23, 2^24), where the spacing is 1, so its rounding is 1.5 2^23 +
// rne(y) (ties to even, 1.5 2^23 being even), and removing 1.5 2^23 is exact.
__device__ __forceinline__ float2 rne2_small(float2 y) {
  const float2 m = make_float2(12582912.0f, 12582912.0f);
  return __fadd2_rn(__fadd2_rn(y, m), make_float2(-12582912.0f, -12582912.0f));
}

// (q - z) = clamp(rne(RN32(wt/delta)), -z, qmax - z) for 2 NP values of one
// group whose quotients all lie below 63 in magnitude (the caller checks
// max|wt| * rcp < 63 for the group, else passes half_lo = -1): proposed by
// the approximate reciprocal and the small-number rounding, proven by one
// remainder test for all of them (see round_quotient), decided by the
// correctly rounded division otherwise.
template <int NP>
__device__ __forceinline__ void quant_qz_pairs(const float2 (&wt)[NP], const GroupQ &g,
                                               float2 (&qz)[NP]) {
  const float2 rc = make_float2(g.rcp, g.rcp), dl = make_float2(g.delta, g.delta);
  float rmax = 0.0f;
#pragma unroll
  for (int h = 0; h < NP; ++h) {
    qz[h] = rne2_small(__fmul2_rn(wt[h], rc));
    const float2 rem = __ffma2_rn(make_float2(-qz[h].x, -qz[h].y), dl, wt[h]);
    rmax = fmaxf(rmax, fmaxf(fabsf(rem.x), fabsf(rem.y)));
  }
  if (!(rmax < g.half_lo)) {
#pragma unroll
    for (int h = 0; h < NP; ++h)
      qz[h] = make_float2(rintf(__fdiv_rn(wt[h].x, g.delta)), rintf(__fdiv_rn(wt[h].y, g.delta)));
  }
  const float lo = -g.zero, hi = g.qmax - g.zero;  // exact (small integers)
#pragma unroll
  for (int h = 0; h < NP; ++h)
    qz[h] = make_float2(fminf(fmaxf(qz[h].x, lo), hi), fminf(fmaxf(qz[h].y, lo), hi));
}

// Three-input max / min (one instruction on sm_100a; same NaN rule as fmaxf).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ float fmin3(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// the group check of quant_qz_pairs: every |wt| <= max(|mx|, |mn|)
__device__ __forceinline__ void fast_path_check(GroupQ &g, float mx, float mn) {
  if (!(fmaxf(fabsf(mx), fabsf(mn)) * g.rcp < 63.0f)) g.half_lo = -1.0f;
}

__device__ __forceinline__ float quant_code(float wt, const GroupQ &g) {
  float q = __fadd_rn(round_quotient(wt, g), g.zero);
  return fminf(fmaxf(q, 0.0f), g.qmax);
}


// ---------------------------------------------------------------------------
// Bounded waits.  A wait that exceeds its poll budget records kDevTimeout and
// returns false; callers stop issuing work and drain what is in flight.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits until the phase with `parity` of `bar` has completed.  Gives up after
// `max_polls` polls or as soon as *abort is set; returns true on success.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  uint32_t max_polls,
                                                  volatile int *abort) {
  for (uint32_t i = 0; i < max_polls; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (abort && *abort) return false;
    if (i > 64) __nanosleep(32);
  }
  return false;
}

// try_wait with a suspend-time hint: the thread sleeps until the phase
// completes or about `ns` nanoseconds pass, instead of spinning (spinning
// warps take issue slots from the warps that do the work).
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t *bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait for waits expected to be long (a role idle for most of a
// tile): each poll sleeps until the phase completes or up to ~1 us, and the
// bound is in time, max_polls x 64 ns (about 1 s for the default 2^24; one
// poll when max_polls is 1), since how long a hinted poll sleeps varies.
__device__ __forceinline__ bool mbar_wait_long(uint64_t *bar, uint32_t parity, uint32_t max_polls,
                                               volatile int *abort) {
  const uint64_t limit_ns = (uint64_t)max_polls * 64u;
  const uint64_t t0 = global_ns();
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity, 1000u)) return true;
    if (abort && *abort) return false;
    if (global_ns() - t0 > limit_ns) return false;
  }
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// ---------------------------------------------------------------------------
// TMA (cp.async.bulk.tensor), 2-D tiles, no multicast.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const void *tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void *smem_dst, const void *tmap, uint64_t *bar,
                                            int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05 / TMEM.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t *smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_result)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16, one CTA.
__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrives on `bar` once every tcgen05 operation this thread issued so far has
// completed.
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 32 lanes x 32 consecutive fp32 columns: thread i of the warp gets lane
// (base lane + i), columns [col, col + 32).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile written by TMA
// with 128-byte swizzling: rows of 64 fp16 (128 B), 8-row core groups 1024 B
// apart.  Fields: start address >> 4 (bits 0-13), leading byte offset >> 4
// (bits 16-29, unused for swizzled K-major, set to 1), stride byte offset >> 4
// (bits 32-45), descriptor version 1 (bits 46-47), base offset 0, swizzle mode
// 2 = 128B (bits 61-63).
__device__ __forceinline__ uint64_t smem_desc_k_sw128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}

// Instruction descriptor, kind::f16: fp16 A and B (format 0), fp32 accumulator
// (bits 4-5 = 1), both K-major, N >> 3 at bits 17-22, M >> 4 at bits 24-28.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

}  // namespace awq
