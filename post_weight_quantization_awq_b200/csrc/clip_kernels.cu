// K6 — per-(row, group) clip-ratio search ("05 — AWQ: Activation-Aware Weight
// Scaling" §4, optional clipping: a ratio of 0.5–1.0 of the range is
// grid-searched after alpha).
//
// For group k the output error of row o under clip c is
//   E_okc = sum_t (sum_{j in k} X_tj d_j)^2 = d^T G_k d,   G_k = X_k^T X_k,
// with d = deq_c/s - w over the group's g channels.  G_k does not depend on s
// or on the row, so it is built once per call (K6a) and every (o, k, c) is a
// 128-dimensional fp32 quadratic form (K6b).
//   K6a  gram_tc: tensor-core block Grams over token chunks, one CTA per
//        (group, chunk); chunk partials are summed in a fixed order by
//        gram_reduce, so G is bitwise reproducible.
//   K6b  clip_tc: tensor-core quadratic forms, one CTA per (group, share of
//        the rows); the first c with the smallest E wins.
#include <cuda.h>
#include <cuda_fp16.h>
#include <math.h>

#include "awq_launch.h"

namespace awq {

namespace {
constexpr int G = 128;          // group size handled by these kernels
}  // namespace

// ---------------------------------------------------------------------------
// K6a — block Grams on the tensor cores.  One CTA per (group k, token chunk):
// TMA brings X[t0:t0+64, 128k:128k+128] as two 64-channel boxes with 128-byte
// swizzling (rows = tokens), which is the MN-major layout of X_k^T; the same
// shared-memory tile is both the A (M = 128 channels) and the B (N = 128
// channels) operand of tcgen05.mma kind::f16 (K = 16 tokens per instruction),
// accumulating G_k = X_k^T X_k in fp32 in 128 TMEM columns.  fp16 products
// are exact in fp32.  Warp 0 loads, warp 1 issues MMAs, warps 2..5 write the
// 128 x 128 partial; chunk partials are summed in a fixed order afterwards.
// ---------------------------------------------------------------------------
namespace {
constexpr int GT = 64;                          // tokens per stage
constexpr int GSTAGES = 6;
constexpr uint32_t GBOX_BYTES = 64 * GT * 2;    // 64 channels x 64 tokens fp16
constexpr uint32_t GSTAGE_BYTES = 2 * GBOX_BYTES;
constexpr uint32_t GDRAIN_POLLS = 1u << 22;
// kind::f16, fp16 A/B, fp32 D, A and B MN-major, N = 128, M = 128
constexpr uint32_t IDESC_GRAM =
    (1u << 4) | (1u << 15) | (1u << 16) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

struct __align__(8) GramTail {
  uint64_t full[GSTAGES];
  uint64_t empty[GSTAGES];
  uint64_t done;
  uint32_t tmem_base;
  int abort_flag;
};
constexpr size_t kGramSmemBytes = 1024 + GSTAGES * GSTAGE_BYTES + sizeof(GramTail);

// MN-major operand with 128-byte swizzling: 64 channels (128 B) per token row,
// 8-row core groups 1024 B apart (SBO), the second 64-channel half of the
// group GBOX_BYTES further (LBO).
__device__ __forceinline__ uint64_t smem_desc_mn_sw128(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((GBOX_BYTES >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}
}  // namespace

__global__ void __launch_bounds__(192, 1)
    gram_tc_kernel(const __grid_constant__ CUtensorMap tmX, int64_t T, int64_t chunk_tokens,
                   int64_t n_groups, float *__restrict__ partials, DevStatus *st,
                   uint32_t max_polls) {
  extern __shared__ uint8_t gsm_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(gsm_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  GramTail *tail = reinterpret_cast<GramTail *>(smem + GSTAGES * GSTAGE_BYTES);
  volatile int *abort_flag = &tail->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k = blockIdx.x, chunk = blockIdx.y;
  const int64_t t0 = (int64_t)chunk * chunk_tokens;
  const int64_t t1 = i64min(T, t0 + chunk_tokens);
  const int nsteps = (int)((t1 - t0 + GT - 1) / GT);  // >= 1 by construction of the chunks

  if (threadIdx.x == 0) {
    for (int s = 0; s < GSTAGES; ++s) {
      mbar_init(&tail->full[s], 1);
      mbar_init(&tail->empty[s], 1);
    }
    mbar_init(&tail->done, 1);
    tail->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tmX);
  if (warp == 1) {
    tmem_alloc(&tail->tmem_base, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tail->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_parity = 0;
      bool ok = true;
      for (int step = 0; step < nsteps; ++step) {
        if (!mbar_wait_bounded(&tail->empty[stage], phase ^ 1u, max_polls, abort_flag)) {
          dev_fail(st, kDevTimeout, 0x600u + stage);
          *abort_flag = 1;
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&tail->full[stage], GSTAGE_BYTES);
        const int32_t y = (int32_t)(t0 + (int64_t)step * GT);
        uint8_t *dst = smem + stage * GSTAGE_BYTES;
        tma_load_2d(dst, &tmX, &tail->full[stage], k * 128, y);
        tma_load_2d(dst + GBOX_BYTES, &tmX, &tail->full[stage], k * 128 + 64, y);
        issued |= 1u << stage;
        issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == GSTAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok || *abort_flag)
        for (int s = 0; s < GSTAGES; ++s)
          if (issued & (1u << s))
            (void)mbar_wait_bounded(&tail->full[s], (issued_parity >> s) & 1u, GDRAIN_POLLS, nullptr);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool issued_any = false, ok = true;
      for (int step = 0; step < nsteps; ++step) {
        if (!mbar_wait_bounded(&tail->full[stage], phase, max_polls, abort_flag)) {
          dev_fail(st, kDevTimeout, 0x700u + stage);
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t base = smem_u32(smem + stage * GSTAGE_BYTES);
#pragma unroll
        for (int ks = 0; ks < GT / 16; ++ks) {
          const uint64_t d = smem_desc_mn_sw128(base + ks * 2048);  // 16 token rows per step
          tc_mma_f16(tmem_base, d, d, IDESC_GRAM, (step | ks) != 0 ? 1u : 0u);
        }
        issued_any = true;
        tc_commit(&tail->empty[stage]);
        if (++stage == GSTAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (issued_any) tc_commit(&tail->done);
      if (!ok && issued_any) (void)mbar_wait_bounded(&tail->done, 0, GDRAIN_POLLS, nullptr);
    }
  } else {
    const int q = warp & 3;
    int ok = 1;
    if (lane == 0) ok = mbar_wait_bounded(&tail->done, 0, max_polls, abort_flag);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) {
      if (lane == 0) {
        dev_fail(st, kDevTimeout, 0x800u);
        *abort_flag = 1;
      }
    } else {
      tc_fence_after();
      const int row = q * 32 + lane;
      float *dst = partials + (((int64_t)chunk * n_groups + k) * 128 + row) * 128;
      // the block's (group, chunk) lies in the grid's n_groups x chunks
      const bool dst_ok = AWQ_IN_BOUNDS(k < n_groups && chunk < (int)gridDim.y, 0xB040u);
#pragma unroll 1
      for (int c = 0; c < (dst_ok ? 128 : 0); c += 32) {
        float v[32];
        tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)c, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4 *>(dst + c + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 128);
  }
}

__global__ void gram_reduce_kernel(const float *__restrict__ partials, int n_chunks, int64_t n,
                                   float *__restrict__ Gout) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    float s = 0.0f;
    for (int c = 0; c < n_chunks; ++c) s += partials[(int64_t)c * n + i];
    Gout[i] = s;
  }
}

cudaError_t launch_gram_blocks(const __half *X, int64_t T, int64_t in, int64_t ldx, int group,
                               int n_chunks, float *partials, float *Gout, DevStatus *st,
                               uint32_t max_polls, cudaStream_t stream) {
  (void)group;  // the block Grams are of 128-channel blocks whatever the quantisation group
  if (in % G != 0) return cudaErrorInvalidValue;
  const int64_t n_groups = in / G;
  // chunks are whole multiples of GT tokens so that no TMA box straddles two
  // chunks; only the last chunk ends at T (rows past T read as zero)
  int64_t chunk_tokens = (T + n_chunks - 1) / n_chunks;
  chunk_tokens = (chunk_tokens + GT - 1) / GT * GT;
  const int eff_chunks = (int)((T + chunk_tokens - 1) / chunk_tokens);
  CUtensorMap tm;
  cudaError_t e = make_tmap_f16_box(&tm, X, T, in, ldx, 64, GT);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(gram_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kGramSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)n_groups, (unsigned)eff_chunks);
  gram_tc_kernel<<<grid, 192, kGramSmemBytes, stream>>>(tm, T, chunk_tokens, n_groups, partials, st,
                                                        max_polls);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t n = n_groups * G * G;
  gram_reduce_kernel<<<(unsigned)i64min(4096, (n + 255) / 256), 256, 0, stream>>>(
      partials, eff_chunks, n, Gout);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// K6b — clip scoring on the tensor cores.
//
// With r_i = sqrt(G_ii), G~ = diag(r)^-1 G diag(r)^-1 (|G~_ij| <= 1, zero
// where r vanishes) and d~ = diag(r) d (d = deq_c/s - w of one (row, group,
// clip) candidate), E = d^T G d = d~^T G~ d~.  A CTA owns one group k: it
// builds G~ once in shared memory as two fp16 parts (hi + lo, 22 significant
// bits) and then walks tiles of 128 candidates = R rows x n_clip ratios.  For
// each tile its threads quantise the candidates and write d~ (scaled by a
// per-row power of two to sit inside fp16) as hi + lo parts into a K-major
// 128-byte-swizzled tile; one thread issues
//     Y = A_hi G~_hi + A_lo G~_hi + A_hi G~_lo
// as tcgen05.mma kind::f16 (M = 128 candidates, N = 128, K = 128) into fp32
// TMEM, and every thread dots its candidate's row of Y with its own d~, so no
// cross-thread reduction is needed.  The dropped A_lo G~_lo term is 2^-22 of E.
// ---------------------------------------------------------------------------
namespace {
constexpr int CW_PROD = 12;                       // producer warps 0..11
constexpr int CW_MMA = 12;                        // MMA warp
constexpr int CW_EPI = 13;                        // epilogue warps 13..16
constexpr int CW_NEPI = 4;                        // one per TMEM lane quarter
constexpr int CT_THREADS = (CW_EPI + CW_NEPI) * 32;  // 17 warps: up to 120 registers
constexpr int CT_MAXR = 32;                       // rows per tile at most
constexpr uint32_t CT_ATOM = 128 * 128;           // bytes: 128 rows x 64 fp16
constexpr uint32_t CT_OPND = 2 * CT_ATOM;         // one operand, K = 128
// kind::f16, fp16 A/B, fp32 D, K-major, N = 128, M = 128
constexpr uint32_t IDESC_CLIP = (1u << 4) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t CT_DRAIN = 1u << 22;

struct __align__(16) ClipSmem {
  uint8_t a_hi[2][CT_OPND];  // candidates of two tiles in flight
  uint8_t a_lo[2][CT_OPND];
  uint8_t b_hi[CT_OPND];     // G~ of the current group
  uint8_t b_lo[CT_OPND];
  float s[G], ar[G], r[G];  // s_i, r_i / s_i, r_i = sqrt(G_ii)
  int rexp[2][CT_MAXR];
  float epart[2][4][128];  // per buffer, per group of the block, per candidate
  float ratio[128];  // clip ratio of each index
  uint64_t a_full[2], a_empty[2], acc_full[2], acc_empty[2], mma_done;
  uint32_t tmem_base;
  int prod_ok, epi_ok;  // outcome of a group's wait, broadcast through its named barrier
  int abort_flag;
};
constexpr size_t kClipSmemBytes = sizeof(ClipSmem) + 1024;

// byte offset of 16-byte chunk `c` (0..7) of row `row` inside a K-major
// 128-byte-swizzled atom (8-row core groups of 1024 bytes)
__device__ __forceinline__ uint32_t sw128_off(int row, int c) {
  return (uint32_t)row * 128u + (uint32_t)((c ^ (row & 7)) << 4);
}

__device__ __forceinline__ void split_store8(uint8_t *hi, uint8_t *lo, uint32_t off, const float *v) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __half2 hv = __floats2half2_rn(v[2 * e], v[2 * e + 1]);
    const float2 hf = __half22float2(hv);
    const __half2 lv = __floats2half2_rn(v[2 * e] - hf.x, v[2 * e + 1] - hf.y);
    h[e] = *reinterpret_cast<const uint32_t *>(&hv);
    l[e] = *reinterpret_cast<const uint32_t *>(&lv);
  }
  *reinterpret_cast<uint4 *>(hi + off) = make_uint4(h[0], h[1], h[2], h[3]);
  *reinterpret_cast<uint4 *>(lo + off) = make_uint4(l[0], l[1], l[2], l[3]);
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void named_bar(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ float clip_ratio_f(int c, int n_clip, float clip_min) {
  if (n_clip <= 1) return 1.0f;
  double r = 1.0 - (double)c * (1.0 - (double)clip_min) / (double)(n_clip - 1);
  return __double2float_rn(r);
}
}  // namespace

// Warp-specialised pipeline over (group, row tile) items, two tiles in
// flight: producers (warps 0-11, three per SM sub-partition) build tile t's
// candidates while the MMA warp runs tile t-1 and the epilogue warps (13-16)
// score and pick tile t-2.
// GS: the quantisation group (32, 64 or 128 channels).  A CTA item is still a
// 128-channel block of one row tile: for GS < 128 the block holds 128/GS
// groups, G~ keeps only their diagonal GS x GS blocks (the group's own
// output error, no cross-group terms), and the epilogue's dot products are
// taken per GS-column segment, so one candidate row (row, ratio) scores that
// ratio for every group of the block at once.
// kCodes: the producers also store every candidate's codes q [out, n_clip, in]
// and zero points z [out, n_clip, in/GS] (the inspection form; the search
// itself is unchanged).
template <int GS, bool kCodes>
__global__ void __launch_bounds__(CT_THREADS, 1) clip_tc_kernel(
    const __half *__restrict__ W, int64_t out, int64_t in, const float *__restrict__ s,
    const float *__restrict__ Gall, float qmax, int sym, int n_clip, float clip_min, int rows_per_tile,
    uint8_t *__restrict__ clip_idx, float *__restrict__ err, DevStatus *st, uint32_t max_polls,
    uint8_t *__restrict__ cq, uint8_t *__restrict__ cz) {
  extern __shared__ uint8_t csm_raw[];
  ClipSmem &S = *reinterpret_cast<ClipSmem *>(
      (reinterpret_cast<uintptr_t>(csm_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  volatile int *abort_flag = &S.abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int GPB = G / GS;        // quantisation groups per 128-channel block
  constexpr int CPG = GS / 8;        // 8-channel chunks per group
  const int64_t n_blocks = in / G;
  const int64_t n_groups = in / GS;  // groups of the outputs clip_idx, err, cz
  const int R = rows_per_tile;
  const int64_t n_tiles = (out + R - 1) / R;
  // this CTA's share of the (group, row tile) items, group-major, so a CTA
  // meets at most a few groups and builds each G~ once
  const int64_t n_items = n_blocks * n_tiles;
  const int64_t item_begin = n_items * blockIdx.x / gridDim.x;
  const int64_t item_end = n_items * (blockIdx.x + 1) / gridDim.x;

  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&S.a_full[b], CW_PROD);
      mbar_init(&S.a_empty[b], CW_NEPI);
      mbar_init(&S.acc_full[b], 1);
      mbar_init(&S.acc_empty[b], CW_NEPI);
    }
    mbar_init(&S.mma_done, 1);
    S.abort_flag = 0;
    fence_mbar_init();
  }
  if (tid < n_clip) S.ratio[tid] = clip_ratio_f(tid, n_clip, clip_min);
  if (warp == CW_MMA) {
    tmem_alloc(&S.tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = S.tmem_base;

  if (warp < CW_PROD) {
    // ================================================================ producers
    // Work unit: (row rr, 16-byte chunk ch of 8 channels, split sp of the
    // clip ratios).  A thread keeps its chunk's s, r and r/s in registers
    // for the whole group, reduces its row's range over the 16 lanes that
    // share the row, and walks ratios sp, sp + nsp, ... < n_clip; lane l of
    // the 16 computes the group parameters of its split's l-th ratio once,
    // and the others take them by shuffle.
    const int ptid = tid;  // 0..CW_PROD*32-1
    const int ch = ptid & 15;
    const int nrc = 16 * R;                          // (row, chunk) slots
    const int nsp = nrc >= CW_PROD * 32 ? 1 : (CW_PROD * 32) / nrc;
    const int nunits = nrc * nsp;                    // a multiple of 16, <= 512
    const int cper = (n_clip + nsp - 1) / nsp;       // ratios per split, <= 16
    int64_t k_cur = -1;
    float sv[8], rv[8], av[8];                       // s_i, r_i, r_i / s_i of the chunk
    // the unit of each pass (row rr, split sp) does not change from tile to
    // tile: take the divisions by R once
    const int u0 = warp * 32 + lane, u1 = u0 + CW_PROD * 32;
    const int rr0 = (u0 >> 4) % R, sp0 = (u0 >> 4) / R, rr1 = (u1 >> 4) % R, sp1 = (u1 >> 4) / R;
    uint4 wpre[2];
    auto load_rows = [&](int64_t kk, int64_t oo) {
#pragma unroll
      for (int pass = 0; pass < 2; ++pass) {
        const int64_t o = oo + (pass ? rr1 : rr0);
        wpre[pass] = ((pass ? u1 : u0) < nunits && o < out)
                         ? __ldg(reinterpret_cast<const uint4 *>(W + o * in + kk * G + 8 * ch))
                         : make_uint4(0u, 0u, 0u, 0u);
      }
    };
    // (group k, row tile tl) of the current item, stepped without a 64-bit
    // division per tile
    int64_t k = item_begin / n_tiles, tl = item_begin - k * n_tiles;
    if (item_begin < item_end) load_rows(k, tl * R);
    for (int64_t item = item_begin; item < item_end; ++item) {
      const int t = (int)(item - item_begin);
      const int b = t & 1;
      const bool new_group = k != k_cur;
      // buffer b is free once tile t-2 is scored; a new G~ also needs tile t-1 done
      if (ptid == 0) {
        int ok = mbar_wait_bounded(&S.a_empty[b], ((t >> 1) & 1) ^ 1u, max_polls, abort_flag);
        if (ok && new_group && t >= 1)
          ok = mbar_wait_bounded(&S.a_empty[b ^ 1], ((t - 1) >> 1) & 1, max_polls, abort_flag);
        if (!ok) {
          dev_fail(st, kDevTimeout, 0x910u);
          *abort_flag = 1;
        }
        S.prod_ok = ok;
      }
      named_bar(1, CW_PROD * 32);
      if (!S.prod_ok) break;
      if (new_group) {
        // ---- group set-up: s, r = sqrt(G_ii), r/s, then G~ = G_ij / (r_i r_j)
        // as hi + lo fp16, K-major swizzled (row j, channel i)
        k_cur = k;
        const float *Gk = Gall + k * G * G;
        if (ptid < G) {
          const float s0 = s ? s[k * G + ptid] : 1.0f;
          const float r0 = sqrtf(fmaxf(Gk[ptid * G + ptid], 0.0f));
          S.s[ptid] = s0;
          S.r[ptid] = r0;
          S.ar[ptid] = r0 / s0;
        }
        named_bar(1, CW_PROD * 32);
        // row j, channels 64 h .. 64 h + 63 (threads 0..255); a warp shares h,
        // so its swizzled 16-byte stores fall in distinct banks
        const int j = ptid & 127, h = ptid >> 7;
        const float rj = S.r[j];
        const float *grow = Gk + (int64_t)j * G + 64 * h;
#pragma unroll 1
        for (int c = 0; c < (ptid < 256 ? 8 : 0); ++c) {
          float v[8];
          const float4 g0 = __ldg(reinterpret_cast<const float4 *>(grow + 8 * c));
          const float4 g1 = __ldg(reinterpret_cast<const float4 *>(grow + 8 * c + 4));
          const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int i = 64 * h + 8 * c + e;
            const float den = rj * S.r[i];
            // only the group's own block (every entry when GS = 128)
            v[e] = (den > 0.0f && (i / GS) == (j / GS)) ? gv[e] / den : 0.0f;
          }
          split_store8(S.b_hi + h * CT_ATOM, S.b_lo + h * CT_ATOM, sw128_off(j, c), v);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          sv[e] = S.s[8 * ch + e];
          rv[e] = S.r[8 * ch + e];
          av[e] = S.ar[8 * ch + e];
        }
      }
#pragma unroll 1
      for (int pass = 0; pass < 2; ++pass) {
        const int ub = warp * 32 + pass * CW_PROD * 32;  // warp-uniform
        if (ub >= nunits) break;
        const int u = ub + lane;
        const bool live = u < nunits;
        const int rr = pass ? rr1 : rr0, sp = pass ? sp1 : sp0;
        // ---- this row's range (s w) and the exponent of the d~ scaling
        const uint4 wv = pass ? wpre[1] : wpre[0];  // no dynamic register indexing
        const uint32_t wr[4] = {wv.x, wv.y, wv.z, wv.w};
        float2 wt[4];
        float mx = -INFINITY, mn = INFINITY, bmax = 0.0f;
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float2 w2 = __half22float2(*reinterpret_cast<const __half2 *>(&wr[h]));
          wt[h] = __fmul2_rn(make_float2(sv[2 * h], sv[2 * h + 1]), w2);
          mx = fmaxf(mx, fmaxf(wt[h].x, wt[h].y));
          mn = fminf(mn, fminf(wt[h].x, wt[h].y));
          bmax = fmaxf(bmax, fmaxf(rv[2 * h] * fabsf(w2.x), rv[2 * h + 1] * fabsf(w2.y)));
        }
        // the group's range over its CPG lanes, the row's bmax over all 16
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) {
          if (off < CPG) {
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
          }
          bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, off));
        }
        // |d~_i| <= r_i |w_i| (+ rounding): keep 2 bmax 2^e <= 2^14
        int e2 = 0;
        if (bmax > 0.0f) {
          (void)frexpf(2.0f * bmax, &e2);
          e2 = 14 - e2;
        }
        if (live && ch == 0 && sp == 0 && AWQ_IN_BOUNDS(rr < CT_MAXR, 0xB041u)) S.rexp[b][rr] = e2;
        const float sc = ldexpf(1.0f, e2);
        float2 ae[4];  // (r_i / s_i) 2^e, exact power-of-two scaling
#pragma unroll
        for (int h = 0; h < 4; ++h) ae[h] = __fmul2_rn(make_float2(av[2 * h], av[2 * h + 1]), make_float2(sc, sc));
        // ---- GS = 128: parameters of ratio sp + nsp * (lane % 16), computed
        // once and shared by shuffle; smaller groups compute their own below
        GroupQ gq;
        if constexpr (GS == 128) {
          const int cl = sp + nsp * ch;
          gq = group_params(mx, mn, S.ratio[cl < n_clip ? cl : 0], qmax, sym != 0);
          // every quotient of the group stays below 63 in magnitude, which the
          // remainder test below needs; otherwise force the exact path
          if (!(fmaxf(fabsf(mx), fabsf(mn)) * gq.rcp < 63.0f)) gq.half_lo = -1.0f;
        }
        const int p0 = rr * n_clip;
        uint8_t *ahi = S.a_hi[b] + (ch >> 3) * CT_ATOM, *alo = S.a_lo[b] + (ch >> 3) * CT_ATOM;
#pragma unroll 2
        for (int jc = 0; jc < cper; ++jc) {  // two ratios interleaved: more independent work
          const int c = sp + nsp * jc;
          float dl, rc, hl, zz;
          if constexpr (GS == 128) {
            dl = __shfl_sync(0xffffffffu, gq.delta, jc, 16);
            rc = __shfl_sync(0xffffffffu, gq.rcp, jc, 16);
            hl = __shfl_sync(0xffffffffu, gq.half_lo, jc, 16);
            zz = __shfl_sync(0xffffffffu, gq.zero, jc, 16);
          } else {
            GroupQ g2 = group_params(mx, mn, S.ratio[c < n_clip ? c : 0], qmax, sym != 0);
            if (!(fmaxf(fabsf(mx), fabsf(mn)) * g2.rcp < 63.0f)) g2.half_lo = -1.0f;
            dl = g2.delta;
            rc = g2.rcp;
            hl = g2.half_lo;
            zz = g2.zero;
          }
          const bool store = live && c < n_clip;  // past n_clip: lane 0's ratio, not stored
          // (q - z) = clamp(rne(wt / delta), -z, qmax - z), proposed from the
          // approximate reciprocal (one FMA rounds wt rc + 1.5 2^23 straight to
          // an integer) and proven by the remainder
          float2 kq[4];
          float rmax = 0.0f;
#pragma unroll
          for (int h = 0; h < 4; ++h) {  // 12582912 = 1.5 2^23
            kq[h] = __fadd2_rn(__ffma2_rn(wt[h], make_float2(rc, rc), make_float2(12582912.0f, 12582912.0f)),
                               make_float2(-12582912.0f, -12582912.0f));
            const float2 rem = __ffma2_rn(make_float2(-kq[h].x, -kq[h].y), make_float2(dl, dl), wt[h]);
            rmax = fmax3(rmax, fabsf(rem.x), fabsf(rem.y));
          }
          if (!(rmax < hl)) {
#pragma unroll
            for (int h = 0; h < 4; ++h)
              kq[h] = make_float2(rintf(__fdiv_rn(wt[h].x, dl)), rintf(__fdiv_rn(wt[h].y, dl)));
          }
          const float lo = -zz, hi = qmax - zz;
          float v[8];
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const float2 qz = make_float2(fminf(fmaxf(kq[h].x, lo), hi), fminf(fmaxf(kq[h].y, lo), hi));
            // d~ 2^e = ((q - z) delta - s w) (r / s) 2^e
            const float2 tq = __ffma2_rn(qz, make_float2(dl, dl), make_float2(-wt[h].x, -wt[h].y));
            const float2 d2 = __fmul2_rn(tq, ae[h]);
            v[2 * h] = d2.x;
            v[2 * h + 1] = d2.y;
          }
          if (store) split_store8(ahi, alo, sw128_off(p0 + c, ch & 7), v);
          if constexpr (kCodes) {
            const int64_t o = tl * R + rr;
            if (store && o < out) {
              uint32_t cw[2] = {0u, 0u};
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                const float qa = fminf(fmaxf(kq[h].x, lo), hi) + zz;
                const float qb = fminf(fmaxf(kq[h].y, lo), hi) + zz;
                cw[h >> 1] |= ((uint32_t)qa << (16 * (h & 1))) | ((uint32_t)qb << (16 * (h & 1) + 8));
              }
              *reinterpret_cast<uint2 *>(cq + (o * n_clip + c) * in + k * G + 8 * ch) =
                  make_uint2(cw[0], cw[1]);
              if (ch % CPG == 0) cz[(o * n_clip + c) * n_groups + k * GPB + ch / CPG] = (uint8_t)zz;
            }
          }
        }
      }
      if (++tl == n_tiles) {
        tl = 0;
        ++k;
      }
      if (item + 1 < item_end) load_rows(k, tl * R);
      fence_async_smem();  // generic-proxy writes (A and, on a new group, B) -> tensor cores
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.a_full[b]);
    }
  } else if (warp == CW_MMA) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      bool issued_any = false;
      for (int64_t item = item_begin; item < item_end; ++item) {
        const int t = (int)(item - item_begin);
        const int b = t & 1;
        const uint32_t ph = (t >> 1) & 1;
        if (!mbar_wait_bounded(&S.a_full[b], ph, max_polls, abort_flag) ||
            !mbar_wait_bounded(&S.acc_empty[b], ph ^ 1u, max_polls, abort_flag)) {
          dev_fail(st, kDevTimeout, 0x920u);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        // Y = A_hi B_hi + A_lo B_hi + A_hi B_lo
        const uint32_t a_hi = smem_u32(S.a_hi[b]), a_lo = smem_u32(S.a_lo[b]);
        const uint32_t b_hi = smem_u32(S.b_hi), b_lo = smem_u32(S.b_lo);
        const uint32_t as[3] = {a_hi, a_lo, a_hi}, bs[3] = {b_hi, b_hi, b_lo};
        const uint32_t d = tmem_base + (uint32_t)(b * 128);
#pragma unroll
        for (int tt = 0; tt < 3; ++tt)
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint32_t koff = (uint32_t)(ks >> 2) * CT_ATOM + (uint32_t)(ks & 3) * 32u;
            tc_mma_f16(d, smem_desc_k_sw128(as[tt] + koff), smem_desc_k_sw128(bs[tt] + koff),
                       IDESC_CLIP, (tt | ks) != 0 ? 1u : 0u);
          }
        tc_commit(&S.acc_full[b]);
        issued_any = true;
      }
      if (issued_any) {
        tc_commit(&S.mma_done);
        (void)mbar_wait_bounded(&S.mma_done, 0, CT_DRAIN, nullptr);
      }
    }
  } else {
    // ================================================================ epilogue
    const int etid = tid - CW_EPI * 32;  // 0..127
    const int q = warp & 3;              // TMEM lane quarter of this warp
    const int p = q * 32 + lane;         // candidate (accumulator row)
    int64_t k = item_begin / n_tiles, tl = item_begin - k * n_tiles;
    for (int64_t item = item_begin; item < item_end; ++item, ++tl) {
      const int t = (int)(item - item_begin);
      const int b = t & 1;
      const uint32_t ph = (t >> 1) & 1;
      if (tl == n_tiles) {
        tl = 0;
        ++k;
      }
      const int64_t o0 = tl * R;
      if (etid == 0) {
        // acc_full: the products are in TMEM; a_full (already complete) makes
        // the producers' plain stores of A and the row data visible here
        const int ok = mbar_wait_bounded(&S.acc_full[b], ph, max_polls, abort_flag) &&
                       mbar_wait_bounded(&S.a_full[b], ph, max_polls, abort_flag);
        if (!ok) {
          dev_fail(st, kDevTimeout, 0x930u);
          *abort_flag = 1;
        }
        S.epi_ok = ok;
      }
      named_bar(2, CW_NEPI * 32);
      if (!S.epi_ok) break;
      tc_fence_after();
      // E = d~ . y over the 128 columns of this candidate's accumulator row
      float2 e2a = make_float2(0.0f, 0.0f), e2b = make_float2(0.0f, 0.0f);
#pragma unroll 1
      for (int cb = 0; cb < 4; ++cb) {  // 32 columns each; a group ends every GS / 32
        float y[32];
        tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * 128 + 32 * cb), y);
        tmem_ld_wait();
        const uint8_t *ahi = S.a_hi[b] + (cb >> 1) * CT_ATOM, *alo = S.a_lo[b] + (cb >> 1) * CT_ATOM;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int c = (cb & 1) * 4 + cc;
          const uint4 hv = *reinterpret_cast<const uint4 *>(ahi + sw128_off(p, c));
          const uint4 lv = *reinterpret_cast<const uint4 *>(alo + sw128_off(p, c));
          const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w}, lw[4] = {lv.x, lv.y, lv.z, lv.w};
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const float2 fh = __half22float2(*reinterpret_cast<const __half2 *>(&hw[x]));
            const float2 fl = __half22float2(*reinterpret_cast<const __half2 *>(&lw[x]));
            const float2 yy = make_float2(y[8 * cc + 2 * x], y[8 * cc + 2 * x + 1]);
            if (x & 1)
              e2b = __ffma2_rn(__fadd2_rn(fh, fl), yy, e2b);
            else
              e2a = __ffma2_rn(__fadd2_rn(fh, fl), yy, e2a);
          }
        }
        if (((cb + 1) * 32) % GS == 0) {  // this candidate's E for group cb * 32 / GS
          S.epart[b][(cb * 32) / GS][p] = (e2a.x + e2b.x) + (e2a.y + e2b.y);
          e2a = make_float2(0.0f, 0.0f);
          e2b = make_float2(0.0f, 0.0f);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.acc_empty[b]);
      // the argmin below needs only epart (this block's) and its row's
      // exponent: take the exponent now and release A, the row data and the
      // buffer to the producers as soon as every dot is done.  TPP threads
      // share one (row, group) pair.
      constexpr int TPP = 4 / GPB;
      const int pair = etid / TPP, part = etid % TPP;
      const int rr = pair / GPB, kk = pair % GPB;
      const int rexp_row = S.rexp[b][rr];  // rr < 32
      named_bar(2, CW_NEPI * 32);
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.a_empty[b]);
      // ---- per (row, group): first clip index with the smallest E; the pair's
      // threads scan every TPP-th ratio, then combine (ties keep the lower index)
      {
        const bool row_ok = rr < R && o0 + rr < out;
        const int64_t gk = k * GPB + kk;  // group index along in
        float best = INFINITY;
        int bc = 1 << 30;
        if (row_ok) {
          const float unscale = ldexpf(1.0f, -2 * rexp_row);
          for (int c = part; c < n_clip; c += TPP) {
            const float ev = S.epart[b][kk][rr * n_clip + c] * unscale;
            if (err && AWQ_IN_BOUNDS(gk < n_groups, 0xB042u)) err[((o0 + rr) * n_groups + gk) * n_clip + c] = ev;
            if (ev < best) {
              best = ev;
              bc = c;
            }
          }
        }
#pragma unroll
        for (int off = 1; off < TPP; off <<= 1) {
          const float ob = __shfl_xor_sync(0xffffffffu, best, off);
          const int oc = __shfl_xor_sync(0xffffffffu, bc, off);
          if (ob < best || (ob == best && oc < bc)) {
            best = ob;
            bc = oc;
          }
        }
        if (row_ok && part == 0 && AWQ_IN_BOUNDS(gk < n_groups, 0xB043u))
          clip_idx[(o0 + rr) * n_groups + gk] = (uint8_t)bc;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == CW_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 256);
  }
}

cudaError_t launch_clip_eval(const __half *W, int64_t out, int64_t in, const float *s,
                             const float *Gall, int group, int w_bit, int zero_point, int n_clip,
                             float clip_min, uint8_t *clip_idx, float *err, DevStatus *st,
                             uint32_t max_polls, int num_sms, cudaStream_t stream, uint8_t *cq,
                             uint8_t *cz) {
  if ((group != 32 && group != 64 && group != G) || in % G != 0 || n_clip < 1 || n_clip > 128)
    return cudaErrorInvalidValue;
  int R = 128 / n_clip;
  if (R > CT_MAXR) R = CT_MAXR;
  const int64_t n_items = (in / G) * ((out + R - 1) / R);
  const int64_t ctas = i64min(num_sms, n_items);  // one CTA per SM (shared memory bound)
  auto kern = group == 32   ? (cq ? clip_tc_kernel<32, true> : clip_tc_kernel<32, false>)
              : group == 64 ? (cq ? clip_tc_kernel<64, true> : clip_tc_kernel<64, false>)
                            : (cq ? clip_tc_kernel<128, true> : clip_tc_kernel<128, false>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kClipSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)ctas);
  kern<<<grid, CT_THREADS, kClipSmemBytes, stream>>>(
      W, out, in, s, Gall, (float)((1 << w_bit) - 1), zero_point ? 0 : 1, n_clip, clip_min, R,
      clip_idx, err, st, max_polls, cq, cz);
  return cudaGetLastError();
}

AWQ_BOUNDS_READER(bounds_status_clip)

}  // namespace awq
