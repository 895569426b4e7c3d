// K4, fused form: the scored candidate GEMM with the candidates built inside
// it ("05 — AWQ: Activation-Aware Weight Scaling" §4: for each alpha apply
// the scaling, quantise, measure the error).  The direct form writes every
// candidate's effective error dW = (Qdeq(s w)/s - w) 2^k to HBM
// (n_alpha x out x in fp16, 640 MiB for a 4096 x 4096 layer) and streams it
// back as the GEMM's B operand.  Here the B tiles are made in shared memory
// from W itself, so that buffer never exists:
//   K3p  fused_params: per (alpha, row, group) the quantiser's step, its
//        zero point and two flags (8 bytes, 21 MB for the layer above; the
//        approximate reciprocal and the fast-path bound follow), from the group's
//        range of s w -- the values the candidate kernel derives on the way;
//   K4f  fused_search_gemm: the scored GEMM's 256 x 256 tiles (two M = 128
//        tcgen05 MMAs share each B tile), where a TMA load brings the W rows
//        of the B tile instead of dW, and sixteen converter warps turn that
//        tile into dW in place (a thread owns one 8-channel chunk column of 4
//        rows of each 64-channel K slice) before the MMA warp may read it.
// Each value goes through the candidate kernel's exact steps in the same
// order (s 2^k w, the proposed code proven by its remainder or decided by the
// correctly rounded quotient, the clamp, (q - z) delta - s w times 1/s), so
// the B tiles hold the direct form's operand values (an error of exactly
// zero may carry the other sign, which no product or square can see), and
// the epilogue, the tile order and the partial sums are the scored GEMM's:
// the MSE comes out bit for bit the same.  The price is the conversion, once per
// 256-token M tile instead of once per layer.
#include <cuda.h>
#include <cuda_fp16.h>
#include <math.h>

#include "awq_launch.h"

namespace awq {

namespace {

constexpr int FBM = kGemmBM, FBN = kGemmBN, FBK = kGemmBK;  // 128, 256, 64
constexpr int F_STAGES = 3;
constexpr int FBM2 = 2 * FBM;                    // CTA tile rows: two M = 128 accumulators
constexpr uint32_t F_A_HALF = FBM * FBK * 2;     // 16 KiB
constexpr uint32_t F_A_BYTES = FBM2 * FBK * 2;   // 32 KiB
constexpr uint32_t F_B_BYTES = FBN * FBK * 2;    // 32 KiB: W rows, converted to dW in place
constexpr uint32_t F_TMEM_COLS = 512;
constexpr uint32_t F_IDESC = idesc_f16_f32(FBM, FBN);
constexpr uint32_t F_DRAIN_POLLS = 1u << 22;
constexpr int F_GROUP_M = 16;
constexpr int F_EPI_WARPS = 4;   // warps 2..5
constexpr int F_CONV_WARPS = 16;  // warps 6..21: 4 chunks of each B tile slice per thread
constexpr int F_CONV_ROWS = FBN * 8 / (F_CONV_WARPS * 32);  // rows per converter thread
constexpr int F_CONV0 = 2 + F_EPI_WARPS;
constexpr int F_THREADS = (F_CONV0 + F_CONV_WARPS) * 32;
static_assert(F_CONV_ROWS * F_CONV_WARPS * 32 == FBN * 8, "every 16-byte chunk of a B slice once");

struct __align__(8) FusedSmemTail {
  uint64_t full[F_STAGES];  // TMA: A tile and W rows landed
  uint64_t conv[F_STAGES];  // converters: the B tile holds dW
  uint64_t empty[F_STAGES]; // MMAs done: the stage may be refilled
  uint64_t tfull, tempty, mma_done;
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t kFusedSmemBytes =
    1024 /*alignment slack*/ + F_STAGES * (F_A_BYTES + F_B_BYTES) + sizeof(FusedSmemTail);

__device__ __forceinline__ void f_tile_coords(int tile, int num_m, int num_n, int group_m, int &m_blk,
                                              int &n_blk) {
  const int per_group = group_m * num_n;
  const int g = tile / per_group;
  const int first_m = g * group_m;
  const int gm = min(group_m, num_m - first_m);
  const int local = tile - g * per_group;
  m_blk = first_m + local % gm;
  n_blk = local / gm;
}

__device__ __forceinline__ void f_abort(FusedSmemTail *t, DevStatus *st, uint32_t where) {
  dev_fail(st, kDevTimeout, where);
  *reinterpret_cast<volatile int *>(&t->abort_flag) = 1;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// byte offset of 16-byte chunk c (0..7) of row r in a K-major 128-byte-swizzled
// tile of 64-channel rows (the layout the TMA box writes and the MMA reads)
__device__ __forceinline__ uint32_t sw128_chunk(int r, int c) {
  return (uint32_t)r * 128u + (uint32_t)((c ^ (r & 7)) << 4);
}
}  // namespace

// ---------------------------------------------------------------------------
// K3p.  A warp takes one row of W and the 256-channel slab blockIdx.y, and
// walks the alphas with the row's weights in registers: lane l holds
// channels 8l..8l+7, reduces its group's range of RN32(s 2^k w) over
// the group's group / 8 lanes, and the group's first lane writes
//   {delta, bits of (zero | clamp << 8 | no fast path << 9)}
// as the candidate kernel computes them (group_params at ratio 1 with the
// 1e-5 2^k floor, the fast-path bound, and whether the codes of the range's
// ends leave [0, qmax]).  Rows out..out_pad-1 read w = 0.
// ---------------------------------------------------------------------------
template <int group>
__global__ void __launch_bounds__(256) fused_params_kernel(
    const __half *__restrict__ W, int64_t out, int64_t in, int64_t out_pad,
    const float *__restrict__ s, int n_alpha, float qmax, int sym, const DevStatus *__restrict__ st,
    float2 *__restrict__ params) {
  constexpr int lanes = group / 8;
  const int k = kscale_from_wmax(__uint_as_float(__ldcg(&st->wmax_bits)));
  const float two_k = ldexpf(1.0f, k);
  const float guard = __fmul_rn(1e-5f, two_k);  // exact
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t o = (int64_t)blockIdx.x * 8 + warp;  // row of W (rows past out read w = 0)
  if (o >= out_pad) return;                          // whole warps
  const int64_t j0 = (int64_t)blockIdx.y * 256 + lane * 8;
  const bool j_ok = j0 < in;
  // the row's 8 weights of this lane, read once for every alpha
  const uint4 wv = j_ok && o < out ? __ldg(reinterpret_cast<const uint4 *>(W + o * in + j0))
                                   : make_uint4(0u, 0u, 0u, 0u);
  const uint32_t wr[4] = {wv.x, wv.y, wv.z, wv.w};
  float2 w2[4];
#pragma unroll
  for (int h = 0; h < 4; ++h) w2[h] = __half22float2(*reinterpret_cast<const __half2 *>(&wr[h]));
  const float2 tk = make_float2(two_k, two_k);
  for (int a = 0; a < n_alpha; ++a) {
    float m = -INFINITY, n = INFINITY;
    if (j_ok) {
      const float4 *sp = reinterpret_cast<const float4 *>(s + (int64_t)a * in + j0);
      const float4 s0 = __ldg(sp), s1 = __ldg(sp + 1);
      const float2 sk[4] = {__fmul2_rn(make_float2(s0.x, s0.y), tk), __fmul2_rn(make_float2(s0.z, s0.w), tk),
                            __fmul2_rn(make_float2(s1.x, s1.y), tk), __fmul2_rn(make_float2(s1.z, s1.w), tk)};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float2 t = __fmul2_rn(sk[h], w2[h]);
        m = fmax3(m, t.x, t.y);
        n = fmin3(n, t.x, t.y);
      }
    }
#pragma unroll
    for (int off = lanes / 2; off >= 1; off >>= 1) {
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      n = fminf(n, __shfl_xor_sync(0xffffffffu, n, off));
    }
    if (j_ok && (lane & (lanes - 1)) == 0) {
      GroupQ g = group_params(m, n, 1.0f, qmax, sym != 0, guard);
      fast_path_check(g, m, n);
      const float qhi = __fadd_rn(round_quotient(m, g), g.zero);
      const float qlo = __fadd_rn(round_quotient(n, g), g.zero);
      const bool clamp = !(qlo >= 0.0f && qhi <= g.qmax);
      // the reciprocal and the fast-path bound follow from delta (the same
      // instructions give the same bits), unless the bound was disabled
      const int zf = (int)g.zero | (clamp ? 256 : 0) | (g.half_lo < 0.0f ? 512 : 0);
      const int64_t gi = j0 / group;
      if (AWQ_IN_BOUNDS(gi < in / group, 0xB070u))
        params[((int64_t)a * out_pad + o) * (in / group) + gi] = make_float2(g.delta, __int_as_float(zf));
    }
  }
}

// ---------------------------------------------------------------------------
// K4f.  Warp 0 loads the A tile (X, 256 x 64) and the W rows of the B tile
// (256 x 64) by TMA into a 3-stage ring; warps 6..21 wait for a stage, turn
// its W rows into dW in place and arrive on the stage's conversion barrier;
// warp 1 issues the two M = 128 MMAs per K slice once both have happened;
// warps 2..5 square and sum the accumulators as the scored GEMM's epilogue
// does.  Every wait is bounded; a wait that runs out records the timeout and
// every role drains what it has in flight before the CTA frees its TMEM.
// ---------------------------------------------------------------------------
template <int group>
__global__ void __launch_bounds__(F_THREADS, 1)
    fused_search_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                             const __grid_constant__ CUtensorMap tmW, int num_m, int num_n, int num_kb,
                             int64_t in, int64_t out_pad, const float *__restrict__ s,
                             const float *__restrict__ inv_s, const float2 *__restrict__ params,
                             float qmax, double *__restrict__ partials, DevStatus *st,
                             uint32_t max_polls) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sA = smem;
  uint8_t *sB = smem + F_STAGES * F_A_BYTES;
  FusedSmemTail *tail = reinterpret_cast<FusedSmemTail *>(sB + F_STAGES * F_B_BYTES);
  volatile int *abort_flag = &tail->abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_m2 = (num_m + 1) / 2;
  const int num_tiles = num_m2 * num_n;

  if (threadIdx.x == 0) {
    for (int i = 0; i < F_STAGES; ++i) {
      mbar_init(&tail->full[i], 1);
      mbar_init(&tail->conv[i], F_CONV_WARPS);
      mbar_init(&tail->empty[i], 1);
    }
    mbar_init(&tail->tfull, 1);
    mbar_init(&tail->tempty, F_EPI_WARPS);
    mbar_init(&tail->mma_done, 1);
    tail->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(&tail->tmem_base, F_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tail->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_parity = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        int m_blk, n_blk;
        f_tile_coords(tile, num_m2, num_n, F_GROUP_M, m_blk, n_blk);
        // the B tile's candidate rows lie in one alpha (out_pad is a multiple
        // of 256): W rows o0 .. o0 + 255 (rows past out read as zeros)
        const int o0 = (int)(((int64_t)n_blk * FBN) % out_pad);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_long(&tail->empty[stage], phase ^ 1u, max_polls, abort_flag)) {
            f_abort(tail, st, 0x1100u + stage);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&tail->full[stage], F_A_BYTES + F_B_BYTES);
          tma_load_2d(sA + stage * F_A_BYTES, &tmA, &tail->full[stage], kb * FBK, m_blk * FBM2);
          tma_load_2d(sB + stage * F_B_BYTES, &tmW, &tail->full[stage], kb * FBK, o0);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == F_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok || *abort_flag) {
        for (int i = 0; i < F_STAGES; ++i)
          if (issued & (1u << i))
            (void)mbar_wait_bounded(&tail->full[i], (issued_parity >> i) & 1u, F_DRAIN_POLLS, nullptr);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true, issued_any = false;
      int it = 0;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++it) {
        if (!mbar_wait_bounded(&tail->tempty, (it & 1) ^ 1u, max_polls, abort_flag)) {
          f_abort(tail, st, 0x1200u);
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_bounded(&tail->full[stage], phase, max_polls, abort_flag) ||
              !mbar_wait_bounded(&tail->conv[stage], phase, max_polls, abort_flag)) {
            f_abort(tail, st, 0x1300u + stage);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * F_A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * F_B_BYTES);
#pragma unroll
          for (int kk = 0; kk < FBK / 16; ++kk) {
            const uint64_t bd = smem_desc_k_sw128(b_addr + kk * 32);
#pragma unroll
            for (int h = 0; h < 2; ++h)
              tc_mma_f16(tmem_base + h * FBN, smem_desc_k_sw128(a_addr + h * F_A_HALF + kk * 32), bd,
                         F_IDESC, (kb | kk) != 0 ? 1u : 0u);
          }
          issued_any = true;
          tc_commit(&tail->empty[stage]);
          if (++stage == F_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&tail->tfull);
      }
      if (issued_any) {
        tc_commit(&tail->mma_done);
        (void)mbar_wait_bounded(&tail->mma_done, 0, F_DRAIN_POLLS, nullptr);
      }
    }
  } else if (warp < F_CONV0) {
    // ------------------------------------------------------------ epilogue
    // four warps, one per TMEM lane quarter, each drains both row halves
    const int q = warp & 3;
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      int ok = 1;
      if (lane == 0) ok = mbar_wait_long(&tail->tfull, it & 1, max_polls, abort_flag);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        if (lane == 0) f_abort(tail, st, 0x1400u);
        break;
      }
      tc_fence_after();
      int m_blk, n_blk;
      f_tile_coords(tile, num_m2, num_n, F_GROUP_M, m_blk, n_blk);
      float sum[2] = {0.0f, 0.0f};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (2 * m_blk + h >= num_m) continue;  // the last tile's second half may lie past T
        const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(h * FBN);
#pragma unroll 1
        for (int c = 0; c < FBN; c += 32) {  // the scored GEMM's order of squares
          float v[32];
          tmem_ld_32x32b_x32(taddr + (uint32_t)c, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) sum[h] = fmaf(v[i], v[i], sum[h]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tail->tempty);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int m128 = 2 * m_blk + h;
        double ds = (double)sum[h];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ds += __shfl_xor_sync(0xffffffffu, ds, off);
        if (lane == 0 && m128 < num_m && AWQ_IN_BOUNDS(n_blk < num_n, 0xB071u))
          partials[((size_t)n_blk * num_m + m128) * 4 + q] = ds;
      }
    }
  } else {
    // ------------------------------------------------------------ converters
    // thread ct converts 16-byte chunk column cc (channels 8 cc .. 8 cc + 7 of
    // the K slice) of rows r0 + 64 i, i = 0..3, of every B tile: its s 2^k
    // and 1/s are loaded once per K slice, and a warp's 32 chunks are 512
    // contiguous bytes of shared memory (four rows).  Row r of the tile is
    // candidate row n_blk * 256 + r: alpha a and row o0 + r of W.
    const int ct = threadIdx.x - F_CONV0 * 32;
    constexpr int kRowStep = F_CONV_WARPS * 4;  // rows between a thread's chunks
    const int cc = ct & 7, r0 = ct >> 3;        // rows r0 + kRowStep i
    const uint32_t off0 = sw128_chunk(r0, cc);  // kRowStep % 8 == 0: the same swizzle for every i
    const int k = kscale_from_wmax(__uint_as_float(__ldcg(&st->wmax_bits)));
    const float2 tk = make_float2(ldexpf(1.0f, k), ldexpf(1.0f, k));
    const float2 M = make_float2(12582912.0f, 12582912.0f);  // 1.5 2^23
    const int64_t groups = in / group;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
      int m_blk, n_blk;
      f_tile_coords(tile, num_m2, num_n, F_GROUP_M, m_blk, n_blk);
      const int64_t crow0 = (int64_t)n_blk * FBN;  // alpha * out_pad + o0
      const int64_t a = crow0 / out_pad;
      const float2 *prow = params + (crow0 + r0) * groups;
      float2 p[F_CONV_ROWS];  // the rows' group parameters, reloaded when a group starts
      for (int kb = 0; kb < num_kb; ++kb) {
        // every lane waits (each reads what the TMA wrote); the warp gives up together
        const bool w_ok = mbar_wait_bounded(&tail->full[stage], phase, max_polls, abort_flag);
        if (!__all_sync(0xffffffffu, w_ok)) {
          if (lane == 0) f_abort(tail, st, 0x1500u + stage);
          ok = false;
          break;
        }
        const int64_t j = (int64_t)kb * FBK + 8 * cc;  // first channel of the chunk column
        if (group < FBK || (kb * FBK) % group == 0) {
#pragma unroll
          for (int i = 0; i < F_CONV_ROWS; ++i) p[i] = __ldg(prow + (int64_t)(kRowStep * i) * groups + j / group);
        }
        const float4 *sp = reinterpret_cast<const float4 *>(s + a * in + j);
        const float4 *ip = reinterpret_cast<const float4 *>(inv_s + a * in + j);
        const float4 s0 = __ldg(sp), s1 = __ldg(sp + 1), i0 = __ldg(ip), i1 = __ldg(ip + 1);
        const float2 sk[4] = {__fmul2_rn(make_float2(s0.x, s0.y), tk), __fmul2_rn(make_float2(s0.z, s0.w), tk),
                              __fmul2_rn(make_float2(s1.x, s1.y), tk), __fmul2_rn(make_float2(s1.z, s1.w), tk)};
        const float2 iv[4] = {make_float2(i0.x, i0.y), make_float2(i0.z, i0.w), make_float2(i1.x, i1.y),
                              make_float2(i1.z, i1.w)};
        uint8_t *b = sB + stage * F_B_BYTES + off0;
#pragma unroll
        for (int i = 0; i < F_CONV_ROWS; ++i) {
          const float dl = p[i].x;
          const int zf = __float_as_int(p[i].y);
          const float rc = rcp_approx(dl);  // as group_params derives them
          const float hl = (zf & 512) ? -1.0f : __fmul_rn(dl, 0.4999847412109375f /* 0.5 - 2^-16 */);
          uint4 *cp = reinterpret_cast<uint4 *>(b + i * kRowStep * 128);
          const uint4 wv = *cp;
          const uint32_t wr[4] = {wv.x, wv.y, wv.z, wv.w};
          float2 wt[4], qz[4], rem[4];
          float rmax = 0.0f;
#pragma unroll
          for (int hh = 0; hh < 4; ++hh) {
            wt[hh] = __fmul2_rn(sk[hh], __half22float2(*reinterpret_cast<const __half2 *>(&wr[hh])));
            qz[hh] = __fadd2_rn(__ffma2_rn(wt[hh], make_float2(rc, rc), M), make_float2(-M.x, -M.y));
            rem[hh] = __ffma2_rn(qz[hh], make_float2(-dl, -dl), wt[hh]);  // RN(wt - q delta)
            rmax = fmax3(rmax, fabsf(rem[hh].x), fabsf(rem[hh].y));
          }
          uint32_t packed[4];
          if (rmax < hl && !(zf & 256)) {
            // every proposed code is proven and none is clamped: the error
            // (q - z) delta - s w is RN(q delta - wt) = -rem (one rounding
            // either way, up to the sign of a zero), so dW = RN(rem (-1/s))
            // needs no further FMA
#pragma unroll
            for (int hh = 0; hh < 4; ++hh) {
              const float2 d2 = __fmul2_rn(rem[hh], make_float2(-iv[hh].x, -iv[hh].y));
              const __half2 hv = __floats2half2_rn(d2.x, d2.y);
              packed[hh] = *reinterpret_cast<const uint32_t *>(&hv);
            }
          } else {
            if (!(rmax < hl)) {
#pragma unroll
              for (int hh = 0; hh < 4; ++hh)
                qz[hh] = make_float2(rintf(__fdiv_rn(wt[hh].x, dl)), rintf(__fdiv_rn(wt[hh].y, dl)));
            }
            if (zf & 256) {
              const float zero = (float)(zf & 255);
              const float lo = -zero, hi = qmax - zero;
#pragma unroll
              for (int hh = 0; hh < 4; ++hh)
                qz[hh] = make_float2(fminf(fmaxf(qz[hh].x, lo), hi), fminf(fmaxf(qz[hh].y, lo), hi));
            }
#pragma unroll
            for (int hh = 0; hh < 4; ++hh) {
              const float2 t = __ffma2_rn(qz[hh], make_float2(dl, dl), make_float2(-wt[hh].x, -wt[hh].y));
              const float2 d2 = __fmul2_rn(t, iv[hh]);
              const __half2 hv = __floats2half2_rn(d2.x, d2.y);
              packed[hh] = *reinterpret_cast<const uint32_t *>(&hv);
            }
          }
          *cp = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        }
        fence_proxy_async_smem();  // the generic-proxy writes -> the tensor cores
        __syncwarp();
        if (lane == 0) mbar_arrive(&tail->conv[stage]);
        if (++stage == F_STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, F_TMEM_COLS);
  }
}

cudaError_t launch_fused_params(const __half *W, int64_t out, int64_t in, int64_t out_pad,
                                const float *s, int n_alpha, int group, int w_bit, int zero_point,
                                const DevStatus *st, float2 *params, cudaStream_t stream) {
  if (group != 32 && group != 64 && group != 128) return cudaErrorInvalidValue;
  dim3 grid((unsigned)((out_pad + 7) / 8), (unsigned)((in + 255) / 256));
  auto kern = group == 32 ? fused_params_kernel<32> : group == 64 ? fused_params_kernel<64>
                                                                  : fused_params_kernel<128>;
  kern<<<grid, 256, 0, stream>>>(W, out, in, out_pad, s, n_alpha, (float)((1 << w_bit) - 1),
                                 zero_point ? 0 : 1, st, params);
  return cudaGetLastError();
}

cudaError_t launch_fused_search_gemm(const __half *X, int64_t T, int64_t ldx, const __half *W,
                                     int64_t out, int64_t in, int64_t out_pad, int n_alpha,
                                     const float *s, const float *inv_s, const float2 *params,
                                     int group, int w_bit, double *partials, DevStatus *st,
                                     uint32_t max_polls, int num_sms, cudaStream_t stream) {
  if (group != 32 && group != 64 && group != 128) return cudaErrorInvalidValue;
  if (in % FBK != 0 || out_pad % FBN != 0) return cudaErrorInvalidValue;
  CUtensorMap tmA, tmW;
  cudaError_t e = make_tmap_f16_box(&tmA, X, T, in, ldx, FBK, FBM2);
  if (e != cudaSuccess) return e;
  e = make_tmap_f16_box(&tmW, W, out, in, in, FBK, FBN);  // rows >= out read as zeros
  if (e != cudaSuccess) return e;
  auto kern = group == 32   ? fused_search_gemm_kernel<32>
              : group == 64 ? fused_search_gemm_kernel<64>
                            : fused_search_gemm_kernel<128>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kFusedSmemBytes);
  if (e != cudaSuccess) return e;
  const int num_m = (int)((T + FBM - 1) / FBM);
  const int num_n = (int)((int64_t)n_alpha * out_pad / FBN);
  const int num_kb = (int)(in / FBK);
  const int tiles = ((num_m + 1) / 2) * num_n;
  const int grid = tiles < num_sms ? tiles : num_sms;
  kern<<<grid, F_THREADS, kFusedSmemBytes, stream>>>(tmA, tmW, num_m, num_n, num_kb, in, out_pad, s,
                                                       inv_s, params, (float)((1 << w_bit) - 1),
                                                       partials, st, max_polls);
  return cudaGetLastError();
}

AWQ_BOUNDS_READER(bounds_status_fused)

}  // namespace awq
