// Gram-form alpha search: the same MSE as the scored GEMM with ~8x fewer
// flops at the calibration sizes AWQ uses.
//
// "05 — AWQ: Activation-Aware Weight Scaling" §4 scores every alpha by the
// MSE of the candidate output against X W^T; by the scaling invariance of §3
// that error is X dW^T, and
//     sum_t sum_o (X dW^T)_to^2 = sum_o dW_o^T (X^T X) dW_o.
// With r_j = sqrt(G_jj), G~ = diag(r)^-1 G diag(r)^-1 (|G~_ij| <= 1) and
// d~ = dW diag(r), this is sum_o d~_o^T G~ d~_o: one tcgen05 GEMM of the
// stacked candidates d~ [n_alpha * out_pad, in] against G~ [in, in] (held as
// fp16 hi + lo parts, ~22 significant bits) whose epilogue dots each
// accumulator row with the matching tile of d~ itself.
//
//   gram_full_kernel   G = X^T X (fp32) on the tensor cores, one CTA per
//                      256 x 256 block pair (bi <= bj), mirrored store;
//   gram_norm_kernel   r and the hi/lo parts of G~;
//   gram_score_kernel  persistent warp-specialised GEMM + dot epilogue over
//                      the 128-block upper triangle of G~, one partial per
//                      (tile, warp).
#include <cuda.h>
#include <cuda_fp16.h>
#include <math.h>

#include "awq_launch.h"

namespace awq {

namespace {
constexpr int GF_T = 64;                          // tokens per stage
constexpr int GF_STAGES = 3;
constexpr uint32_t GF_BOX = 64 * GF_T * 2;        // 64 channels x 64 tokens fp16 (8 KiB)
constexpr uint32_t GF_A = 2 * GF_BOX;             // one 128-channel A half
constexpr uint32_t GF_B = 4 * GF_BOX;             // the 256-channel B panel
constexpr uint32_t GF_STAGE = 2 * GF_A + GF_B;    // 64 KiB
constexpr uint32_t GF_DRAIN = 1u << 22;
// kind::f16, fp16 A/B, fp32 D, A and B MN-major, N = 256, M = 128
constexpr uint32_t IDESC_GF =
    (1u << 4) | (1u << 15) | (1u << 16) | ((256u >> 3) << 17) | ((128u >> 4) << 24);

struct __align__(8) GramFullTail {
  uint64_t full[GF_STAGES];
  uint64_t empty[GF_STAGES];
  uint64_t done;
  uint32_t tmem_base;
  int abort_flag;
};
constexpr size_t kGramFullSmem = 1024 + GF_STAGES * GF_STAGE + sizeof(GramFullTail);

// MN-major operand with 128-byte swizzling: 64 channels (128 B) per token row,
// 8-row core groups 1024 B apart (SBO), consecutive 64-channel boxes GF_BOX
// apart (LBO).
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((GF_BOX >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}

// (bi, bj) with bi <= bj from a triangular index
__device__ __forceinline__ void tri_pair(int t, int nb, int &bi, int &bj) {
  int i = 0;
  int row_len = nb;
  while (t >= row_len) {
    t -= row_len;
    ++i;
    --row_len;
  }
  bi = i;
  bj = i + t;
}
}  // namespace

// One CTA per pair (BI <= BJ) of 256-channel blocks: A = X[:, 256 BI ...] as
// two 128-channel halves (two TMEM accumulators of 256 columns), B =
// X[:, 256 BJ ... + 256]; channels past `in` read as zero and are not stored.
__global__ void __launch_bounds__(192, 1)
    gram_full_kernel(const __grid_constant__ CUtensorMap tmX, int64_t T, int nb,
                     float *__restrict__ G, int64_t in, DevStatus *st, uint32_t max_polls) {
  extern __shared__ uint8_t gf_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(gf_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  GramFullTail *tail = reinterpret_cast<GramFullTail *>(smem + GF_STAGES * GF_STAGE);
  volatile int *abort_flag = &tail->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int bi, bj;
  tri_pair(blockIdx.x, nb, bi, bj);
  const int nsteps = (int)((T + GF_T - 1) / GF_T);

  if (threadIdx.x == 0) {
    for (int s = 0; s < GF_STAGES; ++s) {
      mbar_init(&tail->full[s], 1);
      mbar_init(&tail->empty[s], 1);
    }
    mbar_init(&tail->done, 1);
    tail->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tmX);
  if (warp == 1) {
    tmem_alloc(&tail->tmem_base, 512);
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
        if (!mbar_wait_long(&tail->empty[stage], phase ^ 1u, max_polls, abort_flag)) {
          dev_fail(st, kDevTimeout, 0xA00u + stage);
          *abort_flag = 1;
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&tail->full[stage], GF_STAGE);
        const int32_t y = step * GF_T;
        uint8_t *dst = smem + stage * GF_STAGE;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          tma_load_2d(dst + b * GF_BOX, &tmX, &tail->full[stage], bi * 256 + 64 * b, y);
          tma_load_2d(dst + 2 * GF_A + b * GF_BOX, &tmX, &tail->full[stage], bj * 256 + 64 * b, y);
        }
        issued |= 1u << stage;
        issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == GF_STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok || *abort_flag)
        for (int s = 0; s < GF_STAGES; ++s)
          if (issued & (1u << s))
            (void)mbar_wait_bounded(&tail->full[s], (issued_parity >> s) & 1u, GF_DRAIN, nullptr);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool issued_any = false, ok = true;
      for (int step = 0; step < nsteps; ++step) {
        if (!mbar_wait_bounded(&tail->full[stage], phase, max_polls, abort_flag)) {
          dev_fail(st, kDevTimeout, 0xB00u + stage);
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t base = smem_u32(smem + stage * GF_STAGE);
#pragma unroll
        for (int ks = 0; ks < GF_T / 16; ++ks) {
          const uint64_t bd = desc_mn_sw128(base + 2 * GF_A + ks * 2048);  // 16 token rows per step
#pragma unroll
          for (int h = 0; h < 2; ++h)
            tc_mma_f16(tmem_base + h * 256, desc_mn_sw128(base + h * GF_A + ks * 2048), bd, IDESC_GF,
                       (step | ks) != 0 ? 1u : 0u);
        }
        issued_any = true;
        tc_commit(&tail->empty[stage]);
        if (++stage == GF_STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (issued_any) tc_commit(&tail->done);
      if (!ok && issued_any) (void)mbar_wait_bounded(&tail->done, 0, GF_DRAIN, nullptr);
    }
  } else {
    const int q = warp & 3;
    int ok = 1;
    if (lane == 0) ok = mbar_wait_long(&tail->done, 0, max_polls, abort_flag);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) {
      if (lane == 0) {
        dev_fail(st, kDevTimeout, 0xC00u);
        *abort_flag = 1;
      }
    } else {
      tc_fence_after();
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        const int64_t gi = (int64_t)bi * 256 + h * 128 + q * 32 + lane;  // this thread's channel
#pragma unroll 1
        for (int c = 0; c < 256; c += 32) {
          float v[32];
          tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(h * 256 + c), v);
          tmem_ld_wait();
          const int64_t gj0 = (int64_t)bj * 256 + c;
          if (gi < in && gj0 < in) {  // in % 128 == 0: a 32-column run is all in or all out
            float *row = G + gi * in + gj0;
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4 *>(row + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
            if (bi != bj && AWQ_IN_BOUNDS(gj0 + 32 <= in, 0xB051u)) {  // mirrored block: column gi of rows gj0 + e
#pragma unroll
              for (int e = 0; e < 32; ++e) G[(gj0 + e) * in + gi] = v[e];
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// r_j = sqrt(G_jj); G~_ij = G_ij / (r_i r_j) (0 where r_i r_j = 0) as fp16
// hi + lo parts, row-major [in][in] (row j, channel i: the K-major B operand).
// Because G~ is symmetric, the scores only read the 128-block upper triangle:
// d^T G~ d = sum_J d_J^T G~_JJ d_J + 2 sum_{J<I} d_J^T G~_JI d_I, so blocks
// right of the diagonal are stored doubled (exact) and blocks left of it are
// never read (stored as zero).
__global__ void gram_norm_kernel(const float *__restrict__ G, int64_t in, float *__restrict__ r,
                                 __half *__restrict__ ghi, __half *__restrict__ glo) {
  const int64_t n = in * in;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < n;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t j = idx / in, i = idx - j * in;
    const float rj = sqrtf(fmaxf(__ldg(G + j * in + j), 0.0f));
    const float ri = sqrtf(fmaxf(__ldg(G + i * in + i), 0.0f));
    const float den = ri * rj;
    const int64_t bi = i >> 7, bj = j >> 7;
    float v = den > 0.0f ? __ldg(G + idx) / den : 0.0f;
    v = bi > bj ? 2.0f * v : (bi < bj ? 0.0f : v);
    const __half h = __float2half_rn(v);
    ghi[idx] = h;
    glo[idx] = __float2half_rn(v - __half2float(h));
    if (i == 0) r[j] = rj;
  }
}

cudaError_t launch_gram_full(const __half *X, int64_t T, int64_t in, int64_t ldx, float *G, float *r,
                             __half *ghi, __half *glo, DevStatus *st, uint32_t max_polls,
                             cudaStream_t stream) {
  const int nb = (int)((in + 255) / 256);
  CUtensorMap tm;
  cudaError_t e = make_tmap_f16_box(&tm, X, T, in, ldx, 64, GF_T);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(gram_full_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kGramFullSmem);
  if (e != cudaSuccess) return e;
  const int pairs = nb * (nb + 1) / 2;
  gram_full_kernel<<<pairs, 192, kGramFullSmem, stream>>>(tm, T, nb, G, in, st, max_polls);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t n = in * in;
  gram_norm_kernel<<<(unsigned)i64min(8192, (n + 255) / 256), 256, 0, stream>>>(G, in, r, ghi, glo);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// gram_score_kernel: sum over tiles of d~ (G~_hi + G~_lo) . d~
// ---------------------------------------------------------------------------
namespace {
constexpr int SM_ = 128, SN = 128, SK = 64;
constexpr int SSTAGES = 3;
constexpr uint32_t SA = SM_ * SK * 2;            // 16 KiB
constexpr uint32_t SB = SN * SK * 2;             // 16 KiB (each of hi, lo)
constexpr uint32_t SSTAGE = SA + 2 * SB;         // 48 KiB
constexpr uint32_t SC_ATOM = SM_ * 128;          // 128 rows x 64 columns fp16
constexpr uint32_t SC = 2 * SC_ATOM;             // C tile: 128 rows x 128 columns
constexpr uint32_t IDESC_S = idesc_f16_f32(SM_, SN);
constexpr uint32_t S_DRAIN = 1u << 22;

struct __align__(8) ScoreTail {
  uint64_t full[SSTAGES];
  uint64_t empty[SSTAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t cfull[2];
  uint64_t cempty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
};
constexpr size_t kScoreSmem = 1024 + SSTAGES * SSTAGE + 2 * SC + sizeof(ScoreTail);

__device__ __forceinline__ uint32_t c_off(int row, int col) {  // byte offset in a C tile
  const int atom = col >> 6, cc = (col & 63) >> 3;
  return (uint32_t)atom * SC_ATOM + (uint32_t)row * 128u + (uint32_t)((cc ^ (row & 7)) << 4);
}
}  // namespace

__global__ void __launch_bounds__(192, 1)
    gram_score_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmH,
                      const __grid_constant__ CUtensorMap tmL, int num_m, int num_n, int num_kb,
                      double *__restrict__ partials, DevStatus *st, uint32_t max_polls) {
  extern __shared__ uint8_t gs_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(gs_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sst = smem;                          // stages
  uint8_t *sc = smem + SSTAGES * SSTAGE;        // two C tiles
  ScoreTail *tail = reinterpret_cast<ScoreTail *>(sc + 2 * SC);
  volatile int *abort_flag = &tail->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_tiles = num_m * num_n;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SSTAGES; ++s) {
      mbar_init(&tail->full[s], 1);
      mbar_init(&tail->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tail->tfull[a], 1);
      mbar_init(&tail->tempty[a], 4);
      mbar_init(&tail->cfull[a], 1);
      mbar_init(&tail->cempty[a], 4);
    }
    mbar_init(&tail->mma_done, 1);
    tail->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmH);
    tma_prefetch_desc(&tmL);
  }
  if (warp == 1) {
    tmem_alloc(&tail->tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tail->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0, it = 0;
      uint32_t phase = 0, issued = 0, issued_parity = 0, c_issued = 0, c_parity = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++it) {
        const int m_blk = tile / num_n, n_blk = tile - m_blk * num_n;
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        // C tile: d~[m rows][n columns], read by the epilogue
        if (!mbar_wait_long(&tail->cempty[acc], acc_phase ^ 1u, max_polls, abort_flag)) {
          dev_fail(st, kDevTimeout, 0xD10u + acc);
          *abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(&tail->cfull[acc], SC);
        tma_load_2d(sc + acc * SC, &tmA, &tail->cfull[acc], n_blk * SN, m_blk * SM_);
        tma_load_2d(sc + acc * SC + SC_ATOM, &tmA, &tail->cfull[acc], n_blk * SN + 64, m_blk * SM_);
        c_issued |= 1u << acc;
        c_parity = (c_parity & ~(1u << acc)) | (acc_phase << acc);
        for (int kb = n_blk * (SN / SK); kb < num_kb; ++kb) {  // upper triangle of G~ only
          if (!mbar_wait_long(&tail->empty[stage], phase ^ 1u, max_polls, abort_flag)) {
            dev_fail(st, kDevTimeout, 0xD00u + stage);
            *abort_flag = 1;
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&tail->full[stage], SSTAGE);
          uint8_t *dst = sst + stage * SSTAGE;
          tma_load_2d(dst, &tmA, &tail->full[stage], kb * SK, m_blk * SM_);
          tma_load_2d(dst + SA, &tmH, &tail->full[stage], kb * SK, n_blk * SN);
          tma_load_2d(dst + SA + SB, &tmL, &tail->full[stage], kb * SK, n_blk * SN);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == SSTAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort_flag) {
        for (int s = 0; s < SSTAGES; ++s)
          if (issued & (1u << s))
            (void)mbar_wait_bounded(&tail->full[s], (issued_parity >> s) & 1u, S_DRAIN, nullptr);
        for (int a = 0; a < 2; ++a)
          if (c_issued & (1u << a))
            (void)mbar_wait_bounded(&tail->cfull[a], (c_parity >> a) & 1u, S_DRAIN, nullptr);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0, it = 0;
      uint32_t phase = 0;
      bool ok = true, issued_any = false;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        const int kb0 = (tile % num_n) * (SN / SK);
        if (!mbar_wait_bounded(&tail->tempty[acc], acc_phase ^ 1u, max_polls, abort_flag)) {
          dev_fail(st, kDevTimeout, 0xE00u + acc);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * SN;
        for (int kb = kb0; kb < num_kb; ++kb) {
          if (!mbar_wait_bounded(&tail->full[stage], phase, max_polls, abort_flag)) {
            dev_fail(st, kDevTimeout, 0xE10u + stage);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a = smem_u32(sst + stage * SSTAGE);
#pragma unroll
          for (int k = 0; k < SK / 16; ++k) {
            const uint64_t ad = smem_desc_k_sw128(a + k * 32);
            tc_mma_f16(d_tmem, ad, smem_desc_k_sw128(a + SA + k * 32), IDESC_S,
                       (kb != kb0 || k != 0) ? 1u : 0u);
            tc_mma_f16(d_tmem, ad, smem_desc_k_sw128(a + SA + SB + k * 32), IDESC_S, 1u);
          }
          issued_any = true;
          tc_commit(&tail->empty[stage]);
          if (++stage == SSTAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&tail->tfull[acc]);
      }
      if (issued_any) {
        tc_commit(&tail->mma_done);
        (void)mbar_wait_bounded(&tail->mma_done, 0, S_DRAIN, nullptr);
      }
    }
  } else {
    const int q = warp & 3;
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      int ok = 1;
      if (lane == 0)
        ok = mbar_wait_long(&tail->tfull[acc], acc_phase, max_polls, abort_flag) &&
             mbar_wait_bounded(&tail->cfull[acc], acc_phase, max_polls, abort_flag);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        if (lane == 0) {
          dev_fail(st, kDevTimeout, 0xF00u + acc);
          *abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      const int row = q * 32 + lane;
      const uint8_t *ct = sc + acc * SC;
      float sum = 0.0f;
#pragma unroll 1
      for (int c = 0; c < SN; c += 32) {
        float y[32];
        tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * SN + c), y);
        tmem_ld_wait();
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const uint4 hv = *reinterpret_cast<const uint4 *>(ct + c_off(row, c + 8 * cc));
          const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&hw[e]));
            sum = fmaf(f.x, y[8 * cc + 2 * e], sum);
            sum = fmaf(f.y, y[8 * cc + 2 * e + 1], sum);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&tail->tempty[acc]);
        mbar_arrive(&tail->cempty[acc]);
      }
      double ds = (double)sum;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ds += __shfl_xor_sync(0xffffffffu, ds, off);
      if (lane == 0 && AWQ_IN_BOUNDS(tile < num_tiles, 0xB050u))
        partials[(size_t)tile * 4 + q] = ds;  // tile = m_blk * num_n + n_blk
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 256);
  }
}

cudaError_t launch_gram_score(const __half *dW, int64_t rows, int64_t in, const __half *ghi,
                              const __half *glo, double *partials, DevStatus *st, uint32_t max_polls,
                              int num_sms, cudaStream_t stream) {
  CUtensorMap tA, tH, tL;
  cudaError_t e = make_tmap_f16_box(&tA, dW, rows, in, in, SK, SM_);
  if (e != cudaSuccess) return e;
  e = make_tmap_f16_box(&tH, ghi, in, in, in, SK, SN);
  if (e != cudaSuccess) return e;
  e = make_tmap_f16_box(&tL, glo, in, in, in, SK, SN);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(gram_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kScoreSmem);
  if (e != cudaSuccess) return e;
  const int num_m = (int)(rows / SM_), num_n = (int)(in / SN), num_kb = (int)(in / SK);
  const int tiles = num_m * num_n;
  const int grid = tiles < num_sms ? tiles : num_sms;
  gram_score_kernel<<<grid, 192, kScoreSmem, stream>>>(tA, tH, tL, num_m, num_n, num_kb, partials,
                                                      st, max_polls);
  return cudaGetLastError();
}

AWQ_BOUNDS_READER(bounds_status_gram)

}  // namespace awq
