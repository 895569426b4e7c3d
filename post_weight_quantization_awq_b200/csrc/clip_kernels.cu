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
//   K6b  clip_eval: one block per (group, 16 rows) holds G_k in shared memory;
//        a warp quantises one row for a batch of clip ratios, writes the error
//        vectors to shared memory and evaluates y = G_k d for the whole batch
//        (each G element read once per batch), then E = d . y by warp
//        shuffles; the first c with the smallest E wins.
#include <cuda.h>
#include <cuda_fp16.h>
#include <math.h>

#include "awq_launch.h"

namespace awq {

namespace {
constexpr int G = 128;          // group size handled by these kernels
constexpr int CLIP_ROWS = 16;   // rows per clip_eval block
constexpr int CLIP_WARPS = 4;
constexpr int CLIP_CB = 10;     // clip ratios per batch
constexpr int GSTRIDE = G + 4;  // shared-memory row stride of G_k (floats)
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
#pragma unroll 1
      for (int c = 0; c < 128; c += 32) {
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
  if (group != G) return cudaErrorInvalidValue;
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
// K6b
// ---------------------------------------------------------------------------
__device__ __forceinline__ float clip_ratio_f(int c, int n_clip, float clip_min) {
  if (n_clip <= 1) return 1.0f;
  double r = 1.0 - (double)c * (1.0 - (double)clip_min) / (double)(n_clip - 1);
  return __double2float_rn(r);
}

__global__ void __launch_bounds__(CLIP_WARPS * 32) clip_eval_kernel(
    const __half *__restrict__ W, int64_t out, int64_t in, const float *__restrict__ s,
    const float *__restrict__ Gall, float qmax, int n_clip, float clip_min,
    uint8_t *__restrict__ clip_idx, float *__restrict__ err) {
  extern __shared__ __align__(16) float csm[];
  float *Gs = csm;                                  // [G][GSTRIDE]
  float *dsh = csm + G * GSTRIDE;                   // [warps][CLIP_CB][G]
  const int k = blockIdx.x;
  const int64_t o_base = (int64_t)blockIdx.y * CLIP_ROWS;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_groups = in / G;
  const float *Gk = Gall + (int64_t)k * G * G;
  for (int i = threadIdx.x; i < G * G / 4; i += blockDim.x) {
    const int r = (4 * i) / G, c = (4 * i) % G;
    *reinterpret_cast<float4 *>(&Gs[r * GSTRIDE + c]) = __ldg(reinterpret_cast<const float4 *>(Gk) + i);
  }
  __syncthreads();
  float *dw = dsh + warp * CLIP_CB * G;
  // lane owns channels j = lane + 32 jj (jj = 0..3) of the group
  float sv[4];
#pragma unroll
  for (int jj = 0; jj < 4; ++jj) sv[jj] = s ? s[(int64_t)k * G + lane + 32 * jj] : 1.0f;

  for (int r = warp; r < CLIP_ROWS; r += CLIP_WARPS) {
    const int64_t o = o_base + r;
    if (o >= out) break;
    float w[4], wt[4];
    float mx = -INFINITY, mn = INFINITY;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      w[jj] = __half2float(W[o * in + (int64_t)k * G + lane + 32 * jj]);
      wt[jj] = __fmul_rn(sv[jj], w[jj]);
      mx = fmaxf(mx, wt[jj]);
      mn = fminf(mn, wt[jj]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
    }
    float best_e = INFINITY;
    int best_c = 0;
    for (int c0 = 0; c0 < n_clip; c0 += CLIP_CB) {
      const int nb = min(CLIP_CB, n_clip - c0);
      // error vectors of this batch -> shared memory
      for (int cc = 0; cc < nb; ++cc) {
        const GroupQ g = group_params(mx, mn, clip_ratio_f(c0 + cc, n_clip, clip_min), qmax);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const float deq = dequant(quant_code(wt[jj], g), g);
          dw[cc * G + lane + 32 * jj] = __fsub_rn(__fdiv_rn(deq, sv[jj]), w[jj]);
        }
      }
      __syncwarp();
      float y[4][CLIP_CB];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj)
#pragma unroll
        for (int cc = 0; cc < CLIP_CB; ++cc) y[jj][cc] = 0.0f;
#pragma unroll 2
      for (int i = 0; i < G; i += 4) {
        float4 gr[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
          gr[jj] = *reinterpret_cast<const float4 *>(&Gs[(lane + 32 * jj) * GSTRIDE + i]);
#pragma unroll
        for (int cc = 0; cc < CLIP_CB; ++cc) {
          if (cc < nb) {
            const float4 d = *reinterpret_cast<const float4 *>(&dw[cc * G + i]);
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              float acc = y[jj][cc];
              acc = fmaf(gr[jj].x, d.x, acc);
              acc = fmaf(gr[jj].y, d.y, acc);
              acc = fmaf(gr[jj].z, d.z, acc);
              acc = fmaf(gr[jj].w, d.w, acc);
              y[jj][cc] = acc;
            }
          }
        }
      }
#pragma unroll
      for (int cc = 0; cc < CLIP_CB; ++cc) {
        if (cc < nb) {
          float e = 0.0f;
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) e = fmaf(dw[cc * G + lane + 32 * jj], y[jj][cc], e);
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) e += __shfl_xor_sync(0xffffffffu, e, off);
          if (err && lane == 0) err[(o * n_groups + k) * n_clip + c0 + cc] = e;
          if (e < best_e) {
            best_e = e;
            best_c = c0 + cc;
          }
        }
      }
      __syncwarp();
    }
    if (lane == 0) clip_idx[o * n_groups + k] = (uint8_t)best_c;
  }
}

cudaError_t launch_clip_eval(const __half *W, int64_t out, int64_t in, const float *s,
                             const float *Gall, int group, int w_bit, int n_clip, float clip_min,
                             uint8_t *clip_idx, float *err, cudaStream_t stream) {
  if (group != G) return cudaErrorInvalidValue;
  const size_t smem = sizeof(float) * ((size_t)G * GSTRIDE + (size_t)CLIP_WARPS * CLIP_CB * G);
  cudaError_t e = cudaFuncSetAttribute(clip_eval_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)(in / G), (unsigned)((out + CLIP_ROWS - 1) / CLIP_ROWS));
  clip_eval_kernel<<<grid, CLIP_WARPS * 32, smem, stream>>>(
      W, out, in, s, Gall, (float)((1 << w_bit) - 1), n_clip, clip_min, clip_idx, err);
  return cudaGetLastError();
}

}  // namespace awq
