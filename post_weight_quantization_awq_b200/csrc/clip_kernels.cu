// K6 — per-(row, group) clip-ratio search ("05 — AWQ: Activation-Aware Weight
// Scaling" §4, optional clipping: a ratio of 0.5–1.0 of the range is
// grid-searched after alpha).
//
// For group k the output error of row o under clip c is
//   E_okc = sum_t (sum_{j in k} X_tj d_j)^2 = d^T G_k d,   G_k = X_k^T X_k,
// with d = deq_c/s - w over the group's g channels.  G_k does not depend on s
// or on the row, so it is built once per call (K6a) and every (o, k, c) is a
// 128-dimensional fp32 quadratic form (K6b).
//   K6a  gram_blocks: fp32 FFMA over token chunks, one block per (group,
//        chunk), 8x8 outputs per thread; chunk partials are summed in a fixed
//        order by gram_reduce, so G is bitwise reproducible.
//   K6b  clip_eval: one block per (group, 16 rows) holds G_k in shared memory;
//        a warp quantises one row for a batch of clip ratios, writes the error
//        vectors to shared memory and evaluates y = G_k d for the whole batch
//        (each G element read once per batch), then E = d . y by warp
//        shuffles; the first c with the smallest E wins.
#include <cuda_fp16.h>
#include <math.h>

#include "awq_launch.h"

namespace awq {

namespace {
constexpr int G = 128;          // group size handled by these kernels
constexpr int GRAM_TT = 32;     // tokens staged per step
constexpr int GRAM_PAD = 4;     // row padding of the staged tile (floats)
constexpr int CLIP_ROWS = 16;   // rows per clip_eval block
constexpr int CLIP_WARPS = 4;
constexpr int CLIP_CB = 10;     // clip ratios per batch
constexpr int GSTRIDE = G + 4;  // shared-memory row stride of G_k (floats)
}  // namespace

// Thread (ty, tx) of a 16x16 block owns rows {4ty..4ty+3, 64+4ty..64+4ty+3} and
// the same split set of columns for tx, so float4 reads of a staged token row
// are bank-conflict free.
__global__ void __launch_bounds__(256) gram_blocks_kernel(const __half *__restrict__ X, int64_t T,
                                                          int64_t ldx, int64_t chunk_tokens,
                                                          int64_t n_groups,
                                                          float *__restrict__ partials) {
  __shared__ __align__(16) float xs[GRAM_TT][G + GRAM_PAD];
  const int k = blockIdx.x;
  const int chunk = blockIdx.y;
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int64_t t0 = (int64_t)chunk * chunk_tokens;
  const int64_t t1 = min(T, t0 + chunk_tokens);
  float acc[8][8];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b) acc[a][b] = 0.0f;

  for (int64_t tb = t0; tb < t1; tb += GRAM_TT) {
    // stage GRAM_TT rows x 128 channels (fp16 -> fp32); 256 threads x 16 values
    {
      const int r = tid >> 3;          // 0..31
      const int c = (tid & 7) * 16;    // 0..112
      const int64_t t = tb + r;
      float v[16];
      if (t < t1) {
        const uint4 *p = reinterpret_cast<const uint4 *>(X + t * ldx + (int64_t)k * G + c);
        uint4 a = __ldg(p), b = __ldg(p + 1);
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[h]));
          v[2 * h] = f.x;
          v[2 * h + 1] = f.y;
        }
      } else {
#pragma unroll
        for (int h = 0; h < 16; ++h) v[h] = 0.0f;
      }
#pragma unroll
      for (int h = 0; h < 16; h += 4)
        *reinterpret_cast<float4 *>(&xs[r][c + h]) = make_float4(v[h], v[h + 1], v[h + 2], v[h + 3]);
    }
    __syncthreads();
#pragma unroll 4
    for (int t = 0; t < GRAM_TT; ++t) {
      const float4 a0 = *reinterpret_cast<const float4 *>(&xs[t][4 * ty]);
      const float4 a1 = *reinterpret_cast<const float4 *>(&xs[t][64 + 4 * ty]);
      const float4 b0 = *reinterpret_cast<const float4 *>(&xs[t][4 * tx]);
      const float4 b1 = *reinterpret_cast<const float4 *>(&xs[t][64 + 4 * tx]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(av[a], bv[b], acc[a][b]);
    }
    __syncthreads();
  }
  float *out = partials + ((int64_t)chunk * n_groups + k) * G * G;
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const int row = (a < 4) ? (4 * ty + a) : (64 + 4 * ty + a - 4);
    *reinterpret_cast<float4 *>(&out[row * G + 4 * tx]) =
        make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
    *reinterpret_cast<float4 *>(&out[row * G + 64 + 4 * tx]) =
        make_float4(acc[a][4], acc[a][5], acc[a][6], acc[a][7]);
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
                               int n_chunks, float *partials, float *Gout, cudaStream_t stream) {
  if (group != G) return cudaErrorInvalidValue;
  const int64_t n_groups = in / G;
  const int64_t chunk_tokens = (T + n_chunks - 1) / n_chunks;
  dim3 grid((unsigned)n_groups, (unsigned)n_chunks);
  gram_blocks_kernel<<<grid, 256, 0, stream>>>(X, T, ldx, chunk_tokens, n_groups, partials);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t n = n_groups * G * G;
  gram_reduce_kernel<<<(unsigned)i64min(4096, (n + 255) / 256), 256, 0, stream>>>(
      partials, n_chunks, n, Gout);
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
