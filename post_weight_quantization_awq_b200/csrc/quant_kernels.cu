// HBM-bound kernels of the AWQ scale search: the activation statistic (K1),
// the candidate scale grid (K2), max |W|, the candidate quantiser that writes
// the tensor-core B operand (K3), final quantisation + packing (K7) and the
// 1/s fold (K8).
#include <cuda_fp16.h>
#include <math.h>

#include "awq_launch.h"

namespace awq {

// ---------------------------------------------------------------------------
// K1 — abar_j = (sum_t |X_tj|) / T, exact  ("AWQ and Activation-Aware
// Scaling", Scaling instead of protecting: abar is the per-channel mean
// activation magnitude; "05 — AWQ" §4 step 1).
//
// A block sweeps whole token rows (contiguous bytes, good DRAM locality):
// thread i owns channels 8i..8i+7 of the block's column range and keeps
// kStatsDepth rows of 16-byte loads in flight in a register ring.  The grid
// is one wave: column tiles x row splits = SMs x resident blocks.
//
// Exact sums without a conversion unit: for an fp16 magnitude h = (e << 10) | m,
// the fp64 whose high word is h << 10 (low word 0) is 2^(e-1023)(1 + m/1024)
// for e >= 1 and the subnormal m 2^-1032 for e = 0, i.e. |x| 2^-1008 exactly.
// These are multiples of 2^-1032 below 2^-992, so fp64 sums of up to 4096 of
// them (< 2^-980) are exact; every 4096 rows the sum is scaled by 2^1008 2^24
// (exact) into int64 units of 2^-24 held in registers, and the block's units
// go to the result with one 64-bit integer atomic per channel (exact in any
// order).
// ---------------------------------------------------------------------------
constexpr int kStatsDepth = 4;        // rows of loads in flight per thread
constexpr int kStatsExactRows = 4096;  // rows per exact fp64 partial (multiple of kStatsDepth)

__device__ __forceinline__ double mag_scaled(uint32_t hi_word) {
  return __hiloint2double((int)hi_word, 0);
}

__global__ void __launch_bounds__(1024) act_stats_kernel(const __half *__restrict__ X, int64_t T,
                                                         int64_t in, int64_t ldx,
                                                         int64_t rows_per_block,
                                                         unsigned long long *__restrict__ acc) {
  const int64_t c0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 8;
  const int64_t t0 = (int64_t)blockIdx.y * rows_per_block;
  const int64_t t1 = min(T, t0 + rows_per_block);
  if (c0 >= in || t0 >= t1) return;  // no block-wide synchronisation below
  const __half *p = X + c0;
  double sb[8];
  unsigned long long units[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    sb[e] = 0.0;
    units[e] = 0ull;
  }
  uint4 v[kStatsDepth];
#pragma unroll
  for (int u = 0; u < kStatsDepth; ++u)
    v[u] = t0 + u < t1 && AWQ_IN_BOUNDS(c0 + 8 <= in && t0 + u < T, 0xB001u)
               ? __ldcs(reinterpret_cast<const uint4 *>(p + (t0 + u) * ldx))
                       : make_uint4(0u, 0u, 0u, 0u);
  int since = 0;
  // the next row to load, and the rows left from the current one (< 2^22)
  const __half *pn = p + (t0 + kStatsDepth) * ldx;
  int left = (int)(t1 - t0);
  for (int64_t t = t0; t < t1; t += kStatsDepth, left -= kStatsDepth) {
#pragma unroll
    for (int u = 0; u < kStatsDepth; ++u) {
      // rows past t1 were loaded as zeros and add nothing
      const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        sb[2 * h] += mag_scaled((w[h] << 10) & 0x01FFFC00u);
        sb[2 * h + 1] += mag_scaled((w[h] >> 6) & 0x01FFFC00u);
      }
      v[u] = u + kStatsDepth < left && AWQ_IN_BOUNDS(t + u + kStatsDepth < T, 0xB002u)
                 ? __ldcs(reinterpret_cast<const uint4 *>(pn))
                 : make_uint4(0u, 0u, 0u, 0u);
      pn += ldx;
    }
    since += kStatsDepth;
    if (since == kStatsExactRows) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        units[e] += __double2ull_rn(__dmul_rn(__dmul_rn(sb[e], 0x1p1008), 0x1p24));
        sb[e] = 0.0;
      }
      since = 0;
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    units[e] += __double2ull_rn(__dmul_rn(__dmul_rn(sb[e], 0x1p1008), 0x1p24));
    if (units[e] && AWQ_IN_BOUNDS(c0 + e < in, 0xB003u)) atomicAdd(&acc[c0 + e], units[e]);
  }
}

// abar_j = RN64(RN64(units_j 2^-24) / T); `units` may alias `abar` (each
// thread reads its element before writing it).
__global__ void act_stats_finish_kernel(const long long *units, double *abar, int64_t in, int64_t T) {
  int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j < in) {
    const long long u = units[j];
    double S = __ll2double_rn(u) * 5.9604644775390625e-08;  // * 2^-24, exact
    abar[j] = __ddiv_rn(S, (double)T);
  }
}

cudaError_t launch_act_sums(const __half *X, int64_t T, int64_t in, int64_t ldx, int64_t *sums,
                            int num_sms, cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(sums, 0, sizeof(int64_t) * in, stream);
  if (e != cudaSuccess) return e;
  // column tiles of at most 1024 threads x 8 channels, split evenly
  const int64_t vec = in / 8;
  const int64_t ntiles = (vec + 1023) / 1024;
  const int64_t nthr = ((vec + ntiles - 1) / ntiles + 31) / 32 * 32;
  const int64_t per_sm = i64max(1, 2048 / nthr);  // resident blocks per SM (64 registers)
  int64_t splits = i64max(1, i64min(T, (int64_t)(num_sms > 0 ? num_sms : 148) * per_sm / ntiles));
  const int64_t rows = (T + splits - 1) / splits;
  splits = (T + rows - 1) / rows;
  dim3 grid((unsigned)ntiles, (unsigned)splits);
  act_stats_kernel<<<grid, (unsigned)nthr, 0, stream>>>(X, T, in, ldx, rows,
                                                        reinterpret_cast<unsigned long long *>(sums));
  return cudaGetLastError();
}

cudaError_t launch_act_finish(const int64_t *sums, int64_t in, int64_t T, double *abar,
                              cudaStream_t stream) {
  act_stats_finish_kernel<<<(unsigned)((in + 255) / 256), 256, 0, stream>>>(
      reinterpret_cast<const long long *>(sums), abar, in, T);
  return cudaGetLastError();
}

cudaError_t launch_act_stats(const __half *X, int64_t T, int64_t in, int64_t ldx, double *abar,
                             int num_sms, cudaStream_t stream) {
  // abar's storage holds the int64 sums until the finish kernel converts them
  cudaError_t e = launch_act_sums(X, T, in, ldx, reinterpret_cast<int64_t *>(abar), num_sms, stream);
  if (e != cudaSuccess) return e;
  return launch_act_finish(reinterpret_cast<const int64_t *>(abar), in, T, abar, stream);
}

// ---------------------------------------------------------------------------
// K2 — s_ij = RN32(pow(max(abar_j, 1e-4), alpha_i)), alpha_i = i/(n-1)
// ("AWQ and Activation-Aware Scaling": s = abar^alpha; "05 — AWQ" §4: ~20
// values of alpha in [0, 1]).  pow is CUDA's double pow.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float scale_value(double abar_j, int i, int n_alpha) {
  const double alpha = n_alpha > 1 ? __ddiv_rn((double)i, (double)(n_alpha - 1)) : 0.0;
  return __double2float_rn(pow(fmax(abar_j, 1e-4), alpha));
}

__global__ void scale_grid_kernel(const double *__restrict__ abar, int64_t in, int n_alpha,
                                  float *__restrict__ s, float *__restrict__ inv_s) {
  int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= in * n_alpha) return;
  int i = (int)(idx / in);
  int64_t j = idx - (int64_t)i * in;
  const float v = scale_value(abar[j], i, n_alpha);
  s[idx] = v;
  if (inv_s) inv_s[idx] = __frcp_rn(v);
}

// The selection step of a token-sharded search: MSE_i = sse_i / (T out) from
// the summed squared errors of all shards, best = the first index of the
// smallest, s_best = the grid's s of that alpha.  Every block finds best on
// its own (n_alpha <= 64 values); block 0 writes mse and best_idx.
__global__ void select_scale_kernel(const double *__restrict__ sse, int n_alpha, int64_t T,
                                    int64_t out, const double *__restrict__ abar, int64_t in,
                                    DevStatus *st, double *__restrict__ mse,
                                    int32_t *__restrict__ best_idx, float *__restrict__ s_best) {
  __shared__ int best_sh;
  if (threadIdx.x == 0) {
    const double norm = (double)T * (double)out;
    int best = 0;
    double bv = sse[0] / norm;
    bool finite = isfinite(bv);
    if (blockIdx.x == 0) mse[0] = bv;
    for (int a = 1; a < n_alpha; ++a) {
      const double v = sse[a] / norm;
      if (blockIdx.x == 0) mse[a] = v;
      if (!isfinite(v)) finite = false;
      if (v < bv) {
        bv = v;
        best = a;
      }
    }
    if (blockIdx.x == 0) {
      *best_idx = best;
      if (!finite) dev_fail(st, kDevNonFinite, 0x510u);
    }
    best_sh = best;
  }
  __syncthreads();
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j < in) s_best[j] = scale_value(abar[j], best_sh, n_alpha);
}

cudaError_t launch_select_scale(const double *sse, int n_alpha, int64_t T, int64_t out,
                                const double *abar, int64_t in, DevStatus *st, double *mse,
                                int32_t *best_idx, float *s_best, cudaStream_t stream) {
  select_scale_kernel<<<(unsigned)((in + 255) / 256), 256, 0, stream>>>(
      sse, n_alpha, T, out, abar, in, st, mse, best_idx, s_best);
  return cudaGetLastError();
}

cudaError_t launch_scale_grid(const double *abar, int64_t in, int n_alpha, float *s, float *inv_s,
                              cudaStream_t stream) {
  int64_t n = in * n_alpha;
  scale_grid_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(abar, in, n_alpha, s, inv_s);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// max |W| (bit pattern of a non-negative float orders like an unsigned int).
// ---------------------------------------------------------------------------
// max |W| (r == NULL) or max_oj r_j |W_oj| (bit pattern of a non-negative
// float orders like an unsigned int).
__global__ void wmax_kernel(const __half *__restrict__ W, int64_t n, int64_t in,
                            const float *__restrict__ r, DevStatus *st) {
  uint32_t m = 0;
  const int64_t n8 = n / 8;  // in % 8 == 0: the 8 values of a vector share a row
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8;
       i += (int64_t)gridDim.x * blockDim.x) {
    uint4 v = __ldg(reinterpret_cast<const uint4 *>(W) + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    const int64_t j0 = (i * 8) % in;
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[h]));
      float a = fabsf(f.x), b = fabsf(f.y);
      if (r) {
        a *= __ldg(r + j0 + 2 * h);
        b *= __ldg(r + j0 + 2 * h + 1);
      }
      m = max(m, __float_as_uint(a));
      m = max(m, __float_as_uint(b));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
  if ((threadIdx.x & 31) == 0 && m) atomicMax(&st->wmax_bits, m);
}

cudaError_t launch_wmax(const __half *W, int64_t n, int64_t in, const float *r, DevStatus *st,
                        int num_sms, cudaStream_t stream) {
  int64_t blocks = i64min((int64_t)num_sms * 4, (n / 8 + 255) / 256 + 1);
  wmax_kernel<<<(unsigned)blocks, 256, 0, stream>>>(W, n, in, r, st);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// K3 — candidate quantiser ("05 — AWQ" §4: for each alpha apply the scaling
// and quantize).  For candidate i, row o and group k it computes wt = s*w, the
// group min/max by warp shuffles over the g/8 lanes that hold the group, the
// step and zero point, the codes, deq = (q - z) delta, and writes the
// effective error (deq/s - w) * 2^k as fp16: row (i * out_pad + o) of the
// tensor-core B operand [n_alpha * out_pad, in].  Rows out..out_pad-1 of each
// candidate are zero.
// A block covers one candidate, 64 rows and a slab of 256 channels: lane l
// owns channels 8l..8l+7 of the slab (16-byte loads and stores) and keeps
// their s and 1/s in registers; each warp holds 8 rows in registers, reduces
// their 8 group ranges together (a transposing butterfly: every lane ends
// with whole ranges of its own rows), computes each group's step and zero
// point on one lane instead of all of its lanes, and quantises the rows with
// the parameters taken by shuffle.
// ---------------------------------------------------------------------------
constexpr int kCandRows = 64;
constexpr int kCandWarpRows = 8;  // rows per warp: 8 warps x 8 rows
constexpr int kCandBatch = 4;     // rows a warp holds in registers at a time

// Transposing butterfly for the group ranges of N rows over the 2 * OFF lanes
// of a group: each round exchanges half of the rows a lane carries with its
// partner (xor OFF) and keeps the max / min of the other half, so the rows
// carried halve while the lanes reduced over double; once one row is left the
// rounds are plain butterflies.  Lane l ends with rows held_by_lane / held_at.
template <int N, int OFF>
__device__ __forceinline__ void transpose_reduce(float (&mx)[kCandBatch], float (&mn)[kCandBatch],
                                                 int lane) {
  if constexpr (OFF >= 1) {
    if constexpr (N > 1) {
      const bool up = (lane & OFF) != 0;
#pragma unroll
      for (int i = 0; i < N / 2; ++i) {
        const float sx = up ? mx[i] : mx[i + N / 2], sn = up ? mn[i] : mn[i + N / 2];
        const float kx = up ? mx[i + N / 2] : mx[i], kn = up ? mn[i + N / 2] : mn[i];
        mx[i] = fmaxf(kx, __shfl_xor_sync(0xffffffffu, sx, OFF));
        mn[i] = fminf(kn, __shfl_xor_sync(0xffffffffu, sn, OFF));
      }
      transpose_reduce<N / 2, OFF / 2>(mx, mn, lane);
    } else {
      mx[0] = fmaxf(mx[0], __shfl_xor_sync(0xffffffffu, mx[0], OFF));
      mn[0] = fminf(mn[0], __shfl_xor_sync(0xffffffffu, mn[0], OFF));
      transpose_reduce<1, OFF / 2>(mx, mn, lane);
    }
  }
}

// After transpose_reduce<N, L/2> over groups of L lanes: the lane (within the
// group) and the element that hold row r.  Round k (OFF = L/2, L/4, ...)
// keeps the upper half of the N_k rows on lanes with bit OFF set.
template <int L, int N>
__device__ __forceinline__ constexpr int held_by_lane(int r) {
  int lane = 0, n = N, base = 0;
  for (int off = L / 2; off >= 1 && n > 1; off /= 2) {
    if (r - base >= n / 2) {
      lane |= off;
      base += n / 2;
    }
    n /= 2;
  }
  return lane;
}

template <int L, int N>
__device__ __forceinline__ constexpr int held_at(int r) {
  int n = N, base = 0;
  for (int off = L / 2; off >= 1 && n > 1; off /= 2) {
    if (r - base >= n / 2) base += n / 2;
    n /= 2;
  }
  return r - base;
}

// kCodes: instead of the B operand, the same candidates' codes q [n_alpha,
// out, in], zero points z and steps delta [n_alpha, out, in/group] (delta of
// s, i.e. the s 2^k step times 2^-k, exact) -- the inspection form of the
// kernel, with every quantisation step shared with the operand form.
template <int group, bool kCodes>  // group 32, 64 or 128: the range shuffles unroll
__global__ void __launch_bounds__(256, 3) cand_quant_kernel(
    const __half *__restrict__ W, int64_t out, int64_t in, int64_t out_pad,
    const float *__restrict__ s, const float *__restrict__ inv_s, const float *__restrict__ rch,
    float qmax, int sym, int weights_only, const DevStatus *__restrict__ st,
    __half *__restrict__ dW, uint8_t *__restrict__ cq, uint8_t *__restrict__ cz,
    float *__restrict__ cdelta) {
  // Everything runs on s 2^k: codes and zero points are those of s (power-of-
  // two invariance), delta comes out times 2^k, and the candidate error
  // (deq - s w) 2^k (r / s) needs one FFMA2 and one FMUL2 per pair.  It drops
  // the rounding residual (RN32(s w)/s - w) 2^k, below 2^-22 of the error
  // it is added to, far under the fp16 rounding that follows.
  const int k = weights_only ? 0 : kscale_from_wmax(__uint_as_float(__ldg(&st->wmax_bits)));
  const float two_k = ldexpf(1.0f, k);
  const float guard = __fmul_rn(1e-5f, two_k);  // exact
  constexpr int lanes = group / 8;  // lanes per group (a power of two <= 16)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t j0 = (int64_t)blockIdx.y * 256 + lane * 8;
  const bool j_ok = j0 < in;
  const int rb_per_alpha = (int)(out_pad / kCandRows);
  const int a = (int)(blockIdx.x / rb_per_alpha);
  // the candidate of this block lies in the grid's n_alpha x (out_pad / 64) blocks
  const bool a_ok = (int64_t)(a + 1) * rb_per_alpha <= (int64_t)gridDim.x;
  (void)a_ok;
  const int64_t o0 = (int64_t)(blockIdx.x - (int64_t)a * rb_per_alpha) * kCandRows;
  float2 sk[4], iv[4];  // s 2^k and r / s of this lane's 8 channels
  if (j_ok) {
    const float4 *sp = reinterpret_cast<const float4 *>(s + (int64_t)a * in + j0);
    const float4 *ip = reinterpret_cast<const float4 *>(inv_s + (int64_t)a * in + j0);
    const float4 s0 = __ldg(sp), s1 = __ldg(sp + 1), i0 = __ldg(ip), i1 = __ldg(ip + 1);
    const float2 tk = make_float2(two_k, two_k);
    sk[0] = __fmul2_rn(make_float2(s0.x, s0.y), tk);
    sk[1] = __fmul2_rn(make_float2(s0.z, s0.w), tk);
    sk[2] = __fmul2_rn(make_float2(s1.x, s1.y), tk);
    sk[3] = __fmul2_rn(make_float2(s1.z, s1.w), tk);
    iv[0] = make_float2(i0.x, i0.y);
    iv[1] = make_float2(i0.z, i0.w);
    iv[2] = make_float2(i1.x, i1.y);
    iv[3] = make_float2(i1.z, i1.w);
    if (rch) {  // Gram form: d~ = r_j (deq/s - w)
      const float4 r0 = __ldg(reinterpret_cast<const float4 *>(rch + j0));
      const float4 r1 = __ldg(reinterpret_cast<const float4 *>(rch + j0) + 1);
      iv[0] = __fmul2_rn(iv[0], make_float2(r0.x, r0.y));
      iv[1] = __fmul2_rn(iv[1], make_float2(r0.z, r0.w));
      iv[2] = __fmul2_rn(iv[2], make_float2(r1.x, r1.y));
      iv[3] = __fmul2_rn(iv[3], make_float2(r1.z, r1.w));
    }
  } else {
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      sk[h] = make_float2(two_k, two_k);
      iv[h] = make_float2(1.0f, 1.0f);
    }
  }
  // ---- the warp's 8 rows (o0 + 8 warp .. + 7) in batches of kCandBatch rows
  // held in registers: pass 1 takes this lane's share of each row's group range
#pragma unroll 1
  for (int bt = 0; bt < kCandWarpRows / kCandBatch; ++bt) {
  uint4 wv[kCandBatch];
  float mx[kCandBatch], mn[kCandBatch];
  const int64_t orow = o0 + (int64_t)warp * kCandWarpRows + bt * kCandBatch;
  // row pointers of the batch: one 64-bit base, rows a 32-bit offset apart
  // (in <= 2^20 channels, kCandBatch rows)
  const int in32 = (int)in;
  const __half *wrow = W + orow * in + j0;
  __half *drow = dW ? dW + ((int64_t)a * out_pad + orow) * in + j0 : nullptr;
#pragma unroll
  for (int r = 0; r < kCandBatch; ++r) {
    const bool live = j_ok && orow + r < out;
    wv[r] = live ? __ldg(reinterpret_cast<const uint4 *>(wrow + r * in32)) : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int r = 0; r < kCandBatch; ++r) {
    const uint32_t wr[4] = {wv[r].x, wv[r].y, wv[r].z, wv[r].w};
    float m = -INFINITY, n = INFINITY;
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const float2 t = __fmul2_rn(sk[h], __half22float2(*reinterpret_cast<const __half2 *>(&wr[h])));
      m = fmax3(m, t.x, t.y);
      n = fmin3(n, t.x, t.y);
    }
    mx[r] = m;
    mn[r] = n;
  }
  // ---- whole-group ranges: a transposing butterfly over the group's lanes
  // leaves each lane kCandBatch / lanes rows (or one row shared by several
  // lanes), and each lane computes the step, zero point, fast-path bound and
  // clamp need of its rows once
  transpose_reduce<kCandBatch, lanes / 2>(mx, mn, lane);
  constexpr int kHeld = kCandBatch >= lanes ? kCandBatch / lanes : 1;
  float pd[kHeld], pr[kHeld], ph[kHeld];
  int pz[kHeld];
#pragma unroll
  for (int i = 0; i < kHeld; ++i) {
    GroupQ g = group_params(mx[i], mn[i], 1.0f, qmax, sym != 0, guard);
    fast_path_check(g, mx[i], mn[i]);
    // every code of the group lies between those of its extremes (the
    // quantiser is monotonic): the clamp is needed only if one leaves [0, qmax]
    const float qhi = __fadd_rn(round_quotient(mx[i], g), g.zero);
    const float qlo = __fadd_rn(round_quotient(mn[i], g), g.zero);
    const bool clamp = !(qlo >= 0.0f && qhi <= g.qmax);
    pd[i] = g.delta;
    pr[i] = g.rcp;
    ph[i] = g.half_lo;
    pz[i] = (int)g.zero | (clamp ? 256 : 0);
  }
  // ---- pass 2: per row, the group's parameters from the lane that holds
  // them, then codes proposed by the approximate reciprocal (one FMA rounds
  // the product to an integer), proven by the remainder test, decided by the
  // correctly rounded division otherwise; the clamp only where needed
  const float2 M = make_float2(12582912.0f, 12582912.0f);  // 1.5 2^23
#pragma unroll
  for (int r = 0; r < kCandBatch; ++r) {
    const int src = held_by_lane<lanes, kCandBatch>(r), el = held_at<lanes, kCandBatch>(r);
    const float dl = __shfl_sync(0xffffffffu, pd[el], src, lanes);
    const float rc = __shfl_sync(0xffffffffu, pr[el], src, lanes);
    const float hl = __shfl_sync(0xffffffffu, ph[el], src, lanes);
    const int zf = __shfl_sync(0xffffffffu, pz[el], src, lanes);
    const float zero = (float)(zf & 255);
    const int64_t o = orow + r;
    const uint32_t wr[4] = {wv[r].x, wv[r].y, wv[r].z, wv[r].w};
    float2 wt[4], qz[4];
    float rmax = 0.0f;
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      wt[h] = __fmul2_rn(sk[h], __half22float2(*reinterpret_cast<const __half2 *>(&wr[h])));
      qz[h] = __fadd2_rn(__ffma2_rn(wt[h], make_float2(rc, rc), M), make_float2(-M.x, -M.y));
      const float2 rem = __ffma2_rn(make_float2(-qz[h].x, -qz[h].y), make_float2(dl, dl), wt[h]);
      rmax = fmax3(rmax, fabsf(rem.x), fabsf(rem.y));
    }
    if (!(rmax < hl)) {
#pragma unroll
      for (int h = 0; h < 4; ++h)
        qz[h] = make_float2(rintf(__fdiv_rn(wt[h].x, dl)), rintf(__fdiv_rn(wt[h].y, dl)));
    }
    if (zf & 256) {
      const float lo = -zero, hi = qmax - zero;  // exact (small integers)
#pragma unroll
      for (int h = 0; h < 4; ++h)
        qz[h] = make_float2(fminf(fmaxf(qz[h].x, lo), hi), fminf(fmaxf(qz[h].y, lo), hi));
    }
    if constexpr (kCodes) {
      if (j_ok && o < out) {
        uint32_t bq[2] = {0u, 0u};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          // q = (q - z) + z, small exact integers in [0, qmax]
          bq[h >> 1] |= (uint32_t)__fadd_rn(qz[h].x, zero) << (16 * (h & 1));
          bq[h >> 1] |= (uint32_t)__fadd_rn(qz[h].y, zero) << (16 * (h & 1) + 8);
        }
        if (AWQ_IN_BOUNDS(a_ok && j0 + 8 <= in, 0xB011u))
          *reinterpret_cast<uint2 *>(cq + ((int64_t)a * out + o) * in + j0) = make_uint2(bq[0], bq[1]);
        if ((lane & (lanes - 1)) == 0 && AWQ_IN_BOUNDS(a_ok, 0xB012u)) {
          const int64_t gi = ((int64_t)a * out + o) * (in / group) + j0 / group;
          cz[gi] = (uint8_t)zero;
          cdelta[gi] = ldexpf(dl, -k);
        }
      }
      continue;
    }
    const float2 dl2 = make_float2(dl, dl);
    uint32_t packed[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      // error form: (deq - s w) 2^k (r / s); weights only: deq / s
      const float2 t = weights_only ? __fmul2_rn(qz[h], dl2)
                                    : __ffma2_rn(qz[h], dl2, make_float2(-wt[h].x, -wt[h].y));
      // rows past `out` and channels past `in` hold w = 0, which gives 0 here
      const float2 d2 = __fmul2_rn(t, iv[h]);
      const __half2 hv = __floats2half2_rn(d2.x, d2.y);
      packed[h] = *reinterpret_cast<const uint32_t *>(&hv);
    }
    if (j_ok && AWQ_IN_BOUNDS(a_ok && o < out_pad && j0 + 8 <= in, 0xB010u))
      *reinterpret_cast<uint4 *>(drow + r * in32) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  }
  }
}

cudaError_t launch_cand_quant(const __half *W, int64_t out, int64_t in, int64_t out_pad,
                              const float *s, const float *inv_s, const float *r, int n_alpha,
                              int group, int w_bit, int zero_point, int weights_only,
                              const DevStatus *st, __half *dW, int num_sms, cudaStream_t stream) {
  (void)num_sms;
  dim3 grid((unsigned)(n_alpha * (out_pad / kCandRows)), (unsigned)((in + 255) / 256));
  if (group != 32 && group != 64 && group != 128) return cudaErrorInvalidValue;
  auto kern = group == 32   ? cand_quant_kernel<32, false>
              : group == 64 ? cand_quant_kernel<64, false>
                            : cand_quant_kernel<128, false>;
  kern<<<grid, 256, 0, stream>>>(W, out, in, out_pad, s, inv_s, r, (float)((1 << w_bit) - 1),
                                 zero_point ? 0 : 1, weights_only, st, dW, nullptr, nullptr,
                                 nullptr);
  return cudaGetLastError();
}

cudaError_t launch_cand_codes(const __half *W, int64_t out, int64_t in, int64_t out_pad,
                              const float *s, const float *inv_s, int n_alpha, int group, int w_bit,
                              int zero_point, const DevStatus *st, uint8_t *q, uint8_t *z,
                              float *delta, cudaStream_t stream) {
  dim3 grid((unsigned)(n_alpha * (out_pad / kCandRows)), (unsigned)((in + 255) / 256));
  if (group != 32 && group != 64 && group != 128) return cudaErrorInvalidValue;
  auto kern = group == 32   ? cand_quant_kernel<32, true>
              : group == 64 ? cand_quant_kernel<64, true>
                            : cand_quant_kernel<128, true>;
  kern<<<grid, 256, 0, stream>>>(W, out, in, out_pad, s, inv_s, nullptr, (float)((1 << w_bit) - 1),
                                 zero_point ? 0 : 1, 0, st, nullptr, q, z, delta);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// K7 — final codes with (s, clip ratio) and the pages' storage layout
// ("05 — AWQ" §5): qweight [in, out/8] int32 with the code of output o in
// nibble o%8 of word [j][o/8]; qzeros [in/g, out/8] likewise; scales
// [in/g, out] fp16.  A block handles 64 output rows x 128 input channels:
// warp w takes rows 8w..8w+7 -- exactly the 8 nibbles of one word column --
// and lane l channels 4l..4l+3, so a lane builds the 4 packed words of its
// channels in registers, with no transpose of codes.
// ---------------------------------------------------------------------------
constexpr int kPackRows = 64;

// Status word of the calls that take no workspace (awq_quant_pack,
// awq_search_clip_noalloc): one per device, zero at load, OR-ed by kernels,
// read and cleared by the host (lib_status_read_clear).
static __device__ DevStatus g_lib_status;

cudaError_t lib_status_address(DevStatus **p) {
  void *a = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&a, g_lib_status);
  *p = static_cast<DevStatus *>(a);
  return e;
}

cudaError_t lib_status_read_clear(DevStatus *h) {
  cudaError_t e = cudaMemcpyFromSymbol(h, g_lib_status, sizeof(DevStatus));
  if (e != cudaSuccess) return e;
  const DevStatus zero = {};
  return cudaMemcpyToSymbol(g_lib_status, &zero, sizeof(DevStatus));
}

__device__ __forceinline__ float clip_ratio(int c, int n_clip, float clip_min) {
  if (n_clip <= 1) return 1.0f;
  double r = 1.0 - (double)c * (1.0 - (double)clip_min) / (double)(n_clip - 1);
  return __double2float_rn(r);
}

// Per warp: the 8 rows' group ranges by a transposing butterfly over the
// group's g/4 lanes (each lane ends with one row's range), the step, zero
// point, fast-path bound and clamp need computed once per (row, group) and
// passed through shared memory, codes proposed by the approximate reciprocal
// and proven by one remainder test per 4 values (the correctly rounded
// division otherwise), and the packed word of each channel summed exactly in
// fp32 as two 16-bit halves (codes times 16^r, integers below 2^16).
constexpr int kPackTile = 128;

template <int N, int OFF>
__device__ __forceinline__ void pack_range_reduce(float (&mx)[8], float (&mn)[8], int lane) {
  if constexpr (OFF >= 1) {
    if constexpr (N > 1) {
      const bool up = (lane & OFF) != 0;
#pragma unroll
      for (int i = 0; i < N / 2; ++i) {
        const float sx = up ? mx[i] : mx[i + N / 2], sn = up ? mn[i] : mn[i + N / 2];
        const float kx = up ? mx[i + N / 2] : mx[i], kn = up ? mn[i + N / 2] : mn[i];
        mx[i] = fmaxf(kx, __shfl_xor_sync(0xffffffffu, sx, OFF));
        mn[i] = fminf(kn, __shfl_xor_sync(0xffffffffu, sn, OFF));
      }
      pack_range_reduce<N / 2, OFF / 2>(mx, mn, lane);
    } else {
      mx[0] = fmaxf(mx[0], __shfl_xor_sync(0xffffffffu, mx[0], OFF));
      mn[0] = fminf(mn[0], __shfl_xor_sync(0xffffffffu, mn[0], OFF));
      pack_range_reduce<1, OFF / 2>(mx, mn, lane);
    }
  }
}

template <int group>  // 32, 64 or 128: divisions and the shuffle rounds become constants
__global__ void __launch_bounds__(256, 4) quant_pack_kernel(
    const __half *__restrict__ W, int64_t out, int64_t in, const float *__restrict__ s,
    const uint8_t *__restrict__ clip_idx, int n_clip, float clip_min, float qmax, int sym,
    int32_t *__restrict__ qweight, int32_t *__restrict__ qzeros, __half *__restrict__ scales) {
  constexpr int TC = kPackTile;
  constexpr int gl = group / 4;      // lanes per group
  constexpr int GPT = TC / group;    // groups per tile
  constexpr int kShare = gl / 8;     // lanes sharing one row's range after the reduction
  __shared__ __align__(16) float4 prm[8][GPT][8];      // per warp, group, row: delta, rcp, half_lo, flags
  __shared__ __align__(16) uint32_t words[TC][8 + 1];  // [channel][word column]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t j_tile = (int64_t)blockIdx.y * TC;  // first channel of the tile
  const int cols = (int)i64min(TC, in - j_tile);    // channels here: a multiple of group
  const int64_t o0 = (int64_t)blockIdx.x * kPackRows;
  const int rows_here = (int)i64min(kPackRows, out - o0);  // a multiple of 8 (out % 8 == 0)
  const int64_t groups = in / group;
  const int64_t wpr = out / 8;                      // words per qweight row
  const bool lane_ok = lane * 4 < cols;             // whole groups of lanes
  const bool warp_ok = 8 * warp < rows_here;
  const int gi = (lane * 4) / group;                // group within the tile
  const int64_t kg = j_tile / group + gi;           // global group index
  const int64_t orow = o0 + 8 * warp;
  if (warp_ok) {  // warp-uniform: every lane of the warp takes part in the shuffles
    float2 sv[2] = {make_float2(1.0f, 1.0f), make_float2(1.0f, 1.0f)};
    if (s && lane_ok) {
      const float4 f = __ldg(reinterpret_cast<const float4 *>(s + j_tile + lane * 4));
      sv[0] = make_float2(f.x, f.y);
      sv[1] = make_float2(f.z, f.w);
    }
    float2 wt[8][2];
    float mx[8], mn[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const uint2 v = lane_ok && AWQ_IN_BOUNDS(orow + r < out && j_tile + lane * 4 + 4 <= in, 0xB023u)
                          ? __ldg(reinterpret_cast<const uint2 *>(W + (orow + r) * in + j_tile + lane * 4))
                              : make_uint2(0u, 0u);
      wt[r][0] = __fmul2_rn(sv[0], __half22float2(*reinterpret_cast<const __half2 *>(&v.x)));
      wt[r][1] = __fmul2_rn(sv[1], __half22float2(*reinterpret_cast<const __half2 *>(&v.y)));
      mx[r] = fmaxf(fmax3(wt[r][0].x, wt[r][0].y, wt[r][1].x), wt[r][1].y);
      mn[r] = fminf(fmin3(wt[r][0].x, wt[r][0].y, wt[r][1].x), wt[r][1].y);
    }
    pack_range_reduce<8, gl / 2>(mx, mn, lane);
    // this lane now holds the range of row (lane within the group) / kShare
    const int rh = (lane & (gl - 1)) / kShare;
    if (lane_ok && (lane & (kShare - 1)) == 0) {
      // an index past the clip grid is the caller's error: that group gets
      // codes and zero 0 and a NaN scale, and the library status word records it
      float r32 = 1.0f;
      bool bad = false;
      if (clip_idx) {
        const int ci = AWQ_IN_BOUNDS(orow + rh < out && kg < groups, 0xB024u)
                           ? __ldg(clip_idx + (orow + rh) * groups + kg)
                           : 0;
        if (ci < n_clip)
          r32 = clip_ratio(ci, n_clip, clip_min);
        else
          bad = true;
      }
      GroupQ g = group_params(mx[0], mn[0], r32, qmax, sym != 0);
      fast_path_check(g, mx[0], mn[0]);
      // every code of the group lies between those of its extremes
      const float qhi = __fadd_rn(round_quotient(mx[0], g), g.zero);
      const float qlo = __fadd_rn(round_quotient(mn[0], g), g.zero);
      const int clamp = !(qlo >= 0.0f && qhi <= g.qmax);
      const int flags = (bad ? 0 : (int)g.zero) | (clamp << 8) | ((int)bad << 9);
      prm[warp][gi][rh] = make_float4(g.delta, g.rcp, g.half_lo, __int_as_float(flags));
      if (AWQ_IN_BOUNDS(kg < groups && orow + rh < out, 0xB020u))
        scales[kg * out + orow + rh] = bad ? __ushort_as_half((unsigned short)0x7E00u) : __float2half_rn(g.delta);
      if (bad) dev_fail(&g_lib_status, kDevBadIndex, 0x4B0u);
    }
    __syncwarp();
    if (lane_ok) {  // lanes past the last channel form whole groups
    // codes; the packed words as exact fp32 sums of code * 16^r, per 4-row half
    float lo[4], hi[4];
    float zlo = 0.0f, zhi = 0.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c) lo[c] = hi[c] = 0.0f;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const float4 pv = prm[warp][gi][r];
      const int flags = __float_as_int(pv.w);
      const float zero = (float)(flags & 255);
      const float dl = pv.x, rc = pv.y, hl = pv.z;
      const float2 M = make_float2(12582912.0f, 12582912.0f);  // 1.5 2^23
      float2 qz[2];
      float rmax = 0.0f;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        qz[h] = __fadd2_rn(__ffma2_rn(wt[r][h], make_float2(rc, rc), M), make_float2(-M.x, -M.y));
        const float2 rem = __ffma2_rn(make_float2(-qz[h].x, -qz[h].y), make_float2(dl, dl), wt[r][h]);
        rmax = fmax3(rmax, fabsf(rem.x), fabsf(rem.y));
      }
      if (!(rmax < hl)) {
#pragma unroll
        for (int h = 0; h < 2; ++h)
          qz[h] = make_float2(rintf(__fdiv_rn(wt[r][h].x, dl)), rintf(__fdiv_rn(wt[r][h].y, dl)));
      }
      if (flags & 256) {
        const float lo_q = -zero, hi_q = qmax - zero;  // exact (small integers)
#pragma unroll
        for (int h = 0; h < 2; ++h)
          qz[h] = make_float2(fminf(fmaxf(qz[h].x, lo_q), hi_q), fminf(fmaxf(qz[h].y, lo_q), hi_q));
      }
      if (flags & 512) qz[0] = qz[1] = make_float2(0.0f, 0.0f);  // code 0 (its zero is 0)
      const float pw = (float)(1 << (4 * (r & 3)));  // 16^(r mod 4)
      const float q4[4] = {qz[0].x, qz[0].y, qz[1].x, qz[1].y};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (r < 4)
          lo[c] = fmaf(q4[c], pw, lo[c]);
        else
          hi[c] = fmaf(q4[c], pw, hi[c]);
      }
      if (r < 4)
        zlo = fmaf(zero, pw, zlo);
      else
        zhi = fmaf(zero, pw, zhi);
    }
    // (q - z) + z summed per half: the codes' half-words, exact
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint32_t wl = (uint32_t)__fadd_rn(lo[c], zlo), wh = (uint32_t)__fadd_rn(hi[c], zhi);
      words[lane * 4 + c][warp] = wl | (wh << 16);
    }
    if ((lane & (gl - 1)) == 0)  // first lane of the group: the zero points' word
      if (AWQ_IN_BOUNDS(kg < groups && orow / 8 < wpr, 0xB021u))
        qzeros[kg * wpr + orow / 8] = (int32_t)((uint32_t)zlo | ((uint32_t)zhi << 16));
    }
  }
  __syncthreads();
  // qweight rows of this tile: 8 consecutive words (32 bytes) per channel
  const int w8 = rows_here / 8;
  for (int t = threadIdx.x; t < cols * 8; t += 256) {
    const int jj = t >> 3, wc = t & 7;
    if (wc < w8 && AWQ_IN_BOUNDS(j_tile + jj < in && o0 / 8 + wc < wpr, 0xB022u))
      qweight[(j_tile + jj) * wpr + o0 / 8 + wc] = (int32_t)words[jj][wc];
  }
}

cudaError_t launch_quant_pack(const __half *W, int64_t out, int64_t in, const float *s,
                              const uint8_t *clip_idx, int group, int w_bit, int zero_point,
                              int n_clip, float clip_min, int32_t *qweight, int32_t *qzeros,
                              __half *scales, cudaStream_t stream) {
  if (group != 32 && group != 64 && group != 128) return cudaErrorInvalidValue;
  dim3 grid((unsigned)((out + kPackRows - 1) / kPackRows), (unsigned)((in + kPackTile - 1) / kPackTile));
  auto kern = group == 32 ? quant_pack_kernel<32> : group == 64 ? quant_pack_kernel<64> : quant_pack_kernel<128>;
  kern<<<grid, 256, 0, stream>>>(W, out, in, s, clip_idx, n_clip, clip_min, (float)((1 << w_bit) - 1),
                                 zero_point ? 0 : 1, qweight, qzeros, scales);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// K8 — fold 1/s into the preceding operation ("AWQ and Activation-Aware
// Scaling": the activation-side division is absorbed by the preceding
// normalisation's scale or linear layer): v[j][:] = RN16(RN32(v[j][:]) / s_j).
// ---------------------------------------------------------------------------
__global__ void fold_kernel(__half *__restrict__ v, int64_t rows, int64_t cols,
                            const float *__restrict__ s) {
  const int64_t n = rows * cols;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t j = i / cols;
    v[i] = __float2half_rn(__fdiv_rn(__half2float(v[i]), s[j]));
  }
}

cudaError_t launch_fold(__half *v, int64_t rows, int64_t cols, const float *s, cudaStream_t stream) {
  const int64_t n = rows * cols;
  int64_t blocks = i64min(4096, (n + 255) / 256);
  if (blocks < 1) blocks = 1;
  fold_kernel<<<(unsigned)blocks, 256, 0, stream>>>(v, rows, cols, s);
  return cudaGetLastError();
}

AWQ_BOUNDS_READER(bounds_status_quant)

}  // namespace awq
