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
constexpr int CT_THREADS = 512;
constexpr int CT_MAXR = 32;                       // rows per tile at most
constexpr uint32_t CT_ATOM = 128 * 128;           // bytes: 128 rows x 64 fp16
constexpr uint32_t CT_OPND = 2 * CT_ATOM;         // one operand, K = 128
constexpr int CT_RS = G + G / 32;                 // skewed row stride (floats)
// kind::f16, fp16 A/B, fp32 D, K-major, N = 128, M = 128
constexpr uint32_t IDESC_CLIP = (1u << 4) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

struct __align__(16) ClipSmem {
  uint8_t a_hi[CT_OPND];
  uint8_t a_lo[CT_OPND];
  uint8_t b_hi[CT_OPND];
  uint8_t b_lo[CT_OPND];
  float wt[CT_MAXR][CT_RS];   // s_i w_i of the tile's rows (fp32, exact products)
  float bw[CT_MAXR][CT_RS];   // r_i w_i 2^e_row
  float s[G], ar[CT_RS], r[G];  // s_i, r_i / s_i (skewed), r_i = sqrt(G_ii)
  float rmx[CT_MAXR], rmn[CT_MAXR];
  int rexp[2][CT_MAXR];  // per-row exponent; the argmin of a tile reads it during the next tile
  float epart[4][128];
  float ratio[128];  // clip ratio of each index
  uint64_t mma_bar;
  uint32_t tmem_base;
  int abort_flag;  // a wait ran out: every thread leaves the tile loop together
};
constexpr size_t kClipSmemBytes = sizeof(ClipSmem) + 1024;

// channel i of a skewed row: one extra float every 32 channels, so the four
// threads that share a candidate (32 channels apart) hit different banks
__device__ __forceinline__ int sk(int i) { return i + (i >> 5); }

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

__device__ __forceinline__ float clip_ratio_f(int c, int n_clip, float clip_min) {
  if (n_clip <= 1) return 1.0f;
  double r = 1.0 - (double)c * (1.0 - (double)clip_min) / (double)(n_clip - 1);
  return __double2float_rn(r);
}
}  // namespace

__global__ void __launch_bounds__(CT_THREADS, 1) clip_tc_kernel(
    const __half *__restrict__ W, int64_t out, int64_t in, const float *__restrict__ s,
    const float *__restrict__ Gall, float qmax, int n_clip, float clip_min, int rows_per_tile,
    uint8_t *__restrict__ clip_idx, float *__restrict__ err, DevStatus *st, uint32_t max_polls) {
  extern __shared__ uint8_t csm_raw[];
  ClipSmem &S = *reinterpret_cast<ClipSmem *>(
      (reinterpret_cast<uintptr_t>(csm_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t n_groups = in / G;
  const int R = rows_per_tile;
  const int npairs = R * n_clip;  // <= 128
  const int64_t n_tiles = (out + R - 1) / R;
  // this CTA's share of the (group, row tile) items, group-major, so a CTA
  // meets at most a few groups and builds each G~ once
  const int64_t n_items = n_groups * n_tiles;
  const int64_t item_begin = n_items * blockIdx.x / gridDim.x;
  const int64_t item_end = n_items * (blockIdx.x + 1) / gridDim.x;

  if (tid == 0) {
    mbar_init(&S.mma_bar, 1);
    S.abort_flag = 0;
    fence_mbar_init();
  }
  if (tid < n_clip) S.ratio[tid] = clip_ratio_f(tid, n_clip, clip_min);
  if (warp == 0) {
    tmem_alloc(&S.tmem_base, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = S.tmem_base;

  uint32_t phase = 0;
  bool committed = false;
  int64_t k_cur = -1;
  constexpr int kRowWarps = 12;  // warps 0..11 run the row pass; warps 12..15 the argmin
  // W rows of the next tile, loaded by the row-pass warps one tile ahead
  uint2 wpre[3] = {make_uint2(0u, 0u), make_uint2(0u, 0u), make_uint2(0u, 0u)};
  auto load_rows = [&](int64_t it) {
    const int64_t kk = it / n_tiles, oo = (it - kk * n_tiles) * R;
#pragma unroll
    for (int m = 0; m < 3; ++m) {
      const int rr = warp + kRowWarps * m;
      const int64_t o = oo + rr;
      wpre[m] = (rr < R && o < out)
                    ? __ldg(reinterpret_cast<const uint2 *>(W + o * in + kk * G + 4 * lane))
                    : make_uint2(0u, 0u);
    }
  };
  // first clip index with the smallest E of each row of a finished tile;
  // four threads per row scan every fourth ratio, then combine (ties keep
  // the lower index)
  auto argmin_rows = [&](int64_t kk, int64_t oo, int b) {
    const int t = tid - kRowWarps * 32, rr = t >> 2, part = t & 3;
    const bool row_ok = rr < R && oo + rr < out;
    float best = INFINITY;
    int bc = 1 << 30;
    if (row_ok) {
      const float unscale = ldexpf(1.0f, -2 * S.rexp[b][rr]);
      for (int c = part; c < n_clip; c += 4) {
        const int p = rr * n_clip + c;
        const float ev = ((S.epart[0][p] + S.epart[1][p]) + (S.epart[2][p] + S.epart[3][p])) * unscale;
        if (err) err[((oo + rr) * n_groups + kk) * n_clip + c] = ev;
        if (ev < best) {
          best = ev;
          bc = c;
        }
      }
    }
#pragma unroll
    for (int off = 1; off < 4; off <<= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, off);
      const int oc = __shfl_xor_sync(0xffffffffu, bc, off);
      if (ob < best || (ob == best && oc < bc)) {
        best = ob;
        bc = oc;
      }
    }
    if (row_ok && part == 0) clip_idx[(oo + rr) * n_groups + kk] = (uint8_t)bc;
  };
  if (warp < kRowWarps && item_begin < item_end) load_rows(item_begin);
  int64_t k_prev = -1, o0_prev = 0;
  int buf = 0;
  for (int64_t item = item_begin; item < item_end; ++item) {
    const int64_t k = item / n_tiles;
    const int64_t o0 = (item - k * n_tiles) * R;
    if (k != k_cur) {
      // ---- group set-up: s, r = sqrt(G_ii), r/s, then G~ = G_ij / (r_i r_j)
      // as hi + lo fp16, K-major swizzled (row j, channel i)
      k_cur = k;
      const float *Gk = Gall + k * G * G;
      if (tid < G) {
        const float sv = s ? s[k * G + tid] : 1.0f;
        const float rv = sqrtf(fmaxf(Gk[tid * G + tid], 0.0f));
        S.s[tid] = sv;
        S.r[tid] = rv;
        S.ar[sk(tid)] = rv / sv;
      }
      __syncthreads();
      const int j = tid >> 2, qq = tid & 3;  // row j, channels 32 qq .. 32 qq + 31
      const float rj = S.r[j];
      const float *grow = Gk + (int64_t)j * G + 32 * qq;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float v[8];
        const float4 g0 = __ldg(reinterpret_cast<const float4 *>(grow + 8 * c));
        const float4 g1 = __ldg(reinterpret_cast<const float4 *>(grow + 8 * c + 4));
        const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float den = rj * S.r[32 * qq + 8 * c + e];
          v[e] = den > 0.0f ? gv[e] / den : 0.0f;
        }
        const int h = qq >> 1, cc = (qq & 1) * 4 + c;
        split_store8(S.b_hi + h * CT_ATOM, S.b_lo + h * CT_ATOM, sw128_off(j, cc), v);
      }
      // (the fence before the first MMA of this group publishes these stores)
    }
    if (warp < kRowWarps) {
      // ---- rows of this tile: s w, range, exponent of the d~ scaling, r w 2^e
#pragma unroll
      for (int m = 0; m < 3; ++m) {
        const int rr = warp + kRowWarps * m;
        if (rr >= R) break;
        const uint2 wv = wpre[m];
        const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&wv.x));
        const float2 b = __half22float2(*reinterpret_cast<const __half2 *>(&wv.y));
        const float w4[4] = {a.x, a.y, b.x, b.y};
        float mx = -INFINITY, mn = INFINITY, bmax = 0.0f, wt4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = 4 * lane + e;
          wt4[e] = __fmul_rn(S.s[i], w4[e]);
          mx = fmaxf(mx, wt4[e]);
          mn = fminf(mn, wt4[e]);
          bmax = fmaxf(bmax, S.r[i] * fabsf(w4[e]));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
          mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
          bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, off));
        }
        // |d~_i| <= 2 r_i |w_i| (+ rounding): keep 2 bmax 2^e <= 2^14
        int e2 = 0;
        if (bmax > 0.0f) {
          (void)frexpf(2.0f * bmax, &e2);
          e2 = 14 - e2;
        }
        const float sc = ldexpf(1.0f, e2);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = 4 * lane + e;
          S.wt[rr][sk(i)] = wt4[e];
          S.bw[rr][sk(i)] = (S.r[i] * w4[e]) * sc;
        }
        if (lane == 0) {
          S.rmx[rr] = mx;
          S.rmn[rr] = mn;
          S.rexp[buf][rr] = e2;
        }
      }
      if (item + 1 < item_end) load_rows(item + 1);
    } else if (k_prev >= 0) {
      argmin_rows(k_prev, o0_prev, buf ^ 1);  // the previous tile, overlapping this row pass
    }
    __syncthreads();
    // ---- candidates: thread (pair p, quarter qq) writes channels 32qq..32qq+31:
    // d~_i 2^e = (q - z) (delta 2^e) (r_i / s_i) - r_i w_i 2^e
    {
      const int p = tid >> 2, qq = tid & 3;
      const int rr = p / n_clip, c = p - rr * n_clip;
      const bool valid = p < npairs && o0 + rr < out;
      const int h = qq >> 1;
      uint8_t *ahi = S.a_hi + h * CT_ATOM, *alo = S.a_lo + h * CT_ATOM;
      if (valid) {
        const GroupQ g = group_params(S.rmx[rr], S.rmn[rr], S.ratio[c], qmax);
        const float de = ldexpf(g.delta, S.rexp[buf][rr]);  // exact power-of-two scaling
        const float *wtr = S.wt[rr];
        const float *bwr = S.bw[rr];
#pragma unroll 1
        for (int c4 = 0; c4 < 4; ++c4) {
          float v[8];
          const int i0 = 32 * qq + 8 * c4;
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            const int i = sk(i0 + e);  // i0 + e and i0 + e + 1 stay in one 32-channel run
            const float2 qz = quant_qz2(make_float2(wtr[i], wtr[i + 1]), g);
            const float2 d2 = __ffma2_rn(__fmul2_rn(qz, make_float2(de, de)),
                                         make_float2(S.ar[i], S.ar[i + 1]),
                                         make_float2(-bwr[i], -bwr[i + 1]));
            v[e] = d2.x;
            v[e + 1] = d2.y;
          }
          split_store8(ahi, alo, sw128_off(p, (qq & 1) * 4 + c4), v);
        }
      } else {
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          *reinterpret_cast<uint4 *>(ahi + sw128_off(p, (qq & 1) * 4 + c4)) = z;
          *reinterpret_cast<uint4 *>(alo + sw128_off(p, (qq & 1) * 4 + c4)) = z;
        }
      }
    }
    fence_async_smem();  // generic-proxy writes -> visible to the tensor cores
    __syncthreads();
    // ---- Y = A_hi B_hi + A_lo B_hi + A_hi B_lo
    if (tid == 0) {
      tc_fence_after();
      const uint32_t a_hi = smem_u32(S.a_hi), a_lo = smem_u32(S.a_lo);
      const uint32_t b_hi = smem_u32(S.b_hi), b_lo = smem_u32(S.b_lo);
      const uint32_t as[3] = {a_hi, a_lo, a_hi}, bs[3] = {b_hi, b_hi, b_lo};
#pragma unroll
      for (int t = 0; t < 3; ++t)
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t koff = (uint32_t)(ks >> 2) * CT_ATOM + (uint32_t)(ks & 3) * 32u;
          tc_mma_f16(tmem_base, smem_desc_k_sw128(as[t] + koff), smem_desc_k_sw128(bs[t] + koff),
                     IDESC_CLIP, (t | ks) != 0 ? 1u : 0u);
        }
      tc_commit(&S.mma_bar);
    }
    committed = true;
    // ---- wait for Y, then E = d~ . y per candidate (warp: lane quarter q,
    // column quarter cq)
    int okw = 1;
    if (lane == 0) okw = mbar_wait_bounded(&S.mma_bar, phase, max_polls, nullptr);
    okw = __shfl_sync(0xffffffffu, okw, 0);
    phase ^= 1u;
    if (!okw) {
      if (lane == 0) {
        dev_fail(st, kDevTimeout, 0x900u);
        *reinterpret_cast<volatile int *>(&S.abort_flag) = 1;
      }
    } else {
      tc_fence_after();
      const int q = warp & 3, cq = warp >> 2;
      const int p = q * 32 + lane;
      const uint8_t *ahi = S.a_hi + (cq >> 1) * CT_ATOM, *alo = S.a_lo + (cq >> 1) * CT_ATOM;
      float y[32];
      tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(32 * cq), y);
      tmem_ld_wait();
      float e = 0.0f;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const int c = (cq & 1) * 4 + cc;
        const uint4 hv = *reinterpret_cast<const uint4 *>(ahi + sw128_off(p, c));
        const uint4 lv = *reinterpret_cast<const uint4 *>(alo + sw128_off(p, c));
        const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w}, lw[4] = {lv.x, lv.y, lv.z, lv.w};
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
          const float2 fh = __half22float2(*reinterpret_cast<const __half2 *>(&hw[e2]));
          const float2 fl = __half22float2(*reinterpret_cast<const __half2 *>(&lw[e2]));
          e = fmaf(fh.x + fl.x, y[8 * cc + 2 * e2], e);
          e = fmaf(fh.y + fl.y, y[8 * cc + 2 * e2 + 1], e);
        }
      }
      S.epart[cq][p] = e;
    }
    tc_fence_before();
    __syncthreads();
    if (*reinterpret_cast<volatile int *>(&S.abort_flag)) break;  // uniform across the CTA
    k_prev = k;
    o0_prev = o0;
    buf ^= 1;
  }
  if (!*reinterpret_cast<volatile int *>(&S.abort_flag) && k_prev >= 0 && warp >= kRowWarps)
    argmin_rows(k_prev, o0_prev, buf ^ 1);  // the last tile
  // after an abort the last MMAs may still be running: let them finish
  // (bounded) before the accumulator is freed
  if (tid == 0 && committed && *reinterpret_cast<volatile int *>(&S.abort_flag))
    (void)mbar_wait_bounded(&S.mma_bar, phase ^ 1u, 1u << 22, nullptr);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 128);
  }
}

cudaError_t launch_clip_eval(const __half *W, int64_t out, int64_t in, const float *s,
                             const float *Gall, int group, int w_bit, int n_clip, float clip_min,
                             uint8_t *clip_idx, float *err, DevStatus *st, uint32_t max_polls,
                             int num_sms, cudaStream_t stream) {
  if (group != G || n_clip < 1 || n_clip > 128) return cudaErrorInvalidValue;
  int R = 128 / n_clip;
  if (R > CT_MAXR) R = CT_MAXR;
  const int64_t n_items = (in / G) * ((out + R - 1) / R);
  const int64_t ctas = i64min(num_sms, n_items);  // one CTA per SM (shared memory bound)
  cudaError_t e = cudaFuncSetAttribute(clip_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kClipSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)ctas);
  clip_tc_kernel<<<grid, CT_THREADS, kClipSmemBytes, stream>>>(
      W, out, in, s, Gall, (float)((1 << w_bit) - 1), n_clip, clip_min, R, clip_idx, err, st,
      max_polls);
  return cudaGetLastError();
}

}  // namespace awq
