// K4 — the scored candidate GEMM of the AWQ alpha search, and K5, its
// deterministic reduction and argmin.
//
// "05 — AWQ: Activation-Aware Weight Scaling" §4: for each alpha apply the
// scaling, quantize, and measure the MSE against the fp16 output.  By the
// scaling invariance of §3, (X diag(s)^-1) Qdeq^T - X W^T = X dW^T with
// dW = Qdeq/s - W, so every candidate's error is one GEMM against the same X.
// All n_alpha candidates are stacked along N (B = dW [n_alpha * out_pad, in])
// and run as one persistent GEMM:  M = T tokens, N = n_alpha * out_pad,
// K = in.  The epilogue squares and sums each accumulator tile straight out
// of tensor memory, so no candidate output is ever written to HBM.
//
// sm_100a design, one CTA per SM (320 threads), 256 x 256 output tiles:
//   warp 0      TMA producer: A tile 256x64 and B tile 256x64 (fp16, 128-byte
//               swizzle) into a 3-stage shared-memory ring;
//   warp 1      allocates 512 TMEM columns; one thread issues two
//               tcgen05.mma.cta_group::1.kind::f16 (M=128, N=256, K=16) per K
//               slice, one per 128-row half of the A tile, both against the one
//               B tile, into the two halves of TMEM, and commits stage and
//               accumulator barriers (TMEM holds one tile: the next tile's
//               MMAs wait for the epilogue);
//   warps 2..9  epilogue, one warp per (TMEM lane quarter, row half):
//               tcgen05.ld 32 lanes x 32 columns, two loads in flight, sum of
//               squares in fp32 per row, fp64 warp reduction, one partial per
//               (128-row block, N tile, lane quarter) into HBM.
// Sharing each B tile between two M halves halves the B traffic from L2 to
// shared memory per flop; under the power cap that bought 4 % more
// throughput than 128 x 256 tiles with a double-buffered accumulator.
// Tiles are visited in groups of `group_m` M-blocks so the A panels of a
// group stay in L2 while all N-blocks stream past.  Every mbarrier wait is
// bounded; a wait that runs out records kDevTimeout, raises a CTA-wide abort
// flag, and every role drains its in-flight copies / MMAs before the CTA frees
// its TMEM and exits.
#include <cuda.h>
#include <cuda_fp16.h>
#include <math.h>

#include "awq_launch.h"

namespace awq {

namespace {

constexpr int BM = kGemmBM, BN = kGemmBN, BK = kGemmBK;
constexpr int STAGES = 3;
constexpr int BM2 = 2 * BM;                  // CTA tile rows: two M = 128 accumulators
constexpr uint32_t A_HALF = BM * BK * 2;     // 16 KiB: rows 128..255 of an A tile start here
constexpr uint32_t A_BYTES = BM2 * BK * 2;   // 32 KiB
constexpr uint32_t B_BYTES = BN * BK * 2;  // 32 KiB
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC = idesc_f16_f32(BM, BN);
constexpr uint32_t DRAIN_POLLS = 1u << 22;
constexpr int GROUP_M = 16;  // 256-row M blocks per group: 4096 rows of A in L2
constexpr int kEpiSse = 0, kEpiStoreY = 1, kEpiSubY = 2;
constexpr int kEpiWarps = 8;                      // two per TMEM lane quarter: one per row half
constexpr int kGemmThreads = (2 + kEpiWarps) * 32;  // producer, MMA issuer, epilogue

struct __align__(8) GemmSmemTail {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t kGemmSmemBytes =
    1024 /*alignment slack*/ + STAGES * (A_BYTES + B_BYTES) + sizeof(GemmSmemTail);

__device__ __forceinline__ void tile_coords(int tile, int num_m, int num_n, int group_m,
                                            int &m_blk, int &n_blk) {
  const int per_group = group_m * num_n;
  const int g = tile / per_group;
  const int first_m = g * group_m;
  const int gm = min(group_m, num_m - first_m);
  const int local = tile - g * per_group;
  m_blk = first_m + local % gm;
  n_blk = local / gm;
}

__device__ __forceinline__ void raise_abort(GemmSmemTail *t, DevStatus *st, uint32_t where) {
  dev_fail(st, kDevTimeout, where);
  *reinterpret_cast<volatile int *>(&t->abort_flag) = 1;
}

}  // namespace

// Epilogue of one accumulator tile (a 128-token x 256-column block of the
// product of X with the B rows):
//   kEpiSse    sum of squares (B = candidate errors dW: X dW^T is the error);
//   kEpiStoreY the tile rounded to fp16 into Y [tokens, ldy] (B = W: the
//              reference output Y = X W^T, computed once);
//   kEpiSubY   sum of (acc - Y)^2 with the cached fp16 Y (B = candidate
//              weights Qdeq/s: the literal "MSE against the fp16 output").
template <int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
    search_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB, int num_m, int num_n, int num_kb,
                       double *__restrict__ partials, __half *__restrict__ Y, int64_t ldy,
                       int64_t y_cols, int64_t y_rows, DevStatus *st, uint32_t max_polls) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sA = smem;
  uint8_t *sB = smem + STAGES * A_BYTES;
  GemmSmemTail *tail = reinterpret_cast<GemmSmemTail *>(sB + STAGES * B_BYTES);
  volatile int *abort_flag = &tail->abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_m2 = (num_m + 1) / 2;  // 256-row M blocks (num_m counts 128-row blocks)
  const int num_tiles = num_m2 * num_n;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&tail->full[s], 1);
      mbar_init(&tail->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tail->tfull[a], 1);
      mbar_init(&tail->tempty[a], kEpiWarps);  // one arrival per epilogue warp
    }
    mbar_init(&tail->mma_done, 1);
    tail->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(&tail->tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tail->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_parity = 0;  // per-stage: a fill is pending / its parity
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        int m_blk, n_blk;
        tile_coords(tile, num_m2, num_n, GROUP_M, m_blk, n_blk);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_long(&tail->empty[stage], phase ^ 1u, max_polls, abort_flag)) {
            raise_abort(tail, st, 0x100u + stage);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&tail->full[stage], A_BYTES + B_BYTES);
          tma_load_2d(sA + stage * A_BYTES, &tmA, &tail->full[stage], kb * BK, m_blk * BM2);
          tma_load_2d(sB + stage * B_BYTES, &tmB, &tail->full[stage], kb * BK, n_blk * BN);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok || *abort_flag) {
        // Let every fill already issued land before the CTA can exit.
        for (int s = 0; s < STAGES; ++s)
          if (issued & (1u << s))
            (void)mbar_wait_bounded(&tail->full[s], (issued_parity >> s) & 1u, DRAIN_POLLS,
                                    nullptr);
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
        const int acc = 0;  // TMEM holds one 256 x 256 tile: columns 0..255 rows 0..127, 256..511 rows 128..255
        const uint32_t acc_phase = it & 1;
        if (!mbar_wait_bounded(&tail->tempty[acc], acc_phase ^ 1u, max_polls, abort_flag)) {
          raise_abort(tail, st, 0x200u + acc);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_bounded(&tail->full[stage], phase, max_polls, abort_flag)) {
            raise_abort(tail, st, 0x300u + stage);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t bd = smem_desc_k_sw128(b_addr + k * 32);
#pragma unroll
            for (int h = 0; h < 2; ++h)  // both row halves share the B tile
              tc_mma_f16(d_tmem + h * BN, smem_desc_k_sw128(a_addr + h * A_HALF + k * 32), bd, IDESC,
                         (kb | k) != 0 ? 1u : 0u);
          }
          issued_any = true;
          tc_commit(&tail->empty[stage]);  // frees the stage once these MMAs finish
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&tail->tfull[acc]);  // accumulator ready for the epilogue
      }
      if (issued_any) {
        tc_commit(&tail->mma_done);
        (void)mbar_wait_bounded(&tail->mma_done, 0, DRAIN_POLLS, nullptr);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;           // TMEM lane quarter this warp may access
    const int h = (warp - 2) >> 2;    // the row half (accumulator) this warp reads
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int acc = 0;
      const uint32_t acc_phase = it & 1;
      int ok = 1;
      if (lane == 0) ok = mbar_wait_long(&tail->tfull[acc], acc_phase, max_polls, abort_flag);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        if (lane == 0) raise_abort(tail, st, 0x400u + acc);
        break;
      }
      tc_fence_after();
      int m_blk, n_blk;
      tile_coords(tile, num_m2, num_n, GROUP_M, m_blk, n_blk);
      float sums[1] = {0.0f};
      const int m128 = 2 * m_blk + h;  // 128-row block of this warp's half
      if (m128 < num_m) {              // the last tile's second half may lie past T (and past Y)
        const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(h * BN);
        // this thread's accumulator row is token 128 m128 + 32 q + lane
        const size_t yrow = (size_t)(m128 * BM + q * 32 + lane) * (size_t)ldy;
        float sum = 0.0f;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          float v[32];
          if constexpr (EPI == kEpiSubY) {
            // fetch the cached fp16 outputs first, so their latency overlaps the TMEM read
            const uint4 *yp = reinterpret_cast<const uint4 *>(
                Y + yrow + (size_t)(((int64_t)n_blk * BN) % y_cols) + c);
            uint4 yv[4];
            const bool y_ok = AWQ_IN_BOUNDS((((int64_t)n_blk * BN) % y_cols) + c + 32 <= y_cols, 0xB031u);
#pragma unroll
            for (int u = 0; u < 4; ++u) yv[u] = y_ok ? __ldg(yp + u) : make_uint4(0u, 0u, 0u, 0u);
            tmem_ld_32x32b_x32(taddr + (uint32_t)c, v);
            tmem_ld_wait();
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const uint32_t yw[4] = {yv[u].x, yv[u].y, yv[u].z, yv[u].w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 yf = __half22float2(*reinterpret_cast<const __half2 *>(&yw[e]));
                const float d0 = v[8 * u + 2 * e] - yf.x, d1 = v[8 * u + 2 * e + 1] - yf.y;
                sum = fmaf(d0, d0, sum);
                sum = fmaf(d1, d1, sum);
              }
            }
          } else if constexpr (EPI == kEpiSse) {
            // two 32-column loads in flight per wait
            float v2[32];
            tmem_ld_32x32b_x32(taddr + (uint32_t)c, v);
            tmem_ld_32x32b_x32(taddr + (uint32_t)(c + 32), v2);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) sum = fmaf(v[i], v[i], sum);
#pragma unroll
            for (int i = 0; i < 32; ++i) sum = fmaf(v2[i], v2[i], sum);
            c += 32;
          } else {
            tmem_ld_32x32b_x32(taddr + (uint32_t)c, v);
            tmem_ld_wait();
            if constexpr (EPI == kEpiStoreY) {
              // rows from y_rows on and columns from y_cols on are not stored
              const int64_t token = (int64_t)m128 * BM + q * 32 + lane;
              const int64_t col0 = (int64_t)n_blk * BN + c;
              uint4 *yp = reinterpret_cast<uint4 *>(Y + yrow + col0);
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                if (token >= y_rows || col0 + 8 * u >= y_cols) break;
                uint32_t hw[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const __half2 hv = __floats2half2_rn(v[8 * u + 2 * e], v[8 * u + 2 * e + 1]);
                  hw[e] = *reinterpret_cast<const uint32_t *>(&hv);
                }
                yp[u] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
              }
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) sum = fmaf(v[i], v[i], sum);
            }
          }
        }
        sums[0] = sum;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tail->tempty[acc]);
      if constexpr (EPI != kEpiStoreY) {
        double ds = (double)sums[0];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ds += __shfl_xor_sync(0xffffffffu, ds, off);
        if (lane == 0 && m128 < num_m && AWQ_IN_BOUNDS(n_blk < num_n, 0xB030u))
          partials[((size_t)n_blk * num_m + m128) * 4 + q] = ds;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Host side: tensor maps and launch.
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D fp16 tensor map over a row-major [rows, cols] matrix with row stride
// `ld` elements, box [box_rows, box_cols], 128-byte swizzle, zero fill.
cudaError_t make_tmap_f16_box(CUtensorMap *m, const void *base, int64_t rows, int64_t cols,
                              int64_t ld, uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int EPI>
static cudaError_t launch_gemm_epi(const CUtensorMap &tmA, const CUtensorMap &tmB,
                                   const SearchGemmShape &sh, double *partials, __half *Y,
                                   int64_t ldy, int64_t y_cols, int64_t y_rows, DevStatus *st,
                                   uint32_t max_polls,
                                   int num_sms, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(search_gemm_kernel<EPI>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kGemmSmemBytes);
  if (e != cudaSuccess) return e;
  const int tiles = ((sh.num_m + 1) / 2) * sh.num_n;  // 256-row tiles
  const int grid = tiles < num_sms ? tiles : num_sms;
  search_gemm_kernel<EPI><<<grid, kGemmThreads, kGemmSmemBytes, stream>>>(
      tmA, tmB, sh.num_m, sh.num_n, sh.num_kb, partials, Y, ldy, y_cols, y_rows, st, max_polls);
  return cudaGetLastError();
}

// 2-D int32 tensor map over a row-major [rows, cols] matrix (row stride `ld`
// elements, a multiple of 4), box [box_rows, box_cols], no swizzle, zero fill.
cudaError_t make_tmap_i32_box(CUtensorMap *m, const void *base, int64_t rows, int64_t cols,
                              int64_t ld, uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * 4)};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_INT32, 2, const_cast<void *>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t launch_search_gemm(const __half *X, int64_t ldx, const __half *dW,
                               const SearchGemmShape &sh, double *partials, const __half *Y,
                               int64_t ldy, DevStatus *st, uint32_t max_polls, int num_sms,
                               cudaStream_t stream) {
  CUtensorMap tmA, tmB;
  cudaError_t e = make_tmap_f16_box(&tmA, X, sh.T, sh.in, ldx, BK, BM2);
  if (e != cudaSuccess) return e;
  e = make_tmap_f16_box(&tmB, dW, sh.rows_b, sh.in, sh.in, BK, BN);
  if (e != cudaSuccess) return e;
  if (Y)
    return launch_gemm_epi<kEpiSubY>(tmA, tmB, sh, partials, const_cast<__half *>(Y), ldy, ldy, 0,
                                     st, max_polls, num_sms, stream);
  return launch_gemm_epi<kEpiSse>(tmA, tmB, sh, partials, nullptr, 0, 1, 0, st, max_polls, num_sms,
                                  stream);
}

cudaError_t launch_ref_output(const __half *X, int64_t T, int64_t in, int64_t ldx, const __half *W,
                              int64_t out, int64_t out_pad, __half *Y, DevStatus *st,
                              uint32_t max_polls, int num_sms, cudaStream_t stream) {
  if (out_pad % BN != 0 || in % BK != 0) return cudaErrorInvalidValue;
  CUtensorMap tmA, tmB;
  cudaError_t e = make_tmap_f16_box(&tmA, X, T, in, ldx, BK, BM2);
  if (e != cudaSuccess) return e;
  e = make_tmap_f16_box(&tmB, W, out, in, in, BK, BN);  // rows >= out read as zeros
  if (e != cudaSuccess) return e;
  SearchGemmShape sh;
  sh.T = T;
  sh.in = in;
  sh.rows_b = out;
  sh.num_m = (int)((T + BM - 1) / BM);
  sh.num_n = (int)(out_pad / BN);
  sh.num_kb = (int)(in / BK);
  return launch_gemm_epi<kEpiStoreY>(tmA, tmB, sh, nullptr, Y, out_pad, out_pad,
                                     (int64_t)sh.num_m * BM, st, max_polls, num_sms, stream);
}

cudaError_t launch_gemm_store(const __half *X, int64_t T, int64_t in, int64_t ldx, const __half *W,
                              int64_t out, __half *Y, int64_t ldy, DevStatus *st, uint32_t max_polls,
                              int num_sms, cudaStream_t stream) {
  if (in % BK != 0 || out % 8 != 0) return cudaErrorInvalidValue;
  CUtensorMap tmA, tmB;
  cudaError_t e = make_tmap_f16_box(&tmA, X, T, in, ldx, BK, BM2);  // rows >= T read as zeros
  if (e != cudaSuccess) return e;
  e = make_tmap_f16_box(&tmB, W, out, in, in, BK, BN);  // rows >= out read as zeros
  if (e != cudaSuccess) return e;
  SearchGemmShape sh;
  sh.T = T;
  sh.in = in;
  sh.rows_b = out;
  sh.num_m = (int)((T + BM - 1) / BM);
  sh.num_n = (int)((out + BN - 1) / BN);
  sh.num_kb = (int)(in / BK);
  return launch_gemm_epi<kEpiStoreY>(tmA, tmB, sh, nullptr, Y, ldy, out, T, st, max_polls, num_sms,
                                     stream);
}

// ---------------------------------------------------------------------------
// K5 — MSE_i = (sum of candidate i's `per` partials, stored contiguously)
// * 2^-2k / (T out).  One block
// per candidate sums its partials in a fixed order (bitwise reproducible);
// the last block to finish picks best = the first index of the smallest MSE
// and copies s_best = s_grid[best].  With best_idx = s_best = NULL it only
// writes the sums (T = out = 1 gives the unnormalised SSE of these tokens).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) mse_argmin_kernel(
    const double *__restrict__ partials, int n_alpha, size_t per, int64_t T,
    int64_t out, const float *__restrict__ s_grid, int64_t in, DevStatus *st,
    double *__restrict__ mse, int32_t *__restrict__ best_idx, float *__restrict__ s_best) {
  __shared__ double red[1024];
  __shared__ int last_sh, best_sh;
  const int i = blockIdx.x;
  const int k = kscale_from_wmax(__uint_as_float(__ldcg(&st->wmax_bits)));
  const double *p = partials + (size_t)i * per;
  double acc = 0.0;
  for (size_t idx = threadIdx.x; idx < per; idx += blockDim.x) acc += __ldcg(p + idx);
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int w = blockDim.x >> 1; w > 0; w >>= 1) {
    if ((int)threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double v = ldexp(red[0], -2 * k) / ((double)T * (double)out);
    if (AWQ_IN_BOUNDS(i < n_alpha, 0xB032u)) __stcg(mse + i, v);
    __threadfence();
    last_sh = atomicAdd(&st->mse_done, 1u) == (unsigned)(n_alpha - 1);
  }
  __syncthreads();
  if (!last_sh) return;
  if (threadIdx.x == 0) {
    __threadfence();
    int best = 0;
    double bv = __ldcg(mse);
    bool finite = isfinite(bv);
    for (int a = 1; a < n_alpha; ++a) {
      const double v = __ldcg(mse + a);
      if (!isfinite(v)) finite = false;
      if (v < bv) {
        bv = v;
        best = a;
      }
    }
    if (!finite) dev_fail(st, kDevNonFinite, 0x500u);
    best_sh = best;
    if (best_idx) *best_idx = best;
  }
  __syncthreads();
  if (!s_best) return;  // partial sums only (token-sharded search)
  const float *src = s_grid + (size_t)best_sh * in;
  for (int64_t j = threadIdx.x; j < in; j += blockDim.x) s_best[j] = src[j];
}

cudaError_t launch_mse_argmin(const double *partials, int n_alpha, size_t per_alpha, int64_t T,
                              int64_t out, const float *s_grid, int64_t in, DevStatus *st,
                              double *mse, int32_t *best_idx, float *s_best, cudaStream_t stream) {
  mse_argmin_kernel<<<n_alpha, 1024, 0, stream>>>(partials, n_alpha, per_alpha, T, out, s_grid, in,
                                                  st, mse, best_idx, s_best);
  return cudaGetLastError();
}

AWQ_BOUNDS_READER(bounds_status_gemm)

}  // namespace awq
