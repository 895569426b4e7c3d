// Internal launchers of the AWQ kernels (host side).  Every launcher only
// enqueues work on `stream` and returns the launch error, if any.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "awq_device.cuh"

namespace awq {

__host__ __device__ constexpr int64_t i64min(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ constexpr int64_t i64max(int64_t a, int64_t b) { return a > b ? a : b; }

// K1: abar (exact mean |x|).  abar doubles as the int64 accumulator.
cudaError_t launch_act_stats(const __half *X, int64_t T, int64_t in, int64_t ldx, double *abar,
                             int num_sms, cudaStream_t stream);

// Token-sharded K1: exact sums of |X| in units of 2^-24 into sums [in]
// (overwritten), and abar = RN64(RN64(sums 2^-24) / T) from summed sums.
cudaError_t launch_act_sums(const __half *X, int64_t T, int64_t in, int64_t ldx, int64_t *sums,
                            int num_sms, cudaStream_t stream);
cudaError_t launch_act_finish(const int64_t *sums, int64_t in, int64_t T, double *abar,
                              cudaStream_t stream);

// Token-sharded K5: mse = sse / (T out), best, s_best = s grid row of best.
cudaError_t launch_select_scale(const double *sse, int n_alpha, int64_t T, int64_t out,
                                const double *abar, int64_t in, DevStatus *st, double *mse,
                                int32_t *best_idx, float *s_best, cudaStream_t stream);

// K2: s[i][j] = RN32(pow(max(abar_j, 1e-4), i/(n-1))); inv_s (optional) = RN(1/s).
cudaError_t launch_scale_grid(const double *abar, int64_t in, int n_alpha, float *s, float *inv_s,
                              cudaStream_t stream);

// max |W| (r == NULL) or max r_j |W_oj| into st->wmax_bits (zero beforehand).
cudaError_t launch_wmax(const __half *W, int64_t n, int64_t in, const float *r, DevStatus *st,
                        int num_sms, cudaStream_t stream);

// K3: candidate effective errors dW[i][o][j] = RN16(2^k r_j (deq/s - w))
// (r = NULL: r_j = 1), rows out..out_pad-1 zero.  zero_point = 0 quantises
// symmetrically (step max|w|/(2^(b-1)-1), z = 2^(b-1)).  weights_only: the
// candidate weights RN16(deq/s) themselves (no 2^k, no - w).
cudaError_t launch_cand_quant(const __half *W, int64_t out, int64_t in, int64_t out_pad,
                              const float *s, const float *inv_s, const float *r, int n_alpha,
                              int group, int w_bit, int zero_point, int weights_only,
                              const DevStatus *st, __half *dW, int num_sms, cudaStream_t stream);

// K3, inspection form: the candidates' codes q [n_alpha, out, in], zero
// points z and steps delta [n_alpha, out, in/group] (direct-form k).
cudaError_t launch_cand_codes(const __half *W, int64_t out, int64_t in, int64_t out_pad,
                              const float *s, const float *inv_s, int n_alpha, int group, int w_bit,
                              int zero_point, const DevStatus *st, uint8_t *q, uint8_t *z,
                              float *delta, cudaStream_t stream);

// K4: scored GEMM, partial sums of squares per (n-tile, m-tile, warp).
struct SearchGemmShape {
  int64_t T, in, rows_b;  // rows_b = n_alpha * out_pad
  int num_m, num_n, num_kb;
};
// Y == NULL: partials of sum acc^2 (dW = candidate errors).  Y != NULL: partials
// of sum (acc - Y)^2 with the cached fp16 output Y [num_m * 128, ldy], the
// columns of N tile n being (n * 256) mod ldy (dW = candidate weights Qdeq/s).
cudaError_t launch_search_gemm(const __half *X, int64_t ldx, const __half *dW,
                               const SearchGemmShape &sh, double *partials, const __half *Y,
                               int64_t ldy, DevStatus *st, uint32_t max_polls, int num_sms,
                               cudaStream_t stream);
// Reference output Y = RN16(X W^T) into Y [ceil(T/128) * 128, out_pad] (padding
// rows and columns come out zero); out_pad % 256 == 0, in % 64 == 0.
cudaError_t launch_ref_output(const __half *X, int64_t T, int64_t in, int64_t ldx, const __half *W,
                              int64_t out, int64_t out_pad, __half *Y, DevStatus *st,
                              uint32_t max_polls, int num_sms, cudaStream_t stream);
// Y = RN16(X W^T) into the caller's Y [T, out] (row stride ldy): the scored
// GEMM's tiles with a bounded store epilogue; W fp16 [out, in] row-major,
// in % 64 == 0, out % 8 == 0.
cudaError_t launch_gemm_store(const __half *X, int64_t T, int64_t in, int64_t ldx, const __half *W,
                              int64_t out, __half *Y, int64_t ldy, DevStatus *st, uint32_t max_polls,
                              int num_sms, cudaStream_t stream);
constexpr int kGemmBM = 128, kGemmBN = 256, kGemmBK = 64;

// 2-D fp16 TMA descriptor over a row-major [rows, cols] matrix (row stride
// `ld` elements), box [box_rows, box_cols], 128-byte swizzle, zero fill.
cudaError_t make_tmap_f16_box(CUtensorMap *m, const void *base, int64_t rows, int64_t cols,
                              int64_t ld, uint32_t box_cols, uint32_t box_rows);
// The same for int32 elements (row stride a multiple of 4), no swizzle.
cudaError_t make_tmap_i32_box(CUtensorMap *m, const void *base, int64_t rows, int64_t cols,
                              int64_t ld, uint32_t box_cols, uint32_t box_rows);

// Fused form, K3p: per (alpha, row < out_pad, group) the candidate quantiser's
// {delta, bits of (zero | clamp << 8 | no fast path << 9)} of s 2^k w into
// params [n_alpha * out_pad, in / group] (rows past out: w = 0).
cudaError_t launch_fused_params(const __half *W, int64_t out, int64_t in, int64_t out_pad,
                                const float *s, int n_alpha, int group, int w_bit, int zero_point,
                                const DevStatus *st, float2 *params, cudaStream_t stream);
// Fused form, K4f: the scored GEMM with each B tile converted from the W rows
// in shared memory (the direct form's operand values, never stored); partials
// as launch_search_gemm's.  in % 64 == 0, out_pad % 256 == 0.
cudaError_t launch_fused_search_gemm(const __half *X, int64_t T, int64_t ldx, const __half *W,
                                     int64_t out, int64_t in, int64_t out_pad, int n_alpha,
                                     const float *s, const float *inv_s, const float2 *params,
                                     int group, int w_bit, double *partials, DevStatus *st,
                                     uint32_t max_polls, int num_sms, cudaStream_t stream);

// K5: mse[i] from `per_alpha` contiguous partials per candidate, best index, s_best.
cudaError_t launch_mse_argmin(const double *partials, int n_alpha, size_t per_alpha, int64_t T,
                              int64_t out, const float *s_grid, int64_t in, DevStatus *st,
                              double *mse, int32_t *best_idx, float *s_best, cudaStream_t stream);

// Gram form: G = X^T X (fp32 [in][in]), r = sqrt(diag G), G~ hi/lo fp16 [in][in].
cudaError_t launch_gram_full(const __half *X, int64_t T, int64_t in, int64_t ldx, float *G, float *r,
                             __half *ghi, __half *glo, DevStatus *st, uint32_t max_polls,
                             cudaStream_t stream);
// Gram form scoring: partials[(m_blk * (in/128) + n_blk) * 4 + warp] of
// d~ (G~_hi + G~_lo) . d~ over 128 x 128 tiles; rows % 128 == 0.
cudaError_t launch_gram_score(const __half *dW, int64_t rows, int64_t in, const __half *ghi,
                              const __half *glo, double *partials, DevStatus *st, uint32_t max_polls,
                              int num_sms, cudaStream_t stream);

// K6a: block Grams G[k] = X_k^T X_k (fp32, tensor cores), via per-chunk
// partials [n_chunks][in/g][g][g] summed in a fixed order.
cudaError_t launch_gram_blocks(const __half *X, int64_t T, int64_t in, int64_t ldx, int group,
                               int n_chunks, float *partials, float *G, DevStatus *st,
                               uint32_t max_polls, cudaStream_t stream);
// K6b: clip choice per (row, group), quadratic forms on the tensor cores.
cudaError_t launch_clip_eval(const __half *W, int64_t out, int64_t in, const float *s,
                             const float *G, int group, int w_bit, int zero_point, int n_clip,
                             float clip_min, uint8_t *clip_idx, float *err, DevStatus *st,
                             uint32_t max_polls, int num_sms, cudaStream_t stream,
                             uint8_t *cand_q = nullptr, uint8_t *cand_z = nullptr);

// K7: final codes + packing.
cudaError_t launch_quant_pack(const __half *W, int64_t out, int64_t in, const float *s,
                              const uint8_t *clip_idx, int group, int w_bit, int zero_point,
                              int n_clip, float clip_min, int32_t *qweight, int32_t *qzeros,
                              __half *scales, cudaStream_t stream);

// The status word of the calls that take no workspace: its device address on
// the current device, and a synchronous read that clears it.
cudaError_t lib_status_address(DevStatus **p);
cudaError_t lib_status_read_clear(DevStatus *h);

// W4A16 GEMM on the packed output: Y = RN16(X Wd^T), Wd = RN16((q - z) scale);
// in % 64 == 0, out % 32 == 0, group in {32, 64, 128}.
// splits > 1: split-K over `splits` K ranges, fp32 partial sums in
// partials [splits][T][out], then a fixed-order reduction into Y.
cudaError_t launch_w4a16_gemm(const __half *X, int64_t T, int64_t in, int64_t ldx,
                              const int32_t *qweight, const int32_t *qzeros, const __half *scales,
                              int64_t out, int group, __half *Y, int64_t ldy, float *partials,
                              int splits, DevStatus *st, uint32_t max_polls, int num_sms,
                              cudaStream_t stream);
// The split count the W4A16 GEMM uses when its workspace allows: 1 when the
// output tiles fill at least half of the SMs, else enough K splits (each of
// at least 4 K steps of 64 channels) to occupy them.
// Decode W4A16 product (T <= 8 tokens) on CUDA cores, streaming the packed
// words once; `partials` ([splits][T][out] fp32, splits = w4a16_gemv_splits:
// one per 256 input rows) enables the K split, NULL runs one block column per
// 256 outputs over all of `in`.  Requires in % 64 == 0, out % 8 == 0,
// group % 32 == 0, ldx % 8 == 0.
int w4a16_gemv_splits(int64_t T, int64_t in, int64_t out, int num_sms);
cudaError_t launch_w4a16_gemv(const __half *X, int64_t T, int64_t in, int64_t ldx,
                              const int32_t *qweight, const int32_t *qzeros, const __half *scales,
                              int64_t out, int group, __half *Y, int64_t ldy, float *partials,
                              int num_sms, cudaStream_t stream);
int w4a16_splits(int64_t T, int64_t in, int64_t out, int num_sms);
// The dequantised weights of a packed layer, Wd [out, in] fp16 row-major,
// Wd[o][j] = RN16((q - z) scale): the operand of the W4A16 product for many
// tokens (dequantised once, then one fp16 GEMM).
cudaError_t launch_w4a16_dequant(const int32_t *qweight, const int32_t *qzeros, const __half *scales,
                                 int64_t in, int64_t out, int group, __half *Wd, cudaStream_t stream);

// K8: v[j][:] = RN16(RN32(v[j][:]) / s_j).
cudaError_t launch_fold(__half *v, int64_t rows, int64_t cols, const float *s, cudaStream_t stream);

// Exponent k of the power-of-two factor applied to the candidate errors, from
// max |W|: |deq/s - w| <= 2|w| (+ rounding), so 2 max|W| 2^k <= 2^14 keeps
// every scaled error inside fp16 with a factor-4 margin.
__host__ __device__ inline int kscale_from_wmax(float wmax) {
  if (!(wmax > 0.0f)) return 0;
  int e;
  (void)frexpf(wmax, &e);  // wmax < 2^e
  int k = 13 - e;
  if (k > 60) k = 60;
  if (k < -60) k = -60;
  return k;
}


#ifdef AWQ_DEBUG_BOUNDS
// bounds words of the translation units with index checks (debug library)
cudaError_t bounds_status_quant(DevStatus *h);
cudaError_t bounds_status_gemm(DevStatus *h);
cudaError_t bounds_status_clip(DevStatus *h);
cudaError_t bounds_status_gram(DevStatus *h);
cudaError_t bounds_status_w4a16(DevStatus *h);
cudaError_t bounds_status_fused(DevStatus *h);
#endif

}  // namespace awq
