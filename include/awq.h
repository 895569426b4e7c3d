/*
 * awq.h — C ABI of the B200 (sm_100a) AWQ per-layer scale search.
 *
 * AWQ ("AWQ and Activation-Aware Scaling", "Scaling instead of protecting";
 * "05 — AWQ: Activation-Aware Weight Scaling" §3–§5) protects the weight
 * channels that meet large activations by a per-input-channel scale
 * s = abar^alpha applied before quantisation, with 1/s folded into the
 * activations.  This library runs the search that picks s for one linear
 * layer (or one group of linears that share an input), then the optional
 * per-group clip search, then packs the result.  Call order per layer:
 *
 *   awq_act_stats -> awq_search_scale -> [awq_search_clip] -> awq_quant_pack
 *
 * Conventions shared by every call
 *   - Pointers named as "device" are CUDA device pointers owned by the caller;
 *     the library allocates no device memory.  Scratch memory comes from the
 *     caller's workspace `ws` of at least awq_workspace_size() bytes,
 *     256-byte aligned.  X and W must be 16-byte aligned.
 *   - Every call is asynchronous and ordered on `stream` (a cudaStream_t; NULL
 *     is the legacy default stream).  Outputs are valid once the stream has
 *     been synchronised.  Calls that share a workspace must not overlap.
 *   - Arguments are checked on the host before anything is launched; a failed
 *     check returns AWQ_ERR_INVALID_ARG or AWQ_ERR_UNSUPPORTED and has no side
 *     effect.  awq_last_error() returns a message for the calling thread.
 *   - Device-side failures (a bounded wait in a kernel that ran out, a
 *     non-finite score) are recorded in a status word inside the workspace;
 *     awq_device_status() synchronises the stream and reports and clears it.
 *     Every call that takes a workspace clears that word first, so it
 *     describes the latest such call.  The calls that take no workspace
 *     (awq_quant_pack, awq_search_clip_noalloc) record theirs in one status
 *     word of the library per device instead, which keeps every failure
 *     until awq_device_status(NULL, stream) reads and clears it.
 *   - With the environment variable AWQ_SYNC_CHECK set, the searches, the
 *     packing and the allocation-free clip search synchronise before
 *     returning and return the device status themselves.
 *   - Fault injection for tests, environment variable AWQ_FAULT (read at
 *     every call): "timeout" makes every bounded device wait give up after
 *     one poll; "alloc" refuses every workspace (AWQ_ERR_WORKSPACE, and
 *     awq_workspace_size returns 0); "launch" fails every call after its
 *     argument checks and before any CUDA call (AWQ_ERR_CUDA); "nonfinite"
 *     makes the alpha selection see non-finite scores (AWQ_ERR_NONFINITE).
 *   - X is [T, in] fp16, token-major, row stride ldx >= in elements (ldx a
 *     multiple of 8).  W is [out, in] fp16, row-major and contiguous, laid out
 *     like nn.Linear.  Linears that share one input and one scale (q|k|v,
 *     gate|up) are passed concatenated along out.
 *   - Quantisation (all calls): groups of g consecutive input channels of one
 *     output row, asymmetric min/max with a zero point, b-bit codes, every
 *     float step in fp32 with round-half-to-even:
 *        wt = s*w;  mx, mn = max, min of wt (times r when clipping);
 *        d = max(mx - mn, 1e-5);  delta = d / (2^b - 1);
 *        z = clamp(rne(-mn/delta), 0, 2^b - 1);
 *        q = clamp(rne(wt/delta) + z, 0, 2^b - 1);  deq = (q - z)*delta.
 */
#ifndef AWQ_H_
#define AWQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void *awq_stream_t; /* a cudaStream_t */

typedef enum {
  AWQ_OK = 0,
  AWQ_ERR_INVALID_ARG = 1, /* a size, stride, pointer or alignment is wrong   */
  AWQ_ERR_UNSUPPORTED = 2, /* a valid setting the library does not implement  */
  AWQ_ERR_WORKSPACE = 3,   /* workspace missing, misaligned or too small      */
  AWQ_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed               */
  AWQ_ERR_TIMEOUT = 5,     /* a bounded device-side wait ran out              */
  AWQ_ERR_NONFINITE = 6    /* a score came out NaN or infinite                */
} awq_status;

/* How awq_search_scale scores the candidates (all give the same MSE in exact
 * arithmetic, by the scaling invariance of "05 — AWQ" §3):
 *   AWQ_SEARCH_DIRECT   the scored GEMM ||X dW^T||^2 over all tokens, dW =
 *                       Qdeq/s - W held as fp16 x 2^k (2 T in out n_alpha flops);
 *   AWQ_SEARCH_GRAM     sum_o dW_o^T (X^T X) dW_o: G = X^T X once (T in^2 flops,
 *                       symmetric), then one GEMM of the candidates against the
 *                       normalised G held as fp16 hi + lo parts
 *                       (4 in^2 out n_alpha flops);
 *   AWQ_SEARCH_CACHED_Y the literal reading of "05 — AWQ" §4 ("measure MSE
 *                       against the fp16 output"): Y = RN16(X W^T) once into the
 *                       workspace, then one GEMM of X against the candidate
 *                       weights RN16(Qdeq/s) whose epilogue subtracts the cached
 *                       Y tile and sums the squares (2 T in out (n_alpha + 1)
 *                       flops; the 1/s of the activation side is folded into
 *                       the candidate weights so that every candidate shares
 *                       one staged X tile);
 *   AWQ_SEARCH_FUSED    the direct form with the candidates made inside the
 *                       GEMM: each B tile is converted from the W rows in
 *                       shared memory (from per-group steps and zero points,
 *                       8 bytes per alpha, row and group in the workspace), so
 *                       the n_alpha x out x in operand is never written; the
 *                       same MSE bits as AWQ_SEARCH_DIRECT, with the conversion
 *                       repeated for every 256-token tile. */
enum { AWQ_SEARCH_DIRECT = 0, AWQ_SEARCH_GRAM = 1, AWQ_SEARCH_CACHED_Y = 2, AWQ_SEARCH_FUSED = 3 };

/* Quantisation and search settings; the first three fields are the pages'
 * quant_config ("05 — AWQ" §9: w_bit, q_group_size, zero_point). */
typedef struct {
  int32_t w_bit;      /* 3 or 4                                                  */
  int32_t group_size; /* 128 (the pages' g), or 32 / 64 ("AWQ and Activation-Aware
                         Scaling", When it breaks, contrasts g = 32); must divide in */
  int32_t zero_point; /* 1 = asymmetric: step (max - min)/(2^b - 1), zero point
                         z = clamp(rne(-min/step), 0, 2^b - 1) ("05 — AWQ" §9
                         zero_point = True).  0 = symmetric, the scheme of
                         "05 — AWQ" §3: step max|w|/(2^(b-1) - 1), z = 2^(b-1)
                         for every group, so codes lie in [0, 2^b - 1] centred on
                         z and qzeros holds 2^(b-1) in every nibble           */
  int32_t n_alpha;    /* alpha grid size, 1..64; alpha_i = i/(n_alpha-1) ("05 — AWQ" §4: ~20) */
  int32_t n_clip;     /* clip grid size, 0 = no clip search, else 1..64          */
  float clip_min;     /* smallest clip ratio, in (0, 1]; ("05 — AWQ" §4: 0.5)    */
  int32_t search_form; /* AWQ_SEARCH_DIRECT (0, default), AWQ_SEARCH_GRAM (1),
                          AWQ_SEARCH_CACHED_Y (2) or AWQ_SEARCH_FUSED (3)        */
} awq_config;

/* Bytes of workspace needed by awq_search_scale and awq_search_clip for a
 * layer with T tokens, `in` input and `out` output channels.  Returns 0 when
 * the arguments are invalid (see awq_last_error()). */
size_t awq_workspace_size(int64_t T, int64_t in, int64_t out, const awq_config *cfg);

/* The smallest workspace the same calls accept.  With less than
 * awq_workspace_size() bytes (but at least this many) the alpha search
 * builds and scores its candidates in chunks, as many at a time as the
 * workspace holds (down to one: the candidate operand then takes
 * out_pad x in fp16 instead of n_alpha times that); the results are the same
 * bit for bit, each candidate's scores coming from the same tiles. */
size_t awq_workspace_size_min(int64_t T, int64_t in, int64_t out, const awq_config *cfg);

/* Per-input-channel mean activation magnitude ("AWQ and Activation-Aware
 * Scaling", Scaling instead of protecting: abar; "05 — AWQ" §4, step 1).
 *   X    device fp16 [T, in], row stride ldx (elements)
 *   abar device fp64 [in] (output): abar_j = (sum_t |X_tj|) / T.  The sum is
 *        exact (each fp16 is an integer multiple of 2^-24, summed as int64),
 *        then converted to fp64 and divided by T with one rounding each.
 *        abar's storage doubles as the int64 accumulator while the call runs.
 * Requires T >= 1, in % 8 == 0, T * 65504 * 2^24 < 2^63 (T <= 2^22). */
awq_status awq_act_stats(const void *X, int64_t T, int64_t in, int64_t ldx,
                         double *abar, awq_stream_t stream);

/* The candidate scale grid s_ij = RN32(pow(max(abar_j, 1e-4), alpha_i)),
 * alpha_i = i/(n_alpha-1) ("AWQ and Activation-Aware Scaling": s = abar^alpha;
 * "05 — AWQ" §4: ~20 values in [0, 1]).
 *   abar device fp64 [in];  s device fp32 [n_alpha, in] (output). */
awq_status awq_scale_grid(const double *abar, int64_t in, int32_t n_alpha, float *s,
                          awq_stream_t stream);

/* alpha-grid search ("05 — AWQ" §4 step 2–3; "AWQ and Activation-Aware
 * Scaling": alpha found by a small per-layer grid search minimising
 * reconstruction error).  For each alpha_i it fake-quantises diag(s_i) W and
 * scores MSE_i = mean over tokens and outputs of
 *   ((X diag(s_i)^-1) Qdeq(diag(s_i) W)^T - X W^T)^2,
 * evaluated as ||X dW_i^T||^2 / (T out) with dW_i = Qdeq/s_i - W (the
 * scaling invariance of "05 — AWQ" §3), on the tensor cores; with
 * cfg->search_form = AWQ_SEARCH_GRAM as sum_o dW_o^T (X^T X) dW_o / (T out);
 * with AWQ_SEARCH_CACHED_Y as ||X RN16(Qdeq/s_i)^T - RN16(X W^T)||^2 / (T out)
 * (the workspace then also holds Y: ceil(T/128) * 128 x round_up(out, 256)
 * fp16).
 *   abar     device fp64 [in] from awq_act_stats
 *   s_best   device fp32 [in]      (output) s of the selected alpha
 *   mse      device fp64 [n_alpha] (output) MSE_i
 *   best_idx device int32 [1]      (output) first index of the smallest MSE
 * Requires out % 8 == 0, ldx % 8 == 0, and in % 64 == 0 (direct and cached-Y
 * forms) or in % 128 == 0 (Gram form). */
awq_status awq_search_scale(const void *X, int64_t T, int64_t in, int64_t ldx,
                            const void *W, int64_t out, const double *abar,
                            const awq_config *cfg, void *ws, size_t ws_bytes,
                            float *s_best, double *mse, int32_t *best_idx,
                            awq_stream_t stream);

/* Clip-ratio search ("05 — AWQ" §4, optional clipping: a ratio of 0.5–1.0 of
 * the range, grid-searched after alpha).  For every output row o and group k
 * it tries r_c = 1 - c (1 - clip_min)/(n_clip - 1), c = 0..n_clip-1, shrinking
 * both ends of the group range, and keeps the first c minimising that
 * group's own output error over all tokens,
 *   E_okc = sum_t (sum_{j in k} X_tj (deq_c,oj / s_j - W_oj))^2
 *         = d^T (X_k^T X_k) d,
 * evaluated with an fp32 block Gram X_k^T X_k and fp32 quadratic forms (the
 * Grams of 128-channel blocks, whose diagonal g x g blocks are the groups'
 * when g = 32 or 64).
 *   s        device fp32 [in] (normally s_best); NULL means s = 1
 *   clip_idx device uint8 [out, in/g] (output)
 *   err      device fp32 [out, in/g, n_clip] (output, optional, may be NULL)
 * Requires cfg->n_clip >= 1 and in % 128 == 0. */
awq_status awq_search_clip(const void *X, int64_t T, int64_t in, int64_t ldx,
                           const void *W, int64_t out, const float *s,
                           const awq_config *cfg, void *ws, size_t ws_bytes,
                           uint8_t *clip_idx, float *err, awq_stream_t stream);

/* Inspection form of the alpha search's candidate quantiser: the codes of
 * every candidate of awq_search_scale's grid, produced by the same kernel and
 * quantisation steps that build the search's scored operand ("05 — AWQ" §4:
 * for each alpha apply the scaling and quantize).  For candidate i, row o and
 * group k of diag(s_i) W:
 *   q     device uint8 [n_alpha, out, in]      codes in [0, 2^b - 1]
 *   z     device uint8 [n_alpha, out, in/g]    zero points
 *   delta device fp32  [n_alpha, out, in/g]    steps
 * abar as for awq_search_scale; ws as for awq_search_scale (the first
 * 2 n_alpha in fp32 values of it are used).  Requires in % 64 == 0. */
awq_status awq_candidate_codes(const void *W, int64_t out, int64_t in, const double *abar,
                               const awq_config *cfg, void *ws, size_t ws_bytes, uint8_t *q,
                               uint8_t *z, float *delta, awq_stream_t stream);

/* awq_search_clip_grams, which also stores the codes of every clip candidate
 * as its quantiser makes them (inspection form of "05 — AWQ" §4's optional
 * clipping):
 *   q device uint8 [out, n_clip, in]     codes of (row o, ratio c, channel j)
 *   z device uint8 [out, n_clip, in/g]   zero points of (o, c, group k)
 * The search's own outputs (clip_idx, err) are those of awq_search_clip_grams. */
awq_status awq_clip_candidate_codes(const void *W, int64_t out, int64_t in, const float *s,
                                    const float *G, const awq_config *cfg, void *ws,
                                    size_t ws_bytes, uint8_t *clip_idx, float *err, uint8_t *q,
                                    uint8_t *z, awq_stream_t stream);

/* Allocation-free variant of awq_search_clip (the AWQ pages have no
 * counterpart: this entry exists for callers, not for the method).  Some
 * callers cannot allocate device memory while the search runs: a host
 * framework that owns every device byte through its own pre-planned arena,
 * or code that must not call cudaMalloc because that call can synchronise the
 * device in the middle of its stream work.  This call takes no workspace and
 * calls no cudaMalloc, cudaFree or allocating library routine: its scratch
 * (the block Grams) lives in a static device array of 24 MiB inside this
 * library, which every GPU that loads the library holds until the process
 * exits.  Arguments and outputs are those of awq_search_clip, with these
 * differences:
 *   - in must be at most 16384; larger layers return AWQ_ERR_INVALID_ARG
 *     (use awq_search_clip with a workspace);
 *   - the first call on a device looks up the device address of the static
 *     array (cudaGetSymbolAddress) with that device current; make that first
 *     call before any stream capture;
 *   - every call shares the one array, so calls that overlap on the GPU (on
 *     different streams, or from different threads) race and must be
 *     serialised by the caller.  Nothing in the array needs clearing: each
 *     call writes every element it reads;
 *   - a device-side failure (a bounded wait that ran out) is recorded in the
 *     library's status word: read it with awq_device_status(NULL, stream)
 *     (or set AWQ_SYNC_CHECK); after AWQ_ERR_TIMEOUT, clip_idx and err of
 *     that call are not to be used.
 * The Grams are summed over min(16, ceil(T/1024), 384/(in/128) - 1) token
 * chunks; where that equals awq_search_clip's min(16, ceil(T/1024)) (every
 * in <= 2048) the results are identical, otherwise they equal up to the
 * fp32 summation order of the block Grams. */
awq_status awq_search_clip_noalloc(const void *X, int64_t T, int64_t in, int64_t ldx,
                                   const void *W, int64_t out, const float *s,
                                   const awq_config *cfg, uint8_t *clip_idx, float *err,
                                   awq_stream_t stream);

/* Final quantisation and packing ("05 — AWQ" §5 bit-level output format).
 *   s        device fp32 [in] or NULL (s = 1)
 *   clip_idx device uint8 [out, in/g] or NULL (ratio 1)
 *   qweight  device int32 [in, out/8]:   code of (o, j) in bits 4(o%8)..+3 of [j][o/8]
 *   qzeros   device int32 [in/g, out/8]: zero of (o, k) in bits 4(o%8)..+3 of [k][o/8]
 *   scales   device fp16 [in/g, out]:    RN16(delta of (o, k))
 * INT3 codes use the same 4-bit container.  A clip index >= cfg->n_clip is
 * an error found on the device: that group gets codes and zero point 0 and a
 * NaN scale, and the library's status word records AWQ_ERR_INVALID_ARG
 * (awq_device_status(NULL, stream)). */
awq_status awq_quant_pack(const void *W, int64_t out, int64_t in, const float *s,
                          const uint8_t *clip_idx, const awq_config *cfg,
                          int32_t *qweight, int32_t *qzeros, void *scales,
                          awq_stream_t stream);

/* Folds 1/s into the operation that feeds the scaled linear ("AWQ and
 * Activation-Aware Scaling": the activation-side division is absorbed by the
 * preceding normalisation's scale or linear layer).  v is device fp16
 * [rows, cols]; row j is replaced by RN16(RN32(v_j) / s_j) (rows = in; cols = 1
 * for a norm's gamma, or the preceding linear's input width). */
awq_status awq_fold_inv_scale(void *v, int64_t rows, int64_t cols, const float *s,
                              awq_stream_t stream);

/* ------------------------------------------------------------------------
 * Token sharding of one layer over several GPUs.  Every statistic the search
 * needs is a sum over tokens: the exact |x| sums behind abar, each alpha's
 * squared error, and the clip search's block Grams.  Each rank computes its
 * tokens' part with the calls below, the caller sums the parts over ranks
 * (an all-reduce; the library itself never communicates), and the finishing
 * calls turn the sums into the results the single-GPU calls give.  Every rank
 * needs the full W.
 * ------------------------------------------------------------------------ */

/* sums_j = sum_t |X_tj| of these tokens in units of 2^-24: exact int64
 * (every fp16 is an integer multiple of 2^-24), so sums add exactly across
 * ranks.  X as in awq_act_stats; sums device int64 [in], overwritten. */
awq_status awq_act_sums(const void *X, int64_t T, int64_t in, int64_t ldx, int64_t *sums,
                        awq_stream_t stream);

/* abar_j = RN64(RN64(sums_j 2^-24) / T_total) from the summed sums: the same
 * bits awq_act_stats gives on all T_total tokens.  sums may alias abar. */
awq_status awq_act_stats_finish(const int64_t *sums, int64_t T_total, int64_t in, double *abar,
                                awq_stream_t stream);

/* Unnormalised squared errors of these tokens for every alpha,
 *   sse_i = sum_{t in this shard} sum_o (candidate i's output error)^2,
 * in the scoring form cfg->search_form (each form's sum splits over tokens;
 * the Gram form builds X^T X of these tokens).  abar must be the global abar
 * (awq_act_stats_finish) so that every rank scores the same candidates.
 * Arguments and workspace as awq_search_scale; sse device fp64 [n_alpha]. */
awq_status awq_search_scale_sse(const void *X, int64_t T, int64_t in, int64_t ldx, const void *W,
                                int64_t out, const double *abar, const awq_config *cfg, void *ws,
                                size_t ws_bytes, double *sse, awq_stream_t stream);

/* The selection from the summed sse: mse_i = sse_i / (T_total out), best_idx =
 * the first index of the smallest, s_best = RN32(pow(max(abar_j, 1e-4),
 * alpha_best)) (the grid's value).  ws: at least 256 bytes (status word). */
awq_status awq_select_scale(const double *sse, int64_t T_total, int64_t in, int64_t out,
                            const double *abar, const awq_config *cfg, void *ws, size_t ws_bytes,
                            float *s_best, double *mse, int32_t *best_idx, awq_stream_t stream);

/* Block Grams of these tokens, G[k] = X_k^T X_k for every block k of 128 input
 * channels (any cfg->group_size: groups of 32 or 64 are the diagonal blocks):
 * device fp32 [in/128][128][128] (output).  in % 128 == 0; workspace as
 * awq_search_clip (the same size). */
awq_status awq_block_grams(const void *X, int64_t T, int64_t in, int64_t ldx, const awq_config *cfg,
                           void *ws, size_t ws_bytes, float *G, awq_stream_t stream);

/* The clip-ratio search of awq_search_clip from block Grams G (summed over
 * ranks) instead of X.  ws: at least 256 bytes (status word). */
awq_status awq_search_clip_grams(const void *W, int64_t out, int64_t in, const float *s,
                                 const float *G, const awq_config *cfg, void *ws, size_t ws_bytes,
                                 uint8_t *clip_idx, float *err, awq_stream_t stream);

/* W4A16 GEMM on the packed output, the step after the search ("05 — AWQ" §5
 * layout; the weights are dequantised on the fly inside the GEMM, as the
 * pages describe for AWQ's inference kernels):
 *   Y[t][o] = RN16( sum_j X[t][j] Wd[o][j] ),  Wd[o][j] = RN16((q - z) scale)
 * with q the 4-bit code of (o, j) (nibble o % 8 of qweight[j][o/8]), z that of
 * qzeros[j/g][o/8] and scale = scales[j/g][o]; fp32 accumulation (on the
 * tensor cores from 9 tokens on; up to 8 tokens, a decode step, the product
 * is bound by reading the packed words and runs on CUDA cores, which stream
 * each word once).  INT3 codes use the same nibbles.
 *   X        device fp16 [T, in], row stride ldx
 *   qweight  device int32 [in, out/8]; qzeros int32 [in/g, out/8]; scales fp16 [in/g, out]
 *   Y        device fp16 [T, out] (output), row stride ldy (multiple of 8)
 *   ws       at least 256 bytes (status word), with which the weights are
 *            dequantised tile by tile inside the GEMM.  With
 *            awq_w4a16_workspace_size() bytes: few tokens (up to 8, or
 *            output tiles filling under half of the SMs) are computed with
 *            split-K (fp32
 *            partial sums of K ranges in the workspace, added in a fixed order
 *            and rounded to fp16 once); 1024 tokens or more dequantise the
 *            weights once into the workspace (the same RN16((q - z) scale)
 *            values) and run one fp16 GEMM on the tensor cores
 * Uses cfg->group_size (32, 64 or 128); requires in % 64 == 0 and out % 32 == 0
 * (the packed words of a row are staged by TMA, whose row stride must be a
 * multiple of 16 bytes). */
awq_status awq_w4a16_gemm(const void *X, int64_t T, int64_t in, int64_t ldx, const int32_t *qweight,
                          const int32_t *qzeros, const void *scales, int64_t out,
                          const awq_config *cfg, void *Y, int64_t ldy, void *ws, size_t ws_bytes,
                          awq_stream_t stream);

/* Workspace bytes with which awq_w4a16_gemm runs its fastest form for this
 * shape: 256 + in * out * 2 (the fp16 weights) from 1024 tokens on, the
 * split-K partial sums for few tokens, else 256.  Returns 0 when the
 * arguments are invalid. */
size_t awq_w4a16_workspace_size(int64_t T, int64_t in, int64_t out, const awq_config *cfg);

/* Synchronises `stream`, then returns and clears the device status recorded in
 * workspace `ws` (AWQ_OK, AWQ_ERR_TIMEOUT or AWQ_ERR_NONFINITE).  With
 * ws = NULL: the library's status word of the current device, which the calls
 * without a workspace use (AWQ_OK, AWQ_ERR_TIMEOUT from
 * awq_search_clip_noalloc, AWQ_ERR_INVALID_ARG from awq_quant_pack). */
awq_status awq_device_status(void *ws, awq_stream_t stream);

/* Message describing the last failure on the calling thread ("" if none). */
const char *awq_last_error(void);

/* Index checks (no counterpart on the pages; a stand-in for a memory
 * sanitizer).  The debug library, libawq_debug.so (built with
 * `python -m post_weight_quantization_awq_b200.build --debug-bounds`), checks
 * the global accesses whose indices the kernels derive from their grids: a
 * failed check skips the access and is recorded.  awq_bounds_checks_enabled
 * returns 1 in that library, 0 in libawq.so.  awq_bounds_status synchronises
 * the device and returns AWQ_ERR_INVALID_ARG (the message names the kernel
 * file and the site) if any check failed since the previous call, which
 * clears them; AWQ_OK otherwise, and always AWQ_OK in libawq.so. */
int32_t awq_bounds_checks_enabled(void);
awq_status awq_bounds_status(void);

/* Per-kernel timing with CUDA events recorded on the launch stream.
 * awq_profile_enable(1) starts recording every kernel this library launches;
 * awq_profile_read() synchronises the recorded events and returns, for the
 * kernel named `name`, the summed device time in ms and the launch count;
 * awq_profile_reset() forgets all records.  Off by default. */
awq_status awq_profile_enable(int32_t on);
awq_status awq_profile_read(const char *name, double *total_ms, int64_t *launches);
awq_status awq_profile_reset(void);

/* Library version string. */
const char *awq_version(void);

#ifdef __cplusplus
}
#endif
#endif /* AWQ_H_ */
