// Host implementation of the C ABI declared in include/awq.h: argument
// checks, workspace carving, kernel launches, per-thread error messages and
// optional per-kernel event timing.
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "awq.h"
#include "awq_launch.h"

using namespace awq;

namespace {

thread_local std::string g_err;

awq_status fail(awq_status st, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return st;
}

awq_status cuda_fail(cudaError_t e, const char *what) {
  return fail(AWQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

int num_sms_current() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

// --------------------------------------------------------------- profiling
struct ProfRec {
  const char *name;
  cudaEvent_t a, b;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRec> g_prof;
std::vector<cudaEvent_t> g_ev_pool;

cudaEvent_t take_event() {
  if (!g_ev_pool.empty()) {
    cudaEvent_t e = g_ev_pool.back();
    g_ev_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

struct ProfScope {
  const char *name;
  cudaStream_t s;
  cudaEvent_t a = nullptr;
  ProfScope(const char *n, cudaStream_t st) : name(n), s(st) {
    nvtxRangePushA(n);  // a no-op unless a profiler is attached
    std::lock_guard<std::mutex> lk(g_prof_mu);
    if (g_prof_on) {
      a = take_event();
      cudaEventRecord(a, s);
    }
  }
  ~ProfScope() {
    nvtxRangePop();
    if (!a) return;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    cudaEvent_t b = take_event();
    cudaEventRecord(b, s);
    g_prof.push_back({name, a, b});
  }
};

// NVTX range around one C-ABI call (a no-op unless a profiler is attached)
struct NvtxCall {
  explicit NvtxCall(const char *name) { nvtxRangePushA(name); }
  ~NvtxCall() { nvtxRangePop(); }
};

// ------------------------------------------------------------ validation
awq_status check_cfg(const awq_config *cfg) {
  if (!cfg) return fail(AWQ_ERR_INVALID_ARG, "cfg is NULL");
  if (cfg->w_bit < 1 || cfg->w_bit > 8) return fail(AWQ_ERR_INVALID_ARG, "w_bit=%d", cfg->w_bit);
  if (cfg->w_bit != 3 && cfg->w_bit != 4)
    return fail(AWQ_ERR_UNSUPPORTED, "w_bit=%d (3 or 4 supported)", cfg->w_bit);
  if (cfg->group_size <= 0) return fail(AWQ_ERR_INVALID_ARG, "group_size=%d", cfg->group_size);
  if (cfg->group_size != 32 && cfg->group_size != 64 && cfg->group_size != 128)
    return fail(AWQ_ERR_UNSUPPORTED, "group_size=%d (32, 64 or 128 supported)", cfg->group_size);
  if (cfg->zero_point != 0 && cfg->zero_point != 1)
    return fail(AWQ_ERR_INVALID_ARG, "zero_point=%d (1 asymmetric, 0 symmetric)", cfg->zero_point);
  if (cfg->n_alpha < 1 || cfg->n_alpha > 64)
    return fail(AWQ_ERR_INVALID_ARG, "n_alpha=%d (1..64)", cfg->n_alpha);
  if (cfg->n_clip < 0 || cfg->n_clip > 64)
    return fail(AWQ_ERR_INVALID_ARG, "n_clip=%d (0..64)", cfg->n_clip);
  if (!(cfg->clip_min > 0.0f && cfg->clip_min <= 1.0f))
    return fail(AWQ_ERR_INVALID_ARG, "clip_min=%g (must be in (0, 1])", (double)cfg->clip_min);
  if (cfg->search_form != AWQ_SEARCH_DIRECT && cfg->search_form != AWQ_SEARCH_GRAM &&
      cfg->search_form != AWQ_SEARCH_CACHED_Y && cfg->search_form != AWQ_SEARCH_FUSED)
    return fail(AWQ_ERR_INVALID_ARG,
                "search_form=%d (0 direct, 1 Gram, 2 cached fp16 output, 3 fused)", cfg->search_form);
  return AWQ_OK;
}

awq_status check_shape(int64_t T, int64_t in, int64_t out, const awq_config *cfg) {
  if (T < 1 || T > (int64_t(1) << 22)) return fail(AWQ_ERR_INVALID_ARG, "T=%lld (1..2^22)", (long long)T);
  if (in < cfg->group_size || in % cfg->group_size != 0)
    return fail(AWQ_ERR_INVALID_ARG, "in=%lld must be a positive multiple of group_size=%d",
                (long long)in, cfg->group_size);
  if (in > (int64_t(1) << 20)) return fail(AWQ_ERR_INVALID_ARG, "in=%lld too large", (long long)in);
  if (out < 8 || out % 8 != 0 || out > (int64_t(1) << 22))
    return fail(AWQ_ERR_INVALID_ARG, "out=%lld must be a positive multiple of 8", (long long)out);
  return AWQ_OK;
}

// The clip search works on 128-channel blocks (their Grams hold every group
// of 32, 64 or 128 channels of the block on the diagonal).
awq_status check_clip_in(int64_t in) {
  if (in % 128 != 0)
    return fail(AWQ_ERR_UNSUPPORTED, "in=%lld: the clip search needs in %% 128 == 0", (long long)in);
  return AWQ_OK;
}

awq_status check_x(const void *X, int64_t in, int64_t ldx) {
  if (!X) return fail(AWQ_ERR_INVALID_ARG, "X is NULL");
  if (!aligned(X, 16)) return fail(AWQ_ERR_INVALID_ARG, "X must be 16-byte aligned");
  if (ldx < in || ldx % 8 != 0)
    return fail(AWQ_ERR_INVALID_ARG, "ldx=%lld must be >= in and a multiple of 8", (long long)ldx);
  return AWQ_OK;
}

// ------------------------------------------------------------ workspace
constexpr size_t kHeader = 256;

struct ScaleWs {
  size_t s_grid, inv_s, dW, partials, G, ghi, glo, r, Y, end;
  int64_t out_pad;
  int num_m, nb_per_alpha;
  size_t per_alpha;  // partials per candidate
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Direct form: candidates padded to the GEMM's 256-row N tiles, partials per
// (n tile, m tile, warp).  Gram form: candidates padded to 128-row M tiles,
// partials per (m tile, n tile, warp), plus G, G~ hi/lo and r.
// n_chunk: candidates whose operand the workspace holds at a time (the
// alpha search runs the grid in chunks of that many when the caller's
// workspace is smaller than the whole grid's).
ScaleWs scale_layout(int64_t T, int64_t in, int64_t out, const awq_config *cfg, int n_chunk) {
  ScaleWs w;
  const bool gram = cfg->search_form == AWQ_SEARCH_GRAM;
  const bool cached_y = cfg->search_form == AWQ_SEARCH_CACHED_Y;
  w.out_pad = round_up(out, gram ? 128 : kGemmBN);
  w.num_m = (int)((T + kGemmBM - 1) / kGemmBM);
  w.nb_per_alpha = (int)(w.out_pad / kGemmBN);
  w.per_alpha = gram ? (size_t)(w.out_pad / 128) * (size_t)(in / 128) * 4
                     : (size_t)w.nb_per_alpha * w.num_m * 4;
  size_t off = kHeader;
  w.s_grid = off;
  off = align256(off + sizeof(float) * (size_t)cfg->n_alpha * in);
  w.inv_s = off;
  off = align256(off + sizeof(float) * (size_t)cfg->n_alpha * in);
  w.dW = off;  // fused form: the per-group parameters instead of the operand
  off = align256(off + (cfg->search_form == AWQ_SEARCH_FUSED
                            ? sizeof(float2) * (size_t)cfg->n_alpha * w.out_pad * (in / cfg->group_size)
                            : sizeof(__half) * (size_t)n_chunk * w.out_pad * in));
  w.partials = off;
  off = align256(off + sizeof(double) * (size_t)cfg->n_alpha * w.per_alpha);
  w.G = w.ghi = w.glo = w.r = w.Y = 0;
  if (cached_y) {  // Y = RN16(X W^T), padded to whole 128-token and 256-column tiles
    w.Y = off;
    off = align256(off + sizeof(__half) * (size_t)w.num_m * kGemmBM * (size_t)w.out_pad);
  }
  if (gram) {
    w.G = off;
    off = align256(off + sizeof(float) * (size_t)in * in);
    w.ghi = off;
    off = align256(off + sizeof(__half) * (size_t)in * in);
    w.glo = off;
    off = align256(off + sizeof(__half) * (size_t)in * in);
    w.r = off;
    off = align256(off + sizeof(float) * (size_t)in);
  }
  w.end = off;
  return w;
}

struct ClipWs {
  size_t gpart, G, end;
  int n_chunks;
};

ClipWs clip_layout(int64_t T, int64_t in) {
  ClipWs w;
  int64_t c = (T + 1023) / 1024;
  w.n_chunks = (int)(c < 1 ? 1 : (c > 16 ? 16 : c));
  const size_t gsz = sizeof(float) * (size_t)(in / 128) * 128 * 128;
  size_t off = kHeader;
  w.gpart = off;
  off = align256(off + gsz * w.n_chunks);
  w.G = off;
  off = align256(off + gsz);
  w.end = off;
  return w;
}

// Fault injection for tests (environment variable AWQ_FAULT, read at every
// call): "timeout" makes every bounded device wait give up after one poll;
// "alloc" makes the workspace unobtainable (awq_workspace_size returns 0 and
// every workspace is refused); "launch" fails every call that would launch,
// after its argument checks and before any CUDA call; "nonfinite" makes the
// alpha selection see non-finite scores (the MSE is divided by zero tokens).
enum class Fault { kNone, kTimeout, kAlloc, kLaunch, kNonFinite };

Fault fault_mode() {
  const char *f = getenv("AWQ_FAULT");
  if (!f) return Fault::kNone;
  if (strcmp(f, "timeout") == 0) return Fault::kTimeout;
  if (strcmp(f, "alloc") == 0) return Fault::kAlloc;
  if (strcmp(f, "launch") == 0) return Fault::kLaunch;
  if (strcmp(f, "nonfinite") == 0) return Fault::kNonFinite;
  return Fault::kNone;
}

// From this many tokens on, the W4A16 product dequantises the weights once
// into the workspace and runs one fp16 GEMM (when the workspace holds them):
// the conversion then costs in x out work once instead of once per 256-token
// tile, and the GEMM runs at the tensor cores' rate.
constexpr int64_t kW4DequantMinT = 1024;
// Up to this many tokens the product is bound by reading the packed words:
// a CUDA-core kernel streams them (the tensor-core forms would run a 128-row
// tile for a handful of rows).
constexpr int64_t kW4GemvMaxT = 8;

// status word plus the fp16 weights [out, in]
size_t w4a16_dequant_ws_bytes(int64_t in, int64_t out) {
  return kHeader + align256(sizeof(__half) * (size_t)in * (size_t)out);
}

// status word plus the fp32 partial sums [splits][T][out] of a split-K W4A16 GEMM
size_t w4a16_ws_bytes(int64_t T, int64_t out, int splits) {
  return kHeader + align256(sizeof(float) * (size_t)splits * (size_t)T * (size_t)out);
}

uint32_t poll_cap() {
  return fault_mode() == Fault::kTimeout ? 1u : 1u << 24;
}

// AWQ_OK, or the injected launch failure
awq_status launch_gate() {
  if (fault_mode() == Fault::kLaunch)
    return fail(AWQ_ERR_CUDA, "injected launch failure (AWQ_FAULT=launch)");
  return AWQ_OK;
}

awq_status check_ws(void *ws, size_t ws_bytes, size_t need) {
  if (fault_mode() == Fault::kAlloc)
    return fail(AWQ_ERR_WORKSPACE, "injected allocation failure (AWQ_FAULT=alloc)");
  if (!ws) return fail(AWQ_ERR_WORKSPACE, "workspace is NULL");
  if (!aligned(ws, 256)) return fail(AWQ_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (ws_bytes < need)
    return fail(AWQ_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu needed", ws_bytes,
                need);
  return AWQ_OK;
}

#define AWQ_LAUNCH_GATE()                   \
  do {                                      \
    const awq_status g_ = launch_gate();    \
    if (g_ != AWQ_OK) return g_;            \
  } while (0)

#define AWQ_TRY_CUDA(expr, what)                  \
  do {                                            \
    cudaError_t e_ = (expr);                      \
    if (e_ != cudaSuccess) return cuda_fail(e_, what); \
  } while (0)

}  // namespace

extern "C" {

const char *awq_version(void) { return "awq-b200 0.1 (sm_100a)"; }

const char *awq_last_error(void) { return g_err.c_str(); }

size_t awq_workspace_size(int64_t T, int64_t in, int64_t out, const awq_config *cfg) {
  g_err.clear();
  NvtxCall nvtx_call_(__func__);
  if (fault_mode() == Fault::kAlloc) {
    fail(AWQ_ERR_WORKSPACE, "injected allocation failure (AWQ_FAULT=alloc)");
    return 0;
  }
  if (check_cfg(cfg) != AWQ_OK) return 0;
  if (check_shape(T, in, out, cfg) != AWQ_OK) return 0;
  size_t need = scale_layout(T, in, out, cfg, cfg->n_alpha).end;
  if (cfg->n_clip > 0 && in % 128 == 0) {
    size_t c = clip_layout(T, in).end;
    if (c > need) need = c;
  }
  return need;
}

size_t awq_workspace_size_min(int64_t T, int64_t in, int64_t out, const awq_config *cfg) {
  g_err.clear();
  NvtxCall nvtx_call_(__func__);
  if (fault_mode() == Fault::kAlloc) {
    fail(AWQ_ERR_WORKSPACE, "injected allocation failure (AWQ_FAULT=alloc)");
    return 0;
  }
  if (check_cfg(cfg) != AWQ_OK) return 0;
  if (check_shape(T, in, out, cfg) != AWQ_OK) return 0;
  size_t need = scale_layout(T, in, out, cfg, 1).end;
  if (cfg->n_clip > 0 && in % 128 == 0) {
    size_t c = clip_layout(T, in).end;
    if (c > need) need = c;
  }
  return need;
}

awq_status awq_act_stats(const void *X, int64_t T, int64_t in, int64_t ldx, double *abar,
                         awq_stream_t stream) {
  g_err.clear();
  NvtxCall nvtx_call_(__func__);
  if (T < 1 || T > (int64_t(1) << 22)) return fail(AWQ_ERR_INVALID_ARG, "T=%lld (1..2^22)", (long long)T);
  if (in < 8 || in % 8 != 0) return fail(AWQ_ERR_INVALID_ARG, "in=%lld must be a multiple of 8", (long long)in);
  awq_status st = check_x(X, in, ldx);
  if (st != AWQ_OK) return st;
  if (!abar || !aligned(abar, 8)) return fail(AWQ_ERR_INVALID_ARG, "abar is NULL or misaligned");
  AWQ_LAUNCH_GATE();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  ProfScope p("act_stats", s);
  AWQ_TRY_CUDA(launch_act_stats(static_cast<const __half *>(X), T, in, ldx, abar,
                                num_sms_current(), s),
               "act_stats launch");
  return AWQ_OK;
}

awq_status awq_scale_grid(const double *abar, int64_t in, int32_t n_alpha, float *s,
                          awq_stream_t stream) {
  g_err.clear();
  NvtxCall nvtx_call_(__func__);
  if (!abar || !s) return fail(AWQ_ERR_INVALID_ARG, "abar or s is NULL");
  if (in < 1 || in > (int64_t(1) << 24)) return fail(AWQ_ERR_INVALID_ARG, "in=%lld", (long long)in);
  if (n_alpha < 1 || n_alpha > 64) return fail(AWQ_ERR_INVALID_ARG, "n_alpha=%d (1..64)", n_alpha);
  AWQ_LAUNCH_GATE();
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ProfScope p("scale_grid", st);
  AWQ_TRY_CUDA(launch_scale_grid(abar, in, n_alpha, s, nullptr, st), "scale_grid launch");
  return AWQ_OK;
}

namespace {
// The alpha search up to the candidate scores.  sse == NULL: MSE, best and
// s_best (awq_search_scale); otherwise the unnormalised sums of squared errors
// of these tokens into sse [n_alpha] (awq_search_scale_sse).
awq_status search_scale_impl(const void *X, int64_t T, int64_t in, int64_t ldx, const void *W,
                             int64_t out, const double *abar, const awq_config *cfg, void *ws,
                             size_t ws_bytes, float *s_best, double *mse, int32_t *best_idx,
                             double *sse, awq_stream_t stream) {
  awq_status st = check_cfg(cfg);
  if (st != AWQ_OK) return st;
  if ((st = check_shape(T, in, out, cfg)) != AWQ_OK) return st;
  if ((st = check_x(X, in, ldx)) != AWQ_OK) return st;
  if (!W || !aligned(W, 16)) return fail(AWQ_ERR_INVALID_ARG, "W is NULL or not 16-byte aligned");
  if (!abar || (!sse && (!s_best || !mse || !best_idx)))
    return fail(AWQ_ERR_INVALID_ARG, "an output pointer is NULL");
  if (in % (cfg->search_form == AWQ_SEARCH_GRAM ? 128 : 64) != 0)
    return fail(AWQ_ERR_UNSUPPORTED, "in=%lld: the %s search needs in %% %d == 0", (long long)in,
                cfg->search_form == AWQ_SEARCH_GRAM ? "Gram-form" : "direct",
                cfg->search_form == AWQ_SEARCH_GRAM ? 128 : 64);
  // the whole grid's candidates at once, or the largest chunk of them the
  // caller's workspace holds (the same results, the candidates in turn)
  ScaleWs L = scale_layout(T, in, out, cfg, cfg->n_alpha);
  int chunk = cfg->n_alpha;
  while (chunk > 1 && ws_bytes < L.end) L = scale_layout(T, in, out, cfg, --chunk);
  if ((st = check_ws(ws, ws_bytes, L.end)) != AWQ_OK) return st;
  const int64_t tiles = (int64_t)L.num_m * L.nb_per_alpha * cfg->n_alpha;
  if (tiles > INT32_MAX) return fail(AWQ_ERR_INVALID_ARG, "problem too large (%lld tiles)", (long long)tiles);
  AWQ_LAUNCH_GATE();

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t *base = static_cast<uint8_t *>(ws);
  DevStatus *dst = reinterpret_cast<DevStatus *>(base);
  float *s_grid = reinterpret_cast<float *>(base + L.s_grid);
  float *inv_s = reinterpret_cast<float *>(base + L.inv_s);
  __half *dW = reinterpret_cast<__half *>(base + L.dW);
  double *partials = reinterpret_cast<double *>(base + L.partials);
  const int nsm = num_sms_current();

  // status of this call only: flags, site, exponent and max |W| start at zero
  AWQ_TRY_CUDA(cudaMemsetAsync(dst, 0, sizeof(DevStatus), s), "workspace reset");
  const bool gram = cfg->search_form == AWQ_SEARCH_GRAM;
  const bool cached_y = cfg->search_form == AWQ_SEARCH_CACHED_Y;
  float *r = gram ? reinterpret_cast<float *>(base + L.r) : nullptr;
  __half *Y = cached_y ? reinterpret_cast<__half *>(base + L.Y) : nullptr;
  if (cached_y) {
    ProfScope p("ref_output", s);
    AWQ_TRY_CUDA(launch_ref_output(static_cast<const __half *>(X), T, in, ldx,
                                   static_cast<const __half *>(W), out, L.out_pad, Y, dst,
                                   poll_cap(), nsm, s),
                 "ref_output launch");
  }
  if (gram) {
    ProfScope p("gram_full", s);
    AWQ_TRY_CUDA(launch_gram_full(static_cast<const __half *>(X), T, in, ldx,
                                  reinterpret_cast<float *>(base + L.G), r,
                                  reinterpret_cast<__half *>(base + L.ghi),
                                  reinterpret_cast<__half *>(base + L.glo), dst, poll_cap(), s),
                 "gram_full launch");
  }
  if (!cached_y) {  // the candidate errors' power-of-two scaling
    ProfScope p("wmax", s);
    AWQ_TRY_CUDA(launch_wmax(static_cast<const __half *>(W), out * in, in, r, dst, nsm, s), "wmax launch");
  }
  {
    ProfScope p("scale_grid", s);
    AWQ_TRY_CUDA(launch_scale_grid(abar, in, cfg->n_alpha, s_grid, inv_s, s), "scale_grid launch");
  }
  if (cfg->search_form == AWQ_SEARCH_FUSED) {
    // every candidate's per-group parameters, then the GEMM that builds its
    // B tiles from them and the W rows (the operand is never stored)
    float2 *params = reinterpret_cast<float2 *>(base + L.dW);
    {
      ProfScope p("fused_params", s);
      AWQ_TRY_CUDA(launch_fused_params(static_cast<const __half *>(W), out, in, L.out_pad, s_grid,
                                       cfg->n_alpha, cfg->group_size, cfg->w_bit, cfg->zero_point, dst,
                                       params, s),
                   "fused_params launch");
    }
    ProfScope p("fused_gemm", s);
    AWQ_TRY_CUDA(launch_fused_search_gemm(static_cast<const __half *>(X), T, ldx,
                                          static_cast<const __half *>(W), out, in, L.out_pad,
                                          cfg->n_alpha, s_grid, inv_s, params, cfg->group_size,
                                          cfg->w_bit, partials, dst, poll_cap(), nsm, s),
                 "fused_search_gemm launch");
  }
  // the candidates in chunks of `chunk` (all at once with a full workspace):
  // each chunk's operand, then its scores into its slots of the partials
  for (int a0 = 0; cfg->search_form != AWQ_SEARCH_FUSED && a0 < cfg->n_alpha; a0 += chunk) {
    const int cnt = cfg->n_alpha - a0 < chunk ? cfg->n_alpha - a0 : chunk;
    double *part = partials + (size_t)a0 * L.per_alpha;
    {
      ProfScope p("cand_quant", s);
      AWQ_TRY_CUDA(launch_cand_quant(static_cast<const __half *>(W), out, in, L.out_pad,
                                     s_grid + (size_t)a0 * in, inv_s + (size_t)a0 * in, r, cnt,
                                     cfg->group_size, cfg->w_bit, cfg->zero_point, cached_y ? 1 : 0,
                                     dst, dW, nsm, s),
                   "cand_quant launch");
    }
    if (gram) {
      ProfScope p("gram_score", s);
      AWQ_TRY_CUDA(launch_gram_score(dW, (int64_t)cnt * L.out_pad, in,
                                     reinterpret_cast<const __half *>(base + L.ghi),
                                     reinterpret_cast<const __half *>(base + L.glo), part, dst,
                                     poll_cap(), nsm, s),
                   "gram_score launch");
    } else {
      SearchGemmShape sh;
      sh.T = T;
      sh.in = in;
      sh.rows_b = (int64_t)cnt * L.out_pad;
      sh.num_m = L.num_m;
      sh.num_n = (int)(sh.rows_b / kGemmBN);
      sh.num_kb = (int)(in / kGemmBK);
      ProfScope p("search_gemm", s);
      AWQ_TRY_CUDA(launch_search_gemm(static_cast<const __half *>(X), ldx, dW, sh, part, Y,
                                      L.out_pad, dst, poll_cap(), nsm, s),
                   "search_gemm launch");
    }
  }
  {
    ProfScope p("mse_argmin", s);
    // AWQ_FAULT=nonfinite: normalising by zero tokens makes every score non-finite
    const int64_t t_norm = fault_mode() == Fault::kNonFinite ? 0 : (sse ? 1 : T);
    if (sse)  // T = out = 1: the plain sums of squared errors
      AWQ_TRY_CUDA(launch_mse_argmin(partials, cfg->n_alpha, L.per_alpha, t_norm, 1, s_grid, in, dst,
                                     sse, nullptr, nullptr, s),
                   "mse_argmin launch");
    else
      AWQ_TRY_CUDA(launch_mse_argmin(partials, cfg->n_alpha, L.per_alpha, t_norm, out, s_grid, in,
                                     dst, mse, best_idx, s_best, s),
                   "mse_argmin launch");
  }
  if (getenv("AWQ_SYNC_CHECK")) return awq_device_status(ws, stream);
  return AWQ_OK;
}
}  // namespace

awq_status awq_search_scale(const void *X, int64_t T, int64_t in, int64_t ldx, const void *W,
                            int64_t out, const double *abar, const awq_config *cfg, void *ws,
                            size_t ws_bytes, float *s_best, double *mse, int32_t *best_idx,
                            awq_stream_t stream) {
  g_err.clear();
  NvtxCall nvtx_call_(__func__);
  return search_scale_impl(X, T, in, ldx, W, out, abar, cfg, ws, ws_bytes, s_best, mse, best_idx,
                           nullptr, stream);
}

awq_status awq_search_scale_sse(const void *X, int64_t T, int64_t in, int64_t ldx, const void *W,
                                int64_t out, const double *abar, const awq_config *cfg, void *ws,
                                size_t ws_bytes, double *sse, awq_stream_t stream) {
  g_err.clear();
  NvtxCall nvtx_call_(__func__);
  if (!sse) return fail(AWQ_ERR_INVALID_ARG, "sse is NULL");
  return search_scale_impl(X, T, in, ldx, W, out, abar, cfg, ws, ws_bytes, nullptr, nullptr, nullptr,
                           sse, stream);
}

awq_status awq_select_scale(const double *sse, int64_t T_total, int64_t in, int64_t out,
                            const double *abar, const awq_config *cfg, void *ws, size_t ws_bytes,
                            float *s_best, double *mse, int32_t *best_idx, awq_stream_t stream) {
  g_err.clear();
  NvtxCall nvtx_call_(__func__);
  awq_status st = check_cfg(cfg);
  if (st != AWQ_OK) return st;
  if ((st = check_shape(T_total, in, out, cfg)) != AWQ_OK) return st;
  if (!sse || !abar || !s_best || !mse || !best_idx)
    return fail(AWQ_ERR_INVALID_ARG, "a pointer argument is NULL");
  if ((st = check_ws(ws, ws_bytes, kHeader)) != AWQ_OK) return st;
  AWQ_LAUNCH_GATE();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DevStatus *dst = static_cast<DevStatus *>(ws);
  AWQ_TRY_CUDA(cudaMemsetAsync(dst, 0, sizeof(DevStatus), s), "workspace reset");
  ProfScope p("select_scale", s);
  const int64_t t_norm = fault_mode() == Fault::kNonFinite ? 0 : T_total;  // see Fault
  AWQ_TRY_CUDA(launch_select_scale(sse, cfg->n_alpha, t_norm, out, abar, in, dst, mse, best_idx,
                                   s_best, s),
               "select_scale launch");
  return AWQ_OK;
}

awq_status awq_act_sums(const void *X, int64_t T, int64_t in, int64_t ldx, int64_t *sums,
                        awq_stream_t stream) {
  g_err.clear();
  NvtxCall nvtx_call_(__func__);
  if (T < 1 || T > (int64_t(1) << 22)) return fail(AWQ_ERR_INVALID_ARG, "T=%lld (1..2^22)", (long long)T);
  if (in < 8 || in % 8 != 0) return fail(AWQ_ERR_INVALID_ARG, "in=%lld must be a multiple of 8", (long long)in);
  awq_status st = check_x(X, in, ldx);
  if (st != AWQ_OK) return st;
  if (!sums || !aligned(sums, 8)) return fail(AWQ_ERR_INVALID_ARG, "sums is NULL or misaligned");
  AWQ_LAUNCH_GATE();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  ProfScope p("act_stats", s);
  AWQ_TRY_CUDA(launch_act_sums(static_cast<const __half *>(X), T, in, ldx, sums, num_sms_current(), s),
               "act_sums launch");
  return AWQ_OK;
}

awq_status awq_act_stats_finish(const int64_t *sums, int64_t T_total, int64_t in, double *abar,
                                awq_stream_t stream) {
  g_err.clear();
  NvtxCall nvtx_call_(__func__);
  if (T_total < 1 || T_total > (int64_t(1) << 22))
    return fail(AWQ_ERR_INVALID_ARG, "T_total=%lld (1..2^22)", (long long)T_total);
  if (in < 1) return fail(AWQ_ERR_INVALID_ARG, "in=%lld", (long long)in);
  if (!sums || !abar) return fail(AWQ_ERR_INVALID_ARG, "sums or abar is NULL");
  AWQ_LAUNCH_GATE();
  AWQ_TRY_CUDA(launch_act_finish(sums, in, T_total, abar, static_cast<cudaStream_t>(stream)),
               "act_finish launch");
  return AWQ_OK;
}

awq_status awq_search_clip(const void *X, int64_t T, int64_t in, int64_t ldx, const void *W,
                           int64_t out, const float *s, const awq_config *cfg, void *ws,
                           size_t ws_bytes, uint8_t *clip_idx, float *err, awq_stream_t stream) {
  g_err.clear();
  NvtxCall nvtx_call_(__func__);
  awq_status st = check_cfg(cfg);
  if (st != AWQ_OK) return st;
  if (cfg->n_clip < 1) return fail(AWQ_ERR_INVALID_ARG, "n_clip=%d: clip search needs n_clip >= 1", cfg->n_clip);
  if ((st = check_shape(T, in, out, cfg)) != AWQ_OK) return st;
  if ((st = check_clip_in(in)) != AWQ_OK) return st;
  if ((st = check_x(X, in, ldx)) != AWQ_OK) return st;
  if (!W || !aligned(W, 16)) return fail(AWQ_ERR_INVALID_ARG, "W is NULL or not 16-byte aligned");
  if (!clip_idx) return fail(AWQ_ERR_INVALID_ARG, "clip_idx is NULL");
  if (s && !aligned(s, 16)) return fail(AWQ_ERR_INVALID_ARG, "s must be 16-byte aligned");
  const ClipWs L = clip_layout(T, in);
  if ((st = check_ws(ws, ws_bytes, L.end)) != AWQ_OK) return st;
  AWQ_LAUNCH_GATE();
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t *base = static_cast<uint8_t *>(ws);
  float *gpart = reinterpret_cast<float *>(base + L.gpart);
  float *Gk = reinterpret_cast<float *>(base + L.G);
  AWQ_TRY_CUDA(cudaMemsetAsync(base, 0, sizeof(DevStatus), cs), "workspace reset");
  {
    ProfScope p("gram_blocks", cs);
    AWQ_TRY_CUDA(launch_gram_blocks(static_cast<const __half *>(X), T, in, ldx, cfg->group_size,
                                    L.n_chunks, gpart, Gk, reinterpret_cast<DevStatus *>(base),
                                    poll_cap(), cs),
                 "gram_blocks launch");
  }
  {
    ProfScope p("clip_eval", cs);
    AWQ_TRY_CUDA(launch_clip_eval(static_cast<const __half *>(W), out, in, s, Gk, cfg->group_size,
                                  cfg->w_bit, cfg->zero_point, cfg->n_clip, cfg->clip_min, clip_idx, err,
                                  reinterpret_cast<DevStatus *>(base), poll_cap(),
                                  num_sms_current(), cs),
                 "clip_eval launch");
  }
  return AWQ_OK;
}

awq_status awq_block_grams(const void *X, int64_t T, int64_t in, int64_t ldx, const awq_config *cfg,
                           void *ws, size_t ws_bytes, float *G, awq_stream_t stream) {
  g_err.clear();
  NvtxCall nvtx_call_(__func__);
  awq_status st = check_cfg(cfg);
  if (st != AWQ_OK) return st;
  if (T < 1 || T > (int64_t(1) << 22)) return fail(AWQ_ERR_INVALID_ARG, "T=%lld (1..2^22)", (long long)T);
  if (in < 128 || in % 128 != 0 || in > (int64_t(1) << 20))
    return fail(AWQ_ERR_INVALID_ARG, "in=%lld must be a positive multiple of 128", (long long)in);
  if ((st = check_x(X, in, ldx)) != AWQ_OK) return st;
  if (!G || !aligned(G, 16)) return fail(AWQ_ERR_INVALID_ARG, "G is NULL or not 16-byte aligned");
  const ClipWs L = clip_layout(T, in);
  if ((st = check_ws(ws, ws_bytes, L.end)) != AWQ_OK) return st;
  AWQ_LAUNCH_GATE();
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t *base = static_cast<uint8_t *>(ws);
  AWQ_TRY_CUDA(cudaMemsetAsync(base, 0, sizeof(DevStatus), cs), "workspace reset");
  ProfScope p("gram_blocks", cs);
  AWQ_TRY_CUDA(launch_gram_blocks(static_cast<const __half *>(X), T, in, ldx, cfg->group_size,
                                  L.n_chunks, reinterpret_cast<float *>(base + L.gpart), G,
                                  reinterpret_cast<DevStatus *>(base), poll_cap(), cs),
               "gram_blocks launch");
  return AWQ_OK;
}

awq_status awq_search_clip_grams(const void *W, int64_t out, int64_t in, const float *s,
                                 const float *G, const awq_config *cfg, void *ws, size_t ws_bytes,
                                 uint8_t *clip_idx, float *err, awq_stream_t stream) {
  g_err.clear();
  NvtxCall nvtx_call_(__func__);
  awq_status st = check_cfg(cfg);
  if (st != AWQ_OK) return st;
  if (cfg->n_clip < 1) return fail(AWQ_ERR_INVALID_ARG, "n_clip=%d: clip search needs n_clip >= 1", cfg->n_clip);
  if ((st = check_shape(1, in, out, cfg)) != AWQ_OK) return st;
  if ((st = check_clip_in(in)) != AWQ_OK) return st;
  if (!W || !aligned(W, 16)) return fail(AWQ_ERR_INVALID_ARG, "W is NULL or not 16-byte aligned");
  if (!G || !aligned(G, 16)) return fail(AWQ_ERR_INVALID_ARG, "G is NULL or not 16-byte aligned");
  if (!clip_idx) return fail(AWQ_ERR_INVALID_ARG, "clip_idx is NULL");
  if (s && !aligned(s, 16)) return fail(AWQ_ERR_INVALID_ARG, "s must be 16-byte aligned");
  if ((st = check_ws(ws, ws_bytes, kHeader)) != AWQ_OK) return st;
  AWQ_LAUNCH_GATE();
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t *base = static_cast<uint8_t *>(ws);
  AWQ_TRY_CUDA(cudaMemsetAsync(base, 0, sizeof(DevStatus), cs), "workspace reset");
  ProfScope p("clip_eval", cs);
  AWQ_TRY_CUDA(launch_clip_eval(static_cast<const __half *>(W), out, in, s, G, cfg->group_size,
                                cfg->w_bit, cfg->zero_point, cfg->n_clip, cfg->clip_min, clip_idx, err,
                                reinterpret_cast<DevStatus *>(base), poll_cap(), num_sms_current(), cs),
               "clip_eval launch");
  return AWQ_OK;
}

awq_status awq_candidate_codes(const void *W, int64_t out, int64_t in, const double *abar,
                               const awq_config *cfg, void *ws, size_t ws_bytes, uint8_t *q,
                               uint8_t *z, float *delta, awq_stream_t stream) {
  g_err.clear();
  NvtxCall nvtx_call_(__func__);
  awq_status st = check_cfg(cfg);
  if (st != AWQ_OK) return st;
  if ((st = check_shape(1, in, out, cfg)) != AWQ_OK) return st;
  if (in % 64 != 0) return fail(AWQ_ERR_UNSUPPORTED, "in=%lld: needs in %% 64 == 0", (long long)in);
  if (!W || !aligned(W, 16)) return fail(AWQ_ERR_INVALID_ARG, "W is NULL or not 16-byte aligned");
  if (!abar || !q || !z || !delta) return fail(AWQ_ERR_INVALID_ARG, "a pointer argument is NULL");
  if (!aligned(q, 8)) return fail(AWQ_ERR_INVALID_ARG, "q must be 8-byte aligned");
  // the s grid and 1/s as the direct-form search lays them out
  awq_config c = *cfg;
  c.search_form = AWQ_SEARCH_DIRECT;
  const ScaleWs L = scale_layout(1, in, out, &c, c.n_alpha);
  if ((st = check_ws(ws, ws_bytes, L.dW)) != AWQ_OK) return st;
  AWQ_LAUNCH_GATE();
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t *base = static_cast<uint8_t *>(ws);
  DevStatus *dst = reinterpret_cast<DevStatus *>(base);
  float *s_grid = reinterpret_cast<float *>(base + L.s_grid);
  float *inv_s = reinterpret_cast<float *>(base + L.inv_s);
  const int nsm = num_sms_current();
  AWQ_TRY_CUDA(cudaMemsetAsync(dst, 0, sizeof(DevStatus), cs), "workspace reset");
  AWQ_TRY_CUDA(launch_wmax(static_cast<const __half *>(W), out * in, in, nullptr, dst, nsm, cs),
               "wmax launch");
  AWQ_TRY_CUDA(launch_scale_grid(abar, in, cfg->n_alpha, s_grid, inv_s, cs), "scale_grid launch");
  ProfScope p("cand_codes", cs);
  AWQ_TRY_CUDA(launch_cand_codes(static_cast<const __half *>(W), out, in, L.out_pad,
                                 s_grid, inv_s, cfg->n_alpha, cfg->group_size, cfg->w_bit,
                                 cfg->zero_point, dst, q, z, delta, cs),
               "cand_codes launch");
  return AWQ_OK;
}

awq_status awq_clip_candidate_codes(const void *W, int64_t out, int64_t in, const float *s,
                                    const float *G, const awq_config *cfg, void *ws,
                                    size_t ws_bytes, uint8_t *clip_idx, float *err, uint8_t *q,
                                    uint8_t *z, awq_stream_t stream) {
  g_err.clear();
  NvtxCall nvtx_call_(__func__);
  awq_status st = check_cfg(cfg);
  if (st != AWQ_OK) return st;
  if (cfg->n_clip < 1) return fail(AWQ_ERR_INVALID_ARG, "n_clip=%d: clip search needs n_clip >= 1", cfg->n_clip);
  if ((st = check_shape(1, in, out, cfg)) != AWQ_OK) return st;
  if ((st = check_clip_in(in)) != AWQ_OK) return st;
  if (!W || !aligned(W, 16)) return fail(AWQ_ERR_INVALID_ARG, "W is NULL or not 16-byte aligned");
  if (!G || !aligned(G, 16)) return fail(AWQ_ERR_INVALID_ARG, "G is NULL or not 16-byte aligned");
  if (!clip_idx || !q || !z) return fail(AWQ_ERR_INVALID_ARG, "clip_idx, q or z is NULL");
  if (!aligned(q, 8)) return fail(AWQ_ERR_INVALID_ARG, "q must be 8-byte aligned");
  if (s && !aligned(s, 16)) return fail(AWQ_ERR_INVALID_ARG, "s must be 16-byte aligned");
  if ((st = check_ws(ws, ws_bytes, kHeader)) != AWQ_OK) return st;
  AWQ_LAUNCH_GATE();
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t *base = static_cast<uint8_t *>(ws);
  AWQ_TRY_CUDA(cudaMemsetAsync(base, 0, sizeof(DevStatus), cs), "workspace reset");
  ProfScope p("clip_eval", cs);
  AWQ_TRY_CUDA(launch_clip_eval(static_cast<const __half *>(W), out, in, s, G, cfg->group_size,
                                cfg->w_bit, cfg->zero_point, cfg->n_clip, cfg->clip_min, clip_idx, err,
                                reinterpret_cast<DevStatus *>(base), poll_cap(), num_sms_current(), cs,
                                q, z),
               "clip_eval launch");
  return AWQ_OK;
}

awq_status awq_quant_pack(const void *W, int64_t out, int64_t in, const float *s,
                          const uint8_t *clip_idx, const awq_config *cfg, int32_t *qweight,
                          int32_t *qzeros, void *scales, awq_stream_t stream) {
  g_err.clear();
  NvtxCall nvtx_call_(__func__);
  awq_status st = check_cfg(cfg);
  if (st != AWQ_OK) return st;
  if ((st = check_shape(1, in, out, cfg)) != AWQ_OK) return st;
  if (!W || !aligned(W, 16)) return fail(AWQ_ERR_INVALID_ARG, "W is NULL or not 16-byte aligned");
  if (s && !aligned(s, 16)) return fail(AWQ_ERR_INVALID_ARG, "s must be 16-byte aligned");
  if (clip_idx && cfg->n_clip < 1)
    return fail(AWQ_ERR_INVALID_ARG, "clip_idx given but n_clip=%d", cfg->n_clip);
  if (!qweight || !qzeros || !scales) return fail(AWQ_ERR_INVALID_ARG, "an output pointer is NULL");
  AWQ_LAUNCH_GATE();
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  ProfScope p("quant_pack", cs);
  AWQ_TRY_CUDA(launch_quant_pack(static_cast<const __half *>(W), out, in, s, clip_idx,
                                 cfg->group_size, cfg->w_bit, cfg->zero_point, cfg->n_clip,
                                 cfg->clip_min, qweight,
                                 qzeros, static_cast<__half *>(scales), cs),
               "quant_pack launch");
  if (getenv("AWQ_SYNC_CHECK")) return awq_device_status(nullptr, stream);
  return AWQ_OK;
}

awq_status awq_w4a16_gemm(const void *X, int64_t T, int64_t in, int64_t ldx, const int32_t *qweight,
                          const int32_t *qzeros, const void *scales, int64_t out,
                          const awq_config *cfg, void *Y, int64_t ldy, void *ws, size_t ws_bytes,
                          awq_stream_t stream) {
  g_err.clear();
  NvtxCall nvtx_call_(__func__);
  awq_status st = check_cfg(cfg);
  if (st != AWQ_OK) return st;
  if ((st = check_shape(T, in, out, cfg)) != AWQ_OK) return st;
  if (in % 64 != 0 || out % 32 != 0)
    return fail(AWQ_ERR_UNSUPPORTED, "in=%lld, out=%lld: the W4A16 GEMM needs in %% 64 == 0 and out %% 32 == 0",
                (long long)in, (long long)out);
  if ((st = check_x(X, in, ldx)) != AWQ_OK) return st;
  if (!qweight || !qzeros || !scales || !aligned(qweight, 16) || !aligned(qzeros, 16) || !aligned(scales, 16))
    return fail(AWQ_ERR_INVALID_ARG, "qweight, qzeros and scales must be non-NULL and 16-byte aligned");
  if (!Y || !aligned(Y, 16)) return fail(AWQ_ERR_INVALID_ARG, "Y is NULL or not 16-byte aligned");
  if (ldy < out || ldy % 8 != 0)
    return fail(AWQ_ERR_INVALID_ARG, "ldy=%lld must be >= out and a multiple of 8", (long long)ldy);
  if ((st = check_ws(ws, ws_bytes, kHeader)) != AWQ_OK) return st;
  AWQ_LAUNCH_GATE();
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  DevStatus *dst = static_cast<DevStatus *>(ws);
  AWQ_TRY_CUDA(cudaMemsetAsync(dst, 0, sizeof(DevStatus), cs), "workspace reset");
  // many tokens, with room for the fp16 weights: dequantise once, one fp16 GEMM
  if (T >= kW4DequantMinT && ws_bytes >= w4a16_dequant_ws_bytes(in, out)) {
    __half *Wd = reinterpret_cast<__half *>(static_cast<uint8_t *>(ws) + kHeader);
    {
      ProfScope p("w4a16_dequant", cs);
      AWQ_TRY_CUDA(launch_w4a16_dequant(qweight, qzeros, static_cast<const __half *>(scales), in, out,
                                        cfg->group_size, Wd, cs),
                   "w4a16_dequant launch");
    }
    ProfScope p("w4a16_gemm", cs);
    AWQ_TRY_CUDA(launch_gemm_store(static_cast<const __half *>(X), T, in, ldx, Wd, out,
                                   static_cast<__half *>(Y), ldy, dst, poll_cap(), num_sms_current(), cs),
                 "w4a16 fp16 GEMM launch");
    return AWQ_OK;
  }
  // a few tokens (decode): the product streams the packed words on CUDA cores,
  // split along K when the workspace holds the fp32 partial sums
  if (T <= kW4GemvMaxT) {
    const int nsm = num_sms_current();
    const int gsplits = w4a16_gemv_splits(T, in, out, nsm);
    float *gpart = gsplits > 1 && ws_bytes >= w4a16_ws_bytes(T, out, gsplits)
                       ? reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + kHeader)
                       : nullptr;
    ProfScope p("w4a16_gemv", cs);
    AWQ_TRY_CUDA(launch_w4a16_gemv(static_cast<const __half *>(X), T, in, ldx, qweight, qzeros,
                                   static_cast<const __half *>(scales), out, cfg->group_size,
                                   static_cast<__half *>(Y), ldy, gpart, nsm, cs),
                 "w4a16_gemv launch");
    return AWQ_OK;
  }
  // split-K for few tokens, when the workspace holds the fp32 partial sums
  int splits = w4a16_splits(T, in, out, num_sms_current());
  if (splits > 1 && ws_bytes < w4a16_ws_bytes(T, out, splits)) splits = 1;
  float *partials = splits > 1 ? reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + kHeader) : nullptr;
  ProfScope p("w4a16_gemm", cs);
  AWQ_TRY_CUDA(launch_w4a16_gemm(static_cast<const __half *>(X), T, in, ldx, qweight, qzeros,
                                 static_cast<const __half *>(scales), out, cfg->group_size,
                                 static_cast<__half *>(Y), ldy, partials, splits, dst, poll_cap(),
                                 num_sms_current(), cs),
               "w4a16_gemm launch");
  return AWQ_OK;
}

size_t awq_w4a16_workspace_size(int64_t T, int64_t in, int64_t out, const awq_config *cfg) {
  g_err.clear();
  NvtxCall nvtx_call_(__func__);
  if (fault_mode() == Fault::kAlloc) {
    fail(AWQ_ERR_WORKSPACE, "injected allocation failure (AWQ_FAULT=alloc)");
    return 0;
  }
  if (check_cfg(cfg) != AWQ_OK) return 0;
  if (check_shape(T, in, out, cfg) != AWQ_OK) return 0;
  if (T >= kW4DequantMinT) return w4a16_dequant_ws_bytes(in, out);
  if (T <= kW4GemvMaxT) {
    const int gsplits = w4a16_gemv_splits(T, in, out, num_sms_current());
    return gsplits > 1 ? w4a16_ws_bytes(T, out, gsplits) : kHeader;
  }
  const int splits = w4a16_splits(T, in, out, num_sms_current());
  return splits > 1 ? w4a16_ws_bytes(T, out, splits) : kHeader;
}

awq_status awq_fold_inv_scale(void *v, int64_t rows, int64_t cols, const float *s,
                              awq_stream_t stream) {
  g_err.clear();
  NvtxCall nvtx_call_(__func__);
  if (!v || !s) return fail(AWQ_ERR_INVALID_ARG, "v or s is NULL");
  if (rows < 1 || cols < 1) return fail(AWQ_ERR_INVALID_ARG, "rows=%lld cols=%lld", (long long)rows, (long long)cols);
  AWQ_LAUNCH_GATE();
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  ProfScope p("fold", cs);
  AWQ_TRY_CUDA(launch_fold(static_cast<__half *>(v), rows, cols, s, cs), "fold launch");
  return AWQ_OK;
}

awq_status awq_device_status(void *ws, awq_stream_t stream) {
  g_err.clear();
  NvtxCall nvtx_call_(__func__);
  if (ws && !aligned(ws, 256)) return fail(AWQ_ERR_WORKSPACE, "workspace is misaligned");
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  AWQ_TRY_CUDA(cudaStreamSynchronize(cs), "stream synchronize");
  DevStatus h;
  if (ws) {
    AWQ_TRY_CUDA(cudaMemcpy(&h, ws, sizeof(h), cudaMemcpyDeviceToHost), "status read");
    const uint32_t zero[2] = {0, 0};
    AWQ_TRY_CUDA(cudaMemcpy(ws, zero, sizeof(zero), cudaMemcpyHostToDevice), "status clear");
  } else {  // the library's own word, used by the calls that take no workspace
    AWQ_TRY_CUDA(lib_status_read_clear(&h), "library status read");
  }
  if (h.flags & kDevTimeout)
    return fail(AWQ_ERR_TIMEOUT, "a bounded device wait ran out (site 0x%x)", h.where);
  if (h.flags & kDevNonFinite) return fail(AWQ_ERR_NONFINITE, "a candidate score is not finite");
  if (h.flags & kDevBadIndex)
    return fail(AWQ_ERR_INVALID_ARG,
                "awq_quant_pack was given a clip index >= n_clip (those groups got a NaN scale)");
  return AWQ_OK;
}

int32_t awq_bounds_checks_enabled(void) {
#ifdef AWQ_DEBUG_BOUNDS
  return 1;
#else
  return 0;
#endif
}

awq_status awq_bounds_status(void) {
  g_err.clear();
  NvtxCall nvtx_call_(__func__);
#ifdef AWQ_DEBUG_BOUNDS
  AWQ_TRY_CUDA(cudaDeviceSynchronize(), "device synchronize");
  struct Unit {
    const char *name;
    cudaError_t (*read)(DevStatus *);
  };
  const Unit units[] = {{"quant_kernels", bounds_status_quant}, {"search_gemm", bounds_status_gemm},
                        {"clip_kernels", bounds_status_clip}, {"gram_search", bounds_status_gram},
                        {"w4a16_gemm", bounds_status_w4a16}, {"fused_search", bounds_status_fused}};
  const char *bad = nullptr;
  uint32_t site = 0;
  for (const Unit &u : units) {
    DevStatus h;
    AWQ_TRY_CUDA(u.read(&h), "bounds word read");
    if ((h.flags & kDevOutOfBounds) && !bad) {
      bad = u.name;
      site = h.where;
    }
  }
  if (bad) return fail(AWQ_ERR_INVALID_ARG, "an index check failed in %s (site 0x%x)", bad, site);
#endif
  return AWQ_OK;
}

awq_status awq_profile_enable(int32_t on) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = on != 0;
  return AWQ_OK;
}

awq_status awq_profile_read(const char *name, double *total_ms, int64_t *launches) {
  g_err.clear();
  NvtxCall nvtx_call_(__func__);
  if (!name || !total_ms || !launches) return fail(AWQ_ERR_INVALID_ARG, "NULL argument");
  std::lock_guard<std::mutex> lk(g_prof_mu);
  double tot = 0.0;
  int64_t n = 0;
  for (const ProfRec &r : g_prof) {
    if (strcmp(r.name, name) != 0) continue;
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e != cudaSuccess) return cuda_fail(e, "event synchronize");
    float ms = 0.0f;
    e = cudaEventElapsedTime(&ms, r.a, r.b);
    if (e != cudaSuccess) return cuda_fail(e, "event elapsed time");
    tot += ms;
    ++n;
  }
  *total_ms = tot;
  *launches = n;
  return AWQ_OK;
}

awq_status awq_profile_reset(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (const ProfRec &r : g_prof) {
    cudaEventSynchronize(r.b);
    g_ev_pool.push_back(r.a);
    g_ev_pool.push_back(r.b);
  }
  g_prof.clear();
  return AWQ_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free clip search.
//
// Some callers cannot allocate device memory while they run this search: a
// host framework that owns every device byte through its own pre-planned
// arena (and forbids stray cudaMalloc calls that would fragment it or
// overlap its budget), or code that must not call cudaMalloc because that
// call can synchronise the whole device in the middle of its pipelined
// stream work.  awq_search_clip_noalloc takes no workspace: its block-Gram
// scratch lives in the file-scope device array below, which holds 384 blocks
// of 128 x 128 fp32 (24 MiB): the Grams of up to kNoAllocMaxIn / 128 groups
// plus the per-chunk partials of as many token chunks as the rest holds.
// The array is part of this library's module, so every GPU that loads the
// library holds it until the process exits.  Device-side failures go to the
// library's status word (the one awq_quant_pack uses), read with
// awq_device_status(NULL, stream).
// ---------------------------------------------------------------------------
namespace {
constexpr int64_t kNoAllocMaxIn = 16384;  // up to 128 groups of 128 channels
constexpr int64_t kNoAllocBlocks = 384;   // 128 x 128 fp32 blocks in the array
constexpr size_t kNoAllocGroupFloats = 128 * 128;
constexpr size_t kNoAllocFloats = (size_t)kNoAllocBlocks * kNoAllocGroupFloats;

struct NoAllocDev {
  float *scratch;
  DevStatus *status;
};
std::mutex g_noalloc_mu;
NoAllocDev g_noalloc_dev[64] = {};
}  // namespace

static __device__ __align__(256) float g_noalloc_scratch[kNoAllocFloats];

extern "C" awq_status awq_search_clip_noalloc(const void *X, int64_t T, int64_t in, int64_t ldx,
                                              const void *W, int64_t out, const float *s,
                                              const awq_config *cfg, uint8_t *clip_idx, float *err,
                                              awq_stream_t stream) {
  g_err.clear();
  NvtxCall nvtx_call_(__func__);
  awq_status st = check_cfg(cfg);
  if (st != AWQ_OK) return st;
  if (cfg->n_clip < 1) return fail(AWQ_ERR_INVALID_ARG, "n_clip=%d: clip search needs n_clip >= 1", cfg->n_clip);
  if ((st = check_shape(T, in, out, cfg)) != AWQ_OK) return st;
  if ((st = check_clip_in(in)) != AWQ_OK) return st;
  if (in > kNoAllocMaxIn)
    return fail(AWQ_ERR_INVALID_ARG,
                "in=%lld exceeds the %lld input channels the allocation-free clip search's "
                "static scratch holds; use awq_search_clip with a workspace",
                (long long)in, (long long)kNoAllocMaxIn);
  if ((st = check_x(X, in, ldx)) != AWQ_OK) return st;
  if (!W || !aligned(W, 16)) return fail(AWQ_ERR_INVALID_ARG, "W is NULL or not 16-byte aligned");
  if (!clip_idx) return fail(AWQ_ERR_INVALID_ARG, "clip_idx is NULL");
  if (s && !aligned(s, 16)) return fail(AWQ_ERR_INVALID_ARG, "s must be 16-byte aligned");
  AWQ_LAUNCH_GATE();

  // Device addresses of the static scratch and of the status word, looked up
  // once per device with that device current (the host-side symbols are not
  // device addresses).
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(AWQ_ERR_UNSUPPORTED, "device ordinal %d", dev);
  NoAllocDev nd;
  {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_dev[dev].scratch) {
      void *p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static clip scratch)");
      DevStatus *sp = nullptr;
      e = lib_status_address(&sp);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(library status word)");
      g_noalloc_dev[dev].status = sp;
      g_noalloc_dev[dev].scratch = static_cast<float *>(p);
    }
    nd = g_noalloc_dev[dev];
  }

  // Token chunks of the block-Gram partials: as many as the workspace form
  // uses (up to 16, one per 1024 tokens) while chunks + 1 sets of the layer's
  // group blocks fit in the array.  Every scratch element a call reads is
  // written earlier in the same call when no wait runs out (all chunk
  // partials of the groups in use, then their sums); after a timeout the
  // status word says so and clip_idx is not to be used.
  const int64_t groups = in / 128;
  const int64_t fit = kNoAllocBlocks / groups - 1;  // >= 2 for in <= kNoAllocMaxIn
  int64_t c = (T + 1023) / 1024;
  if (c > 16) c = 16;
  if (c > fit) c = fit;
  const int n_chunks = (int)(c < 1 ? 1 : c);
  const size_t gsz = (size_t)groups * kNoAllocGroupFloats;
  float *gpart = nd.scratch;
  float *Gk = nd.scratch + gsz * (size_t)n_chunks;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  {
    ProfScope p("gram_blocks", cs);
    e = launch_gram_blocks(static_cast<const __half *>(X), T, in, ldx, cfg->group_size, n_chunks,
                           gpart, Gk, nd.status, poll_cap(), cs);
    if (e != cudaSuccess) return cuda_fail(e, "gram_blocks launch");
  }
  {
    ProfScope p("clip_eval", cs);
    e = launch_clip_eval(static_cast<const __half *>(W), out, in, s, Gk, cfg->group_size, cfg->w_bit,
                         cfg->zero_point, cfg->n_clip, cfg->clip_min, clip_idx, err, nd.status,
                         poll_cap(), num_sms_current(), cs);
    if (e != cudaSuccess) return cuda_fail(e, "clip_eval launch");
  }
  if (getenv("AWQ_SYNC_CHECK")) return awq_device_status(nullptr, stream);
  return AWQ_OK;
}
