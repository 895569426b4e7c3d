/* The four calls of the C ABI (include/awq.h) from plain C, with no Python or
 * PyTorch: a seeded synthetic layer X [T, in] fp16, W [out, in] fp16 is made
 * on the host, copied to the device with the CUDA runtime, and quantised
 * (activation statistic, alpha search, clip search, packing); the packed
 * output and the selected alpha are written to a binary file so that a test
 * compares them with the same calls made through the Python binding.
 *
 *   quantize_layer OUT.bin [T in out]
 *   quantize_layer --inputs OUT.bin [T in out]   (only X and W; no GPU needed)
 *
 * Values: x = (u - 0.5) * c_j with u from a 64-bit LCG and c_j = 1, except
 * every 50th channel scaled by 20 (salient channels); w = (u - 0.5) / 16.
 * fp16 conversion: round to nearest even, written out below. */
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "awq.h"

static uint64_t lcg_state;

static double lcg_uniform(void) {
  lcg_state = lcg_state * 6364136223846793005ULL + 1442695040888963407ULL;
  return (double)(lcg_state >> 11) * (1.0 / 9007199254740992.0); /* [0, 1) */
}

/* float -> IEEE binary16, round to nearest even (normal and subnormal halves;
 * the values used here are far from overflow) */
static uint16_t to_half(float f) {
  uint32_t x;
  memcpy(&x, &f, 4);
  const uint32_t sign = (x >> 16) & 0x8000u;
  const uint32_t ax = x & 0x7FFFFFFFu;
  if (ax >= 0x47800000u) return (uint16_t)(sign | 0x7C00u); /* >= 65536: inf */
  if (ax < 0x38800000u) { /* below 2^-14: a subnormal half (or zero) */
    float a;
    memcpy(&a, &ax, 4);
    /* the subnormal grid step is 2^-24: round a * 2^24 to nearest even */
    const float scaled = a * 16777216.0f;
    uint32_t q = (uint32_t)scaled;
    const float rem = scaled - (float)q;
    if (rem > 0.5f || (rem == 0.5f && (q & 1u))) ++q;
    return (uint16_t)(sign | q);
  }
  /* normal: keep 10 mantissa bits, round on the 13 dropped ones */
  uint32_t h = ((ax - 0x38000000u) >> 13); /* rebias exponent 127 -> 15 */
  const uint32_t dropped = ax & 0x1FFFu;
  if (dropped > 0x1000u || (dropped == 0x1000u && (h & 1u))) ++h;
  return (uint16_t)(sign | h);
}

#define CHECK(call)                                                                   \
  do {                                                                                \
    awq_status st_ = (call);                                                          \
    if (st_ != AWQ_OK) {                                                              \
      fprintf(stderr, "%s failed: %d %s\n", #call, (int)st_, awq_last_error());       \
      return 1;                                                                       \
    }                                                                                 \
  } while (0)

#define CUDA(call)                                                                    \
  do {                                                                                \
    cudaError_t e_ = (call);                                                          \
    if (e_ != cudaSuccess) {                                                          \
      fprintf(stderr, "%s failed: %s\n", #call, cudaGetErrorString(e_));              \
      return 1;                                                                       \
    }                                                                                 \
  } while (0)

int main(int argc, char **argv) {
  const int inputs_only = argc > 1 && strcmp(argv[1], "--inputs") == 0;
  if (inputs_only) {
    ++argv;
    --argc;
  }
  if (argc < 2) {
    fprintf(stderr, "usage: quantize_layer [--inputs] OUT.bin [T in out]\n");
    return 2;
  }
  const int64_t T = argc > 2 ? atoll(argv[2]) : 1000;
  const int64_t in = argc > 3 ? atoll(argv[3]) : 512;
  const int64_t out = argc > 4 ? atoll(argv[4]) : 264;
  awq_config cfg = {4, 128, 1, 20, 20, 0.5f, AWQ_SEARCH_DIRECT};

  uint16_t *hX = (uint16_t *)malloc(sizeof(uint16_t) * T * in);
  uint16_t *hW = (uint16_t *)malloc(sizeof(uint16_t) * out * in);
  lcg_state = 12345u;
  for (int64_t t = 0; t < T; ++t)
    for (int64_t j = 0; j < in; ++j) {
      const double c = (j % 50 == 7) ? 20.0 : 1.0;
      hX[t * in + j] = to_half((float)((lcg_uniform() - 0.5) * c));
    }
  for (int64_t i = 0; i < out * in; ++i) hW[i] = to_half((float)((lcg_uniform() - 0.5) / 16.0));
  if (inputs_only) {
    FILE *f = fopen(argv[1], "wb");
    if (!f) {
      perror(argv[1]);
      return 1;
    }
    fwrite(hX, sizeof(uint16_t), T * in, f);
    fwrite(hW, sizeof(uint16_t), out * in, f);
    fclose(f);
    return 0;
  }

  void *dX, *dW, *ws, *scales;
  double *abar, *mse;
  float *s_best;
  int32_t *best, *qweight, *qzeros;
  uint8_t *clip_idx;
  const int64_t groups = in / cfg.group_size;
  const size_t ws_bytes = awq_workspace_size(T, in, out, &cfg);
  if (ws_bytes == 0) {
    fprintf(stderr, "awq_workspace_size: %s\n", awq_last_error());
    return 1;
  }
  CUDA(cudaMalloc(&dX, sizeof(uint16_t) * T * in));
  CUDA(cudaMalloc(&dW, sizeof(uint16_t) * out * in));
  CUDA(cudaMalloc(&ws, ws_bytes));
  CUDA(cudaMalloc((void **)&abar, sizeof(double) * in));
  CUDA(cudaMalloc((void **)&mse, sizeof(double) * cfg.n_alpha));
  CUDA(cudaMalloc((void **)&s_best, sizeof(float) * in));
  CUDA(cudaMalloc((void **)&best, sizeof(int32_t)));
  CUDA(cudaMalloc((void **)&clip_idx, (size_t)out * groups));
  CUDA(cudaMalloc((void **)&qweight, sizeof(int32_t) * in * (out / 8)));
  CUDA(cudaMalloc((void **)&qzeros, sizeof(int32_t) * groups * (out / 8)));
  CUDA(cudaMalloc(&scales, sizeof(uint16_t) * groups * out));
  CUDA(cudaMemcpy(dX, hX, sizeof(uint16_t) * T * in, cudaMemcpyHostToDevice));
  CUDA(cudaMemcpy(dW, hW, sizeof(uint16_t) * out * in, cudaMemcpyHostToDevice));

  CHECK(awq_act_stats(dX, T, in, in, abar, NULL));
  CHECK(awq_search_scale(dX, T, in, in, dW, out, abar, &cfg, ws, ws_bytes, s_best, mse, best, NULL));
  CHECK(awq_search_clip(dX, T, in, in, dW, out, s_best, &cfg, ws, ws_bytes, clip_idx, NULL, NULL));
  CHECK(awq_quant_pack(dW, out, in, s_best, clip_idx, &cfg, qweight, qzeros, scales, NULL));
  CHECK(awq_device_status(ws, NULL));
  CHECK(awq_device_status(NULL, NULL));

  int32_t hbest = -1;
  double *hmse = (double *)malloc(sizeof(double) * cfg.n_alpha);
  int32_t *hqw = (int32_t *)malloc(sizeof(int32_t) * in * (out / 8));
  int32_t *hqz = (int32_t *)malloc(sizeof(int32_t) * groups * (out / 8));
  uint16_t *hsc = (uint16_t *)malloc(sizeof(uint16_t) * groups * out);
  uint8_t *hci = (uint8_t *)malloc((size_t)out * groups);
  CUDA(cudaMemcpy(&hbest, best, sizeof(int32_t), cudaMemcpyDeviceToHost));
  CUDA(cudaMemcpy(hmse, mse, sizeof(double) * cfg.n_alpha, cudaMemcpyDeviceToHost));
  CUDA(cudaMemcpy(hqw, qweight, sizeof(int32_t) * in * (out / 8), cudaMemcpyDeviceToHost));
  CUDA(cudaMemcpy(hqz, qzeros, sizeof(int32_t) * groups * (out / 8), cudaMemcpyDeviceToHost));
  CUDA(cudaMemcpy(hsc, scales, sizeof(uint16_t) * groups * out, cudaMemcpyDeviceToHost));
  CUDA(cudaMemcpy(hci, clip_idx, (size_t)out * groups, cudaMemcpyDeviceToHost));

  FILE *f = fopen(argv[1], "wb");
  if (!f) {
    perror(argv[1]);
    return 1;
  }
  /* layout: best (int32), mse [n_alpha] f64, clip_idx [out, in/g] u8, qweight
   * [in, out/8] i32, qzeros [in/g, out/8] i32, scales [in/g, out] f16, then
   * X [T, in] and W [out, in] f16 */
  fwrite(&hbest, sizeof(int32_t), 1, f);
  fwrite(hmse, sizeof(double), cfg.n_alpha, f);
  fwrite(hci, 1, (size_t)out * groups, f);
  fwrite(hqw, sizeof(int32_t), in * (out / 8), f);
  fwrite(hqz, sizeof(int32_t), groups * (out / 8), f);
  fwrite(hsc, sizeof(uint16_t), groups * out, f);
  fwrite(hX, sizeof(uint16_t), T * in, f); /* the inputs, so the generator can be checked */
  fwrite(hW, sizeof(uint16_t), out * in, f);
  fclose(f);
  printf("best alpha index %d, mse %.6e, %s\n", hbest, hmse[hbest], awq_version());
  return 0;
}
