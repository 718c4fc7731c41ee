/*
 * A decode step driven from plain C through include/dllm.h only (no Python, no torch):
 * cudaMalloc'd buffers, deterministic synthetic inputs, dllm_decode_step, then checks of
 * what holds at any size: the compaction equals the mask, every selected position is a
 * masked one, confidences lie in [1/V, 1], the selection is ordered by confidence, and the
 * invalid-argument paths return their status codes.  Prints "ok" and exits 0 on success.
 */
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "dllm.h"

#define CHECK_CUDA(x) do { cudaError_t e_ = (x); if (e_ != cudaSuccess) { \
    fprintf(stderr, "CUDA %s at line %d\n", cudaGetErrorString(e_), __LINE__); return 2; } } while (0)
#define EXPECT(c) do { if (!(c)) { fprintf(stderr, "failed: %s (line %d)\n", #c, __LINE__); \
    return 1; } } while (0)

static uint16_t to_bf16(float f) {          /* round to nearest even */
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

static uint32_t lcg(uint32_t* s) { *s = *s * 1664525u + 1013904223u; return *s; }
static float unif(uint32_t* s) { return (float)(lcg(s) >> 8) / 16777216.0f; }

int main(void) {
  const int B = 2, L = 700, d = 128, V = 3001, k = 16;
  const int n = B * L;
  uint32_t seed = 12345u;
  uint16_t* H = malloc(sizeof(uint16_t) * (size_t)n * d);
  uint16_t* W = malloc(sizeof(uint16_t) * (size_t)V * d);
  uint8_t* M = malloc((size_t)n);
  for (size_t i = 0; i < (size_t)n * d; ++i) H[i] = to_bf16(2.0f * unif(&seed) - 1.0f);
  for (size_t i = 0; i < (size_t)V * d; ++i) W[i] = to_bf16(0.2f * (unif(&seed) - 0.5f));
  int masked = 0;
  for (int i = 0; i < n; ++i) { M[i] = unif(&seed) < 0.6f; masked += M[i]; }

  void *dH, *dW, *dM, *ws;
  int32_t *tok, *row_idx, *seq_off, *count, *idx, *n_sel, *tok_sel;
  float *conf, *lse, *conf_sel;
  const size_t ws_bytes = dllm_workspace_bytes(B, L, d, V);
  EXPECT(ws_bytes > 0);
  CHECK_CUDA(cudaMalloc(&dH, sizeof(uint16_t) * (size_t)n * d));
  CHECK_CUDA(cudaMalloc(&dW, sizeof(uint16_t) * (size_t)V * d));
  CHECK_CUDA(cudaMalloc(&dM, (size_t)n));
  CHECK_CUDA(cudaMalloc(&ws, ws_bytes));
  CHECK_CUDA(cudaMalloc((void**)&tok, sizeof(int32_t) * n));
  CHECK_CUDA(cudaMalloc((void**)&conf, sizeof(float) * n));
  CHECK_CUDA(cudaMalloc((void**)&lse, sizeof(float) * n));
  CHECK_CUDA(cudaMalloc((void**)&row_idx, sizeof(int32_t) * n));
  CHECK_CUDA(cudaMalloc((void**)&seq_off, sizeof(int32_t) * (B + 1)));
  CHECK_CUDA(cudaMalloc((void**)&count, 16));
  CHECK_CUDA(cudaMalloc((void**)&idx, sizeof(int32_t) * B * k));
  CHECK_CUDA(cudaMalloc((void**)&n_sel, sizeof(int32_t) * B));
  CHECK_CUDA(cudaMalloc((void**)&tok_sel, sizeof(int32_t) * B * k));
  CHECK_CUDA(cudaMalloc((void**)&conf_sel, sizeof(float) * B * k));
  CHECK_CUDA(cudaMemcpy(dH, H, sizeof(uint16_t) * (size_t)n * d, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(dW, W, sizeof(uint16_t) * (size_t)V * d, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(dM, M, (size_t)n, cudaMemcpyHostToDevice));
  cudaStream_t s;
  CHECK_CUDA(cudaStreamCreate(&s));

  /* host-side validation: nothing is launched for a bad call */
  EXPECT(dllm_decode_step(dH, dM, dW, B, L, d, V, 0, NULL, NULL, tok, conf, lse, row_idx, seq_off,
                          count, idx, n_sel, tok_sel, conf_sel, ws, ws_bytes, s) == DLLM_ERR_SHAPE);
  EXPECT(dllm_decode_step(dH, dM, dW, B, L, d, V, k, NULL, NULL, tok, conf, lse, row_idx, seq_off,
                          count, idx, n_sel, tok_sel, conf_sel, ws, 16, s) == DLLM_ERR_WORKSPACE);
  EXPECT(dllm_decode_step(dH, dM, dW, B, L, 100, V, k, NULL, NULL, tok, conf, lse, row_idx, seq_off,
                          count, idx, n_sel, tok_sel, conf_sel, ws, ws_bytes, s) == DLLM_ERR_SHAPE);

  EXPECT(dllm_decode_step(dH, dM, dW, B, L, d, V, k, NULL, NULL, tok, conf, lse, row_idx, seq_off,
                          count, idx, n_sel, tok_sel, conf_sel, ws, ws_bytes, s) == DLLM_OK);
  EXPECT(dllm_get_status(s) == DLLM_OK);

  int32_t c = 0, h_seq[3], h_idx[2 * 16], h_nsel[2], h_tok_sel[2 * 16];
  float h_conf_sel[2 * 16];
  int32_t* h_rows = malloc(sizeof(int32_t) * n);
  float* h_conf = malloc(sizeof(float) * n);
  float* h_lse = malloc(sizeof(float) * n);
  int32_t* h_tok = malloc(sizeof(int32_t) * n);
  CHECK_CUDA(cudaMemcpy(&c, count, 4, cudaMemcpyDeviceToHost));
  EXPECT(c == masked);
  CHECK_CUDA(cudaMemcpy(h_rows, row_idx, sizeof(int32_t) * c, cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(h_conf, conf, sizeof(float) * c, cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(h_lse, lse, sizeof(float) * c, cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(h_tok, tok, sizeof(int32_t) * c, cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(h_seq, seq_off, sizeof(h_seq), cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(h_idx, idx, sizeof(h_idx), cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(h_nsel, n_sel, sizeof(h_nsel), cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(h_tok_sel, tok_sel, sizeof(h_tok_sel), cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(h_conf_sel, conf_sel, sizeof(h_conf_sel), cudaMemcpyDeviceToHost));

  /* compaction = the mask, ascending; per-sequence offsets */
  int r = 0;
  for (int p = 0; p < n; ++p)
    if (M[p]) { EXPECT(h_rows[r] == p); ++r; }
  EXPECT(h_seq[0] == 0 && h_seq[B] == c);
  for (int i = 0; i < c; ++i) {
    EXPECT(h_conf[i] >= 1.0f / V * 0.999f && h_conf[i] <= 1.0f);
    EXPECT(h_tok[i] >= 0 && h_tok[i] < V);
    EXPECT(isfinite(h_lse[i]));
  }
  /* the selection: masked positions of its sequence, ordered, consistent with conf and tok */
  for (int b = 0; b < B; ++b) {
    const int cand = h_seq[b + 1] - h_seq[b];
    EXPECT(h_nsel[b] == (cand < k ? cand : k));
    for (int j = 0; j < k; ++j) {
      if (j >= h_nsel[b]) { EXPECT(h_idx[b * k + j] == -1); continue; }
      const int pos = h_idx[b * k + j];
      EXPECT(pos >= 0 && pos < L && M[b * L + pos]);
      int row = -1;
      for (int i = h_seq[b]; i < h_seq[b + 1]; ++i) if (h_rows[i] == b * L + pos) row = i;
      EXPECT(row >= 0 && h_conf_sel[b * k + j] == h_conf[row] && h_tok_sel[b * k + j] == h_tok[row]);
      if (j > 0) EXPECT(h_conf_sel[b * k + j] <= h_conf_sel[b * k + j - 1]);
      /* nothing left out beats the last one taken */
      if (j == h_nsel[b] - 1)
        for (int i = h_seq[b]; i < h_seq[b + 1]; ++i) {
          int taken = 0;
          for (int q = 0; q <= j; ++q) taken |= (h_rows[i] == b * L + h_idx[b * k + q]);
          if (!taken) EXPECT(h_conf[i] <= h_conf_sel[b * k + j]);
        }
    }
  }
  printf("ok %d masked rows, version %d\n", c, dllm_version());
  return 0;
}
