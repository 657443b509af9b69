/* A plain C99 caller of the C ABI (include/flce.h): no Python, no torch.  Builds a small
 * problem on the host, copies it to the device, runs the fused forward with gradients and the
 * statistics-only forward through the library, and prints the loss, the number of rows in the
 * loss and the status word.  Then the same rows taken as the rows before the model's final
 * RMSNorm (gain 1.25): flce_forward_rmsnorm against flce_forward on the rows normalised here on
 * the host.  Exit code 0 when the calls agree and the status is clean. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "flce.h"

static uint16_t to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

#define CHECK_CUDA(x)                                                      \
  do {                                                                     \
    cudaError_t e_ = (x);                                                  \
    if (e_ != cudaSuccess) {                                               \
      fprintf(stderr, "%s: %s\n", #x, cudaGetErrorString(e_));             \
      return 2;                                                            \
    }                                                                      \
  } while (0)

#define CHECK_FLCE(x)                                                      \
  do {                                                                     \
    int r_ = (x);                                                          \
    if (r_ != FLCE_OK) {                                                   \
      fprintf(stderr, "%s: %s\n", #x, flce_status_string(r_));             \
      return 3;                                                            \
    }                                                                      \
  } while (0)

int main(void) {
  const int64_t N = 200, d = 128, Vreal = 1000, Vpad = 1024;
  flce_shape s;
  s.N = N;
  s.d = d;
  s.Vpad = Vpad;
  s.Vreal = Vreal;
  s.cap = 15.0f;
  s.ignore_index = -1;
  s.chunk_rows = 0;

  uint16_t* hX = (uint16_t*)malloc(sizeof(uint16_t) * N * d);
  uint16_t* hW = (uint16_t*)malloc(sizeof(uint16_t) * Vpad * d);
  int64_t* ht = (int64_t*)malloc(sizeof(int64_t) * N);
  uint32_t state = 12345u;
  for (int64_t i = 0; i < N * d; ++i) {
    state = state * 1664525u + 1013904223u;
    hX[i] = to_bf16(((float)(state >> 8) / 16777216.0f - 0.5f) * 2.0f);
  }
  for (int64_t i = 0; i < Vpad * d; ++i) {
    state = state * 1664525u + 1013904223u;
    hW[i] = to_bf16(((float)(state >> 8) / 16777216.0f - 0.5f) * 0.1f);
  }
  for (int64_t i = 0; i < N; ++i) ht[i] = (i % 17 == 0) ? -1 : (i * 37) % Vreal;

  void *X, *W, *ws, *dX;
  int64_t* t;
  float *loss, *lse, *dW;
  const size_t ws_bytes = flce_workspace_bytes(&s, 1);
  if (ws_bytes == 0) return 4;
  CHECK_CUDA(cudaMalloc(&X, sizeof(uint16_t) * N * d));
  CHECK_CUDA(cudaMalloc(&W, sizeof(uint16_t) * Vpad * d));
  CHECK_CUDA(cudaMalloc((void**)&t, sizeof(int64_t) * N));
  CHECK_CUDA(cudaMalloc((void**)&loss, 2 * sizeof(float)));
  CHECK_CUDA(cudaMalloc((void**)&lse, sizeof(float) * N));
  CHECK_CUDA(cudaMalloc(&dX, sizeof(uint16_t) * N * d));
  CHECK_CUDA(cudaMalloc((void**)&dW, sizeof(float) * Vpad * d));
  CHECK_CUDA(cudaMalloc(&ws, ws_bytes));
  CHECK_CUDA(cudaMemcpy(X, hX, sizeof(uint16_t) * N * d, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(W, hW, sizeof(uint16_t) * Vpad * d, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(t, ht, sizeof(int64_t) * N, cudaMemcpyHostToDevice));

  CHECK_FLCE(flce_forward(&s, X, W, t, loss, lse, 1, NULL, dX, dW, FLCE_DTYPE_F32, 0, ws,
                          ws_bytes, NULL));
  CHECK_FLCE(flce_forward(&s, X, W, t, loss + 1, lse, 0, NULL, NULL, NULL, FLCE_DTYPE_F32, 0, ws,
                          ws_bytes, NULL));
  uint32_t status = 0;
  int64_t n_valid = 0;
  CHECK_FLCE(flce_read_status(ws, &status, &n_valid, NULL));
  float hl[2];
  CHECK_CUDA(cudaMemcpy(hl, loss, sizeof(hl), cudaMemcpyDeviceToHost));
  printf("loss %.6f (stats-only %.6f) n_valid %lld status %u\n", hl[0], hl[1],
         (long long)n_valid, status);
  int ok = status == 0 && n_valid == N - (N + 16) / 17 && isfinite(hl[0]) &&
           fabsf(hl[0] - hl[1]) < 1e-6f;

  /* the final RMSNorm in front of the head, in one call; X serves as the rows before the norm */
  uint16_t* hg = (uint16_t*)malloc(sizeof(uint16_t) * d);
  uint16_t* hXn = (uint16_t*)malloc(sizeof(uint16_t) * N * d);
  for (int64_t k = 0; k < d; ++k) hg[k] = to_bf16(1.25f);
  for (int64_t i = 0; i < N; ++i) {
    double ss = 0.0;
    for (int64_t k = 0; k < d; ++k) {
      uint32_t u = (uint32_t)hX[i * d + k] << 16;
      float f;
      memcpy(&f, &u, 4);
      ss += (double)f * f;
    }
    const double rstd = 1.0 / sqrt(ss / (double)d + 1e-6);
    for (int64_t k = 0; k < d; ++k) {
      uint32_t u = (uint32_t)hX[i * d + k] << 16;
      float f;
      memcpy(&f, &u, 4);
      hXn[i * d + k] = to_bf16((float)(f * rstd * 1.25));
    }
  }
  void *gamma, *Xn, *dH, *ws_r;
  float *dgamma, *g_one;
  const size_t ws_r_bytes = flce_workspace_bytes_rmsnorm(&s, 1);
  if (ws_r_bytes <= ws_bytes) return 4;
  CHECK_CUDA(cudaMalloc(&gamma, sizeof(uint16_t) * d));
  CHECK_CUDA(cudaMalloc(&Xn, sizeof(uint16_t) * N * d));
  CHECK_CUDA(cudaMalloc(&dH, sizeof(uint16_t) * N * d));
  CHECK_CUDA(cudaMalloc((void**)&dgamma, sizeof(float) * d));
  CHECK_CUDA(cudaMalloc((void**)&g_one, sizeof(float)));
  CHECK_CUDA(cudaMalloc(&ws_r, ws_r_bytes));
  const float one = 1.0f;
  CHECK_CUDA(cudaMemcpy(g_one, &one, sizeof(float), cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(gamma, hg, sizeof(uint16_t) * d, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(Xn, hXn, sizeof(uint16_t) * N * d, cudaMemcpyHostToDevice));
  CHECK_FLCE(flce_forward_rmsnorm(&s, X, gamma, 1e-6f, W, t, loss, lse, 1, NULL, dH, dgamma, dW,
                                  FLCE_DTYPE_F32, 0, ws_r, ws_r_bytes, NULL));
  CHECK_FLCE(flce_scale_grads_rmsnorm(&s, g_one, dH, dgamma, dW, FLCE_DTYPE_F32, NULL));
  CHECK_FLCE(flce_forward(&s, Xn, W, t, loss + 1, lse, 0, NULL, NULL, NULL, FLCE_DTYPE_F32, 0, ws,
                          ws_bytes, NULL));
  uint32_t status_r = 0;
  CHECK_FLCE(flce_read_status(ws_r, &status_r, &n_valid, NULL));
  CHECK_CUDA(cudaMemcpy(hl, loss, sizeof(hl), cudaMemcpyDeviceToHost));
  printf("rmsnorm + head: loss %.6f (head on host-normalised rows %.6f) status %u\n", hl[0],
         hl[1], status_r);
  ok = ok && status_r == 0 && isfinite(hl[0]) && fabsf(hl[0] - hl[1]) < 1e-3f;
  cudaFree(gamma);
  cudaFree(Xn);
  cudaFree(dH);
  cudaFree(dgamma);
  cudaFree(g_one);
  cudaFree(ws_r);
  free(hg);
  free(hXn);
  cudaFree(X);
  cudaFree(W);
  cudaFree(t);
  cudaFree(loss);
  cudaFree(lse);
  cudaFree(dX);
  cudaFree(dW);
  cudaFree(ws);
  free(hX);
  free(hW);
  free(ht);
  return ok ? 0 : 1;
}
