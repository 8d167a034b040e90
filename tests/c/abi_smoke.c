/* A C program that uses libdpo through include/dpo.h only (no Python, no torch).
 *
 *   abi_smoke host   argument checks that return before any CUDA call
 *   abi_smoke gpu    one DPO step on the current GPU with policy == reference:
 *                    the loss must be ln 2, every weight 1/2, the accuracy 0,
 *                    and no device error may be reported.
 * Exit status 0 on success; the failing check is printed otherwise. */
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime.h>

#include "dpo.h"

#define CHECK(cond)                                                         \
  do {                                                                      \
    if (!(cond)) {                                                          \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond);   \
      return 1;                                                             \
    }                                                                       \
  } while (0)

static int host_checks(void) {
  int32_t P[4] = {4, 4, 4, 4}, C[4] = {10, 10, 10, 10};
  dpo_batch b;
  memset(&b, 0, sizeof b);
  b.R = 4; b.L = 32; b.d = 64; b.V = 100; b.dtype = DPO_BF16;
  b.H = (const void*)0x10000; b.W = (const void*)0x10000; b.tokens = (const int32_t*)0x10000;
  b.prompt_len = P; b.completion_len = C;
  size_t f = 0, bw = 0, mn = 0;
  CHECK(dpo_workspace_size(&b, &f, &bw, &mn) == DPO_OK);
  CHECK(f > 0 && bw >= mn && mn > 0 && f % 256 == 0);
  b.dtype = DPO_F16;
  CHECK(dpo_workspace_size(&b, &f, &bw, &mn) == DPO_ERR_UNSUPPORTED);
  b.dtype = DPO_BF16;
  P[0] = 0;
  CHECK(dpo_workspace_size(&b, &f, NULL, NULL) == DPO_ERR_INVALID_ARG);
  P[0] = 4;
  float out[4];
  CHECK(dpo_seq_logprobs(&b, 0, out, NULL, NULL, NULL, 0, NULL) == DPO_ERR_WORKSPACE);
  CHECK(dpo_loss(0, DPO_PAIRS_HALVES, out, out, 0.1f, 1.0f, out, NULL, NULL, NULL, NULL, NULL,
                 NULL, NULL) == DPO_ERR_INVALID_ARG);
  CHECK(strcmp(dpo_status_string(DPO_OK), "ok") == 0);
  CHECK(dpo_version() > 0);
  printf("host checks ok\n");
  return 0;
}

static uint16_t bf16(float x) {       /* round to nearest even */
  uint32_t u;
  memcpy(&u, &x, 4);
  return (uint16_t)((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

static int gpu_step(void) {
  const int R = 4, L = 96, d = 128, V = 700, B = R / 2;
  int32_t P[4] = {5, 9, 1, 30}, C[4] = {60, 40, 95, 10};
  size_t nh = (size_t)R * L * d, nw = (size_t)V * d;
  uint16_t* h = (uint16_t*)malloc(nh * 2);
  uint16_t* w = (uint16_t*)malloc(nw * 2);
  int32_t* tok = (int32_t*)malloc(sizeof(int32_t) * R * L);
  srand(7);
  for (size_t i = 0; i < nh; ++i) h[i] = bf16((float)rand() / RAND_MAX - 0.5f);
  for (size_t i = 0; i < nw; ++i) w[i] = bf16(((float)rand() / RAND_MAX - 0.5f) * 0.2f);
  for (int i = 0; i < R * L; ++i) tok[i] = rand() % V;

  void *dH_in, *dW_in, *dtok, *ws, *dlse, *dpol, *dref, *dloss, *dacc, *dw8, *dcoef, *dH, *dW;
  CHECK(cudaMalloc(&dH_in, nh * 2) == cudaSuccess);
  CHECK(cudaMalloc(&dW_in, nw * 2) == cudaSuccess);
  CHECK(cudaMalloc(&dtok, sizeof(int32_t) * R * L) == cudaSuccess);
  cudaMemcpy(dH_in, h, nh * 2, cudaMemcpyHostToDevice);
  cudaMemcpy(dW_in, w, nw * 2, cudaMemcpyHostToDevice);
  cudaMemcpy(dtok, tok, sizeof(int32_t) * R * L, cudaMemcpyHostToDevice);

  dpo_batch b;
  memset(&b, 0, sizeof b);
  b.R = R; b.L = L; b.d = d; b.V = V; b.dtype = DPO_BF16;
  b.H = dH_in; b.W = dW_in; b.tokens = (const int32_t*)dtok;
  b.prompt_len = P; b.completion_len = C;
  size_t f = 0, bw = 0;
  CHECK(dpo_workspace_size(&b, &f, &bw, NULL) == DPO_OK);
  int nc = 0;
  for (int r = 0; r < R; ++r) nc += C[r];
  CHECK(cudaMalloc(&ws, f > bw ? f : bw) == cudaSuccess);
  CHECK(cudaMalloc(&dlse, sizeof(float) * nc) == cudaSuccess);
  CHECK(cudaMalloc(&dpol, sizeof(float) * R) == cudaSuccess);
  CHECK(cudaMalloc(&dref, sizeof(float) * R) == cudaSuccess);
  CHECK(cudaMalloc(&dloss, sizeof(float)) == cudaSuccess);
  CHECK(cudaMalloc(&dacc, sizeof(float)) == cudaSuccess);
  CHECK(cudaMalloc(&dw8, sizeof(float) * B) == cudaSuccess);
  CHECK(cudaMalloc(&dcoef, sizeof(float) * R) == cudaSuccess);
  CHECK(cudaMalloc(&dH, sizeof(float) * nh) == cudaSuccess);
  CHECK(cudaMalloc(&dW, sizeof(float) * nw) == cudaSuccess);

  /* policy == reference: same weights for both forwards */
  CHECK(dpo_seq_logprobs(&b, 1, (float*)dpol, NULL, (float*)dlse, ws, f > bw ? f : bw, NULL) == DPO_OK);
  CHECK(dpo_seq_logprobs(&b, 0, (float*)dref, NULL, NULL, ws, f > bw ? f : bw, NULL) == DPO_OK);
  CHECK(dpo_loss(B, DPO_PAIRS_HALVES, (float*)dpol, (float*)dref, 0.1f, 1.0f, (float*)dloss,
                 (float*)dacc, NULL, NULL, NULL, (float*)dw8, (float*)dcoef, NULL) == DPO_OK);
  CHECK(dpo_backward(&b, (float*)dlse, (float*)dcoef, (float*)dH, (float*)dW, 0, ws,
                     f > bw ? f : bw, NULL) == DPO_OK);
  CHECK(dpo_check(NULL) == DPO_OK);
  float loss, acc, wts[2], pol[4];
  cudaMemcpy(&loss, dloss, 4, cudaMemcpyDeviceToHost);
  cudaMemcpy(&acc, dacc, 4, cudaMemcpyDeviceToHost);
  cudaMemcpy(wts, dw8, sizeof wts, cudaMemcpyDeviceToHost);
  cudaMemcpy(pol, dpol, sizeof pol, cudaMemcpyDeviceToHost);
  CHECK(fabsf(loss - (float)log(2.0)) < 1e-6f);
  CHECK(acc == 0.0f && wts[0] == 0.5f && wts[1] == 0.5f);
  for (int r = 0; r < R; ++r) CHECK(pol[r] < 0.0f && pol[r] > -20.0f * C[r]);
  printf("gpu step ok: loss %.7f, sums %.3f %.3f %.3f %.3f\n", loss, pol[0], pol[1], pol[2], pol[3]);
  return 0;
}

int main(int argc, char** argv) {
  if (argc > 1 && strcmp(argv[1], "gpu") == 0) return gpu_step();
  return host_checks();
}
