/* A C program that uses libdpo through include/dpo.h only (no Python, no torch).
 *
 *   abi_smoke host   argument checks that return before any CUDA call
 *   abi_smoke gpu    one DPO step on the current GPU with policy == reference:
 *                    the loss must be ln 2, every weight 1/2, the accuracy 0,
 *                    and no device error may be reported.
 *   abi_smoke case DIR   one DPO step (policy forward, reference forward, loss,
 *                    backward) on the inputs in DIR, checked against the expected
 *                    values in DIR (written by the Python test from the fp64 oracle):
 *                    sequence sums |err| <= 5e-2 and <= 1e-4 relative, loss |err|
 *                    <= 1e-4, dH and dW relative Frobenius error <= 1e-2.
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

  /* reference-free objective: no reference buffer at all, the same bits as a reference of
     zeros through dpo_loss */
  float loss_free, loss_zero;
  dpo_loss_options opt = {0};
  opt.reference_free = 1;
  CHECK(dpo_loss_ex(B, DPO_PAIRS_HALVES, (float*)dpol, NULL, 0.1f, 1.0f, &opt, (float*)dloss,
                    NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL) == DPO_OK);
  cudaMemcpy(&loss_free, dloss, 4, cudaMemcpyDeviceToHost);
  CHECK(cudaMemset(dref, 0, sizeof(float) * R) == cudaSuccess);
  CHECK(dpo_loss(B, DPO_PAIRS_HALVES, (float*)dpol, (float*)dref, 0.1f, 1.0f, (float*)dloss, NULL,
                 NULL, NULL, NULL, NULL, NULL, NULL) == DPO_OK);
  cudaMemcpy(&loss_zero, dloss, 4, cudaMemcpyDeviceToHost);
  CHECK(loss_free == loss_zero);
  opt.reference_free = 0;
  CHECK(dpo_loss_ex(B, DPO_PAIRS_HALVES, (float*)dpol, NULL, 0.1f, 1.0f, &opt, (float*)dloss,
                    NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL) == DPO_ERR_INVALID_ARG);
  CHECK(dpo_check(NULL) == DPO_OK);
  printf("gpu step ok: loss %.7f, sums %.3f %.3f %.3f %.3f, reference-free loss %.7f\n", loss,
         pol[0], pol[1], pol[2], pol[3], loss_free);
  return 0;
}

/* Read exactly n bytes of DIR/name into a new host buffer (NULL on failure). */
static void* read_file(const char* dir, const char* name, size_t n) {
  char path[4096];
  snprintf(path, sizeof path, "%s/%s", dir, name);
  FILE* f = fopen(path, "rb");
  if (!f) return NULL;
  void* p = malloc(n > 0 ? n : 1);
  size_t got = fread(p, 1, n, f);
  fclose(f);
  if (got != n) {
    free(p);
    return NULL;
  }
  return p;
}

/* Relative Frobenius error of a float array against a double array. */
static double rel_frob(const float* a, const double* b, size_t n) {
  double num = 0.0, den = 0.0;
  for (size_t i = 0; i < n; ++i) {
    const double e = (double)a[i] - b[i];
    num += e * e;
    den += b[i] * b[i];
  }
  return sqrt(num / (den > 0.0 ? den : 1e-300));
}

static int case_step(const char* dir) {
  /* meta: R L d V beta (pairs in halves layout) */
  char path[4096];
  snprintf(path, sizeof path, "%s/meta.txt", dir);
  FILE* mf = fopen(path, "r");
  CHECK(mf != NULL);
  int R = 0, L = 0, d = 0, V = 0;
  double beta = 0.0;
  CHECK(fscanf(mf, "%d %d %d %d %lf", &R, &L, &d, &V, &beta) == 5);
  fclose(mf);
  CHECK(R > 0 && R % 2 == 0 && L > 1 && d > 0 && V > 0);
  const int B = R / 2;
  const size_t nh = (size_t)R * L * d, nw = (size_t)V * d;
  uint16_t* h = (uint16_t*)read_file(dir, "H.bin", nh * 2);
  uint16_t* w = (uint16_t*)read_file(dir, "W.bin", nw * 2);
  uint16_t* wr = (uint16_t*)read_file(dir, "W_ref.bin", nw * 2);
  int32_t* tok = (int32_t*)read_file(dir, "tokens.bin", sizeof(int32_t) * R * L);
  int32_t* P = (int32_t*)read_file(dir, "prompt_len.bin", sizeof(int32_t) * R);
  int32_t* C = (int32_t*)read_file(dir, "completion_len.bin", sizeof(int32_t) * R);
  double* e_pol = (double*)read_file(dir, "pol.bin", sizeof(double) * R);
  double* e_ref = (double*)read_file(dir, "ref.bin", sizeof(double) * R);
  double* e_loss = (double*)read_file(dir, "loss.bin", sizeof(double));
  double* e_dH = (double*)read_file(dir, "dH.bin", sizeof(double) * nh);
  double* e_dW = (double*)read_file(dir, "dW.bin", sizeof(double) * nw);
  CHECK(h && w && wr && tok && P && C && e_pol && e_ref && e_loss && e_dH && e_dW);

  void *dHin, *dWin, *dWr, *dtok, *ws, *dlse, *dpol, *dref, *dloss, *dcoef, *ddH, *ddW;
  CHECK(cudaMalloc(&dHin, nh * 2) == cudaSuccess);
  CHECK(cudaMalloc(&dWin, nw * 2) == cudaSuccess);
  CHECK(cudaMalloc(&dWr, nw * 2) == cudaSuccess);
  CHECK(cudaMalloc(&dtok, sizeof(int32_t) * R * L) == cudaSuccess);
  CHECK(cudaMemcpy(dHin, h, nh * 2, cudaMemcpyHostToDevice) == cudaSuccess);
  CHECK(cudaMemcpy(dWin, w, nw * 2, cudaMemcpyHostToDevice) == cudaSuccess);
  CHECK(cudaMemcpy(dWr, wr, nw * 2, cudaMemcpyHostToDevice) == cudaSuccess);
  CHECK(cudaMemcpy(dtok, tok, sizeof(int32_t) * R * L, cudaMemcpyHostToDevice) == cudaSuccess);

  dpo_batch b, br;
  memset(&b, 0, sizeof b);
  b.R = R; b.L = L; b.d = d; b.V = V; b.dtype = DPO_BF16;
  b.H = dHin; b.W = dWin; b.tokens = (const int32_t*)dtok;
  b.prompt_len = P; b.completion_len = C;
  br = b;
  br.W = dWr;
  size_t f = 0, bw = 0;
  CHECK(dpo_workspace_size(&b, &f, &bw, NULL) == DPO_OK);
  const size_t wsb = f > bw ? f : bw;
  int nc = 0;
  for (int r = 0; r < R; ++r) nc += C[r];
  CHECK(cudaMalloc(&ws, wsb) == cudaSuccess);
  CHECK(cudaMalloc(&dlse, sizeof(float) * (nc > 0 ? nc : 1)) == cudaSuccess);
  CHECK(cudaMalloc(&dpol, sizeof(float) * R) == cudaSuccess);
  CHECK(cudaMalloc(&dref, sizeof(float) * R) == cudaSuccess);
  CHECK(cudaMalloc(&dloss, sizeof(float)) == cudaSuccess);
  CHECK(cudaMalloc(&dcoef, sizeof(float) * R) == cudaSuccess);
  CHECK(cudaMalloc(&ddH, sizeof(float) * nh) == cudaSuccess);
  CHECK(cudaMalloc(&ddW, sizeof(float) * nw) == cudaSuccess);

  CHECK(dpo_seq_logprobs(&b, 1, (float*)dpol, NULL, (float*)dlse, ws, wsb, NULL) == DPO_OK);
  CHECK(dpo_seq_logprobs(&br, 0, (float*)dref, NULL, NULL, ws, wsb, NULL) == DPO_OK);
  CHECK(dpo_loss(B, DPO_PAIRS_HALVES, (float*)dpol, (float*)dref, (float)beta, 1.0f,
                 (float*)dloss, NULL, NULL, NULL, NULL, NULL, (float*)dcoef, NULL) == DPO_OK);
  CHECK(dpo_backward(&b, (float*)dlse, (float*)dcoef, (float*)ddH, (float*)ddW, 0, ws, wsb,
                     NULL) == DPO_OK);
  CHECK(dpo_check(NULL) == DPO_OK);

  float* pol = (float*)malloc(sizeof(float) * R);
  float* ref = (float*)malloc(sizeof(float) * R);
  float* gH = (float*)malloc(sizeof(float) * nh);
  float* gW = (float*)malloc(sizeof(float) * nw);
  float loss = 0.f;
  CHECK(cudaMemcpy(pol, dpol, sizeof(float) * R, cudaMemcpyDeviceToHost) == cudaSuccess);
  CHECK(cudaMemcpy(ref, dref, sizeof(float) * R, cudaMemcpyDeviceToHost) == cudaSuccess);
  CHECK(cudaMemcpy(&loss, dloss, sizeof(float), cudaMemcpyDeviceToHost) == cudaSuccess);
  CHECK(cudaMemcpy(gH, ddH, sizeof(float) * nh, cudaMemcpyDeviceToHost) == cudaSuccess);
  CHECK(cudaMemcpy(gW, ddW, sizeof(float) * nw, cudaMemcpyDeviceToHost) == cudaSuccess);
  for (int r = 0; r < R; ++r) {
    const double ep = fabs((double)pol[r] - e_pol[r]), er = fabs((double)ref[r] - e_ref[r]);
    CHECK(ep <= 5e-2 && ep <= 1e-4 * fmax(1.0, fabs(e_pol[r])));
    CHECK(er <= 5e-2 && er <= 1e-4 * fmax(1.0, fabs(e_ref[r])));
  }
  CHECK(fabs((double)loss - e_loss[0]) <= 1e-4);
  const double rh = rel_frob(gH, e_dH, nh), rw = rel_frob(gW, e_dW, nw);
  CHECK(rh <= 1e-2 && rw <= 1e-2);
  printf("case ok: loss %.7f (oracle %.7f), dH rel %.2e, dW rel %.2e\n", loss, e_loss[0], rh, rw);
  return 0;
}

int main(int argc, char** argv) {
  if (argc > 1 && strcmp(argv[1], "gpu") == 0) return gpu_step();
  if (argc > 2 && strcmp(argv[1], "case") == 0) return case_step(argv[2]);
  return host_checks();
}
