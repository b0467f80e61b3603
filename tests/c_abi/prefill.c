/*
 * prefill.c -- the prefill step driven from plain C through include/xattn.h
 * alone: device buffers from the CUDA runtime, the two calls of the fused
 * path (xattn_score_select, xattn_sparse_attn), and the error path.
 *
 *   prefill <in.bin> <out.bin> batch hq hkv L d B S causal tau
 *
 * in.bin holds Q, K, V as raw bf16 [batch, heads, L, d], one after another;
 * out.bin receives O (raw bf16, same layout as Q). Exit status 0 on success;
 * every failure prints the call and its status text.
 */
#include <stdio.h>
#include <stdlib.h>

#include <cuda_runtime_api.h>

#include "xattn.h"

#define CHECK_CUDA(x)                                                     \
  do {                                                                    \
    cudaError_t e_ = (x);                                                 \
    if (e_ != cudaSuccess) {                                              \
      fprintf(stderr, "%s: %s\n", #x, cudaGetErrorString(e_));            \
      return 2;                                                           \
    }                                                                     \
  } while (0)

#define CHECK_XATTN(x)                                                    \
  do {                                                                    \
    int s_ = (x);                                                         \
    if (s_ != XATTN_OK) {                                                 \
      fprintf(stderr, "%s: %s (%d)\n", #x, xattn_strerror(s_), s_);       \
      return 3;                                                           \
    }                                                                     \
  } while (0)

int main(int argc, char** argv) {
  if (argc != 12) {
    fprintf(stderr, "usage: prefill in.bin out.bin batch hq hkv L d B S causal tau\n");
    return 1;
  }
  xattn_shape sh;
  sh.batch = atoi(argv[3]);
  sh.hq = atoi(argv[4]);
  sh.hkv = atoi(argv[5]);
  sh.L = atoi(argv[6]);
  sh.d = atoi(argv[7]);
  sh.B = atoi(argv[8]);
  sh.S = atoi(argv[9]);
  sh.causal = atoi(argv[10]);
  sh.dtype = XATTN_BF16;
  const float tau1 = (float)atof(argv[11]);

  /* the error path first: a length that is not a multiple of S is refused
     before anything runs */
  xattn_shape bad = sh;
  bad.L = sh.L + 1;
  if (xattn_score_workspace_bytes(&bad) != 0 ||
      xattn_score(NULL, NULL, &bad, NULL, NULL, 0, NULL) != XATTN_ERR_INVALID_ARG) {
    fprintf(stderr, "bad shape not refused\n");
    return 4;
  }

  const size_t nq = (size_t)sh.batch * sh.hq * sh.L * sh.d;
  const size_t nkv = (size_t)sh.batch * sh.hkv * sh.L * sh.d;
  const int NB = (sh.L + sh.B - 1) / sh.B;
  const size_t rows = (size_t)sh.batch * sh.hq * NB;
  unsigned short* host = (unsigned short*)malloc((nq + 2 * nkv) * 2);
  float* tau = (float*)malloc(sizeof(float) * sh.hq);
  if (!host || !tau) return 5;
  for (int h = 0; h < sh.hq; ++h) tau[h] = tau1;
  FILE* f = fopen(argv[1], "rb");
  if (!f || fread(host, 2, nq + 2 * nkv, f) != nq + 2 * nkv) {
    fprintf(stderr, "cannot read %s\n", argv[1]);
    return 6;
  }
  fclose(f);

  void *Q, *K, *V, *O, *ws_s, *ws_a;
  uint32_t* mask;
  int32_t *counts, *idx;
  const size_t ws_s_bytes = xattn_score_workspace_bytes(&sh);
  const size_t ws_a_bytes = xattn_attn_workspace_bytes(&sh);
  if (ws_s_bytes == 0 || ws_a_bytes == 0) {
    fprintf(stderr, "shape refused\n");
    return 7;
  }
  CHECK_CUDA(cudaMalloc(&Q, nq * 2));
  CHECK_CUDA(cudaMalloc(&K, nkv * 2));
  CHECK_CUDA(cudaMalloc(&V, nkv * 2));
  CHECK_CUDA(cudaMalloc(&O, nq * 2));
  CHECK_CUDA(cudaMalloc(&ws_s, ws_s_bytes));
  CHECK_CUDA(cudaMalloc(&ws_a, ws_a_bytes));
  CHECK_CUDA(cudaMalloc((void**)&mask, rows * ((NB + 31) / 32) * 4));
  CHECK_CUDA(cudaMalloc((void**)&counts, rows * 4));
  CHECK_CUDA(cudaMalloc((void**)&idx, rows * NB * 4));
  CHECK_CUDA(cudaMemcpy(Q, host, nq * 2, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(K, host + nq, nkv * 2, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(V, host + nq + nkv, nkv * 2, cudaMemcpyHostToDevice));

  cudaStream_t st;
  CHECK_CUDA(cudaStreamCreate(&st));
  /* per-head thresholds live in device memory (the kernels read them there) */
  float* tau_d;
  CHECK_CUDA(cudaMalloc((void**)&tau_d, sizeof(float) * sh.hq));
  CHECK_CUDA(cudaMemcpy(tau_d, tau, sizeof(float) * sh.hq, cudaMemcpyHostToDevice));
  CHECK_XATTN(xattn_score_select(Q, K, &sh, tau_d, NULL, mask, counts, idx, ws_s, ws_s_bytes,
                                 st));
  CHECK_XATTN(xattn_sparse_attn(Q, K, V, &sh, counts, idx, O, NULL, ws_a, ws_a_bytes, st));
  CHECK_XATTN(xattn_get_device_status(st));

  CHECK_CUDA(cudaMemcpy(host, O, nq * 2, cudaMemcpyDeviceToHost));
  f = fopen(argv[2], "wb");
  if (!f || fwrite(host, 2, nq, f) != nq) return 8;
  fclose(f);
  cudaFree(Q); cudaFree(K); cudaFree(V); cudaFree(O); cudaFree(ws_s); cudaFree(ws_a);
  cudaFree(mask); cudaFree(counts); cudaFree(idx); cudaFree(tau_d);
  cudaStreamDestroy(st);
  free(host);
  free(tau);
  printf("ok\n");
  return 0;
}
