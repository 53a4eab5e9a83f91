/*
 * The whole path called from C through include/psa.h: pool -> top-k route ->
 * attention, with caller-owned device buffers and a caller stream.
 *
 * usage: psa_from_c B H N d density in.bin out.bin
 *   in.bin  : q, k, v as raw bf16 [B, H, N, d] each, back to back
 *   out.bin : the attention output, raw bf16 [B, H, N, d]
 * Exit status 0 on success; otherwise the failing call and its status text
 * are printed to stderr.
 */
#include <stdio.h>
#include <stdlib.h>

#include <cuda_runtime.h>

#include "psa.h"

#define CHECK_CUDA(x)                                                                   \
  do {                                                                                  \
    cudaError_t e_ = (x);                                                               \
    if (e_ != cudaSuccess) {                                                            \
      fprintf(stderr, "%s: %s\n", #x, cudaGetErrorString(e_));                          \
      return 2;                                                                         \
    }                                                                                   \
  } while (0)

#define CHECK_PSA(x)                                                                    \
  do {                                                                                  \
    int s_ = (x);                                                                       \
    if (s_ != PSA_OK) {                                                                 \
      fprintf(stderr, "%s: %s\n", #x, psa_status_string(s_));                           \
      return 3;                                                                         \
    }                                                                                   \
  } while (0)

int main(int argc, char** argv) {
  if (argc != 8) {
    fprintf(stderr, "usage: %s B H N d density in.bin out.bin\n", argv[0]);
    return 1;
  }
  const int B = atoi(argv[1]), H = atoi(argv[2]), N = atoi(argv[3]), d = atoi(argv[4]);
  const float density = (float)atof(argv[5]);
  const int M = N / 64;
  const size_t n = (size_t)B * H * N * d, m = (size_t)B * H * M;

  psa_bf16_t* host = (psa_bf16_t*)malloc(3 * n * sizeof(psa_bf16_t));
  FILE* f = fopen(argv[6], "rb");
  if (!host || !f || fread(host, sizeof(psa_bf16_t), 3 * n, f) != 3 * n) {
    fprintf(stderr, "cannot read %s\n", argv[6]);
    return 1;
  }
  fclose(f);

  cudaStream_t stream;
  CHECK_CUDA(cudaStreamCreate(&stream));
  psa_bf16_t *q, *k, *v, *out;
  float *qbar, *kbar, *vsum, *row_max;
  int *row_ptr, *col_idx, *nnz;
  void* ws;
  const size_t cap = psa_route_capacity(B, H, M, 0);
  const size_t ws_bytes = psa_workspace_size(B, H, N, d);
  CHECK_CUDA(cudaMalloc((void**)&q, 3 * n * sizeof(psa_bf16_t)));
  k = q + n;
  v = k + n;
  CHECK_CUDA(cudaMalloc((void**)&out, n * sizeof(psa_bf16_t)));
  CHECK_CUDA(cudaMalloc((void**)&qbar, 3 * m * d * sizeof(float)));
  kbar = qbar + m * d;
  vsum = kbar + m * d;
  CHECK_CUDA(cudaMalloc((void**)&row_max, m * sizeof(float)));
  CHECK_CUDA(cudaMalloc((void**)&row_ptr, (m + 1) * sizeof(int)));
  CHECK_CUDA(cudaMalloc((void**)&col_idx, cap * sizeof(int)));
  CHECK_CUDA(cudaMalloc((void**)&nnz, sizeof(int)));
  CHECK_CUDA(cudaMalloc(&ws, ws_bytes));
  CHECK_CUDA(cudaMemcpyAsync(q, host, 3 * n * sizeof(psa_bf16_t), cudaMemcpyHostToDevice, stream));

  CHECK_PSA(psa_pool(q, k, v, B, H, N, d, 64, qbar, kbar, vsum, stream));
  CHECK_PSA(psa_route_topk(qbar, kbar, B, H, M, d, density, 0, row_ptr, col_idx, cap, nnz, row_max, ws,
                           ws_bytes, stream));
  CHECK_PSA(psa_attn(q, k, v, kbar, vsum, row_ptr, col_idx, cap, row_max, B, H, N, d, 64, 0, out, NULL, ws,
                     ws_bytes, stream));
  int device_status = -1;
  CHECK_PSA(psa_read_status(ws, &device_status, stream));
  CHECK_PSA(device_status);

  CHECK_CUDA(cudaMemcpyAsync(host, out, n * sizeof(psa_bf16_t), cudaMemcpyDeviceToHost, stream));
  CHECK_CUDA(cudaStreamSynchronize(stream));
  f = fopen(argv[7], "wb");
  if (!f || fwrite(host, sizeof(psa_bf16_t), n, f) != n) {
    fprintf(stderr, "cannot write %s\n", argv[7]);
    return 1;
  }
  fclose(f);
  printf("ok: psa version %d\n", psa_version());
  cudaFree(q);
  cudaFree(out);
  cudaFree(qbar);
  cudaFree(row_max);
  cudaFree(row_ptr);
  cudaFree(col_idx);
  cudaFree(nnz);
  cudaFree(ws);
  cudaStreamDestroy(stream);
  free(host);
  return 0;
}
