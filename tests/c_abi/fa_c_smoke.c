/* Plain-C use of the exact-attention library: no torch, no C++.
 *
 * Builds Q, K, V (bf16, [B, N, H, d]) on the host from a closed formula,
 * copies them to device buffers from cudaMalloc, calls fa_fwd, checks the
 * device error word, and prints O (as raw bf16 bits) and LSE (as float bits)
 * in hexadecimal, one value per line, so a caller can compare them exactly
 * with another route to the same library.
 *
 * Usage: fa_c_smoke B N H d causal   (d must be 64 or 128)
 * Exit status: 0 on success, 1 on a bad argument, 2 on a library error,
 * 3 on a CUDA runtime error. */
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "fa.h"

/* float -> bf16 bits, round to nearest even (finite inputs) */
static uint16_t to_bf16(float x) {
  uint32_t u;
  memcpy(&u, &x, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* the input value of tensor `which` (0 q, 1 k, 2 v) at flat index i: an
 * integer pattern divided by 1024, exact in float, so any other program can
 * build bitwise the same inputs */
float input_value(int which, long i) {
  const long k = (i * 7919L + 104729L * which) % 2001L;
  return (float)(k - 1000) / 1024.0f;
}

int main(int argc, char** argv) {
  if (argc != 6) {
    fprintf(stderr, "usage: %s B N H d causal\n", argv[0]);
    return 1;
  }
  const int B = atoi(argv[1]), N = atoi(argv[2]), H = atoi(argv[3]), d = atoi(argv[4]), causal = atoi(argv[5]);
  if (B < 1 || N < 1 || H < 1 || (d != 64 && d != 128)) return 1;
  const long n = (long)B * N * H * d, nl = (long)B * H * N;
  uint16_t* host = (uint16_t*)malloc((size_t)n * 2);
  float* lse_h = (float*)malloc((size_t)nl * 4);
  void *q, *k, *v, *o;
  float* lse;
  if (cudaMalloc(&q, n * 2) || cudaMalloc(&k, n * 2) || cudaMalloc(&v, n * 2) || cudaMalloc(&o, n * 2) ||
      cudaMalloc((void**)&lse, nl * 4))
    return 3;
  void* dst[3] = {q, k, v};
  for (int w = 0; w < 3; ++w) {
    for (long i = 0; i < n; ++i) host[i] = to_bf16(input_value(w, i));
    if (cudaMemcpy(dst[w], host, (size_t)n * 2, cudaMemcpyHostToDevice)) return 3;
  }
  fa_status st = fa_fwd(q, k, v, o, lse, B, N, H, d, 1.0f / sqrtf((float)d), causal, NULL);
  if (st != FA_OK) {
    fprintf(stderr, "fa_fwd: %s\n", fa_status_string(st));
    return 2;
  }
  st = fa_get_device_error(NULL);
  if (st != FA_OK) {
    fprintf(stderr, "device: %s\n", fa_status_string(st));
    return 2;
  }
  if (cudaMemcpy(host, o, (size_t)n * 2, cudaMemcpyDeviceToHost) ||
      cudaMemcpy(lse_h, lse, (size_t)nl * 4, cudaMemcpyDeviceToHost))
    return 3;
  for (long i = 0; i < n; ++i) printf("%04x\n", host[i]);
  for (long i = 0; i < nl; ++i) {
    uint32_t u;
    memcpy(&u, &lse_h[i], 4);
    printf("%08x\n", u);
  }
  cudaFree(q);
  cudaFree(k);
  cudaFree(v);
  cudaFree(o);
  cudaFree(lse);
  free(host);
  free(lse_h);
  return 0;
}
