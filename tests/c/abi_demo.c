/*
 * abi_demo.c -- the sparse FFN forward called from plain C through the C ABI
 * (include/sfn.h, libsfn.so) with the CUDA runtime for device memory.
 *
 * usage: abi_demo <inputs.bin> <outputs.bin>
 *   inputs.bin : int64 T, d, d_i, r, bank, k, then float32 x [T][d], A [r][d],
 *                B [d_i][r], Wg, Wu, Wd [d_i][d]
 *   outputs.bin: float32 y [T][d], then uint64 mask [T][d_i/bank]
 * Runs sfn_sparse_ffn_forward_f32_ws on a caller-owned stream and scratch.
 * Exit status 0 on success; the caller compares the outputs with the oracle.
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include <cuda_runtime.h>

#include "sfn.h"

static int fail(const char *what, int code) {
  fprintf(stderr, "abi_demo: %s (%d)\n", what, code);
  return 1;
}

int main(int argc, char **argv) {
  if (argc != 3) return fail("usage: abi_demo <inputs.bin> <outputs.bin>", 0);
  FILE *fi = fopen(argv[1], "rb");
  if (!fi) return fail("cannot open inputs", 0);
  int64_t dims[6];
  if (fread(dims, sizeof dims, 1, fi) != 1) return fail("short header", 0);
  const int64_t T = dims[0];
  const int d = (int)dims[1], d_i = (int)dims[2], r = (int)dims[3];
  const int bank = (int)dims[4], k = (int)dims[5];
  const size_t n[6] = {(size_t)T * d, (size_t)r * d, (size_t)d_i * r,
                       (size_t)d_i * d, (size_t)d_i * d, (size_t)d_i * d};
  void *dev[6];
  for (int i = 0; i < 6; ++i) {
    float *h = (float *)malloc(n[i] * sizeof(float));
    if (!h || fread(h, sizeof(float), n[i], fi) != n[i]) return fail("short input", i);
    if (cudaMalloc(&dev[i], n[i] * sizeof(float)) != cudaSuccess) return fail("cudaMalloc", i);
    cudaMemcpy(dev[i], h, n[i] * sizeof(float), cudaMemcpyHostToDevice);
    free(h);
  }
  fclose(fi);
  const int n_banks = d_i / bank;
  void *y, *mask, *ws;
  const size_t ws_bytes = sfn_workspace_bytes(T, d, d_i, r, bank, k, SFN_DTYPE_F32);
  if (cudaMalloc(&y, (size_t)T * d * sizeof(float)) != cudaSuccess ||
      cudaMalloc(&mask, (size_t)T * n_banks * sizeof(uint64_t)) != cudaSuccess ||
      cudaMalloc(&ws, ws_bytes ? ws_bytes : 1) != cudaSuccess)
    return fail("cudaMalloc outputs", 0);
  cudaStream_t st;
  cudaStreamCreate(&st);
  const sfn_status s = sfn_sparse_ffn_forward_f32_ws(
      (const float *)dev[0], (const float *)dev[1], (const float *)dev[2],
      (const float *)dev[3], (const float *)dev[4], (const float *)dev[5], (float *)y,
      (uint64_t *)mask, T, d, d_i, r, bank, k, ws, ws_bytes, (sfn_stream_t)st);
  if (s != SFN_OK) return fail(sfn_status_string(s), (int)s);
  if (cudaStreamSynchronize(st) != cudaSuccess) return fail("stream", 0);
  float *yh = (float *)malloc((size_t)T * d * sizeof(float));
  uint64_t *mh = (uint64_t *)malloc((size_t)T * n_banks * sizeof(uint64_t));
  cudaMemcpy(yh, y, (size_t)T * d * sizeof(float), cudaMemcpyDeviceToHost);
  cudaMemcpy(mh, mask, (size_t)T * n_banks * sizeof(uint64_t), cudaMemcpyDeviceToHost);
  FILE *fo = fopen(argv[2], "wb");
  if (!fo) return fail("cannot open outputs", 0);
  fwrite(yh, sizeof(float), (size_t)T * d, fo);
  fwrite(mh, sizeof(uint64_t), (size_t)T * n_banks, fo);
  fclose(fo);
  printf("abi_demo: T=%lld d=%d d_i=%d abi=%d ok\n", (long long)T, d, d_i, sfn_abi_version());
  return 0;
}
