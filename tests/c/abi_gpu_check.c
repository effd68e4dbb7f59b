/* The whole path from plain C on a GPU: device buffers from the CUDA runtime, one
 * fused_norm_launch, results copied back. LayerNorm with a broadcast gate, a bf16 weight
 * and per-token scale and shift, B = 1, L rows of D = 5120.
 *
 *   abi_gpu_check <L> <inputs.bin> <outputs.bin>
 *
 * The inputs (x, residual, gate, weight, scale, shift as bf16 bit patterns, in that order)
 * are drawn from a fixed 64-bit linear congruential sequence and written to inputs.bin;
 * y and r are written to outputs.bin, for the caller to compare with an independent
 * evaluation of the same inputs. Exit status 0 when every CUDA and library call succeeded.
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "fused_norm.h"

enum { D = 5120 };

static uint64_t state = 0x2545F4914F6CDD1Dull;

/* A value of about the given magnitude as a bf16 bit pattern: a uniform draw in
 * [-scale, scale) plus an offset, truncated to the top 16 bits of its binary32 form. */
static uint16_t draw(float offset, float scale) {
  state = state * 6364136223846793005ull + 1442695040888963407ull;
  const float u = (float)((state >> 40) & 0xFFFFFF) / 16777216.0f;  /* [0, 1) */
  const float v = offset + scale * (2.0f * u - 1.0f);
  uint32_t bits;
  memcpy(&bits, &v, sizeof(bits));
  return (uint16_t)(bits >> 16);
}

static int cuda_ok(cudaError_t e, const char* what) {
  if (e != cudaSuccess) {
    fprintf(stderr, "%s: %s\n", what, cudaGetErrorString(e));
    return 0;
  }
  return 1;
}

int main(int argc, char** argv) {
  if (argc != 4) {
    fprintf(stderr, "usage: %s L inputs.bin outputs.bin\n", argv[0]);
    return 2;
  }
  const int64_t L = atoll(argv[1]);
  if (L < 1 || L > 100000) return 2;
  const size_t row = (size_t)D * 2, full = (size_t)L * row;

  /* host inputs: x, residual (L rows), gate (1 row), weight (1 row), scale, shift (L rows) */
  const size_t n_host = 4 * full + 2 * row;
  uint16_t* h = (uint16_t*)malloc(n_host);
  uint16_t* out = (uint16_t*)malloc(2 * full);
  if (!h || !out) return 3;
  uint16_t *hx = h, *hres = hx + L * D, *hgate = hres + L * D, *hw = hgate + D;
  uint16_t *hs = hw + D, *ht = hs + L * D;
  for (int64_t i = 0; i < L * D; ++i) hx[i] = draw(0.0f, 1.7f);
  for (int64_t i = 0; i < L * D; ++i) hres[i] = draw(0.0f, 1.7f);
  for (int i = 0; i < D; ++i) hgate[i] = draw(0.0f, 0.8f);
  for (int i = 0; i < D; ++i) hw[i] = draw(1.0f, 0.2f);
  for (int64_t i = 0; i < L * D; ++i) hs[i] = draw(0.0f, 0.2f);
  for (int64_t i = 0; i < L * D; ++i) ht[i] = draw(0.0f, 0.2f);

  void *dbuf = NULL, *dout = NULL;
  if (!cuda_ok(cudaMalloc(&dbuf, n_host), "cudaMalloc inputs")) return 4;
  if (!cuda_ok(cudaMalloc(&dout, 2 * full), "cudaMalloc outputs")) return 4;
  if (!cuda_ok(cudaMemcpy(dbuf, h, n_host, cudaMemcpyHostToDevice), "copy in")) return 4;
  uint16_t* d = (uint16_t*)dbuf;

  fn_config cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.D = D;
  cfg.has_gate = 1;
  cfg.has_weight = 1;
  cfg.eps = 1e-6;
  fused_norm_t handle = NULL;
  fn_status st = fused_norm_create(&handle, &cfg);
  if (st != FN_OK) {
    fprintf(stderr, "create: %s\n", fused_norm_status_string(st));
    return 5;
  }

  fn_args a;
  memset(&a, 0, sizeof(a));
  a.B = 1;
  a.L = L;
  a.x.ptr = d;
  a.x.stride_l = D;
  a.residual.ptr = d + L * D;
  a.residual.stride_l = D;
  a.gate.ptr = d + 2 * L * D;                 /* broadcast: all strides 0 */
  a.weight = d + 2 * L * D + D;
  a.scale.ptr = d + 2 * L * D + 2 * D;
  a.scale.stride_l = D;
  a.shift.ptr = d + 3 * L * D + 2 * D;
  a.shift.stride_l = D;
  a.y = dout;
  a.y_stride_b = L * D;
  a.y_stride_l = D;
  a.r = (uint16_t*)dout + L * D;
  a.r_stride_b = L * D;
  a.r_stride_l = D;

  cudaStream_t stream;
  if (!cuda_ok(cudaStreamCreate(&stream), "stream")) return 4;
  st = fused_norm_launch(handle, &a, (fn_stream_t)stream);
  if (st != FN_OK) {
    fprintf(stderr, "launch: %s (cuda %d)\n", fused_norm_status_string(st), fused_norm_last_cuda_error());
    return 5;
  }
  if (!cuda_ok(cudaStreamSynchronize(stream), "synchronize")) return 4;
  if (!cuda_ok(cudaMemcpy(out, dout, 2 * full, cudaMemcpyDeviceToHost), "copy out")) return 4;

  FILE* fi = fopen(argv[2], "wb");
  FILE* fo = fopen(argv[3], "wb");
  if (!fi || !fo) return 6;
  if (fwrite(h, 1, n_host, fi) != n_host || fwrite(out, 1, 2 * full, fo) != 2 * full) return 6;
  fclose(fi);
  fclose(fo);

  fused_norm_destroy(handle);
  cudaStreamDestroy(stream);
  cudaFree(dbuf);
  cudaFree(dout);
  free(h);
  free(out);
  printf("ok %lld rows\n", (long long)L);
  return 0;
}
