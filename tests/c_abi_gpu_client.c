/* A plain C user of libkca.so on the GPU, built and run by
 * tests/test_c_abi_gpu.py: device memory from the CUDA runtime, the library
 * through include/kca.h alone.  It reads its inputs from files the test
 * wrote (the seeded draws, in their stored formats), runs one chunked
 * prefill (bf16, 300 rows at position 1000 of a 1300-row cache) and one
 * decode batch (f32 queries, f16 cache of 5000 rows, contexts 5000 and 77),
 * checks every status, and writes the f32 outputs back for the test to
 * compare with the oracle.
 * usage: c_abi_gpu_client DIR */
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include "kca.h"

static char g_dir[4096];

static void *load(const char *name, size_t bytes) {
  char path[4200];
  snprintf(path, sizeof path, "%s/%s", g_dir, name);
  FILE *f = fopen(path, "rb");
  void *h = malloc(bytes);
  if (f == NULL || h == NULL || fread(h, 1, bytes, f) != bytes) {
    fprintf(stderr, "cannot read %s\n", path);
    exit(2);
  }
  fclose(f);
  return h;
}

static void save(const char *name, const void *h, size_t bytes) {
  char path[4200];
  snprintf(path, sizeof path, "%s/%s", g_dir, name);
  FILE *f = fopen(path, "wb");
  if (f == NULL || fwrite(h, 1, bytes, f) != bytes) {
    fprintf(stderr, "cannot write %s\n", path);
    exit(2);
  }
  fclose(f);
}

static void *to_device(const void *h, size_t bytes) {
  void *d = NULL;
  if (cudaMalloc(&d, bytes) != cudaSuccess || cudaMemcpy(d, h, bytes, cudaMemcpyHostToDevice) != cudaSuccess) {
    fprintf(stderr, "device copy failed\n");
    exit(3);
  }
  return d;
}

static void check(const char *what, int status) {
  printf("%s %d %s\n", what, status, attn_status_string(status));
  if (status != KCA_OK) exit(4);
}

int main(int argc, char **argv) {
  if (argc != 2) return 1;
  snprintf(g_dir, sizeof g_dir, "%s", argv[1]);
  const float scale = 1.0f / 16.0f;

  /* chunked prefill: bf16 Q / K / V */
  const int64_t cs = 1000, cap = 1300;
  const int32_t rows = 300;
  const size_t qb = (size_t)rows * 8 * 256 * 2, kb = (size_t)cap * 256 * 2, ob = (size_t)rows * 8 * 256 * 4;
  void *q = to_device(load("q.bin", qb), qb);
  void *k = to_device(load("k.bin", kb), kb);
  void *v = to_device(load("v.bin", kb), kb);
  const size_t wsb = attn_prefill_workspace_bytes(KCA_BF16, KCA_BF16, cs, rows, 0);
  void *ws = NULL;
  float *out = NULL;
  if (wsb == 0 || cudaMalloc(&ws, wsb) != cudaSuccess || cudaMalloc((void **)&out, ob) != cudaSuccess) return 3;
  check("workspace_init", attn_workspace_init(ws, wsb, NULL));
  check("prefill", attn_prefill(q, KCA_BF16, k, v, KCA_BF16, 8, 1, 256, cap, cs, rows, cs + rows, 0, scale, out, ws,
                                wsb, NULL));
  uint32_t detail = 0;
  check("prefill_device_status", attn_device_status(ws, NULL, &detail));
  void *h = malloc(ob);
  if (h == NULL || cudaMemcpy(h, out, ob, cudaMemcpyDeviceToHost) != cudaSuccess) return 3;
  save("out_prefill.bin", h, ob);

  /* decode: f32 queries over an f16 cache of two sequences */
  const int64_t dcap = 5000, ctx[2] = {5000, 77};
  const size_t dqb = 2 * 8 * 256 * 4, dkb = (size_t)2 * dcap * 256 * 2, dob = 2 * 8 * 256 * 4;
  void *dq = to_device(load("dq.bin", dqb), dqb);
  void *dk = to_device(load("dk.bin", dkb), dkb);
  void *dv = to_device(load("dv.bin", dkb), dkb);
  const size_t dwsb = attn_decode_workspace_bytes(2, ctx, 0);
  void *dws = NULL;
  float *dout = NULL;
  if (dwsb == 0 || cudaMalloc(&dws, dwsb) != cudaSuccess || cudaMalloc((void **)&dout, dob) != cudaSuccess) return 3;
  check("decode_workspace_init", attn_workspace_init(dws, dwsb, NULL));
  check("decode", attn_decode(dq, KCA_F32, dk, dv, KCA_F16, 8, 1, 256, dcap, 2, ctx, 0, scale, dout, dws, dwsb,
                              NULL));
  check("decode_device_status", attn_device_status(dws, NULL, &detail));
  void *hd = malloc(dob);
  if (hd == NULL || cudaMemcpy(hd, dout, dob, cudaMemcpyDeviceToHost) != cudaSuccess) return 3;
  save("out_decode.bin", hd, dob);
  printf("done\n");
  return 0;
}
