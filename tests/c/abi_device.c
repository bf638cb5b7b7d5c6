/* A whole anchor step through the C ABI from plain C on the GPU (CUDA
 * runtime for memory, no Python): plan -> partial attention into the cache
 * slots -> merge.  Reads Q, K, V (bf16 bits, [B, H, N, d]) from files, writes
 * the fp32 output and lse to files for the caller to check.
 * usage: abi_device <dir>  (dir holds q.bin k.bin v.bin; gets out.bin lse.bin)
 * Geometry: B = 1, H = 2, N = 1024, d = 64, 4 partitions of 256. */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime.h>

#include "ditango.h"

#define CK(x)                                                        \
  do {                                                               \
    cudaError_t e_ = (x);                                            \
    if (e_ != cudaSuccess) {                                         \
      fprintf(stderr, "%s: %s\n", #x, cudaGetErrorString(e_));       \
      return 2;                                                      \
    }                                                                \
  } while (0)
#define DK(x)                                                        \
  do {                                                               \
    ditango_status s_ = (x);                                         \
    if (s_ != DITANGO_OK) {                                          \
      fprintf(stderr, "%s: %s\n", #x, ditango_status_string(s_));    \
      return 3;                                                      \
    }                                                                \
  } while (0)

static int read_file(const char *dir, const char *name, void *buf, size_t n) {
  char path[4096];
  snprintf(path, sizeof(path), "%s/%s", dir, name);
  FILE *f = fopen(path, "rb");
  if (!f) return 1;
  const size_t got = fread(buf, 1, n, f);
  fclose(f);
  return got != n;
}

static int write_file(const char *dir, const char *name, const void *buf, size_t n) {
  char path[4096];
  snprintf(path, sizeof(path), "%s/%s", dir, name);
  FILE *f = fopen(path, "wb");
  if (!f) return 1;
  const size_t put = fwrite(buf, 1, n, f);
  fclose(f);
  return put != n;
}

int main(int argc, char **argv) {
  if (argc < 2) return 1;
  enum { B = 1, H = 2, N = 1024, D = 64, P = 4 };
  int32_t off[P + 1] = {0, 256, 512, 768, 1024};
  ditango_geom g;
  memset(&g, 0, sizeof(g));
  g.B = B; g.H = H; g.N = N; g.d = D; g.P = P; g.F = 0;
  g.part_off = off;
  for (int k = 0; k < 3; ++k)
    g.q_strides[k] = g.k_strides[k] = g.v_strides[k] =
        k == 0 ? (int64_t)H * N * D : (k == 1 ? (int64_t)N * D : D);
  const int64_t slots = ditango_num_active(&g), Lmax = ditango_state_rows(&g);
  const size_t nqkv = (size_t)B * H * N * D;
  uint16_t *hq = malloc(nqkv * 2), *hk = malloc(nqkv * 2), *hv = malloc(nqkv * 2);
  float *hout = malloc(nqkv * 4), *hlse = malloc((size_t)B * H * N * 4);
  if (read_file(argv[1], "q.bin", hq, nqkv * 2) || read_file(argv[1], "k.bin", hk, nqkv * 2) ||
      read_file(argv[1], "v.bin", hv, nqkv * 2))
    return 4;
  uint16_t *q, *k, *v;
  float *sO, *slse, *out, *olse;
  uint8_t *valid;
  int8_t *plan;
  int32_t *fresh, *counts, *status, *work;
  CK(cudaMalloc((void **)&q, nqkv * 2));
  CK(cudaMalloc((void **)&k, nqkv * 2));
  CK(cudaMalloc((void **)&v, nqkv * 2));
  CK(cudaMalloc((void **)&sO, (size_t)slots * B * H * Lmax * D * 4));
  CK(cudaMalloc((void **)&slse, (size_t)slots * B * H * Lmax * 4));
  CK(cudaMalloc((void **)&valid, slots));
  CK(cudaMalloc((void **)&plan, P * P));
  CK(cudaMalloc((void **)&fresh, slots * 4));
  CK(cudaMalloc((void **)&counts, 8));
  CK(cudaMalloc((void **)&status, 4));
  CK(cudaMalloc((void **)&work, 8));
  CK(cudaMalloc((void **)&out, nqkv * 4));
  CK(cudaMalloc((void **)&olse, (size_t)B * H * N * 4));
  CK(cudaMemset(status, 0, 4));
  CK(cudaMemset(work, 0, 8));   /* the attention kernel's work counter, zeroed once */
  CK(cudaMemset(valid, 0, slots));
  CK(cudaMemcpy(q, hq, nqkv * 2, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(k, hk, nqkv * 2, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(v, hv, nqkv * 2, cudaMemcpyHostToDevice));
  cudaStream_t st;
  CK(cudaStreamCreate(&st));
  /* an anchor step: every pair fresh, states written into the cache slots */
  DK(ditango_plan(&g, NULL, valid, 0, 1.0, 1, plan, fresh, counts, NULL, NULL, 0, st));
  DK(ditango_attn_partial(&g, q, k, v, fresh, counts, 0.0f, sO, slse, 1, 0, valid, NULL, status, work,
                          st));
  DK(ditango_merge(&g, plan, NULL, NULL, sO, slse, valid, 0, 0, out, 1, NULL, olse, NULL, st));
  CK(cudaStreamSynchronize(st));
  int32_t hstatus = -1;
  CK(cudaMemcpy(&hstatus, status, 4, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(hout, out, nqkv * 4, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(hlse, olse, (size_t)B * H * N * 4, cudaMemcpyDeviceToHost));
  if (write_file(argv[1], "out.bin", hout, nqkv * 4) || write_file(argv[1], "lse.bin", hlse, (size_t)B * H * N * 4))
    return 5;
  printf("status %d slots %lld\n", hstatus, (long long)slots);
  return hstatus != 0;
}
