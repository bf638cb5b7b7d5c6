/* The allocation-free plan across a device reset, from plain C.
 *
 * ditango_plan_noalloc keeps the device address of the library's fixed
 * scratch array between calls.  cudaDeviceReset destroys the context that
 * address belongs to; the next call must look the address up again in the
 * new context instead of launching on freed memory.  Each round: upload a
 * seeded cache lse, plan with ditango_plan (caller workspace) and with
 * ditango_plan_noalloc, require identical plans, fresh lists, counts and
 * scores, free everything and reset the device.
 * usage: noalloc_reset   (exit 0 = equal in every round) */
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

enum { B = 1, H = 4, P = 8, LP = 512, N = P * LP, D = 64, UNITS = P * P };

/* uniform in [-4, 4) from a 64-bit LCG (Knuth's MMIX constants) */
static float next_val(unsigned long long *s) {
  *s = *s * 6364136223846793005ULL + 1442695040888963407ULL;
  return (float)((double)(*s >> 11) * (1.0 / 9007199254740992.0) * 8.0 - 4.0);
}

static int one_round(const ditango_geom *g, int round) {
  const size_t slots = (size_t)ditango_num_active(g);
  const size_t rows = (size_t)B * H * (size_t)ditango_state_rows(g);
  const size_t nlse = slots * rows;
  float *h_lse = (float *)malloc(nlse * sizeof(float));
  if (!h_lse) return 4;
  unsigned long long seed = 0x9e3779b97f4a7c15ULL + (unsigned long long)round;
  for (size_t k = 0; k < nlse; ++k) h_lse[k] = next_val(&seed);

  const size_t nws = ditango_plan_workspace_size(g);
  float *lse = NULL;
  void *ws = NULL;
  int8_t *plan[2] = {NULL, NULL};
  int32_t *fresh[2] = {NULL, NULL}, *counts[2] = {NULL, NULL};
  float *score[2] = {NULL, NULL};
  CK(cudaMalloc((void **)&lse, nlse * sizeof(float)));
  CK(cudaMalloc(&ws, nws));
  for (int k = 0; k < 2; ++k) {
    CK(cudaMalloc((void **)&plan[k], UNITS));
    CK(cudaMalloc((void **)&fresh[k], slots * sizeof(int32_t)));
    CK(cudaMalloc((void **)&counts[k], 2 * sizeof(int32_t)));
    CK(cudaMalloc((void **)&score[k], UNITS * sizeof(float)));
    CK(cudaMemset(plan[k], 0x7f, UNITS));
    CK(cudaMemset(fresh[k], 0x7f, slots * sizeof(int32_t)));
    CK(cudaMemset(counts[k], 0x7f, 2 * sizeof(int32_t)));
    CK(cudaMemset(score[k], 0x7f, UNITS * sizeof(float)));
  }
  CK(cudaMemcpy(lse, h_lse, nlse * sizeof(float), cudaMemcpyHostToDevice));
  DK(ditango_plan(g, lse, NULL, 1, 0.5, 0, plan[0], fresh[0], counts[0], score[0], ws, nws, NULL));
  DK(ditango_plan_noalloc(g, lse, NULL, 1, 0.5, 0, plan[1], fresh[1], counts[1], score[1], NULL));
  CK(cudaDeviceSynchronize());

  int8_t hp[2][UNITS];
  int32_t hc[2][2], hf[2][UNITS];
  float hs[2][UNITS];
  for (int k = 0; k < 2; ++k) {
    CK(cudaMemcpy(hp[k], plan[k], UNITS, cudaMemcpyDeviceToHost));
    CK(cudaMemcpy(hc[k], counts[k], sizeof(hc[k]), cudaMemcpyDeviceToHost));
    CK(cudaMemcpy(hf[k], fresh[k], slots * sizeof(int32_t), cudaMemcpyDeviceToHost));
    CK(cudaMemcpy(hs[k], score[k], sizeof(hs[k]), cudaMemcpyDeviceToHost));
  }
  int bad = memcmp(hp[0], hp[1], UNITS) != 0 || memcmp(hc[0], hc[1], sizeof(hc[0])) != 0 ||
            memcmp(hs[0], hs[1], sizeof(hs[0])) != 0;
  if (!bad && (hc[0][0] < 0 || hc[0][0] > (int32_t)slots)) bad = 1;
  if (!bad && memcmp(hf[0], hf[1], (size_t)hc[0][0] * sizeof(int32_t)) != 0) bad = 1;
  printf("round %d: fresh %d reuse %d %s\n", round, hc[0][0], hc[0][1], bad ? "DIFFER" : "equal");

  for (int k = 0; k < 2; ++k) {
    CK(cudaFree(plan[k]));
    CK(cudaFree(fresh[k]));
    CK(cudaFree(counts[k]));
    CK(cudaFree(score[k]));
  }
  CK(cudaFree(lse));
  CK(cudaFree(ws));
  free(h_lse);
  return bad ? 1 : 0;
}

int main(void) {
  int32_t off[P + 1];
  for (int p = 0; p <= P; ++p) off[p] = p * LP;
  ditango_geom g;
  memset(&g, 0, sizeof(g));
  g.B = B; g.H = H; g.N = N; g.d = D; g.P = P; g.F = 0;
  g.part_off = off;
  g.q_strides[0] = g.k_strides[0] = g.v_strides[0] = (int64_t)H * N * D;
  g.q_strides[1] = g.k_strides[1] = g.v_strides[1] = (int64_t)N * D;
  g.q_strides[2] = g.k_strides[2] = g.v_strides[2] = D;
  for (int round = 0; round < 3; ++round) {
    const int rc = one_round(&g, round);
    if (rc != 0) return rc;
    CK(cudaDeviceReset());   /* a new context for the next round */
  }
  return 0;
}
