// Log-sum-exp weights of a block of query rows, and the block's sums of
// them: the one definition both the merge and the plan's mass score use,
// so that the importance w the merge emits and the w the plan computes from
// the cache are the same bits.
//
// DiTango, "Riepilogo Tecnico" -> Metodologia -> 2. State-Centric Parallel
// Runtime, "Composizione dello Stato": a row's output is the composition of
// its units' states, with weights exp(lse_a - L), L = log sum_a exp(lse_a).
// 1. Anchor-Guided Selection Planner, "Modellazione dell'Errore": the
// importance w of unit a is the mean of that weight (its share of the
// row's softmax denominator) over the rows of its query partition.
//
// Arithmetic of one row, states a = 0 .. n-1 in ascending unit order:
//   M  = max_a lse_a;  Ms = M if finite, else 0 (a row with no state)
//   e_a = expf(lse_a - Ms)
//   S  = a fixed binary tree over 64 leaves e_0 .. e_63 (absent states are
//        +0): level sums t[a] + t[a + h] for h = 32, 16, 8, 4, 2, 1
//   share_a = e_a * (1 / S)  (0 for a row with no state)
//   L  = Ms + logf(S)  (-inf for a row with no state)
// Block sums: a block covers kWRows consecutive rows of one (b*h, query
// partition); a unit's sum is ((x_l + x_{l+32}) + x_{l+64}) + x_{l+96} per
// lane l, then a butterfly over the 32 lanes (rows past the partition's end
// hold 0).  Everything is in a fixed order: no atomics.
#pragma once

#include "common.cuh"

namespace ditango {
namespace weights {

constexpr int kWRows = 128;   // rows per block: the chunk of the mass sums

// Row t of the block: lse of n states (src_lse[a][row]) -> their shares in
// sh[a * kWRows + t] (shared memory, n <= 64) and the row's L.  A row past
// the end of the partition (live = false) gets shares 0 for every state.
__device__ __forceinline__ float row_shares(const float *const *src_lse, int n, int row, bool live,
                                            float *sh, int t) {
  if (!live) {
    for (int a = 0; a < n; ++a) sh[a * kWRows + t] = 0.f;
    return -INFINITY;
  }
  float M = -INFINITY;
  for (int a = 0; a < n; ++a) {
    const float l = __ldg(src_lse[a] + row);
    sh[a * kWRows + t] = l;
    M = fmaxf(M, l);
  }
  const bool dead = !(M > -INFINITY);
  const float Ms = dead ? 0.f : M;
  for (int a = 0; a < n; ++a) sh[a * kWRows + t] = expf(sh[a * kWRows + t] - Ms);
  // fixed tree over 64 leaves; leaves a >= n are +0 (adding them is exact)
  float s[32];
#pragma unroll
  for (int a = 0; a < 32; ++a) {
    const float lo = (a < n) ? sh[a * kWRows + t] : 0.f;
    const float hi = (a + 32 < n) ? sh[(a + 32) * kWRows + t] : 0.f;
    s[a] = lo + hi;
  }
#pragma unroll
  for (int h = 16; h >= 1; h >>= 1)
#pragma unroll
    for (int a = 0; a < h; ++a) s[a] = s[a] + s[a + h];
  const float S = s[0];
  const float inv = dead ? 0.f : 1.f / S;
  for (int a = 0; a < n; ++a) sh[a * kWRows + t] = sh[a * kWRows + t] * inv;
  return dead ? -INFINITY : Ms + logf(S);
}

// Sum of x[0 .. kWRows) in the block-sum order; called by a whole warp,
// every lane returns the sum.
__device__ __forceinline__ float block_sum(const float *x, int lane) {
  float v = ((x[lane] + x[lane + 32]) + x[lane + 64]) + x[lane + 96];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Layout of the block sums ("mass partials"): float32
// [P][B*H][nrb][G + 1], nrb = ceil(Lmax / kWRows); column c < G is unit
// (i, c)'s sum of shares over the block's rows, column G the sum of the
// local drift rows (error planner).  Entries of blocks past a partition's
// end and of masked units are never read.
__host__ __device__ inline int n_row_blocks(int Lmax) { return (Lmax + kWRows - 1) / kWRows; }
__host__ __device__ inline size_t partial_index(const DevGeom &g, int i, int bh, int rb, int col) {
  return (((size_t)i * g.BH + bh) * n_row_blocks(g.Lmax) + rb) * (size_t)(g.G + 1) + col;
}
// Floats of the block sums (the mass partials a merge writes).
__host__ __device__ inline size_t n_partials(const DevGeom &g) {
  return (size_t)g.P * g.BH * n_row_blocks(g.Lmax) * (size_t)(g.G + 1);
}

}  // namespace weights
}  // namespace ditango
