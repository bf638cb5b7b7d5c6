// Fresh-versus-reuse plan (DiTango, "Riepilogo Tecnico" -> Metodologia ->
// 1. Anchor-Guided Selection Planner).
//
// The candidates are units (query partition i, KV group c); without KV
// groups a unit is the pair (i, j) ("Strategia per Gruppi": decisions per
// group of adjacent partitions).
// Stage 1 (mass_partial_kernel): importance of each active unit from the
// cached log-sum-exps.  For every cached row r of query partition i the
// share of unit (i, c) in that row's softmax denominator is
//   e_c / sum_c' e_c',  e_c = exp(lse_ic[r] - max_c' lse_ic'[r]),
// and each block sums these shares over a fixed chunk of (b*h, r) rows with
// a fixed-order tree (warp shuffles, then warps in index order).  Invalid
// (never written) slots hold no mass.
// Stage 2 (plan_select_kernel, one block): chunk sums are added in chunk
// order in double precision and divided by the row count (w = mean share),
// then the band, the invalid slots and the top-w units up to the budget are
// marked fresh.  Ranking sorts 64-bit keys (~bits(w) << 32 | i*G + c) with a
// bitonic network: larger w first, ties to the lower linear index.
// Error mode (DiTango, "Modellazione dell'Errore", "Predizione Online"):
// stage 1 also sums each partition's local drift rows (written by the
// attention kernel) into the extra column G of the chunk sums; stage 2 turns
// them into delta_i, ages every cached state (0 if the previous plan made it
// fresh, + delta_i if it reused it) and ranks by w * (age + delta_i), with w
// recomputed only on the step after an anchor and held otherwise.
// Everything is deterministic; no floating-point atomics.
#include "common.cuh"

namespace ditango {
namespace plan {

constexpr int kMassThreads = 256;
constexpr int kRowsPerThread = 4;
constexpr int kRowsPerBlock = kMassThreads * kRowsPerThread;
constexpr int kSelThreads = 1024;

__device__ __forceinline__ float warp_sum_fixed(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Error-mode arguments of the plan (all null in the plain mode).
struct ErrorArgs {
  const float *drift_rows;     // [P][B*H][Lmax]
  float *w;                    // [P*G] importance held between anchors
  float *age;                  // [slots]
  float *delta;                // [P] output
  unsigned char *local_ok;     // [P] read (last step), then rewritten
  int refresh_w;
};

__global__ void __launch_bounds__(kMassThreads)
mass_partial_kernel(DevGeom g, const float *__restrict__ cache_lse,
                    const unsigned char *__restrict__ cache_valid, float *__restrict__ partial,
                    int nchunks_max, int do_mass, const float *__restrict__ drift_rows,
                    const unsigned char *__restrict__ local_ok) {
  const int i = blockIdx.y;
  const int chunk = blockIdx.x;
  const int Li = g.part_off[i + 1] - g.part_off[i];
  const long long nrows = (long long)g.BH * Li;
  const long long row0 = (long long)chunk * kRowsPerBlock;
  if (row0 >= nrows) return;  // uniform per block
  const unsigned long long mask = g.row_mask[i];
  const int nact = __popcll(mask);
  if (nact == 0) return;
  const int s0 = g.row_start[i];
  const int GC = g.G + 1;       // columns of the chunk sums: G units + the drift
  const size_t slot_stride = (size_t)g.BH * g.Lmax;

  // per-thread rows: row0 + threadIdx.x + t * kMassThreads
  long long roff[kRowsPerThread];
  bool rok[kRowsPerThread];
  float rmax[kRowsPerThread], rinv[kRowsPerThread];
#pragma unroll
  for (int t = 0; t < kRowsPerThread; ++t) {
    long long q = row0 + threadIdx.x + (long long)t * kMassThreads;
    rok[t] = q < nrows;
    long long bh = rok[t] ? q / Li : 0;
    long long r = rok[t] ? q - bh * Li : 0;
    roff[t] = bh * g.Lmax + r;
    rmax[t] = -INFINITY;
    rinv[t] = 0.f;
  }
  // pass 1: per-row maximum and denominator over the valid active slots
  const int nact_m = do_mass ? nact : 0;
  for (int a = 0; a < nact_m; ++a) {
    const bool valid = cache_valid == nullptr || cache_valid[s0 + a] != 0;
    if (!valid) continue;
    const float *src = cache_lse + (size_t)(s0 + a) * slot_stride;
#pragma unroll
    for (int t = 0; t < kRowsPerThread; ++t)
      if (rok[t]) rmax[t] = fmaxf(rmax[t], __ldg(src + roff[t]));
  }
  for (int a = 0; a < nact_m; ++a) {
    const bool valid = cache_valid == nullptr || cache_valid[s0 + a] != 0;
    if (!valid) continue;
    const float *src = cache_lse + (size_t)(s0 + a) * slot_stride;
#pragma unroll
    for (int t = 0; t < kRowsPerThread; ++t)
      if (rok[t] && rmax[t] > -INFINITY) rinv[t] += expf(__ldg(src + roff[t]) - rmax[t]);
  }
#pragma unroll
  for (int t = 0; t < kRowsPerThread; ++t) rinv[t] = (rinv[t] > 0.f) ? 1.f / rinv[t] : 0.f;

  // pass 2: per active unit, the block's sum of shares
  __shared__ float warp_part[kMassThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (drift_rows != nullptr) {
    // the block's sum of the local drift rows of partition i
    float v = 0.f;
    if (local_ok == nullptr || local_ok[i]) {
      const float *src = drift_rows + (size_t)i * g.BH * g.Lmax;
#pragma unroll
      for (int t = 0; t < kRowsPerThread; ++t)
        if (rok[t]) v += __ldg(src + roff[t]);
    }
    v = warp_sum_fixed(v);
    if (lane == 0) warp_part[warp] = v;
    __syncthreads();
    if (threadIdx.x == 0) {
      float s = 0.f;
      for (int w = 0; w < kMassThreads / 32; ++w) s += warp_part[w];
      partial[((size_t)i * nchunks_max + chunk) * GC + g.G] = s;
    }
    __syncthreads();
  }
  unsigned long long m = mask;
  for (int a = 0; a < nact_m; ++a) {
    const int j = __ffsll((long long)m) - 1;
    m &= m - 1;
    const bool valid = cache_valid == nullptr || cache_valid[s0 + a] != 0;
    float v = 0.f;
    if (valid) {
      const float *src = cache_lse + (size_t)(s0 + a) * slot_stride;
#pragma unroll
      for (int t = 0; t < kRowsPerThread; ++t)
        if (rok[t] && rmax[t] > -INFINITY) v += expf(__ldg(src + roff[t]) - rmax[t]) * rinv[t];
    }
    v = warp_sum_fixed(v);
    if (lane == 0) warp_part[warp] = v;
    __syncthreads();
    if (threadIdx.x == 0) {
      float s = 0.f;
      for (int w = 0; w < kMassThreads / 32; ++w) s += warp_part[w];
      partial[((size_t)i * nchunks_max + chunk) * GC + j] = s;
    }
    __syncthreads();
  }
}

__global__ void __launch_bounds__(kSelThreads)
plan_select_kernel(DevGeom g, const float *__restrict__ partial, int nchunks_max,
                   const unsigned char *__restrict__ cache_valid, int band_k, int target,
                   int anchor, signed char *__restrict__ plan_out, int *__restrict__ fresh_list,
                   int *__restrict__ counts, float *__restrict__ score_out, ErrorArgs ea) {
  __shared__ unsigned long long keys[kMaxP * kMaxP];
  __shared__ unsigned char fresh[kMaxP * kMaxP];
  __shared__ int scan[kSelThreads / 32];
  __shared__ int n_forced;
  __shared__ float s_delta[kMaxP];
  const int G = g.G;
  const int GC = G + 1;
  const int PP = g.P * G;
  const bool err = ea.age != nullptr;
  int n = 1;
  while (n < PP) n <<= 1;
  if (threadIdx.x == 0) n_forced = 0;
  if (err && !anchor && threadIdx.x < g.P) {
    // local drift of partition i in the last step (0 if it had no earlier state)
    const int i = threadIdx.x;
    float d = 0.f;
    if (ea.local_ok[i]) {
      const int Li = g.part_off[i + 1] - g.part_off[i];
      const int nch = (int)(((long long)g.BH * Li + kRowsPerBlock - 1) / kRowsPerBlock);
      double acc = 0.0;
      for (int ch = 0; ch < nch; ++ch) acc += (double)partial[((size_t)i * nchunks_max + ch) * GC + G];
      d = (float)(acc / ((double)g.BH * Li));
    }
    s_delta[i] = d;
    ea.delta[i] = d;
  }
  __syncthreads();

  int my_forced = 0;
  for (int p = threadIdx.x; p < n; p += kSelThreads) {
    unsigned long long key = ~0ull;
    if (p < PP) {
      const int i = p / G, c = p - (p / G) * G;
      const bool act = (g.row_mask[i] >> c) & 1ull;
      bool f = false;
      float w = 0.f;
      if (act) {
        const int slot = slot_of(g, i, c);
        const bool valid = cache_valid == nullptr || cache_valid[slot] != 0;
        if (!anchor) {
          if (!err || ea.refresh_w) {
            const int Li = g.part_off[i + 1] - g.part_off[i];
            const int nch = (int)(((long long)g.BH * Li + kRowsPerBlock - 1) / kRowsPerBlock);
            double acc = 0.0;
            for (int ch = 0; ch < nch; ++ch)
              acc += (double)partial[((size_t)i * nchunks_max + ch) * GC + c];
            w = (float)(acc / ((double)g.BH * Li));
            if (err) ea.w[p] = w;
          } else {
            w = ea.w[p];
          }
          if (err) {
            // age of the cached state, then the predicted error of reusing it
            const float a = (plan_out[p] == DITANGO_PLAN_FRESH) ? 0.f : ea.age[slot] + s_delta[i];
            ea.age[slot] = a;
            w = w * (a + s_delta[i]);
          }
        }
        if (anchor || !valid || unit_in_band(g, i, c, band_k)) {
          f = true;
          ++my_forced;
        } else {
          key = ((unsigned long long)(~__float_as_uint(w)) << 32) | (unsigned)p;
        }
      }
      fresh[p] = f ? 1 : 0;
      if (score_out) score_out[p] = w;
    }
    keys[p] = key;
  }
  if (my_forced) atomicAdd(&n_forced, my_forced);  // integer count: order-free
  __syncthreads();

  // bitonic sort of keys[0, n) ascending
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = threadIdx.x; t < (n >> 1); t += kSelThreads) {
        const int lo = 2 * t - (t & (stride - 1));
        const int hi = lo + stride;
        const bool up = ((lo & size) == 0);
        const unsigned long long a = keys[lo], b = keys[hi];
        if ((a > b) == up) {
          keys[lo] = b;
          keys[hi] = a;
        }
      }
      __syncthreads();
    }
  }
  const int need = anchor ? 0 : target - n_forced;
  for (int s = threadIdx.x; s < need && s < n; s += kSelThreads) {
    const unsigned long long key = keys[s];
    if (key != ~0ull) fresh[(int)(key & 0xffffffffu)] = 1;
  }
  __syncthreads();

  // plan codes and the row-major fresh list (block-wide exclusive scan)
  const int per = (PP + kSelThreads - 1) / kSelThreads;
  const int p0 = threadIdx.x * per;
  int cnt = 0;
  for (int p = p0; p < p0 + per && p < PP; ++p) cnt += fresh[p];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) scan[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int v = (lane < kSelThreads / 32) ? scan[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    if (lane < kSelThreads / 32) scan[lane] = v;
  }
  __syncthreads();
  int pos = incl - cnt + (warp > 0 ? scan[warp - 1] : 0);
  for (int p = p0; p < p0 + per && p < PP; ++p) {
    const int i = p / G, c = p - (p / G) * G;
    const bool act = (g.row_mask[i] >> c) & 1ull;
    plan_out[p] = fresh[p] ? (signed char)DITANGO_PLAN_FRESH
                           : (act ? (signed char)DITANGO_PLAN_REUSE : (signed char)DITANGO_PLAN_SKIP);
    if (fresh[p]) fresh_list[pos++] = p;
  }
  if (threadIdx.x == kSelThreads - 1) {
    counts[0] = pos;
    counts[1] = g.n_active - pos;
  }
  if (err && threadIdx.x < g.P) {
    // for the next step: did the local unit hold a state before this step?
    const int i = threadIdx.x, c = g.part_group[i];
    bool ok = (g.row_mask[i] >> c) & 1ull;
    if (ok && cache_valid) ok = cache_valid[slot_of(g, i, c)] != 0;
    ea.local_ok[i] = ok ? 1 : 0;
  }
}

}  // namespace plan

size_t plan_workspace_bytes(const DevGeom &g) {
  const int nchunks_max =
      (int)(((long long)g.BH * g.Lmax + plan::kRowsPerBlock - 1) / plan::kRowsPerBlock);
  return (size_t)g.P * nchunks_max * (g.G + 1) * sizeof(float);
}

cudaError_t launch_plan(const DevGeom &g, const float *cache_lse, const unsigned char *cache_valid,
                        int band_k, int target, int anchor, signed char *plan_out, int *fresh_list,
                        int *counts, float *score_out, void *workspace, cudaStream_t stream,
                        const float *drift_rows, float *w_hold, float *age, float *delta,
                        unsigned char *local_ok, int refresh_w) {
  const int nchunks_max =
      (int)(((long long)g.BH * g.Lmax + plan::kRowsPerBlock - 1) / plan::kRowsPerBlock);
  float *partial = static_cast<float *>(workspace);
  plan::ErrorArgs ea{drift_rows, w_hold, age, delta, local_ok, refresh_w};
  const bool err = age != nullptr;
  const int do_mass = err ? refresh_w : 1;
  if (!anchor && (do_mass || err)) {
    dim3 grid(nchunks_max, g.P);
    plan::mass_partial_kernel<<<grid, plan::kMassThreads, 0, stream>>>(
        g, cache_lse, cache_valid, partial, nchunks_max, do_mass, err ? drift_rows : nullptr,
        local_ok);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  plan::plan_select_kernel<<<1, plan::kSelThreads, 0, stream>>>(
      g, partial, nchunks_max, cache_valid, band_k, target, anchor, plan_out, fresh_list, counts,
      score_out, ea);
  return cudaGetLastError();
}

}  // namespace ditango
