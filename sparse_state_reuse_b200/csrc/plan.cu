// Fresh-versus-reuse plan (DiTango, "Riepilogo Tecnico" -> Metodologia ->
// 1. Anchor-Guided Selection Planner).
//
// The candidates are units (query partition i, KV group c); without KV
// groups a unit is the pair (i, j) ("Strategia per Gruppi": decisions per
// group of adjacent partitions).
// Stage 1 (mass_kernel): importance of each active unit from the cached
// log-sum-exps.  For every cached row r of query partition i the share of
// unit (i, c) in that row's softmax denominator is e_c / sum_c' e_c',
// e_c = exp(lse_ic[r] - max_c' lse_ic'[r]); each block of 128 rows of one
// (b*h, i) sums these shares in a fixed order (weights.cuh -- the same
// arithmetic, and the same blocks, as the merge's mass partials, so the
// merge of the previous step can stand in for this stage).  Invalid (never
// written) slots hold no mass.
// Stage 2 (plan_select_kernel, one block): the block sums are added in
// (b*h, block) order in double precision and divided by the row count
// (w = mean share), then the band, the invalid slots and the top-w units up
// to the budget are marked fresh.  Ranking sorts 64-bit keys
// (~bits(w) << 32 | i*G + c) with a bitonic network: larger w first, ties to
// the lower linear index.
// Error mode (DiTango, "Modellazione dell'Errore", "Predizione Online"):
// stage 1 also sums each partition's local drift rows (written by the
// attention kernel) into the extra column G of the block sums; stage 2 turns
// them into delta_i, ages every cached state (0 if the previous plan made it
// fresh, + delta_i if it reused it) and ranks by w * (age + delta_i), with w
// recomputed only on the step after an anchor and held otherwise.
// Everything is deterministic; no floating-point atomics.
#include "common.cuh"
#include "weights.cuh"

namespace ditango {
namespace plan {

constexpr int kSelThreads = 1024;
using weights::kWRows;

// Error-mode arguments of the plan (all null in the plain mode).
struct ErrorArgs {
  const float *drift_rows;     // [P][B*H][Lmax]
  float *w;                    // [P*G] importance held between anchors
  float *age;                  // [slots]
  float *delta;                // [P] output
  unsigned char *local_ok;     // [P] read (last step), then rewritten
  int refresh_w;
};

// Block sums of one (row block, query partition, b*h): the shares of the
// valid active units of each row (do_mass), and the rows' local drift
// (drift_rows non-null).  One thread per row; dynamic shared memory holds the
// shares [units][kWRows] and the drift [kWRows].
__global__ void __launch_bounds__(kWRows)
mass_kernel(DevGeom g, const float *__restrict__ cache_lse,
            const unsigned char *__restrict__ cache_valid, float *__restrict__ partial, int do_mass,
            const float *__restrict__ drift_rows, const unsigned char *__restrict__ local_ok) {
  const int i = blockIdx.y;
  const int bh = blockIdx.z;
  const int Li = g.part_off[i + 1] - g.part_off[i];
  const int r0 = blockIdx.x * kWRows;
  if (r0 >= Li) return;   // uniform per block
  const int nrows = (Li - r0 < kWRows) ? Li - r0 : kWRows;
  const int G = g.G;
  extern __shared__ float sh[];
  __shared__ const float *s_lse[kMaxP];
  __shared__ signed char s_state_of[kMaxP];
  __shared__ int s_n;
  const size_t slot_stride = (size_t)g.BH * g.Lmax;
  if (threadIdx.x == 0) {
    int a = 0;
    for (int c = 0; c < G; ++c) {
      s_state_of[c] = -1;
      if (!do_mass || !((g.row_mask[i] >> c) & 1ull)) continue;
      const int slot = slot_of(g, i, c);
      if (cache_valid != nullptr && cache_valid[slot] == 0) continue;   // no state, no mass
      s_lse[a] = cache_lse + (size_t)slot * slot_stride + (size_t)bh * g.Lmax + r0;
      s_state_of[c] = (signed char)a;
      ++a;
    }
    s_n = a;
  }
  __syncthreads();
  const int n = s_n;
  const int t = threadIdx.x;
  float *drift_sh = sh + (size_t)n * kWRows;
  weights::row_shares(s_lse, n, t, t < nrows, sh, t);
  if (drift_rows != nullptr) {
    const bool use = (local_ok == nullptr || local_ok[i]) && t < nrows;
    drift_sh[t] = use ? __ldg(drift_rows + ((size_t)i * g.BH + bh) * g.Lmax + r0 + t) : 0.f;
  }
  __syncthreads();
  const int warp = t >> 5, lane = t & 31;
  for (int c = warp; c <= G; c += kWRows / 32) {
    float v;
    if (c < G) {
      if (!((g.row_mask[i] >> c) & 1ull)) continue;
      const int a = s_state_of[c];
      v = (a >= 0) ? weights::block_sum(sh + a * kWRows, lane) : 0.f;
    } else {
      if (drift_rows == nullptr) continue;
      v = weights::block_sum(drift_sh, lane);
    }
    if (lane == 0) partial[weights::partial_index(g, i, bh, blockIdx.x, c)] = v;
  }
}

// Mean over the rows of query partition i of a unit's (or the drift
// column's) per-row values, from its block sums: one warp; lane l adds the
// blocks j = l + 32 m of the (b*h, block) sequence into accumulator m % 4
// (four loads in flight), the four accumulators are added in order, then a
// butterfly; every lane returns the same value.  Double precision.
__device__ __forceinline__ float mean_blocks(const DevGeom &g, const float *partial, int i, int col,
                                             int lane) {
  const int Li = g.part_off[i + 1] - g.part_off[i];
  const int nrb_i = weights::n_row_blocks(Li);
  const int n = g.BH * nrb_i;
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int j0 = lane; j0 < n; j0 += 4 * 32) {
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int j = j0 + m * 32;
      if (j < n) {
        const int bh = j / nrb_i;
        acc[m] += (double)partial[weights::partial_index(g, i, bh, j - bh * nrb_i, col)];
      }
    }
  }
  double a = (acc[0] + acc[1]) + (acc[2] + acc[3]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
  return (float)(a / ((double)g.BH * Li));
}

// Second stage of the mass score: one warp per active unit -- and, in error
// mode, per partition's drift column -- turns the block sums into the mean
// (w, or delta), written to the end of the workspace: [P*G] then [P].
constexpr int kReduceWarps = 8;
__global__ void __launch_bounds__(kReduceWarps * 32)
mass_reduce_kernel(DevGeom g, const float *__restrict__ partial, float *__restrict__ means,
                   int do_mass, int do_drift, const unsigned char *__restrict__ local_ok) {
  const int lane = threadIdx.x & 31;
  const int v = blockIdx.x * kReduceWarps + (threadIdx.x >> 5);
  const int PG = g.P * g.G;
  if (v < PG) {
    const int i = v / g.G, c = v - (v / g.G) * g.G;
    float m = 0.f;
    if (do_mass && ((g.row_mask[i] >> c) & 1ull)) m = mean_blocks(g, partial, i, c, lane);
    if (lane == 0) means[v] = m;
  } else if (v < PG + g.P && do_drift) {
    const int i = v - PG;
    const float d = (local_ok == nullptr || local_ok[i]) ? mean_blocks(g, partial, i, g.G, lane) : 0.f;
    if (lane == 0) means[v] = d;
  }
}

__global__ void __launch_bounds__(kSelThreads)
plan_select_kernel(DevGeom g, const float *__restrict__ partial,
                   const unsigned char *__restrict__ cache_valid, int band_k, int target,
                   int anchor, signed char *__restrict__ plan_out, int *__restrict__ fresh_list,
                   int *__restrict__ counts, float *__restrict__ score_out, ErrorArgs ea) {
  __shared__ unsigned long long keys[kMaxP * kMaxP];
  __shared__ unsigned char fresh[kMaxP * kMaxP];
  __shared__ int scan[kSelThreads / 32];
  __shared__ int n_forced;
  __shared__ float s_delta[kMaxP];
  const int G = g.G;
  const int PP = g.P * G;
  const bool err = ea.age != nullptr;
  int n = 1;
  while (n < PP) n <<= 1;
  if (threadIdx.x == 0) n_forced = 0;
  // the importance w of every active unit (when it is computed from the
  // block sums) and the local drift of every partition (error mode), as the
  // reduction kernel left them at the end of the workspace
  const bool sum_w = !anchor && (!err || ea.refresh_w);
  const float *means = partial + weights::n_partials(g);
  if (err && !anchor && threadIdx.x < g.P) {
    const float d = means[PP + threadIdx.x];
    s_delta[threadIdx.x] = d;
    ea.delta[threadIdx.x] = d;
  }
  __syncthreads();
  constexpr int kPerThread = kMaxP * kMaxP / kSelThreads;
  int my_forced = 0;
#pragma unroll
  for (int q = 0; q < kPerThread; ++q) {
    const int p = threadIdx.x + q * kSelThreads;
    if (p >= n) break;
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
          if (sum_w) {
            w = means[p];
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
  // the block sums, then the means of the units and of the drift columns
  return (weights::n_partials(g) + (size_t)g.P * g.G + g.P) * sizeof(float);
}

// mass_source: the block sums are already in `workspace` (written by the
// merge of the previous step), so stage 1 is skipped.
cudaError_t launch_plan(const DevGeom &g, const float *cache_lse, const unsigned char *cache_valid,
                        int band_k, int target, int anchor, signed char *plan_out, int *fresh_list,
                        int *counts, float *score_out, void *workspace, cudaStream_t stream,
                        const float *drift_rows, float *w_hold, float *age, float *delta,
                        unsigned char *local_ok, int refresh_w, int mass_given) {
  float *partial = static_cast<float *>(workspace);
  plan::ErrorArgs ea{drift_rows, w_hold, age, delta, local_ok, refresh_w};
  const bool err = age != nullptr;
  const int do_mass = err ? refresh_w : 1;
  if (!anchor && !mass_given && (do_mass || err)) {
    int most = 0;
    for (int i = 0; i < g.P; ++i) {
      const int c = __builtin_popcountll(g.row_mask[i]);
      most = c > most ? c : most;
    }
    const size_t smem = ((size_t)(do_mass ? most : 0) + 1) * weights::kWRows * sizeof(float);
    dim3 grid(weights::n_row_blocks(g.Lmax), g.P, g.BH);
    plan::mass_kernel<<<grid, weights::kWRows, smem, stream>>>(
        g, cache_lse, cache_valid, partial, do_mass, err ? drift_rows : nullptr, local_ok);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (!anchor && (do_mass || err)) {
    // block sums -> per-unit means (and per-partition drift), in parallel
    const int nv = g.P * g.G + (err ? g.P : 0);
    const int blocks = (nv + plan::kReduceWarps - 1) / plan::kReduceWarps;
    plan::mass_reduce_kernel<<<blocks, plan::kReduceWarps * 32, 0, stream>>>(
        g, partial, partial + weights::n_partials(g), do_mass, err ? 1 : 0, local_ok);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  plan::plan_select_kernel<<<1, plan::kSelThreads, 0, stream>>>(
      g, partial, cache_valid, band_k, target, anchor, plan_out, fresh_list, counts, score_out, ea);
  return cudaGetLastError();
}

}  // namespace ditango
