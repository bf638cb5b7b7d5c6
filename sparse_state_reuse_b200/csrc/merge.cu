// Log-sum-exp merge of attention states and the cache write-back.
//
// DiTango, "Riepilogo Tecnico" -> Metodologia -> 2. State-Centric Parallel
// Runtime, "Composizione dello Stato": the output of a query row is the
// composition of the states of all active units (KV partitions, or KV
// groups) of its partition,
//   L = M + log sum_c exp(lse_c - M),  O = sum_c exp(lse_c - L) O_c,
// fresh states coming from this step's partial buffer and reused ones from
// the cache.  "Anchor Steps": the states computed fresh refresh the cache.
//
// The merge is HBM bound.  A block takes 128 rows of one (b*h, query
// partition).  Phase 1: one thread per row reads the row's lse of every
// state and writes the weights to shared memory (weights.cuh, the same
// arithmetic as the plan's mass score).  Phase 2: the block's rows of each
// state are one contiguous run of memory, streamed as a flat array of 16-byte
// groups (4 fp32 or 8 bf16 values) by all threads -- coalesced whatever d is,
// no idle lanes -- with several states' loads of several groups in flight per
// thread.  Optionally
// the block also writes its sums of the weights ("mass partials"): the
// importance w of the next step's plan, so that the plan need not read the
// cache again.
#include <cuda_bf16.h>

#include "common.cuh"
#include "weights.cuh"

namespace ditango {
namespace merge {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// Checked builds record a bad plan code here; read and cleared by
// ditango_check_status.
__device__ int g_merge_check_status;

// Four bf16 values (two packed pairs, low element first) as floats.
__device__ __forceinline__ float4 widen_bf16x4(uint32_t lo, uint32_t hi) {
  return make_float4(__uint_as_float(lo << 16), __uint_as_float(lo & 0xffff0000u),
                     __uint_as_float(hi << 16), __uint_as_float(hi & 0xffff0000u));
}

__device__ __forceinline__ void store_out(void *out, int is_fp32, size_t off, float4 v) {
  if (is_fp32) {
    *reinterpret_cast<float4 *>(static_cast<float *>(out) + off) = v;
  } else {
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
    __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t *>(&a);
    u.y = *reinterpret_cast<uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(out) + off) = u;
  }
}

__device__ __forceinline__ void fma4(float4 &acc, float w, const float4 &v) {
  acc.x = fmaf(w, v.x, acc.x);
  acc.y = fmaf(w, v.y, acc.y);
  acc.z = fmaf(w, v.z, acc.z);
  acc.w = fmaf(w, v.w, acc.w);
}

// The merge's unit of streaming: 16 bytes of one stored state row, i.e. 4
// fp32 values or 8 bf16 values, kept packed until used.
template <bool SB>
struct Grp {
  static constexpr int V = 4;               // values per group
  using Raw = float4;
  struct Acc { float4 a; };
};
template <>
struct Grp<true> {
  static constexpr int V = 8;
  using Raw = uint4;
  struct Acc { float4 a, b; };
};
template <bool SB>
__device__ __forceinline__ typename Grp<SB>::Raw load_grp(const char *p) {
  return __ldg(reinterpret_cast<const typename Grp<SB>::Raw *>(p));
}
template <bool SB>
__device__ __forceinline__ typename Grp<SB>::Raw zero_grp() {
  typename Grp<SB>::Raw r;
  if constexpr (SB) r = make_uint4(0u, 0u, 0u, 0u); else r = make_float4(0.f, 0.f, 0.f, 0.f);
  return r;
}
template <bool SB>
__device__ __forceinline__ void store_grp(char *p, typename Grp<SB>::Raw u) {
  *reinterpret_cast<typename Grp<SB>::Raw *>(p) = u;
}
template <bool SB>
__device__ __forceinline__ void zero_acc(typename Grp<SB>::Acc &acc) {
  acc.a = make_float4(0.f, 0.f, 0.f, 0.f);
  if constexpr (SB) acc.b = make_float4(0.f, 0.f, 0.f, 0.f);
}
template <bool SB>
__device__ __forceinline__ void fma_grp(typename Grp<SB>::Acc &acc, float w, typename Grp<SB>::Raw u) {
  if constexpr (SB) {
    fma4(acc.a, w, widen_bf16x4(u.x, u.y));
    fma4(acc.b, w, widen_bf16x4(u.z, u.w));
  } else {
    fma4(acc.a, w, u);
  }
}
// The merged group to the output (fp32 or bf16 elements at element offset off).
template <bool SB>
__device__ __forceinline__ void store_out_grp(void *out, int is_fp32, size_t off,
                                              const typename Grp<SB>::Acc &acc) {
  if constexpr (SB) {
    if (is_fp32) {
      *reinterpret_cast<float4 *>(static_cast<float *>(out) + off) = acc.a;
      *reinterpret_cast<float4 *>(static_cast<float *>(out) + off + 4) = acc.b;
    } else {
      uint4 u;
      __nv_bfloat162 t;
      t = __floats2bfloat162_rn(acc.a.x, acc.a.y); u.x = *reinterpret_cast<uint32_t *>(&t);
      t = __floats2bfloat162_rn(acc.a.z, acc.a.w); u.y = *reinterpret_cast<uint32_t *>(&t);
      t = __floats2bfloat162_rn(acc.b.x, acc.b.y); u.z = *reinterpret_cast<uint32_t *>(&t);
      t = __floats2bfloat162_rn(acc.b.z, acc.b.w); u.w = *reinterpret_cast<uint32_t *>(&t);
      *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(out) + off) = u;
    }
  } else {
    store_out(out, is_fp32, off, acc.a);
  }
}

// Merge of one block of rows (see the file comment).  Dynamic shared memory:
// the weights, [states][kWRows] floats.
template <int D, bool SB>
__global__ void __launch_bounds__(kThreads, 3)
merge_kernel(DevGeom g, const signed char *__restrict__ plan, const char *__restrict__ part_O,
             const float *__restrict__ part_lse, char *cache_O, float *cache_lse,
             unsigned char *cache_valid, int writeback, void *out, int out_is_fp32, long long osb,
             long long osh, long long osn, float *__restrict__ out_lse, float *__restrict__ mass) {
  constexpr int VG = Grp<SB>::V;            // values per 16-byte group
  constexpr int QG = D / VG;                // groups per row
  constexpr int ES = SB ? 2 : 4;            // bytes per stored O element
  constexpr size_t ROWB = (size_t)D * ES;   // bytes per state row
  constexpr int U = 2;                      // groups per thread per pass
  constexpr int SBATCH = 4;                 // states per batch of loads
  using weights::kWRows;
  const int i = blockIdx.y;
  const int bh = blockIdx.z;
  const int Li = g.part_off[i + 1] - g.part_off[i];
  const int r0 = blockIdx.x * kWRows;
  if (r0 >= Li) return;
  const int nrows = (Li - r0 < kWRows) ? Li - r0 : kWRows;
  const int G = g.G;
  extern __shared__ float sh[];             // weights [n][kWRows]
  __shared__ const char *s_O[kMaxP];        // state rows of this block
  __shared__ const float *s_lse[kMaxP];
  __shared__ char *s_wbO[kMaxP];            // write-back targets (fresh states) or null
  __shared__ float *s_wblse[kMaxP];
  __shared__ signed char s_state_of[kMaxP]; // column -> state index, -1: none
  __shared__ int s_n;
  __shared__ int warp_cnt[kWarps];

  // fresh units before row i (row-major), for fresh-list positions
  int cnt = 0;
  for (int p = threadIdx.x; p < i * G; p += kThreads) cnt += (plan[p] == DITANGO_PLAN_FRESH);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if ((threadIdx.x & 31) == 0) warp_cnt[threadIdx.x >> 5] = cnt;
  __syncthreads();
  if (threadIdx.x == 0) {
    int fpos = 0;
    for (int w = 0; w < kWarps; ++w) fpos += warp_cnt[w];
    const size_t blk = (size_t)g.BH * g.Lmax;
    const size_t row0 = (size_t)bh * g.Lmax + r0;   // this block's first row in a state block
    int a = 0;
    for (int c = 0; c < G; ++c) {
      s_state_of[c] = -1;
#ifdef DITANGO_CHECK
      {
        // a plan code outside {skip, fresh, reuse}, or anything but skip on a
        // masked unit: recorded (the unit is then left out, as always)
        const int code = plan[i * G + c];
        const bool act = (g.row_mask[i] >> c) & 1ull;
        if (code < 0 || code > 2 || (!act && code != 0))
          atomicExch(&g_merge_check_status, (int)DITANGO_ERR_BOUNDS);
      }
#endif
      if (!((g.row_mask[i] >> c) & 1ull)) continue;
      const int code = plan[i * G + c];
      const int slot = slot_of(g, i, c);
      char *wbO = nullptr;
      float *wblse = nullptr;
      const char *O;
      const float *lse;
      if (code == DITANGO_PLAN_FRESH && part_O != nullptr) {
        O = part_O + ((size_t)fpos * blk + row0) * ROWB;
        lse = part_lse + (size_t)fpos * blk + row0;
        if (writeback) {
          wbO = cache_O + ((size_t)slot * blk + row0) * ROWB;
          wblse = cache_lse + (size_t)slot * blk + row0;
          if (cache_valid && bh == 0 && blockIdx.x == 0) cache_valid[slot] = 1;
        }
      } else if (code == DITANGO_PLAN_FRESH || code == DITANGO_PLAN_REUSE) {
        O = cache_O + ((size_t)slot * blk + row0) * ROWB;
        lse = cache_lse + (size_t)slot * blk + row0;
      } else {
        continue;  // active unit the plan skipped: contributes nothing
      }
      if (code == DITANGO_PLAN_FRESH) ++fpos;
      s_O[a] = O;
      s_lse[a] = lse;
      s_wbO[a] = wbO;
      s_wblse[a] = wblse;
      s_state_of[c] = (signed char)a;
      ++a;
    }
    s_n = a;
  }
  __syncthreads();
  const int n = s_n;
  const int b = bh / g.H, h = bh - (bh / g.H) * g.H;
  const int tok0 = g.part_off[i] + r0;

  // ---- phase 1: weights of every row (one thread per row)
  if (threadIdx.x < kWRows) {
    const int t = threadIdx.x;
    const float L = weights::row_shares(s_lse, n, t, t < nrows, sh, t);
    if (t < nrows) {
      if (out_lse) out_lse[(size_t)bh * g.N + tok0 + t] = L;
      for (int a = 0; a < n; ++a)
        if (s_wblse[a]) s_wblse[a][t] = __ldg(s_lse[a] + t);
    }
  }
  __syncthreads();

  // the block's sums of the weights: the next plan's importance w
  if (mass != nullptr) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int c = warp; c < G; c += kWarps) {
      const int a = s_state_of[c];
      const float v = (a >= 0) ? weights::block_sum(sh + a * kWRows, lane) : 0.f;
      if (lane == 0) mass[weights::partial_index(g, i, bh, blockIdx.x, c)] = v;
    }
  }

  // ---- phase 2: stream the states' rows as one flat array of 16-byte groups
  const int ng = nrows * QG;
  const size_t obase = (size_t)b * osb + (size_t)h * osh;
  for (int f0 = threadIdx.x; f0 < ng; f0 += kThreads * U) {
    typename Grp<SB>::Acc acc[U];
    int row[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      zero_acc<SB>(acc[u]);
      row[u] = (f0 + u * kThreads) / QG;
    }
    for (int a0 = 0; a0 < n; a0 += SBATCH) {
      typename Grp<SB>::Raw v[SBATCH][U];
#pragma unroll
      for (int q = 0; q < SBATCH; ++q) {
        const char *src = (a0 + q < n) ? s_O[a0 + q] : nullptr;
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int f = f0 + u * kThreads;
          v[q][u] = zero_grp<SB>();
          if (src != nullptr && f < ng) v[q][u] = load_grp<SB>(src + (size_t)f * 16);
        }
      }
#pragma unroll
      for (int q = 0; q < SBATCH; ++q) {
        if (a0 + q >= n) break;
        const float *wq = sh + (a0 + q) * kWRows;
        char *wb = s_wbO[a0 + q];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int f = f0 + u * kThreads;
          if (f < ng) {
            fma_grp<SB>(acc[u], wq[row[u]], v[q][u]);
            if (wb != nullptr) store_grp<SB>(wb + (size_t)f * 16, v[q][u]);
          }
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int f = f0 + u * kThreads;
      if (f < ng)
        store_out_grp<SB>(out, out_is_fp32,
                          obase + (size_t)(tok0 + row[u]) * osn + (size_t)(f - row[u] * QG) * VG, acc[u]);
    }
  }
}

// Copy the fresh states (fresh-list positions) into their cache slots.
// blockIdx.y = slot; the block finds its unit, and if the plan marks it fresh
// counts the fresh units before it (row-major) to find its fresh position.
__global__ void __launch_bounds__(256)
cache_update_kernel(DevGeom g, const signed char *__restrict__ plan,
                    const char *__restrict__ part_O, const float *__restrict__ part_lse,
                    char *cache_O, float *cache_lse, unsigned char *cache_valid, int row_bytes) {
  const int slot = blockIdx.y;
  int i = 0;
  while (i + 1 < g.P && g.row_start[i + 1] <= slot) ++i;
  int rank = slot - g.row_start[i];
  unsigned long long m = g.row_mask[i];
  for (int t = 0; t < rank; ++t) m &= m - 1;
  const int c = __ffsll((long long)m) - 1;
  const int pair = i * g.G + c;
  if (plan[pair] != DITANGO_PLAN_FRESH) return;
  __shared__ int warp_cnt[8];
  __shared__ int s_fpos;
  int cnt = 0;
  for (int p = threadIdx.x; p < pair; p += blockDim.x) cnt += (plan[p] == DITANGO_PLAN_FRESH);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if ((threadIdx.x & 31) == 0) warp_cnt[threadIdx.x >> 5] = cnt;
  __syncthreads();
  if (threadIdx.x == 0) {
    int c = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) c += warp_cnt[w];
    s_fpos = c;
  }
  __syncthreads();
  const int f = s_fpos;
  const size_t blk = (size_t)g.BH * g.Lmax;
  const float4 *s = reinterpret_cast<const float4 *>(part_O + (size_t)f * blk * row_bytes);
  float4 *d = reinterpret_cast<float4 *>(cache_O + (size_t)slot * blk * row_bytes);
  const size_t n4 = blk * row_bytes / 16;
  for (size_t t = (size_t)blockIdx.x * blockDim.x + threadIdx.x; t < n4;
       t += (size_t)gridDim.x * blockDim.x)
    d[t] = __ldg(s + t);
  const float *sl = part_lse + (size_t)f * blk;
  float *dl = cache_lse + (size_t)slot * blk;
  for (size_t t = (size_t)blockIdx.x * blockDim.x + threadIdx.x; t < blk;
       t += (size_t)gridDim.x * blockDim.x)
    dl[t] = __ldg(sl + t);
  if (cache_valid && blockIdx.x == 0 && threadIdx.x == 0) cache_valid[slot] = 1;
}

// Dynamic group composition (DiTango, 2. State-Centric Parallel Runtime,
// "Composizione Dinamica dei Gruppi"): the cached state of coarse unit
// (i, C) is the log-sum-exp composition of the cached states of the fine
// units (i, c), c inside C -- no attention is recomputed.  Those fine units
// are consecutive slots of the fine cache.  blockIdx.y = coarse slot,
// blockIdx.z = b*h, blockIdx.x = a block of kWRows rows.  The same two
// phases as the merge: the rows' weights (and the coarse lse) in shared
// memory, then the fine states' rows streamed as a flat array of 4-value
// groups into the coarse state's rows, which are contiguous too.  A coarse
// slot is valid only if every fine slot it covers is; an invalid one is
// marked and left unwritten.
template <int D, bool SB>
__global__ void __launch_bounds__(kThreads, 3)
compose_kernel(DevGeom fine, DevGeom coarse, const char *__restrict__ fO,
               const float *__restrict__ flse, const unsigned char *__restrict__ fvalid,
               char *__restrict__ cO, float *__restrict__ clse, unsigned char *cvalid) {
  constexpr int VG = Grp<SB>::V;            // values per 16-byte group
  constexpr int QG = D / VG;                // groups per row
  constexpr int ES = SB ? 2 : 4;
  constexpr size_t ROWB = (size_t)D * ES;
  constexpr int U = 2;                      // groups per thread per pass
  constexpr int SBATCH = 4;                 // states per batch of loads
  using weights::kWRows;
  const int cslot = blockIdx.y;
  const int bh = blockIdx.z;
  int i = 0;
  while (i + 1 < coarse.P && coarse.row_start[i + 1] <= cslot) ++i;
  unsigned long long m = coarse.row_mask[i];
  for (int t = cslot - coarse.row_start[i]; t > 0; --t) m &= m - 1;
  const int C = __ffsll((long long)m) - 1;
  const int Li = coarse.part_off[i + 1] - coarse.part_off[i];
  const int r0 = blockIdx.x * kWRows;
  if (r0 >= Li) return;
  const int nrows = (Li - r0 < kWRows) ? Li - r0 : kWRows;
  // the fine units inside C that are active: consecutive fine slots
  int fs0 = -1, nf = 0;
  for (int c = 0; c < fine.G; ++c) {
    if (fine.group_off[c] < coarse.group_off[C] || fine.group_off[c + 1] > coarse.group_off[C + 1]) continue;
    if (!((fine.row_mask[i] >> c) & 1ull)) continue;
    if (fs0 < 0) fs0 = slot_of(fine, i, c);
    ++nf;
  }
  bool valid = nf > 0;
  if (fvalid)
    for (int a = 0; a < nf; ++a) valid = valid && fvalid[fs0 + a] != 0;
  if (cvalid && bh == 0 && blockIdx.x == 0) cvalid[cslot] = valid ? 1 : 0;
  if (!valid) return;   // uniform per block

  extern __shared__ float sh[];             // weights [nf][kWRows]
  __shared__ const char *s_O[kMaxP];
  __shared__ const float *s_lse[kMaxP];
  const size_t blk = (size_t)fine.BH * fine.Lmax;
  const size_t row0 = (size_t)bh * fine.Lmax + r0;   // this block's first row in a state block
  if (threadIdx.x < nf) {
    s_O[threadIdx.x] = fO + ((size_t)(fs0 + threadIdx.x) * blk + row0) * ROWB;
    s_lse[threadIdx.x] = flse + (size_t)(fs0 + threadIdx.x) * blk + row0;
  }
  __syncthreads();
  char *dstO = cO + ((size_t)cslot * blk + row0) * ROWB;
  float *dstl = clse + (size_t)cslot * blk + row0;

  // ---- phase 1: weights and the coarse lse of every row
  if (threadIdx.x < kWRows) {
    const int t = threadIdx.x;
    const float L = weights::row_shares(s_lse, nf, t, t < nrows, sh, t);
    if (t < nrows) dstl[t] = L;
  }
  __syncthreads();

  // ---- phase 2: the fine rows, weighted, into the coarse rows (16-byte groups)
  const int ng = nrows * QG;
  for (int f0 = threadIdx.x; f0 < ng; f0 += kThreads * U) {
    typename Grp<SB>::Acc acc[U];
    int row[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      zero_acc<SB>(acc[u]);
      row[u] = (f0 + u * kThreads) / QG;
    }
    for (int a0 = 0; a0 < nf; a0 += SBATCH) {
      typename Grp<SB>::Raw v[SBATCH][U];
#pragma unroll
      for (int q = 0; q < SBATCH; ++q) {
        const char *src = (a0 + q < nf) ? s_O[a0 + q] : nullptr;
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int f = f0 + u * kThreads;
          v[q][u] = zero_grp<SB>();
          if (src != nullptr && f < ng) v[q][u] = load_grp<SB>(src + (size_t)f * 16);
        }
      }
#pragma unroll
      for (int q = 0; q < SBATCH; ++q) {
        if (a0 + q >= nf) break;
        const float *wq = sh + (a0 + q) * kWRows;
#pragma unroll
        for (int u = 0; u < U; ++u)
          if (f0 + u * kThreads < ng) fma_grp<SB>(acc[u], wq[row[u]], v[q][u]);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int f = f0 + u * kThreads;
      if (f < ng) store_out_grp<SB>(dstO, SB ? 0 : 1, (size_t)f * VG, acc[u]);
    }
  }
}

}  // namespace merge

cudaError_t launch_merge(const DevGeom &g, const signed char *plan, const void *part_O,
                         const float *part_lse, void *cache_O, float *cache_lse,
                         unsigned char *cache_valid, int writeback, int state_bf16, void *out,
                         int out_is_fp32,
                         long long osb, long long osh, long long osn, float *out_lse,
                         float *mass_partials, cudaStream_t stream) {
  dim3 grid(weights::n_row_blocks(g.Lmax), g.P, g.BH);
  int most = 1;   // most active units of any row: the states a row can merge
  for (int i = 0; i < g.P; ++i) {
    const int c = __builtin_popcountll(g.row_mask[i]);
    most = c > most ? c : most;
  }
  const size_t smem = (size_t)most * weights::kWRows * sizeof(float);
  switch (g.d) {
#define DITANGO_MERGE(DD)                                                                        \
  case DD:                                                                                       \
    if (state_bf16)                                                                              \
      merge::merge_kernel<DD, true><<<grid, merge::kThreads, smem, stream>>>(                    \
          g, plan, static_cast<const char *>(part_O), part_lse, static_cast<char *>(cache_O),   \
          cache_lse, cache_valid, writeback, out, out_is_fp32, osb, osh, osn, out_lse,           \
          mass_partials);                                                                        \
    else                                                                                         \
      merge::merge_kernel<DD, false><<<grid, merge::kThreads, smem, stream>>>(                   \
          g, plan, static_cast<const char *>(part_O), part_lse, static_cast<char *>(cache_O),   \
          cache_lse, cache_valid, writeback, out, out_is_fp32, osb, osh, osn, out_lse,           \
          mass_partials);                                                                        \
    return cudaGetLastError();
    DITANGO_MERGE(64)
    DITANGO_MERGE(96)
    DITANGO_MERGE(128)
#undef DITANGO_MERGE
    default:
      return cudaErrorInvalidValue;
  }
}

cudaError_t launch_cache_update(const DevGeom &g, const signed char *plan, const void *part_O,
                                const float *part_lse, void *cache_O, float *cache_lse,
                                unsigned char *cache_valid, int state_bf16, int num_sms,
                                cudaStream_t stream) {
  if (g.n_active == 0) return cudaSuccess;
  const int row_bytes = g.d * (state_bf16 ? 2 : 4);
  const size_t n4 = (size_t)g.BH * g.Lmax * row_bytes / 16;
  int bx = (int)((n4 + 255) / 256);
  const int cap = (num_sms * 8 + g.n_active - 1) / g.n_active;
  if (bx > cap) bx = cap < 1 ? 1 : cap;
  dim3 grid(bx, g.n_active);
  merge::cache_update_kernel<<<grid, 256, 0, stream>>>(
      g, plan, static_cast<const char *>(part_O), part_lse, static_cast<char *>(cache_O), cache_lse,
      cache_valid, row_bytes);
  return cudaGetLastError();
}

cudaError_t launch_cache_compose(const DevGeom &fine, const DevGeom &coarse, const void *fine_O,
                                 const float *fine_lse, const unsigned char *fine_valid,
                                 void *coarse_O, float *coarse_lse, unsigned char *coarse_valid,
                                 int state_bf16, cudaStream_t stream) {
  if (coarse.n_active == 0) return cudaSuccess;
  dim3 grid(weights::n_row_blocks(coarse.Lmax), coarse.n_active, coarse.BH);
  int most = 1;   // most fine units one coarse unit covers
  for (int i = 0; i < coarse.P; ++i)
    for (int C = 0; C < coarse.G; ++C) {
      int n = 0;
      for (int c = 0; c < fine.G; ++c)
        if (fine.group_off[c] >= coarse.group_off[C] && fine.group_off[c + 1] <= coarse.group_off[C + 1] &&
            ((fine.row_mask[i] >> c) & 1ull))
          ++n;
      most = n > most ? n : most;
    }
  const size_t smem = (size_t)most * weights::kWRows * sizeof(float);
  switch (coarse.d) {
#define DITANGO_COMPOSE(DD)                                                                      \
  case DD:                                                                                       \
    if (state_bf16)                                                                              \
      merge::compose_kernel<DD, true><<<grid, merge::kThreads, smem, stream>>>(                  \
          fine, coarse, static_cast<const char *>(fine_O), fine_lse, fine_valid,                 \
          static_cast<char *>(coarse_O), coarse_lse, coarse_valid);                              \
    else                                                                                         \
      merge::compose_kernel<DD, false><<<grid, merge::kThreads, smem, stream>>>(                 \
          fine, coarse, static_cast<const char *>(fine_O), fine_lse, fine_valid,                 \
          static_cast<char *>(coarse_O), coarse_lse, coarse_valid);                              \
    return cudaGetLastError();
    DITANGO_COMPOSE(64)
    DITANGO_COMPOSE(96)
    DITANGO_COMPOSE(128)
#undef DITANGO_COMPOSE
    default:
      return cudaErrorInvalidValue;
  }
}

// Read (and optionally clear) this file's check word.
cudaError_t merge_check_status(int *out, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(out, merge::g_merge_check_status, sizeof(int));
  if (e != cudaSuccess || !reset) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(merge::g_merge_check_status, &zero, sizeof(int));
}

}  // namespace ditango
