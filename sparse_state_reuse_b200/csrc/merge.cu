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
// The merge is HBM bound: one warp per token row, d/4 lanes each holding a
// float4 of d; the loads of up to 8 states are issued before they are
// consumed so that enough bytes are in flight.  The per-block table of
// source pointers (fresh -> partial buffer at its fresh-list position,
// reuse -> cache slot) is built once per (b*h, partition) in shared memory.
#include <cuda_bf16.h>

#include "common.cuh"

namespace ditango {
namespace merge {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRowsPerBlock = 128;
constexpr int kBatch = 4;    // O vectors per row in flight per lane
constexpr int kSmallStates = 4;  // rows of at most this many states: per-lane weights

struct Src {
  const char *O;     // [Lmax][d] block of this (index, b*h): float32, or bf16 (SB)
  const float *lse;  // [Lmax]
  char *wbO;         // cache block to write back into, or null
  float *wblse;
};

// Four consecutive O values of a state row (float32, or bf16 when SB).
template <bool SB>
__device__ __forceinline__ float4 load_o4(const char *p) {
  if constexpr (SB) {
    const uint2 u = __ldg(reinterpret_cast<const uint2 *>(p));
    return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                       __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
  } else {
    return __ldg(reinterpret_cast<const float4 *>(p));
  }
}

// Raw form of four stored O values (kept packed until used).
template <bool SB>
struct Raw4 {
  using T = float4;
};
template <>
struct Raw4<true> {
  using T = uint2;
};
template <bool SB>
__device__ __forceinline__ typename Raw4<SB>::T load_raw4(const char *p) {
  if constexpr (SB)
    return __ldg(reinterpret_cast<const uint2 *>(p));
  else
    return __ldg(reinterpret_cast<const float4 *>(p));
}
template <bool SB>
__device__ __forceinline__ float4 widen4(typename Raw4<SB>::T u) {
  if constexpr (SB)
    return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                       __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
  else
    return u;
}
template <bool SB>
__device__ __forceinline__ typename Raw4<SB>::T zero_raw4() {
  if constexpr (SB)
    return make_uint2(0u, 0u);
  else
    return make_float4(0.f, 0.f, 0.f, 0.f);
}
template <bool SB>
__device__ __forceinline__ void store_raw4(char *p, typename Raw4<SB>::T u) {
  if constexpr (SB)
    *reinterpret_cast<uint2 *>(p) = u;
  else
    *reinterpret_cast<float4 *>(p) = u;
}

// Store four values that came from load_o4 (exact in either format).
template <bool SB>
__device__ __forceinline__ void store_o4(char *p, float4 v) {
  if constexpr (SB) {
    uint2 u;
    u.x = (__float_as_uint(v.x) >> 16) | (__float_as_uint(v.y) & 0xffff0000u);
    u.y = (__float_as_uint(v.z) >> 16) | (__float_as_uint(v.w) & 0xffff0000u);
    *reinterpret_cast<uint2 *>(p) = u;
  } else {
    *reinterpret_cast<float4 *>(p) = v;
  }
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

// Weights of one row: lane a holds lse of state a (l0) and a + 32 (l1);
// returns exp(lse_a - L) for both and L = log sum_a exp(lse_a).
__device__ __forceinline__ void lse_weights(float l0, float l1, float &w0, float &w1, float &L) {
  float M = fmaxf(l0, l1);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const bool dead = !(M > -INFINITY);
  const float Ms = dead ? 0.f : M;
  const float e0 = expf(l0 - Ms), e1 = expf(l1 - Ms);
  float S = e0 + e1;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) S += __shfl_xor_sync(0xffffffffu, S, o);
  const float invS = dead ? 0.f : 1.f / S;
  w0 = e0 * invS;
  w1 = e1 * invS;
  L = dead ? -INFINITY : Ms + logf(S);
}

// MS > 0: every row has at most MS states (frame-tile rows hold 2 to 4;
// measured on B200, rows of 8 states merge faster on the general path).
// Then each lane loads all of a row's lse (one broadcast load each) and
// computes the row's weights itself: no shuffles, and the weights overwrite
// the loaded lse in place.  MS = 0: any number of states (up to 64), weights
// by warp reductions over one state per lane.
template <int D, bool SB, int MS>
__global__ void __launch_bounds__(kThreads, SB ? 3 : 4)
merge_kernel(DevGeom g, const signed char *__restrict__ plan, const char *__restrict__ part_O,
             const float *__restrict__ part_lse, char *cache_O, float *cache_lse,
             unsigned char *cache_valid, int writeback, void *out, int out_is_fp32, long long osb,
             long long osh, long long osn, float *__restrict__ out_lse) {
  constexpr int G4 = D / 4;  // lanes carrying one row
  constexpr int ES = SB ? 2 : 4;            // bytes per stored O element
  constexpr size_t ROWB = (size_t)D * ES;   // bytes per state row
  const int i = blockIdx.y;
  const int bh = blockIdx.z;
  const int Li = g.part_off[i + 1] - g.part_off[i];
  const int r0 = blockIdx.x * kRowsPerBlock;
  if (r0 >= Li) return;
  const int G = g.G;
  __shared__ Src src[kMaxP];
  __shared__ int s_nact, s_fresh_before;
  __shared__ int warp_cnt[kWarps];
  __shared__ signed char s_plan[kMaxP];
  if (threadIdx.x < G) s_plan[threadIdx.x] = plan[i * G + threadIdx.x];

  // fresh units before row i (row-major), for fresh-list positions
  int cnt = 0;
  for (int p = threadIdx.x; p < i * G; p += kThreads) cnt += (plan[p] == DITANGO_PLAN_FRESH);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if ((threadIdx.x & 31) == 0) warp_cnt[threadIdx.x >> 5] = cnt;
  __syncthreads();
  if (threadIdx.x == 0) {
    int fb = 0;
    for (int w = 0; w < kWarps; ++w) fb += warp_cnt[w];
    s_fresh_before = fb;
    const size_t blk = (size_t)g.BH * g.Lmax;
    int a = 0;
    const int slot0 = g.row_start[i];
    int fpos = fb;
    for (int c = 0; c < G; ++c) {
      if (!((g.row_mask[i] >> c) & 1ull)) continue;
      const int code = s_plan[c];
      const int slot = slot0 + __popcll(g.row_mask[i] & ((c == 0) ? 0ull : (~0ull >> (64 - c))));
      Src s;
      s.wbO = nullptr;
      s.wblse = nullptr;
      if (code == DITANGO_PLAN_FRESH) {
        if (part_O != nullptr) {
          s.O = part_O + ((size_t)fpos * blk + (size_t)bh * g.Lmax) * ROWB;
          s.lse = part_lse + (size_t)fpos * blk + (size_t)bh * g.Lmax;
          if (writeback) {
            s.wbO = cache_O + ((size_t)slot * blk + (size_t)bh * g.Lmax) * ROWB;
            s.wblse = cache_lse + (size_t)slot * blk + (size_t)bh * g.Lmax;
            if (cache_valid && bh == 0 && blockIdx.x == 0) cache_valid[slot] = 1;
          }
        } else {
          s.O = cache_O + ((size_t)slot * blk + (size_t)bh * g.Lmax) * ROWB;
          s.lse = cache_lse + (size_t)slot * blk + (size_t)bh * g.Lmax;
        }
        ++fpos;
      } else if (code == DITANGO_PLAN_REUSE) {
        s.O = cache_O + ((size_t)slot * blk + (size_t)bh * g.Lmax) * ROWB;
        s.lse = cache_lse + (size_t)slot * blk + (size_t)bh * g.Lmax;
      } else {
        continue;  // active unit the plan skipped: contributes nothing
      }
      src[a++] = s;
    }
    s_nact = a;
  }
  __syncthreads();
  const int nact = s_nact;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = bh / g.H, h = bh - (bh / g.H) * g.H;
  const int rend = (r0 + kRowsPerBlock < Li) ? r0 + kRowsPerBlock : Li;

  // R rows per warp iteration (2 for fp32 states, 4 for bf16 states, so both
  // keep the same bytes in flight); every load of a row -- its states' lse
  // and the first kBatch O vectors -- is issued before any of it is used.
  constexpr int R = SB ? 4 : 2;
  if constexpr (MS > 0) {
    constexpr int RS = 2;   // rows per warp iteration (the weights live in registers)
    const bool act = lane < G4;
    for (int r = r0 + RS * warp; r < rend; r += RS * kWarps) {
      constexpr int R = RS;
      float wt[R][MS];   // the states' lse, then their weights
#pragma unroll
      for (int q = 0; q < R; ++q)
#pragma unroll
        for (int a = 0; a < MS; ++a)
          wt[q][a] = (a < nact && (r + q) < rend) ? __ldg(src[a].lse + r + q) : -INFINITY;
      typename Raw4<SB>::T v[R][kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
#pragma unroll
        for (int q = 0; q < R; ++q) {
          v[q][u] = zero_raw4<SB>();
          if (act && u < nact && (r + q) < rend)
            v[q][u] = load_raw4<SB>(src[u].O + (size_t)(r + q) * ROWB + lane * 4 * ES);
        }
      float L[R];
#pragma unroll
      for (int q = 0; q < R; ++q) {
        // write back the lse of fresh states (lane a for state a)
#pragma unroll
        for (int a = 0; a < MS; ++a)
          if (lane == a && a < nact && (r + q) < rend && src[a].wblse) src[a].wblse[r + q] = wt[q][a];
        float M = wt[q][0];
#pragma unroll
        for (int a = 1; a < MS; ++a) M = fmaxf(M, wt[q][a]);
        const bool dead = !(M > -INFINITY);
        const float Ms = dead ? 0.f : M;
        float S = 0.f;
#pragma unroll
        for (int a = 0; a < MS; ++a) {
          wt[q][a] = expf(wt[q][a] - Ms);   // exp(-inf) = 0 for absent states
          S += wt[q][a];
        }
        const float invS = dead ? 0.f : 1.f / S;
#pragma unroll
        for (int a = 0; a < MS; ++a) wt[q][a] *= invS;
        L[q] = dead ? -INFINITY : Ms + logf(S);
      }
      float4 acc[R];
#pragma unroll
      for (int q = 0; q < R; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int a0 = 0; a0 < MS; a0 += kBatch) {
        if (a0 >= nact) break;
        if (a0 > 0) {
#pragma unroll
          for (int u = 0; u < kBatch; ++u)
#pragma unroll
            for (int q = 0; q < R; ++q)
              if (act && a0 + u < nact && (r + q) < rend)
                v[q][u] = load_raw4<SB>(src[a0 + u].O + (size_t)(r + q) * ROWB + lane * 4 * ES);
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          const int a = a0 + u;
          if (a >= nact) break;
#pragma unroll
          for (int q = 0; q < R; ++q) {
            fma4(acc[q], wt[q][a], widen4<SB>(v[q][u]));
            if (act && src[a].wbO && (r + q) < rend)
              store_raw4<SB>(src[a].wbO + (size_t)(r + q) * ROWB + lane * 4 * ES, v[q][u]);
          }
        }
      }
      const int n = g.part_off[i] + r;
      const size_t obase = (size_t)b * osb + (size_t)h * osh + lane * 4;
#pragma unroll
      for (int q = 0; q < R; ++q) {
        if ((r + q) >= rend) continue;
        if (act) store_out(out, out_is_fp32, obase + (size_t)(n + q) * osn, acc[q]);
        if (out_lse && lane == 0) out_lse[((size_t)b * g.H + h) * g.N + n + q] = L[q];
      }
    }
  } else {
  for (int r = r0 + R * warp; r < rend; r += R * kWarps) {
    float l0[R], l1[R];
#pragma unroll
    for (int q = 0; q < R; ++q) {
      const bool ok = (r + q) < rend;
      l0[q] = (ok && lane < nact) ? __ldg(src[lane].lse + r + q) : -INFINITY;
      l1[q] = (ok && lane + 32 < nact) ? __ldg(src[lane + 32].lse + r + q) : -INFINITY;
    }
    const bool act = lane < G4;
    typename Raw4<SB>::T v[R][kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u)
#pragma unroll
      for (int q = 0; q < R; ++q) {
        v[q][u] = zero_raw4<SB>();
        if (act && u < nact && (r + q) < rend)
          v[q][u] = load_raw4<SB>(src[u].O + (size_t)(r + q) * ROWB + lane * 4 * ES);
      }
    float w0[R], w1[R], L[R];
#pragma unroll
    for (int q = 0; q < R; ++q) lse_weights(l0[q], l1[q], w0[q], w1[q], L[q]);
    float4 acc[R];
#pragma unroll
    for (int q = 0; q < R; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int a0 = 0; a0 < nact; a0 += kBatch) {
      if (a0 > 0) {
#pragma unroll
        for (int u = 0; u < kBatch; ++u)
#pragma unroll
          for (int q = 0; q < R; ++q)
            if (act && a0 + u < nact && (r + q) < rend)
              v[q][u] = load_raw4<SB>(src[a0 + u].O + (size_t)(r + q) * ROWB + lane * 4 * ES);
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int a = a0 + u;
#pragma unroll
        for (int q = 0; q < R; ++q) {
          const float wq = __shfl_sync(0xffffffffu, (a < 32) ? w0[q] : w1[q], a & 31);
          if (a < nact) {
            fma4(acc[q], wq, widen4<SB>(v[q][u]));
            if (act && src[a].wbO && (r + q) < rend)
              store_raw4<SB>(src[a].wbO + (size_t)(r + q) * ROWB + lane * 4 * ES, v[q][u]);
          }
        }
      }
    }
    // write back the lse of fresh states
#pragma unroll
    for (int q = 0; q < R; ++q) {
      if ((r + q) >= rend) continue;
      if (lane < nact && src[lane].wblse) src[lane].wblse[r + q] = l0[q];
      if (lane + 32 < nact && src[lane + 32].wblse) src[lane + 32].wblse[r + q] = l1[q];
    }
    const int n = g.part_off[i] + r;
    const size_t obase = (size_t)b * osb + (size_t)h * osh + lane * 4;
#pragma unroll
    for (int q = 0; q < R; ++q) {
      if ((r + q) >= rend) continue;
      if (act) store_out(out, out_is_fp32, obase + (size_t)(n + q) * osn, acc[q]);
      if (out_lse && lane == 0) out_lse[((size_t)b * g.H + h) * g.N + n + q] = L[q];
    }
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
// blockIdx.z = b*h, blockIdx.x = a block of kRowsPerBlock rows; one warp
// merges R rows at a time with d/4 lanes per row, as in the merge.  A
// coarse slot is valid only if every fine slot it covers is; an invalid one
// is marked and left unwritten.
template <int D, bool SB>
__global__ void __launch_bounds__(kThreads, SB ? 3 : 4)
compose_kernel(DevGeom fine, DevGeom coarse, const char *__restrict__ fO,
               const float *__restrict__ flse, const unsigned char *__restrict__ fvalid,
               char *__restrict__ cO, float *__restrict__ clse, unsigned char *cvalid) {
  constexpr int G4 = D / 4;                 // lanes carrying one row
  constexpr int ES = SB ? 2 : 4;
  constexpr size_t ROWB = (size_t)D * ES;
  const int cslot = blockIdx.y;
  const int bh = blockIdx.z;
  int i = 0;
  while (i + 1 < coarse.P && coarse.row_start[i + 1] <= cslot) ++i;
  unsigned long long m = coarse.row_mask[i];
  for (int t = cslot - coarse.row_start[i]; t > 0; --t) m &= m - 1;
  const int C = __ffsll((long long)m) - 1;
  const int Li = coarse.part_off[i + 1] - coarse.part_off[i];
  const int r0 = blockIdx.x * kRowsPerBlock;
  if (r0 >= Li) return;
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

  const size_t blk = (size_t)fine.BH * fine.Lmax;
  const size_t base = (size_t)bh * fine.Lmax;
  const char *srcO = fO + ((size_t)fs0 * blk + base) * ROWB;   // fine slot a: + a * blk * ROWB
  const float *srcl = flse + (size_t)fs0 * blk + base;
  char *dstO = cO + ((size_t)cslot * blk + base) * ROWB;
  float *dstl = clse + (size_t)cslot * blk + base;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rend = (r0 + kRowsPerBlock < Li) ? r0 + kRowsPerBlock : Li;
  const bool act = lane < G4;
  constexpr int R = SB ? 4 : 2;
  for (int r = r0 + R * warp; r < rend; r += R * kWarps) {
    float l0[R], l1[R];
#pragma unroll
    for (int q = 0; q < R; ++q) {
      const bool ok = (r + q) < rend;
      l0[q] = (ok && lane < nf) ? __ldg(srcl + (size_t)lane * blk + r + q) : -INFINITY;
      l1[q] = (ok && lane + 32 < nf) ? __ldg(srcl + (size_t)(lane + 32) * blk + r + q) : -INFINITY;
    }
    typename Raw4<SB>::T v[R][kBatch];
    float w0[R], w1[R], L[R];
    float4 acc[R];
#pragma unroll
    for (int q = 0; q < R; ++q) {
      lse_weights(l0[q], l1[q], w0[q], w1[q], L[q]);
      acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int a0 = 0; a0 < nf; a0 += kBatch) {
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
#pragma unroll
        for (int q = 0; q < R; ++q) {
          v[q][u] = zero_raw4<SB>();
          if (act && a0 + u < nf && (r + q) < rend)
            v[q][u] = load_raw4<SB>(srcO + ((size_t)(a0 + u) * blk + r + q) * ROWB + lane * 4 * ES);
        }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int a = a0 + u;
#pragma unroll
        for (int q = 0; q < R; ++q) {
          const float wq = __shfl_sync(0xffffffffu, (a < 32) ? w0[q] : w1[q], a & 31);
          if (a < nf) fma4(acc[q], wq, widen4<SB>(v[q][u]));
        }
      }
    }
#pragma unroll
    for (int q = 0; q < R; ++q) {
      if ((r + q) >= rend) continue;
      if (act) store_out(dstO, SB ? 0 : 1, (size_t)(r + q) * D + lane * 4, acc[q]);
      if (lane == 0) dstl[r + q] = L[q];
    }
  }
}

}  // namespace merge

cudaError_t launch_merge(const DevGeom &g, const signed char *plan, const void *part_O,
                         const float *part_lse, void *cache_O, float *cache_lse,
                         unsigned char *cache_valid, int writeback, int state_bf16, void *out,
                         int out_is_fp32,
                         long long osb, long long osh, long long osn, float *out_lse,
                         cudaStream_t stream) {
  dim3 grid((g.Lmax + merge::kRowsPerBlock - 1) / merge::kRowsPerBlock, g.P, g.BH);
  int most = 0;   // most active units of any row: the states a row can merge
  for (int i = 0; i < g.P; ++i) {
    const int c = __builtin_popcountll(g.row_mask[i]);
    most = c > most ? c : most;
  }
  const int ms = most <= merge::kSmallStates ? merge::kSmallStates : 0;
  switch (g.d) {
#define DITANGO_MERGE_MS(DD, SB, MS)                                                             \
  merge::merge_kernel<DD, SB, MS><<<grid, merge::kThreads, 0, stream>>>(                         \
      g, plan, static_cast<const char *>(part_O), part_lse, static_cast<char *>(cache_O),       \
      cache_lse, cache_valid, writeback, out, out_is_fp32, osb, osh, osn, out_lse);
#define DITANGO_MERGE_SB(DD, SB)                                                                 \
  if (ms == merge::kSmallStates) {                                                               \
    DITANGO_MERGE_MS(DD, SB, merge::kSmallStates)                                                \
  } else {                                                                                       \
    DITANGO_MERGE_MS(DD, SB, 0)                                                                  \
  }
#define DITANGO_MERGE(DD)                                                                        \
  case DD:                                                                                       \
    if (state_bf16) {                                                                            \
      DITANGO_MERGE_SB(DD, true)                                                                 \
    } else {                                                                                     \
      DITANGO_MERGE_SB(DD, false)                                                                \
    }                                                                                            \
    return cudaGetLastError();
    DITANGO_MERGE(64)
    DITANGO_MERGE(96)
    DITANGO_MERGE(128)
#undef DITANGO_MERGE
#undef DITANGO_MERGE_SB
#undef DITANGO_MERGE_MS
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
  dim3 grid((coarse.Lmax + merge::kRowsPerBlock - 1) / merge::kRowsPerBlock, coarse.n_active,
            coarse.BH);
  switch (coarse.d) {
#define DITANGO_COMPOSE(DD)                                                                      \
  case DD:                                                                                       \
    if (state_bf16)                                                                              \
      merge::compose_kernel<DD, true><<<grid, merge::kThreads, 0, stream>>>(                     \
          fine, coarse, static_cast<const char *>(fine_O), fine_lse, fine_valid,                 \
          static_cast<char *>(coarse_O), coarse_lse, coarse_valid);                              \
    else                                                                                         \
      merge::compose_kernel<DD, false><<<grid, merge::kThreads, 0, stream>>>(                    \
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

}  // namespace ditango
