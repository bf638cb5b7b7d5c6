// Partial attention states of the fresh (query partition, KV partition)
// pairs on B200: tcgen05 MMA with TMEM accumulators, TMA-staged Q/K/V tiles.
//
// What a work unit computes (DiTango, "Riepilogo Tecnico" -> Metodologia ->
// 2. State-Centric Parallel Runtime, "Composizione dello Stato"): for up to
// 256 query rows of partition i and all keys of partition j of one (b, h),
// the state O = softmax(Q K^T * scale) V (normalised) and
// lse = log sum exp(Q K^T * scale), by an online softmax over 128-key tiles.
//
// CTA organisation (one CTA per SM, persistent over work units):
//   warps 0-3  softmax warpgroup 0: rows   0..127 of the unit (Q tile 0)
//   warps 4-7  softmax warpgroup 1: rows 128..255 of the unit (Q tile 1)
//   warp  8    TMA producer (Q tiles, then a 2-stage K ring and V ring)
//   warp  9    TMEM owner and MMA issuer (one thread)
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+d) O1 [384,384+d).
// The bf16 probabilities P_k overwrite the first 64 columns of S_k and feed
// the P V product straight from TMEM.  The two Q tiles ping-pong: while one
// warpgroup exponentiates its S tile, the tensor pipe runs the other tile's
// P V and next Q K^T.  One thread owns one query row, so row max and row sum
// need no cross-thread reduction.  O is rescaled only when a row's running
// maximum grows by more than 2^8 (exact: O and l share the stale maximum).
#include "common.cuh"

namespace ditango {
namespace attn {

constexpr int BM = 128;            // query rows per tile
constexpr int BN = 128;            // keys per tile
constexpr int kThreads = 320;
constexpr int kStages = 2;         // K ring and V ring depth
constexpr float kRescaleLog2 = 8.0f;

template <int D>
struct Cfg {
  static constexpr int NCH = (D + 63) / 64;          // 64-column chunks
  static constexpr int CHUNK = BM * 128;             // bytes of one 128 x 64 bf16 chunk
  static constexpr int TILE = NCH * CHUNK;
  static constexpr int OFF_Q = 0;                    // Q0, Q1
  static constexpr int OFF_K = 2 * TILE;
  static constexpr int OFF_V = OFF_K + kStages * TILE;
  static constexpr int OFF_BAR = OFF_V + kStages * TILE;
  static constexpr int BAR_BYTES = 256;
  static constexpr int USED = OFF_BAR + BAR_BYTES;
  // >= 116 KB keeps one CTA per SM (each CTA allocates all 512 TMEM columns).
  static constexpr int SMEM = (USED + 1024 > 120 * 1024 ? USED + 1024 : 120 * 1024);
};

struct Params {
  DevGeom g;
  const int *fresh_list;
  const int *counts;
  float scale_log2;       // logit scale * log2(e)
  float *out_O;
  float *out_lse;
  int out_by_slot;
  unsigned char *out_valid;
  int *dev_status;
  long long wait_limit_ns;
};

struct Unit {
  bool live;
  int f, i, j, bh, b, h;
  int q0;          // first query token of the unit
  int rloc0;       // row of q0 inside partition i
  int rows0, rows1;
  int k0, Lk, T;   // first key token, keys, key tiles
};

__device__ __forceinline__ Unit decode(const Params &p, int u, int nqt2) {
  Unit w;
  const DevGeom &g = p.g;
  int qt2 = u % nqt2;
  int rest = u / nqt2;
  w.bh = rest % g.BH;
  w.f = rest / g.BH;
  int pair = __ldg(p.fresh_list + w.f);
  w.i = pair / g.P;
  w.j = pair - w.i * g.P;
  w.b = w.bh / g.H;
  w.h = w.bh - w.b * g.H;
  w.rloc0 = qt2 * 2 * BM;
  w.q0 = g.part_off[w.i] + w.rloc0;
  int rem = g.part_off[w.i + 1] - w.q0;
  w.rows0 = rem < BM ? rem : BM;
  int r1 = rem - BM;
  w.rows1 = r1 <= 0 ? 0 : (r1 < BM ? r1 : BM);
  w.k0 = g.part_off[w.j];
  w.Lk = g.part_off[w.j + 1] - w.k0;
  w.T = (w.Lk + BN - 1) / BN;
  w.live = (w.rows0 > 0) && (w.Lk > 0);
  return w;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_partial_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ Params p) {
  using C = Cfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the 128B-swizzled operand tiles
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::OFF_Q;
  const uint32_t sK = sbase + C::OFF_K;
  const uint32_t sV = sbase + C::OFF_V;
  const uint32_t bar = sbase + C::OFF_BAR;
  // barrier addresses (8 bytes each)
  const uint32_t q_full = bar + 0, q_empty = bar + 8;
  auto k_full = [&](int s) { return bar + 16 + 8 * s; };
  auto k_empty = [&](int s) { return bar + 32 + 8 * s; };
  auto v_full = [&](int s) { return bar + 48 + 8 * s; };
  auto v_empty = [&](int s) { return bar + 64 + 8 * s; };
  auto s_full = [&](int k) { return bar + 80 + 8 * k; };
  auto p_full = [&](int k) { return bar + 96 + 8 * k; };
  auto o_full = [&](int k) { return bar + 112 + 8 * k; };
  auto o_empty = [&](int k) { return bar + 128 + 8 * k; };
  const uint32_t drain = bar + 144;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_BAR + 192);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_BAR + 200);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  WaitCtl ctl{abort_flag, p.dev_status, p.wait_limit_ns};

  const int nqt2 = (p.g.Lmax + 2 * BM - 1) / (2 * BM);
  const int n_units = __ldg(p.counts) * p.g.BH * nqt2;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(s_full(k), 1);
      mbar_init(p_full(k), 128);
      mbar_init(o_full(k), 1);
      mbar_init(o_empty(k), 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t kc = 0, vc = 0, uc = 0;
      // last armed phase per full barrier (for a clean stop on abort)
      int q_armed = -1, k_armed[kStages], v_armed[kStages];
      for (int s = 0; s < kStages; ++s) k_armed[s] = v_armed[s] = -1;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        Unit w = decode(p, u, nqt2);
        if (!w.live) continue;
        if (!(ok = wait_bounded(q_empty, (uc & 1) ^ 1, ctl))) break;
        const uint32_t qbytes = C::TILE * (w.rows1 > 0 ? 2 : 1);
        mbar_arrive_expect_tx(q_full, qbytes);
        q_armed = uc & 1;
        for (int c = 0; c < C::NCH; ++c)
          tma_load_4d(sQ + c * C::CHUNK, &tmQ, q_full, c * 64, w.q0, w.h, w.b);
        if (w.rows1 > 0)
          for (int c = 0; c < C::NCH; ++c)
            tma_load_4d(sQ + C::TILE + c * C::CHUNK, &tmQ, q_full, c * 64, w.q0 + BM, w.h, w.b);
        for (int t = 0; t < w.T && ok; ++t) {
          const int row = w.k0 + t * BN;
          int s = kc % kStages;
          if (!(ok = wait_bounded(k_empty(s), ((kc / kStages) & 1) ^ 1, ctl))) break;
          mbar_arrive_expect_tx(k_full(s), C::TILE);
          k_armed[s] = (kc / kStages) & 1;
          for (int c = 0; c < C::NCH; ++c)
            tma_load_4d(sK + s * C::TILE + c * C::CHUNK, &tmK, k_full(s), c * 64, row, w.h, w.b);
          ++kc;
          s = vc % kStages;
          if (!(ok = wait_bounded(v_empty(s), ((vc / kStages) & 1) ^ 1, ctl))) break;
          mbar_arrive_expect_tx(v_full(s), C::TILE);
          v_armed[s] = (vc / kStages) & 1;
          for (int c = 0; c < C::NCH; ++c)
            tma_load_4d(sV + s * C::TILE + c * C::CHUNK, &tmV, v_full(s), c * 64, row, w.h, w.b);
          ++vc;
        }
        ++uc;
      }
      if (!ok) {
        // stop cleanly: let every load already issued land before exiting
        WaitCtl drain_ctl{nullptr, nullptr, 100000000LL};
        volatile int never = 0;
        drain_ctl.abort_flag = &never;
        if (q_armed >= 0) wait_bounded(q_full, (uint32_t)q_armed, drain_ctl);
        for (int s = 0; s < kStages; ++s) {
          if (k_armed[s] >= 0) wait_bounded(k_full(s), (uint32_t)k_armed[s], drain_ctl);
          if (v_armed[s] >= 0) wait_bounded(v_full(s), (uint32_t)v_armed[s], drain_ctl);
        }
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, BN, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, D, 0, 1);
      uint32_t kc = 0, vc = 0, uc = 0;
      uint32_t pc[2] = {0, 0}, oc[2] = {0, 0};
      bool ok = true;
      auto qk = [&](int k, int ks) {
        // S_k = Q_k K^T : K-major A and B, 16 columns of d per instruction
        const uint32_t qa = sQ + k * C::TILE;
        const uint32_t kb = sK + ks * C::TILE;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::CHUNK + (kk & 3) * 32;
          mma_ss(tmem + k * 128, smem_desc_sw128(qa + off, 16, 1024),
                 smem_desc_sw128(kb + off, 16, 1024), idesc_qk, kk > 0);
        }
      };
      auto pv = [&](int k, int vs, bool acc) {
        // O_k (+)= P_k V : P from TMEM (K-major), V MN-major (d contiguous)
        const uint32_t vb = sV + vs * C::TILE;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          mma_ts(tmem + 256 + k * 128, tmem + k * 128 + kk * 8,
                 smem_desc_sw128(vb + kk * 2048, C::CHUNK, 1024), idesc_pv, (acc || kk > 0));
        }
      };
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        Unit w = decode(p, u, nqt2);
        if (!w.live) continue;
        const bool has1 = w.rows1 > 0;
        if (!(ok = wait_bounded(q_full, uc & 1, ctl))) break;
        int ks = kc % kStages;
        if (!(ok = wait_bounded(k_full(ks), (kc / kStages) & 1, ctl))) break;
        tc_fence_after();
        qk(0, ks);
        tc_commit(s_full(0));
        if (has1) {
          qk(1, ks);
          tc_commit(s_full(1));
        }
        tc_commit(k_empty(ks));
        ++kc;
        if (w.T == 1) tc_commit(q_empty);
        for (int t = 0; t < w.T && ok; ++t) {
          const int vs = vc % kStages;
          if (!(ok = wait_bounded(v_full(vs), (vc / kStages) & 1, ctl))) break;
          const bool more = (t + 1 < w.T);
          // ---- Q tile 0
          if (!(ok = wait_bounded(p_full(0), pc[0] & 1, ctl))) break;
          ++pc[0];
          if (t == 0) {
            if (!(ok = wait_bounded(o_empty(0), (oc[0] & 1) ^ 1, ctl))) break;
            ++oc[0];
          }
          tc_fence_after();
          pv(0, vs, t > 0);
          if (!more) tc_commit(o_full(0));
          int ks2 = kc % kStages;
          if (more) {
            if (!(ok = wait_bounded(k_full(ks2), (kc / kStages) & 1, ctl))) break;
            tc_fence_after();
            qk(0, ks2);
            tc_commit(s_full(0));
          }
          // ---- Q tile 1
          if (has1) {
            if (!(ok = wait_bounded(p_full(1), pc[1] & 1, ctl))) break;
            ++pc[1];
            if (t == 0) {
              if (!(ok = wait_bounded(o_empty(1), (oc[1] & 1) ^ 1, ctl))) break;
              ++oc[1];
            }
            tc_fence_after();
            pv(1, vs, t > 0);
            if (!more) tc_commit(o_full(1));
            if (more) {
              qk(1, ks2);
              tc_commit(s_full(1));
            }
          }
          tc_commit(v_empty(vs));
          ++vc;
          if (more) {
            tc_commit(k_empty(ks2));
            ++kc;
            if (t + 2 == w.T) tc_commit(q_empty);
          }
        }
        ++uc;
      }
      // drain: every MMA issued so far must finish before TMEM is released
      tc_commit(drain);
      WaitCtl drain_ctl{nullptr, nullptr, 100000000LL};
      volatile int never = 0;
      drain_ctl.abort_flag = &never;
      wait_bounded(drain, 0, drain_ctl);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int k = warp >> 2;                 // Q tile of this warpgroup
    const int r = threadIdx.x & 127;         // row within the tile = TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + k * 128;
    const uint32_t tO = tmem + lane_base + 256 + k * 128;
    const float sl2 = p.scale_log2;
    uint32_t sc = 0, ofc = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      Unit w = decode(p, u, nqt2);
      if (!w.live) continue;
      const int rows_k = (k == 0) ? w.rows0 : w.rows1;
      if (rows_k <= 0) continue;
      float m_used = -INFINITY;   // running maximum used for exponentiation (log2 units)
      float l = 0.f;
      for (int t = 0; t < w.T; ++t) {
        if (!(ok = wait_bounded(s_full(k), sc & 1, ctl))) break;
        ++sc;
        tc_fence_after();
        float s[BN];
        {
          uint32_t v[32];
#pragma unroll
          for (int c = 0; c < BN / 32; ++c) {
            tmem_ld32(tS + c * 32, v);
            tc_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) s[c * 32 + e] = __uint_as_float(v[e]);
          }
        }
        const int valid = w.Lk - t * BN;
        if (valid < BN) {
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (c >= valid) s[c] = -INFINITY;
        }
        float mx = s[0];
#pragma unroll
        for (int c = 1; c < BN; ++c) mx = fmaxf(mx, s[c]);
        const float mx2 = mx * sl2;
        if (t == 0) {
          m_used = mx2;
        } else {
          const bool need = mx2 > m_used + kRescaleLog2;
          if (__any_sync(0xffffffffu, need)) {
            // O of this row already holds every P V of earlier tiles: the
            // commit that released S(t) covers all earlier MMAs.
            const float m_new = need ? mx2 : m_used;
            const float alpha = ex2(m_used - m_new);
            l *= alpha;
            m_used = m_new;
            uint32_t v[32];
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              tmem_ld32(tO + c * 32, v);
              tc_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
              tmem_st32(tO + c * 32, v);
            }
          }
        }
        const float neg = -m_used;
        uint32_t pk[32];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float a = ex2(fmaf(s[h2 * 64 + 2 * e], sl2, neg));
            const float b = ex2(fmaf(s[h2 * 64 + 2 * e + 1], sl2, neg));
            l += a + b;
            pk[e] = pack_bf16(a, b);
          }
          tmem_st32(tS + h2 * 32, pk);
        }
        tc_wait_st();
        tc_fence_before();
        mbar_arrive(p_full(k));
      }
      if (!ok) break;
      // ---- epilogue: normalise and store the state of this row
      if (!(ok = wait_bounded(o_full(k), ofc & 1, ctl))) break;
      ++ofc;
      tc_fence_after();
      const int idx = p.out_by_slot ? slot_of(p.g, w.i, w.j) : w.f;
      const int rloc = w.rloc0 + k * BM + r;
      const size_t row_off = ((size_t)idx * p.g.BH + w.bh) * (size_t)p.g.Lmax + rloc;
      const bool row_ok = r < rows_k;
      const float inv_l = 1.f / l;
      float4 *dst = reinterpret_cast<float4 *>(p.out_O + row_off * D);
      uint32_t v[32];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        tmem_ld32(tO + c * 32, v);
        tc_wait_ld();
        if (row_ok) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            float4 o;
            o.x = __uint_as_float(v[4 * e + 0]) * inv_l;
            o.y = __uint_as_float(v[4 * e + 1]) * inv_l;
            o.z = __uint_as_float(v[4 * e + 2]) * inv_l;
            o.w = __uint_as_float(v[4 * e + 3]) * inv_l;
            dst[c * 8 + e] = o;
          }
        }
      }
      if (row_ok) p.out_lse[row_off] = (m_used + __log2f(l)) * 0.69314718055994531f;
      if (p.out_by_slot && p.out_valid && k == 0 && r == 0) p.out_valid[idx] = 1;
      tc_fence_before();
      mbar_arrive(o_empty(k));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace attn

// Host launcher (called from the C ABI after validation).
cudaError_t launch_attn_partial(const DevGeom &g, const CUtensorMap &tq, const CUtensorMap &tk,
                                const CUtensorMap &tv, const int *fresh_list, const int *counts,
                                float scale, float *out_O, float *out_lse, int out_by_slot,
                                unsigned char *out_valid, int *dev_status, long long wait_limit_ns,
                                int num_sms, cudaStream_t stream) {
  attn::Params p;
  p.g = g;
  p.fresh_list = fresh_list;
  p.counts = counts;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.out_O = out_O;
  p.out_lse = out_lse;
  p.out_by_slot = out_by_slot;
  p.out_valid = out_valid;
  p.dev_status = dev_status;
  p.wait_limit_ns = wait_limit_ns;
  const long long nqt2 = (g.Lmax + 255) / 256;
  const long long max_units = (long long)g.n_active * g.BH * nqt2;
  if (max_units == 0) return cudaSuccess;
  const int grid = (int)(max_units < num_sms ? max_units : num_sms);
  cudaError_t e = cudaSuccess;
  switch (g.d) {
#define DITANGO_LAUNCH(DD)                                                                       \
  case DD: {                                                                                     \
    auto kfn = attn::attn_partial_kernel<DD>;                                                    \
    e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize,                   \
                             attn::Cfg<DD>::SMEM);                                               \
    if (e != cudaSuccess) return e;                                                              \
    kfn<<<grid, attn::kThreads, attn::Cfg<DD>::SMEM, stream>>>(tq, tk, tv, p);                    \
    return cudaGetLastError();                                                                   \
  }
    DITANGO_LAUNCH(64)
    DITANGO_LAUNCH(96)
    DITANGO_LAUNCH(128)
#undef DITANGO_LAUNCH
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace ditango
