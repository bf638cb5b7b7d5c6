// Partial attention states of the fresh (query partition, KV group) units
// on B200: tcgen05 MMA with TMEM accumulators, TMA-staged Q/K/V tiles.
//
// What a work item computes (DiTango, "Riepilogo Tecnico" -> Metodologia ->
// 2. State-Centric Parallel Runtime, "Composizione dello Stato" and
// "Calcolo dello Stato di Gruppo"): for up to 256 query rows of partition i
// and all keys of the active partitions of KV group c of one (b, h), the
// state O = softmax(Q K^T * scale) V (normalised) and
// lse = log sum exp(Q K^T * scale), by an online softmax over key tiles
// (96 keys at d = 96, else 128).
// Without KV groups a group is one partition and a unit is a pair (i, j).
// A group's active partitions are walked as runs of adjacent partitions,
// each run one contiguous key range whose last tile is masked at its end.
//
// CTA organisation (one CTA per SM, persistent over work units, 384 threads):
//   warps 0-3  softmax warpgroup 0: rows   0..127 of the unit (Q tile 0)
//   warps 4-7  softmax warpgroup 1: rows 128..255 of the unit (Q tile 1)
//   warp  8    TMA producer (Q tiles, then a 2-stage K ring and V ring)
//   warp  9    TMEM owner and MMA issuer (one thread); d = 64 and 96: the
//              MMA issuer of Q tile 0
//   warp  10   d = 64 and 96: the MMA issuer of Q tile 1; else idle
//   warp  11   idle
// Registers are rebalanced with setmaxnreg: the softmax warpgroups, which
// hold a whole S row per thread, get softmax_regs; warpgroup 2 drops to
// control_regs.  2 * 128 * 216 + 128 * 72 = 2 * 128 * 192 + 128 * 120 =
// 384 * 168, the registers the CTA is launched with; the launcher refuses to
// launch a build whose register count differs (an unbalanced split would
// block forever).
// One thread owns one query row (TMEM lane), so row max and row sum need no
// cross-thread reduction.  O is rescaled only when a row's running maximum
// grows by more than 2^8 (exact: O and l share the stale maximum).
// d = 128: TMEM S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512); the bf16
// probabilities P_k overwrite the first 64 columns of S_k and feed the P V
// product straight from TMEM.  The two Q tiles ping-pong: while one
// warpgroup exponentiates its S tile, the tensor pipe runs the other tile's
// P V and next Q K^T (which waits for that P V, since P lives in S).
// d = 64 and 96 ("free S"): P_k has TMEM columns of its own (Cfg::P_COL),
// so each softmax warp signals s_free as soon as S is in its registers and
// the next Q K^T runs under its exponentials; it forms the whole P row in
// registers and only then waits on p_free (the P V that read the previous P
// is done, normally long before) to overwrite P_k.  Each Q tile
// has its own MMA warp, so neither tile waits for the other's events.
// Work items go from the producer warp to the other roles through a 2-slot
// ring in shared memory; with a work counter each CTA takes the next item
// when it is ready for it (balanced whatever the items' sizes), otherwise
// items are taken in a fixed stride.  Items are numbered in (b*h, partition,
// rows) order, every partition's last block of rows after all the others:
// the CTAs running at the same time share one (b, h)'s K/V in L2, and the
// small items fill the end of the schedule.
#include <mutex>
#include <set>
#include <utility>

#include "common.cuh"

namespace ditango {
namespace attn {

constexpr int BM = 128;            // query rows per tile
constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;   // 65536 / 384, rounded down to a multiple of 8
// Registers per thread after setmaxnreg: the softmax warpgroups hold a whole
// S row (128 columns; 96 at d = 96), the control warpgroup the producer and
// MMA loops.  At d = 96 the two MMA warps of the free-S pipeline need more
// than 72 (they spilled inside their loops) and the 96-column softmax rows
// fewer than 216.
template <int D> __host__ __device__ constexpr int softmax_regs() { return D == 96 ? 192 : 216; }
template <int D> __host__ __device__ constexpr int control_regs() { return D == 96 ? 120 : 72; }
template <int D> __host__ __device__ constexpr bool split_ok() {
  return 2 * 128 * softmax_regs<D>() + 128 * control_regs<D>() == kThreads * kLaunchRegs;
}
static_assert(split_ok<64>() && split_ok<96>() && split_ok<128>(),
              "register split must equal the launch budget");
constexpr int kStages = 2;         // K ring and V ring depth
constexpr float kRescaleLog2 = 8.0f;

// Key tile and TMEM plan per head dimension.
//   d = 128: 128-key tiles; S_k [128k, 128k+128), O_k [256+128k, ...); the
//     bf16 P_k overwrites the first 64 columns of S_k, so the next Q K^T of
//     tile k waits for its P V.
//   d = 64 and 96 (FS, "free S"): P_k has columns of its own, so the next
//     Q K^T of tile k is issued as soon as S_k is in the softmax registers and
//     runs under the exponentials.  d = 96 takes 96-key tiles to fit:
//     S0 [0,96) P0 [96,144) S1 [160,256) P1 [256,304) O0 [320,416) O1 [416,512);
//     d = 64, 128-key tiles: S0 [0,128) P0 [128,192) S1 [192,320) P1 [320,384)
//     O0 [384,448) O1 [448,512).  Every region starts on a multiple of 32.
template <int D>
struct Cfg {
  static constexpr bool FS = (D != 128);
  static constexpr int BN = (D == 96) ? 96 : 128;    // keys per tile
  static constexpr int NCH = (D + 63) / 64;          // 64-column chunks
  static constexpr int QCHUNK = BM * 128;            // bytes of one 128-row x 64-column bf16 chunk
  static constexpr int KCHUNK = BN * 128;            // bytes of one BN-row chunk
  static constexpr int QTILE = NCH * QCHUNK;
  static constexpr int KTILE = NCH * KCHUNK;
  static constexpr int OFF_Q = 0;                    // Q0, Q1
  static constexpr int OFF_K = 2 * QTILE;
  static constexpr int OFF_V = OFF_K + kStages * KTILE;
  static constexpr int OFF_EPI = OFF_V + kStages * KTILE;     // 8 warps x 32 rows x 128 B
  static constexpr int EPI_BYTES = 8 * 32 * 128;
  static constexpr int OFF_BAR = OFF_EPI + EPI_BYTES;
  static constexpr int BAR_BYTES = 256;
  static constexpr int USED = OFF_BAR + BAR_BYTES;
  // >= 116 KB keeps one CTA per SM (each CTA allocates all 512 TMEM columns).
  static constexpr int SMEM = (USED + 1024 > 120 * 1024 ? USED + 1024 : 120 * 1024);
  // TMEM columns of S_k, P_k and O_k
  __host__ __device__ static constexpr int S_COL(int k) { return !FS ? 128 * k : (D == 96 ? 160 * k : 192 * k); }
  __host__ __device__ static constexpr int P_COL(int k) { return !FS ? 128 * k : S_COL(k) + BN; }
  __host__ __device__ static constexpr int O_COL(int k) { return !FS ? 256 + 128 * k : (D == 96 ? 320 + 96 * k : 384 + 64 * k); }
  static_assert(KCHUNK % 1024 == 0, "128B-swizzled tiles start on 1024-byte boundaries");
};
template <int D>
constexpr bool tmem_plan_ok() {
  using C = Cfg<D>;
  return C::O_COL(1) + D <= 512 && C::O_COL(0) + D <= C::O_COL(1) &&
         (C::FS ? (C::S_COL(0) + C::BN <= C::P_COL(0) && C::P_COL(0) + C::BN / 2 <= C::S_COL(1) &&
                   C::S_COL(1) + C::BN <= C::P_COL(1) && C::P_COL(1) + C::BN / 2 <= C::O_COL(0))
                : (C::S_COL(1) + C::BN <= C::O_COL(0))) &&
         C::S_COL(1) % 32 == 0 && C::P_COL(0) % 32 == 0 && C::P_COL(1) % 32 == 0 &&
         C::O_COL(0) % 32 == 0 && C::O_COL(1) % 32 == 0;
}
static_assert(tmem_plan_ok<64>() && tmem_plan_ok<96>() && tmem_plan_ok<128>(), "TMEM plan");

struct Params {
  DevGeom g;
  const int *fresh_list;
  const int *counts;
  float scale_log2;       // logit scale * log2(e)
  void *out_O;             // float32, or bf16 when the state format is bf16
  float *out_lse;
  int out_by_slot;
  unsigned char *out_valid;
  float *drift_rows;       // [P][B*H][Lmax] local-state drift, or null
  int *dev_status;
  long long wait_limit_ns;
  int *sched;              // [2] work counter (next item, CTAs done) or null: fixed stride
};

// A work item: up to 256 query rows of partition i for one (b, h).  The item
// visits every fresh unit (i, c) of row i in fresh-list order, so its Q tiles
// are loaded once and reused for all of them.
struct Item {
  bool live;
  int i, bh, b, h;
  int q0;          // first query token of the item
  int rloc0;       // row of q0 inside partition i
  int rows0, rows1;
  int f0, f1;      // fresh-list range of row i
};

struct UnitRange {
  int f, c;
  int T;                     // key tiles over all runs of adjacent partitions
  int k0, Lk;                // key range of the first run (the only one unless MR)
};

// Partitions whose keys unit (i, c) attends: its active pairs; for a masked
// unit in the fresh list (never from the planner) the group's partitions
// unmasked, so that every role still sees at least one tile.
__device__ __forceinline__ unsigned long long unit_key_bits(const DevGeom &g, int i, int c) {
  const unsigned long long b = unit_pairs(g, i, c);
  return b ? b : bit_range(g.group_off[c], g.group_off[c + 1]);
}

// The first run of adjacent partitions in `bits` (nonzero): its key range
// [k0, k0 + Lk) and the partition after it.
__device__ __forceinline__ void first_run(const DevGeom &g, unsigned long long bits, int &k0,
                                          int &Lk, int &jend) {
  const int j0 = __ffsll((long long)bits) - 1;
  const unsigned long long sh = bits >> j0;
  const int len = (~sh == 0ull) ? 64 - j0 : __ffsll((long long)~sh) - 1;
  jend = j0 + len;
  k0 = g.part_off[j0];
  Lk = g.part_off[jend] - k0;
}

// Key tiles of unit (i, c) in order: tile t of the current run.  Only the
// end of the current run is held; the next run is found again from the
// geometry (kernel parameters), which keeps the softmax warps' registers.
template <int BN>
struct KeyCursor {
  int k0, Lk, t, jend;
  __device__ __forceinline__ void start(const DevGeom &g, int i, int c) {
    first_run(g, unit_key_bits(g, i, c), k0, Lk, jend);
    t = 0;
  }
  __device__ __forceinline__ int row() const { return k0 + t * BN; }
  __device__ __forceinline__ int valid() const { return Lk - t * BN; }
  __device__ __forceinline__ void next(const DevGeom &g, int i, int c) {
    ++t;
    if (t * BN >= Lk) {
      const unsigned long long rest = unit_key_bits(g, i, c) & ~bit_range(0, jend);
      if (rest) {
        first_run(g, rest, k0, Lk, jend);
        t = 0;
      }
    }
  }
};

__device__ __forceinline__ Item decode_item(const Params &p, const int *row_fresh, int it, int nqt2) {
  Item w;
  const DevGeom &g = p.g;
  const int n_main = g.P * g.BH * (nqt2 - 1);
  int qt2, rest;
  if (it < n_main) {
    qt2 = it % (nqt2 - 1);
    rest = it / (nqt2 - 1);
  } else {
    qt2 = nqt2 - 1;   // the last block of rows of every partition, after all the others
    rest = it - n_main;
  }
  w.i = rest % g.P;   // b*h-major: the CTAs running together share one (b, h)'s K/V
  w.bh = rest / g.P;
  w.b = w.bh / g.H;
  w.h = w.bh - w.b * g.H;
  w.rloc0 = qt2 * 2 * BM;
  w.q0 = g.part_off[w.i] + w.rloc0;
  const int rem = g.part_off[w.i + 1] - w.q0;
  w.rows0 = rem < BM ? rem : BM;
  const int r1 = rem - BM;
  w.rows1 = r1 <= 0 ? 0 : (r1 < BM ? r1 : BM);
  w.f0 = row_fresh[w.i];
  w.f1 = row_fresh[w.i + 1];
  w.live = (w.rows0 > 0) && (w.f1 > w.f0);
  return w;
}

// MR, the general variant: units may hold several runs of adjacent
// partitions (a frame mask that leaves a gap inside a KV group), and the
// frame mask may forbid single token pairs inside an active pair (partitions
// that straddle frames); otherwise every unit is one key range attended by
// all its rows.
template <bool MR, int BN>
__device__ __forceinline__ UnitRange unit_at(const Params &p, int i, int f) {
  UnitRange u;
  const int unit = __ldg(p.fresh_list + f);
  u.f = f;
  u.c = unit % p.g.G;
  unsigned long long rest = unit_key_bits(p.g, i, u.c);
  if constexpr (!MR) {
    // one run: from the first to the last active partition
    u.k0 = p.g.part_off[__ffsll((long long)rest) - 1];
    u.Lk = p.g.part_off[64 - __clzll((long long)rest)] - u.k0;
    u.T = (u.Lk + BN - 1) / BN;
  } else {
    int jend = 0;
    first_run(p.g, rest, u.k0, u.Lk, jend);
    u.T = (u.Lk + BN - 1) / BN;
    rest &= ~bit_range(0, jend);
    while (rest) {
      int k0, Lk;
      first_run(p.g, rest, k0, Lk, jend);
      rest &= ~bit_range(0, jend);
      u.T += (Lk + BN - 1) / BN;
    }
  }
  return u;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA/ALU pipes, to take part of the exponentials off the
// special-function unit.  Range reduction in the style of Cody and Waite, to
// the nearest integer with the 1.5 * 2^23 rounding constant (x = n + f,
// f in [-1/2, 1/2]); 2^f by a cubic whose constant term is fixed at 1 (so
// integer inputs are exact) and whose other coefficients are the minimax
// (Chebyshev) fit of the relative error on [-1/2, 1/2], computed as a linear
// program over a dense grid -- the optimum the Remez exchange algorithm
// converges to; max relative error 1.013e-4, far below the bf16 rounding P
// gets next; 2^n by adding n to the exponent field.  Inputs below -126
// give ~0.
constexpr float kExpC1 = 0.6932829022f;
constexpr float kExpC2 = 0.2422109693f;
constexpr float kExpC3 = 0.0550090596f;
__device__ __forceinline__ float exp2_poly(float x) {
  x = fmaxf(x, -126.0f);
  const float kRound = 12582912.0f;  // 1.5 * 2^23
  const float t = x + kRound;        // t = 1.5 * 2^23 + round(x), exactly
  const float n = t - kRound;
  const float f = x - n;
  const float p = fmaf(fmaf(fmaf(kExpC3, f, kExpC2), f, kExpC1), f, 1.0f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// Of every 16 probabilities of a row, this many use exp2_poly, the rest the
// ex2 instruction.  Measured on B200: moving exponentials off the special
// function unit does not pay at the current pipeline depth, so 0 by default.
#ifndef DITANGO_EMU_D64
#define DITANGO_EMU_D64 0
#endif
#ifndef DITANGO_EMU_D96
#define DITANGO_EMU_D96 0
#endif
#ifndef DITANGO_EMU_D128
#define DITANGO_EMU_D128 0
#endif
template <int D>
__host__ __device__ constexpr int emu_per16() {
  return D == 64 ? DITANGO_EMU_D64 : (D == 96 ? DITANGO_EMU_D96 : DITANGO_EMU_D128);
}

// Packed pairs of fp32 (sm_100 f32x2 arithmetic: one instruction, two lanes).
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unf2(uint64_t v, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Checked builds record a bad device-resident input here (and in the
// caller's dev_status); read and cleared by ditango_check_status.
__device__ int g_attn_check_status;

__device__ __forceinline__ void record_check_failure(int *dev_status) {
  atomicExch(&g_attn_check_status, (int)DITANGO_ERR_BOUNDS);
  if (dev_status) atomicExch(dev_status, (int)DITANGO_ERR_BOUNDS);
}

// Frame of a token (tokens past the end count in the last frame).
__device__ __forceinline__ int frame_of(const DevGeom &g, int tok) {
  int lo = 0, hi = g.F - 1;
  while (lo < hi) {            // the last frame whose start is <= tok
    const int mid = (lo + hi + 1) >> 1;
    if (g.frame_off[mid] <= tok) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Token-level frame mask (Efficient-vDiT's frame tiles, with partitions that
// straddle frames): in the key tile starting at token k0 (valid keys), the
// logits of keys whose frame this row may not attend become -inf.
template <int BN>
__device__ __forceinline__ void mask_frames(const DevGeom &g, int k0, int valid,
                                            unsigned long long allow, uint32_t (&sv)[BN]) {
  for (int f = frame_of(g, k0); f < g.F && g.frame_off[f] < k0 + valid; ++f) {
    if ((allow >> f) & 1ull) continue;
    const int c0 = (g.frame_off[f] > k0 ? g.frame_off[f] : k0) - k0;
    const int e = g.frame_off[f + 1] < k0 + valid ? g.frame_off[f + 1] : k0 + valid;
    const int c1 = e - k0;
#pragma unroll
    for (int c = 0; c < BN; ++c)
      if (c >= c0 && c < c1) sv[c] = __float_as_uint(-INFINITY);
  }
}

// SB: states stored with bf16 O (compressed cache); MR: see unit_at.
template <int D, bool SB, bool MR>
__global__ void __launch_bounds__(kThreads, 1)
attn_partial_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ Params p) {
  using C = Cfg<D>;
  constexpr int BN = C::BN;
  constexpr bool FS = C::FS;
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
  // work items pass from the producer to the other roles through a 2-slot ring
  auto item_full = [&](int s) { return bar + 152 + 8 * s; };
  auto item_empty = [&](int s) { return bar + 168 + 8 * s; };
  volatile int *item_slot = reinterpret_cast<volatile int *>(smem + C::OFF_BAR + 208);
  // FS: S_k read into registers (the next Q K^T may overwrite it) / P_k V done
  auto s_free = [&](int k) { return bar + 216 + 8 * k; };
  auto p_free = [&](int k) { return bar + 232 + 8 * k; };

  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_BAR + 192);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_BAR + 200);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  WaitCtl ctl{abort_flag, p.dev_status, p.wait_limit_ns};

  const int nqt2 = (p.g.Lmax + 2 * BM - 1) / (2 * BM);
  const int n_items = p.g.P * p.g.BH * nqt2;
  // fresh-list range of every query partition (the list is row-major)
  __shared__ int row_fresh[kMaxP + 1];
  if (threadIdx.x <= p.g.P) row_fresh[threadIdx.x] = 0;
#ifdef DITANGO_CHECK
  // Checked build: the device-resident inputs are validated before any use.
  // A count beyond the active units, a unit index out of range or inactive,
  // or a list that is not strictly row-major: nothing is computed and
  // DITANGO_ERR_BOUNDS is recorded.
  __shared__ int s_bad;
  if (threadIdx.x == 0) s_bad = 0;
  __syncthreads();
  {
    const int n_fresh = __ldg(p.counts);
    if (n_fresh < 0 || n_fresh > p.g.n_active) {
      s_bad = 1;   // every thread writes the same value
    } else {
      for (int f = threadIdx.x; f < n_fresh; f += blockDim.x) {
        const int u = __ldg(p.fresh_list + f);
        bool ok = u >= 0 && u < p.g.P * p.g.G;
        if (ok) ok = ((p.g.row_mask[u / p.g.G] >> (u % p.g.G)) & 1ull) != 0ull;
        if (ok && f > 0) ok = __ldg(p.fresh_list + f - 1) < u;
        if (!ok) s_bad = 1;
      }
    }
  }
  __syncthreads();
  const bool bad_input = s_bad != 0;
  if (bad_input && threadIdx.x == 0) record_check_failure(p.dev_status);
#else
  constexpr bool bad_input = false;
#endif
  __syncthreads();
  {
    const int n_fresh = bad_input ? 0 : __ldg(p.counts);
    const int n_units = p.g.P * p.g.G;
    for (int f = threadIdx.x; f < n_fresh; f += blockDim.x) {
      const int u = __ldg(p.fresh_list + f);
      if (u >= 0 && u < n_units) atomicAdd(&row_fresh[u / p.g.G + 1], 1);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0)
    for (int i = 1; i <= p.g.P; ++i) row_fresh[i] += row_fresh[i - 1];

  if (threadIdx.x == 0) {
    // FS: each of the two MMA warps releases every Q, K and V stage once
    mbar_init(q_full, 1);
    mbar_init(q_empty, FS ? 2 : 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), FS ? 2 : 1);
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), FS ? 2 : 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(s_full(k), 1);
      mbar_init(p_full(k), 4);    // one arrival per softmax warp
      mbar_init(o_full(k), 1);
      mbar_init(o_empty(k), 4);
      mbar_init(s_free(k), 4);    // one arrival per softmax warp
      mbar_init(p_free(k), 1);
    }
    mbar_init(drain, FS ? 2 : 1);   // one commit per MMA warp
    for (int s = 0; s < 2; ++s) {
      mbar_init(item_full(s), 1);
      mbar_init(item_empty(s), FS ? 10 : 9);   // the MMA warp(s) and the eight softmax warps
    }

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

  if (warp >= 8) {
   asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(control_regs<D>()));
   if (warp == 8) {
    // ------------------------------------------------------------ producer
    // Warp-uniform loop; one elected lane arms the barriers and issues TMA.
    {
      const bool leader = elect_one();
      uint32_t kc = 0, vc = 0, uc = 0;
      // last armed phase per full barrier (drained before the warp exits)
      // bit 2s: stage s armed at least once; bit 2s+1: parity of its last arming
      int q_armed = -1;
      uint32_t k_armed = 0, v_armed = 0;
      bool ok = true;
      uint32_t ic = 0;                 // items published to the other roles
      int next_static = blockIdx.x;
      while (ok) {
        // the next live item: from the work counter (each CTA takes the next
        // one when it is ready for it), or in a fixed stride without one
        int it;
        Item w;
        for (;;) {
          if (p.sched != nullptr) {
            int v = 0;
            if (lane == 0) v = atomicAdd(p.sched, 1);
            it = __shfl_sync(0xffffffffu, v, 0);
          } else {
            it = next_static;
            next_static += gridDim.x;
          }
          if (it >= n_items) {
            it = -1;
            break;
          }
          w = decode_item(p, row_fresh, it, nqt2);
          if (w.live) break;
        }
        // publish it (or the end, -1) to the MMA and softmax warps
        const int is = ic & 1;
        if (!(ok = wait_warp(item_empty(is), ((ic >> 1) & 1) ^ 1, ctl))) break;
        if (leader) {
          item_slot[is] = it;
          mbar_arrive(item_full(is));
        }
        ++ic;
        if (it < 0) break;
        if (!(ok = wait_warp(q_empty, (uc & 1) ^ 1, ctl))) break;
        const uint32_t qbytes = C::QTILE * (w.rows1 > 0 ? 2 : 1);
        if (leader) mbar_arrive_expect_tx(q_full, qbytes);
        q_armed = uc & 1;
        if (leader) {
          for (int c = 0; c < C::NCH; ++c)
            tma_load_4d(sQ + c * C::QCHUNK, &tmQ, q_full, c * 64, w.q0, w.h, w.b);
          if (w.rows1 > 0)
            for (int c = 0; c < C::NCH; ++c)
              tma_load_4d(sQ + C::QTILE + c * C::QCHUNK, &tmQ, q_full, c * 64, w.q0 + BM, w.h, w.b);
        }
        for (int f = w.f0; f < w.f1 && ok; ++f) {
          const UnitRange pr = unit_at<MR, BN>(p, w.i, f);
          KeyCursor<BN> cur;
          if constexpr (MR) cur.start(p.g, w.i, pr.c);
          for (int t = 0; t < pr.T && ok; ++t) {
            if constexpr (MR) {
              if (t > 0) cur.next(p.g, w.i, pr.c);
            }
            const int row = MR ? cur.row() : pr.k0 + t * BN;
            int s = kc % kStages;
            if (!(ok = wait_warp(k_empty(s), ((kc / kStages) & 1) ^ 1, ctl))) break;
            if (leader) mbar_arrive_expect_tx(k_full(s), C::KTILE);
            k_armed = (k_armed & ~(3u << (2 * s))) | ((1u | (((kc / kStages) & 1u) << 1)) << (2 * s));
            if (leader)
              for (int c = 0; c < C::NCH; ++c)
                tma_load_4d(sK + s * C::KTILE + c * C::KCHUNK, &tmK, k_full(s), c * 64, row, w.h, w.b);
            ++kc;
            s = vc % kStages;
            if (!(ok = wait_warp(v_empty(s), ((vc / kStages) & 1) ^ 1, ctl))) break;
            if (leader) mbar_arrive_expect_tx(v_full(s), C::KTILE);
            v_armed = (v_armed & ~(3u << (2 * s))) | ((1u | (((vc / kStages) & 1u) << 1)) << (2 * s));
            if (leader)
              for (int c = 0; c < C::NCH; ++c)
                tma_load_4d(sV + s * C::KTILE + c * C::KCHUNK, &tmV, v_full(s), c * 64, row, w.h, w.b);
            ++vc;
          }
        }
        ++uc;
      }
      // Every load issued lands before the warp exits, on both paths.  When
      // another role gave up, this warp can still finish its loop with
      // ok == true (each wait of its last tiles completed at once and never
      // looked at the abort flag) while nothing consumes its last loads.  On
      // the normal path these waits pass at once or as the loads land: only
      // this warp arms the full barriers, so none runs past its last arming.
      {
        WaitCtl drain_ctl{nullptr, nullptr, 100000000LL};
        volatile int never = 0;
        drain_ctl.abort_flag = &never;
        if (q_armed >= 0) wait_bounded(q_full, (uint32_t)q_armed, drain_ctl);
#pragma unroll
        for (int s = 0; s < kStages; ++s) {
          if ((k_armed >> (2 * s)) & 1u) wait_bounded(k_full(s), (k_armed >> (2 * s + 1)) & 1u, drain_ctl);
          if ((v_armed >> (2 * s)) & 1u) wait_bounded(v_full(s), (v_armed >> (2 * s + 1)) & 1u, drain_ctl);
        }
      }
    }
  } else if (warp == 9 || (FS && warp == 10)) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop (warp-uniform control flow keeps the
    // descriptors in uniform registers); one elected lane issues every MMA
    // and commit, so the commits track exactly the MMAs that lane issued.
    {
      const bool leader = elect_one();
      constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, BN, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, D, 0, 1);
      uint32_t kc = 0, vc = 0, uc = 0;
      uint32_t pc[2] = {0, 0}, oc[2] = {0, 0};
      bool ok = true;
      // Descriptors are built once; a k-step only adds a compile-time offset
      // to the start-address field (all addresses stay below 256 KB, so the
      // 14-bit field never carries).
      const uint64_t dQ0 = smem_desc_sw128(sQ, 16, 1024);
      const uint64_t dQ1 = smem_desc_sw128(sQ + C::QTILE, 16, 1024);
      const uint64_t dK0 = smem_desc_sw128(sK, 16, 1024);
      const uint64_t dK1 = smem_desc_sw128(sK + C::KTILE, 16, 1024);
      // V: MN-major; the leading offset steps from one 64-column chunk of d
      // to the next (BN rows of 128 bytes each)
      const uint64_t dV0 = smem_desc_sw128(sV, C::KCHUNK, 1024);
      const uint64_t dV1 = smem_desc_sw128(sV + C::KTILE, C::KCHUNK, 1024);
      static_assert(kStages == 2, "descriptor selection assumes two stages");
      auto qk = [&](int k, int ks) {
        // S_k = Q_k K^T : K-major A and B, 16 columns of d per instruction
        uint64_t a0 = k ? dQ1 : dQ0;
        uint64_t b0 = ks ? dK1 : dK0;
        // opaque to the compiler: the per-step descriptors are formed at each
        // use instead of all being hoisted into registers of this warp
        asm volatile("mov.b64 %0, %0;" : "+l"(a0));
        asm volatile("mov.b64 %0, %0;" : "+l"(b0));
        const uint32_t d_tmem = tmem + C::S_COL(k);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t offa = (uint64_t)(((kk >> 2) * C::QCHUNK + (kk & 3) * 32) >> 4);
          const uint64_t offb = (uint64_t)(((kk >> 2) * C::KCHUNK + (kk & 3) * 32) >> 4);
          if (leader) mma_ss(d_tmem, a0 + offa, b0 + offb, idesc_qk, kk > 0);
        }
      };
      auto pv = [&](int k, int vs, bool acc) {
        // O_k (+)= P_k V : P from TMEM (K-major), V MN-major (d contiguous)
        uint64_t b0 = vs ? dV1 : dV0;
        asm volatile("mov.b64 %0, %0;" : "+l"(b0));
        const uint32_t d_tmem = tmem + C::O_COL(k);
        const uint32_t a_tmem = tmem + C::P_COL(k);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          if (leader) mma_ts(d_tmem, a_tmem + kk * 8, b0 + (uint64_t)((kk * 2048) >> 4), idesc_pv, (acc || kk > 0));
      };
      uint32_t ic = 0;
      if constexpr (!FS) {
        while (ok) {
          const int is = ic & 1;
          if (!(ok = wait_warp(item_full(is), (ic >> 1) & 1, ctl))) break;
          const int it = item_slot[is];
          __syncwarp();
          if (lane == 0) mbar_arrive(item_empty(is));
          ++ic;
          if (it < 0) break;
          const Item w = decode_item(p, row_fresh, it, nqt2);
          const bool has1 = w.rows1 > 0;
          if (!(ok = wait_warp(q_full, uc & 1, ctl))) break;
          for (int f = w.f0; f < w.f1 && ok; ++f) {
            const UnitRange pr = unit_at<MR, BN>(p, w.i, f);
            const bool last_pair = (f + 1 == w.f1);
            int ks = kc % kStages;
            if (!(ok = wait_warp(k_full(ks), (kc / kStages) & 1, ctl))) break;
            tc_fence_after();
            qk(0, ks);
            commit_by(leader, s_full(0));
            if (has1) {
              qk(1, ks);
              commit_by(leader, s_full(1));
            }
            commit_by(leader, k_empty(ks));
            ++kc;
            if (pr.T == 1 && last_pair) commit_by(leader, q_empty);
            for (int t = 0; t < pr.T && ok; ++t) {
              const int vs = vc % kStages;
              if (!(ok = wait_warp(v_full(vs), (vc / kStages) & 1, ctl))) break;
              const bool more = (t + 1 < pr.T);
              // ---- Q tile 0
              if (!(ok = wait_warp(p_full(0), pc[0] & 1, ctl))) break;
              ++pc[0];
              if (t == 0) {
                if (!(ok = wait_warp(o_empty(0), (oc[0] & 1) ^ 1, ctl))) break;
                ++oc[0];
              }
              tc_fence_after();
              pv(0, vs, t > 0);
              if (!more) commit_by(leader, o_full(0));
              const int ks2 = kc % kStages;
              if (more) {
                if (!(ok = wait_warp(k_full(ks2), (kc / kStages) & 1, ctl))) break;
                tc_fence_after();
                qk(0, ks2);
                commit_by(leader, s_full(0));
              }
              // ---- Q tile 1
              if (has1) {
                if (!(ok = wait_warp(p_full(1), pc[1] & 1, ctl))) break;
                ++pc[1];
                if (t == 0) {
                  if (!(ok = wait_warp(o_empty(1), (oc[1] & 1) ^ 1, ctl))) break;
                  ++oc[1];
                }
                tc_fence_after();
                pv(1, vs, t > 0);
                if (!more) commit_by(leader, o_full(1));
                if (more) {
                  qk(1, ks2);
                  commit_by(leader, s_full(1));
                }
              }
              commit_by(leader, v_empty(vs));
              ++vc;
              if (more) {
                commit_by(leader, k_empty(ks2));
                ++kc;
                if (t + 2 == pr.T && last_pair) commit_by(leader, q_empty);
              }
            }
          }
          ++uc;
        }
      } else {
        // FS: one MMA warp per Q tile (warp 9: tile 0, warp 10: tile 1), each
        // waiting in its tile's own order, so neither tile waits for the
        // other's events.  Units and their key tiles form one stream of steps
        // per item; at step n the Q K^T of step n + 1 is issued as soon as the
        // softmax has read S of step n, and the P V of step n once P is
        // written.  Each warp releases every Q, K and V stage once (the
        // barriers count two); for an item without a second Q tile warp 10
        // only follows the stages and releases them.
        const int k = warp - 9;
        uint32_t sf = 0;             // s_free completions consumed
        while (ok) {
          const int is = ic & 1;
          if (!(ok = wait_warp(item_full(is), (ic >> 1) & 1, ctl))) break;
          const int it = item_slot[is];
          __syncwarp();
          if (lane == 0) mbar_arrive(item_empty(is));
          ++ic;
          if (it < 0) break;
          const Item w = decode_item(p, row_fresh, it, nqt2);
          const bool active = (k == 0) || (w.rows1 > 0);
          int n_steps = 0;
          for (int f = w.f0; f < w.f1; ++f) n_steps += unit_at<MR, BN>(p, w.i, f).T;
          if (!(ok = wait_warp(q_full, uc & 1, ctl))) break;
          ++uc;
          if (!active) {
            commit_by(leader, q_empty);
            for (int n = 0; n < n_steps && ok; ++n) {
              if (!(ok = wait_warp(k_full(kc % kStages), (kc / kStages) & 1, ctl))) break;
              commit_by(leader, k_empty(kc % kStages));
              ++kc;
              if (!(ok = wait_warp(v_full(vc % kStages), (vc / kStages) & 1, ctl))) break;
              commit_by(leader, v_empty(vc % kStages));
              ++vc;
            }
            continue;
          }
          // Q K^T of step 0 (S_k is free: the softmax's read of the last S
          // of the previous item was waited for)
          if (!(ok = wait_warp(k_full(kc % kStages), (kc / kStages) & 1, ctl))) break;
          tc_fence_after();
          qk(k, kc % kStages);
          commit_by(leader, s_full(k));
          commit_by(leader, k_empty(kc % kStages));
          ++kc;
          if (n_steps == 1) commit_by(leader, q_empty);
          int f = w.f0, t = 0;
          int T = unit_at<MR, BN>(p, w.i, f).T;
          for (int n = 0; n < n_steps && ok; ++n) {
            if (!(ok = wait_warp(s_free(k), sf & 1, ctl))) break;
            ++sf;
            if (n + 1 < n_steps) {
              if (!(ok = wait_warp(k_full(kc % kStages), (kc / kStages) & 1, ctl))) break;
              tc_fence_after();
              qk(k, kc % kStages);
              commit_by(leader, s_full(k));
              commit_by(leader, k_empty(kc % kStages));
              ++kc;
              if (n + 2 == n_steps) commit_by(leader, q_empty);   // the item's last Q K^T
            }
            if (!(ok = wait_warp(v_full(vc % kStages), (vc / kStages) & 1, ctl))) break;
            if (!(ok = wait_warp(p_full(k), pc[k] & 1, ctl))) break;
            ++pc[k];
            if (t == 0) {
              if (!(ok = wait_warp(o_empty(k), (oc[k] & 1) ^ 1, ctl))) break;
              ++oc[k];
            }
            tc_fence_after();
            pv(k, vc % kStages, t > 0);
            commit_by(leader, p_free(k));
            commit_by(leader, v_empty(vc % kStages));
            ++vc;
            if (t + 1 == T) {
              commit_by(leader, o_full(k));
              t = 0;
              if (++f < w.f1) T = unit_at<MR, BN>(p, w.i, f).T;
            } else {
              ++t;
            }
          }
        }
      }
      // drain: every MMA issued so far must finish before TMEM is released
      commit_by(leader, drain);
      WaitCtl drain_ctl{nullptr, nullptr, 100000000LL};
      volatile int never = 0;
      drain_ctl.abort_flag = &never;
      wait_bounded(drain, 0, drain_ctl);
    }
   }
    // end of the control warpgroup: warp 9 frees TMEM once every warp is done
    if (warp == 9) {
      named_bar_sync(1, kThreads);
      tc_fence_after();
      tmem_dealloc(tmem, 512);
      if (p.sched != nullptr && lane == 0) {
        // the last CTA to finish (every producer has taken its last item by
        // then) leaves the counter at zero for the next launch
        __threadfence();
        if (atomicAdd(p.sched + 1, 1) == (int)gridDim.x - 1) {
          p.sched[0] = 0;
          p.sched[1] = 0;
          __threadfence();
        }
      }
    } else {
      tc_fence_before();
      named_bar_arrive(1, kThreads);
    }
    return;
  } else {
    // ------------------------------------------------------------ softmax
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(softmax_regs<D>()));
    const int k = warp >> 2;                 // Q tile of this warpgroup
    const int r = threadIdx.x & 127;         // row within the tile = TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + C::S_COL(k);
    const uint32_t tP = tmem + lane_base + C::P_COL(k);   // = tS unless FS
    const uint32_t tO = tmem + lane_base + C::O_COL(k);
    const float sl2 = p.scale_log2;
    uint32_t sc = 0, ofc = 0;
    uint32_t pst = 0;   // FS: P tiles stored so far (each one's P V completes p_free)
    bool ok = true;
    uint32_t ic = 0;
    while (ok) {
      const int is = ic & 1;
      if (!(ok = wait_warp(item_full(is), (ic >> 1) & 1, ctl))) break;
      const int it = item_slot[is];
      __syncwarp();
      if (lane == 0) mbar_arrive(item_empty(is));
      ++ic;
      if (it < 0) break;
      const Item w = decode_item(p, row_fresh, it, nqt2);
      const int rows_k = (k == 0) ? w.rows0 : w.rows1;
      if (rows_k <= 0) continue;
      // key frames this row may attend (partitions that straddle frames)
      unsigned long long allow = ~0ull;
      if constexpr (MR) {
        if (p.g.token_mask) allow = p.g.frame_allow[frame_of(p.g, w.q0 + k * BM + r)];
      }
     for (int f = w.f0; f < w.f1 && ok; ++f) {
      const UnitRange pr = unit_at<MR, BN>(p, w.i, f);
      KeyCursor<BN> cur;
      if constexpr (MR) cur.start(p.g, w.i, pr.c);
      float m_used = -INFINITY;   // running maximum used for exponentiation (log2 units)
      float l = 0.f;
      for (int t = 0; t < pr.T; ++t) {
        if constexpr (MR) {
          if (t > 0) cur.next(p.g, w.i, pr.c);
        }
        if (!(ok = wait_bounded(s_full(k), sc & 1, ctl))) break;
        ++sc;
        tc_fence_after();
        // the whole S row of this thread: eight loads in flight, one wait
        uint32_t sv[BN];
#pragma unroll
        for (int c = 0; c < BN / 16; ++c) tmem_ld16p(tS + c * 16, &sv[c * 16]);
        tc_wait_ld();
        bool pv_done = true;   // the previous P V of this tile has completed
        if constexpr (FS) {
          // S is in registers: the next Q K^T may overwrite it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(s_free(k));
          pv_done = (pst == 0);
        }
        const int valid = MR ? cur.valid() : pr.Lk - t * BN;
        if (valid < BN) {
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (c >= valid) sv[c] = __float_as_uint(-INFINITY);
        }
        if constexpr (MR) {
          if (p.g.token_mask) mask_frames(p.g, cur.row(), valid, allow, sv);
        }
        // row maximum: 8 independent chains of 3-input max, then a tree
        float m8[8];
#pragma unroll
        for (int q = 0; q < 8; ++q)
          m8[q] = max3(__uint_as_float(sv[q]), __uint_as_float(sv[q + 8]), __uint_as_float(sv[q + 16]));
#pragma unroll
        for (int c = 24; c + 16 <= BN; c += 16)
#pragma unroll
          for (int q = 0; q < 8; ++q)
            m8[q] = max3(m8[q], __uint_as_float(sv[c + q]), __uint_as_float(sv[c + q + 8]));
        static_assert(BN % 16 == 0 && BN >= 32, "key tile: a multiple of 16 columns");
#pragma unroll
        for (int q = 0; q < 8; ++q)   // the last 8 columns (BN - 24 is 8 more than a multiple of 16)
          m8[q] = fmaxf(m8[q], __uint_as_float(sv[BN - 8 + q]));
        const float mx = max3(max3(m8[0], m8[1], m8[2]), max3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
        const float mx2 = mx * sl2;
        if (t == 0) {
          m_used = mx2;
        } else {
          const bool need = mx2 > m_used + kRescaleLog2;
          if (__any_sync(0xffffffffu, need)) {
            // O of this row must hold every P V of earlier tiles: without FS
            // the commit that released S(t) covers all earlier MMAs; with FS
            // the last one is waited for here.
            if constexpr (FS) {
              if (!pv_done) {
                if (!(ok = wait_bounded(p_free(k), (pst - 1) & 1, ctl))) break;
                tc_fence_after();
                pv_done = true;
              }
            }
            const float m_new = need ? mx2 : m_used;
            const float alpha = need ? ex2(m_used - m_new) : 1.f;   // 1, not NaN, for a row still at -inf
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
        // P = 2^(s*scale*log2e - m), rounded to bf16 into P_k (the first BN/2
        // columns of S_k unless FS)
        // (general variant) a row with no admissible key so far exponentiates against 0
        const float neg = (MR && !(m_used > -INFINITY)) ? 0.f : -m_used;
        const uint64_t sl2x2 = f2(sl2, sl2), negx2 = f2(neg, neg);
        uint64_t lsum0 = 0, lsum1 = 0;   // packed partial row sums (+0.0f bits)
        if constexpr (FS) {
          // The whole P row is formed in registers first.  P_k is then
          // overwritten, once the P V that read it is done: by the end of the
          // exponentials it normally is, so this wait no longer sits between
          // the row maximum and the exponentials.
          uint32_t pk[BN / 2];
#pragma unroll
          for (int e = 0; e < BN / 2; ++e) {
            const int c = 2 * e;
            float xa, xb;
            unf2(fma2(f2(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), sl2x2, negx2), xa, xb);
            const float a = (2 * (e % 8) < emu_per16<D>()) ? exp2_poly(xa) : ex2(xa);
            const float b = (2 * (e % 8) + 1 < emu_per16<D>()) ? exp2_poly(xb) : ex2(xb);
            if (e & 1) lsum1 = add2(lsum1, f2(a, b)); else lsum0 = add2(lsum0, f2(a, b));
            pk[e] = pack_bf16(a, b);
          }
          if (!pv_done) {
            if (!(ok = wait_bounded(p_free(k), (pst - 1) & 1, ctl))) break;
            tc_fence_after();
          }
#pragma unroll
          for (int g8 = 0; g8 < BN / 16; ++g8)
            tmem_st8(tP + g8 * 8, pk[g8 * 8 + 0], pk[g8 * 8 + 1], pk[g8 * 8 + 2], pk[g8 * 8 + 3],
                     pk[g8 * 8 + 4], pk[g8 * 8 + 5], pk[g8 * 8 + 6], pk[g8 * 8 + 7]);
        } else {
          // P overwrites S_k: stored 16 probabilities at a time, under the
          // exponentials
#pragma unroll
          for (int g8 = 0; g8 < BN / 16; ++g8) {
            // 16 probabilities -> 8 packed bf16 pairs -> TMEM columns [8*g8, 8*g8+8)
            uint32_t pk[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int c = g8 * 16 + 2 * e;
              float xa, xb;
              unf2(fma2(f2(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), sl2x2, negx2), xa, xb);
              const float a = (2 * e < emu_per16<D>()) ? exp2_poly(xa) : ex2(xa);
              const float b = (2 * e + 1 < emu_per16<D>()) ? exp2_poly(xb) : ex2(xb);
              if (e & 1) lsum1 = add2(lsum1, f2(a, b)); else lsum0 = add2(lsum0, f2(a, b));
              pk[e] = pack_bf16(a, b);
            }
            tmem_st8(tP + g8 * 8, pk[0], pk[1], pk[2], pk[3], pk[4], pk[5], pk[6], pk[7]);
          }
        }
        {
          float s0, s1, s2, s3;
          unf2(lsum0, s0, s1);
          unf2(lsum1, s2, s3);
          l += (s0 + s1) + (s2 + s3);
        }
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full(k));   // one arrival per warp
        ++pst;
      }
      if (!ok) break;
      // ---- epilogue: O of this row into registers, release the TMEM
      // accumulator to the next pair at once, then normalise and store.
      if (!(ok = wait_bounded(o_full(k), ofc & 1, ctl))) break;
      ++ofc;
      tc_fence_after();
      // O is read in halves of up to 64 columns (fewer live registers); the
      // accumulator is released to the next pair once the last half is in
      // registers.  The 32 rows of this warp are one contiguous block of the
      // state buffer: each half is transposed through this warp's 4 KB of
      // shared memory, 32 columns at a time, so that every store writes whole
      // 128-byte row segments (XOR swizzle: both phases free of bank
      // conflicts).
      constexpr int HALF = (D > 64) ? 64 : D;
      const int idx = p.out_by_slot ? slot_of(p.g, w.i, pr.c) : pr.f;
      const int rloc = w.rloc0 + k * BM + r;
      const size_t row_off = ((size_t)idx * p.g.BH + w.bh) * (size_t)p.g.Lmax + rloc;
      const float inv_l = (l > 0.f) ? 1.f / l : 0.f;   // a row with no admissible key: O = 0
      float4 *epi = reinterpret_cast<float4 *>(smem + C::OFF_EPI + (warp & 7) * 4096);
      // a masked unit in the fresh list has no slot: nothing is stored by slot
      const bool store = !p.out_by_slot || unit_pairs(p.g, w.i, pr.c) != 0ull;
      const int row_valid = store ? rows_k - (r & ~31) : 0;   // rows of this warp to store
#pragma unroll
      for (int h0 = 0; h0 < D; h0 += HALF) {
        constexpr int W = HALF;
        const int width = (D - h0 < W) ? (D - h0) : W;  // 64, or 32 for the tail of d = 96
        uint32_t ov[W];
#pragma unroll
        for (int c = 0; c < W / 16; ++c)
          if (c * 16 < width) tmem_ld16p(tO + h0 + c * 16, &ov[c * 16]);
        tc_wait_ld();
        if (h0 + HALF >= D) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(o_empty(k));
        }
#pragma unroll
        for (int c = 0; c < W / 32; ++c) {
          if (c * 32 >= width) break;
          if constexpr (!SB) {
            float *blk = static_cast<float *>(p.out_O) + (row_off - lane) * D;  // row 0 of the warp's block
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              float4 o;
              o.x = __uint_as_float(ov[c * 32 + 4 * q + 0]) * inv_l;
              o.y = __uint_as_float(ov[c * 32 + 4 * q + 1]) * inv_l;
              o.z = __uint_as_float(ov[c * 32 + 4 * q + 2]) * inv_l;
              o.w = __uint_as_float(ov[c * 32 + 4 * q + 3]) * inv_l;
              epi[lane * 8 + (q ^ (lane & 7))] = o;
            }
            __syncwarp();
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const int row = (lane >> 3) + 4 * q;
              const int seg = lane & 7;
              if (row < row_valid)
                reinterpret_cast<float4 *>(blk + (size_t)row * D + h0 + c * 32)[seg] =
                    epi[row * 8 + (seg ^ (row & 7))];
            }
          } else {
            // bf16 O: 32 columns = 64 bytes per row; 4 stores of 8 rows each
            uint16_t *blk = static_cast<uint16_t *>(p.out_O) + (row_off - lane) * D;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint4 u;
              u.x = pack_bf16(__uint_as_float(ov[c * 32 + 8 * q + 0]) * inv_l, __uint_as_float(ov[c * 32 + 8 * q + 1]) * inv_l);
              u.y = pack_bf16(__uint_as_float(ov[c * 32 + 8 * q + 2]) * inv_l, __uint_as_float(ov[c * 32 + 8 * q + 3]) * inv_l);
              u.z = pack_bf16(__uint_as_float(ov[c * 32 + 8 * q + 4]) * inv_l, __uint_as_float(ov[c * 32 + 8 * q + 5]) * inv_l);
              u.w = pack_bf16(__uint_as_float(ov[c * 32 + 8 * q + 6]) * inv_l, __uint_as_float(ov[c * 32 + 8 * q + 7]) * inv_l);
              reinterpret_cast<uint4 *>(epi)[lane * 4 + (q ^ ((lane >> 1) & 3))] = u;
            }
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int row = (lane >> 2) + 8 * i;
              const int seg = lane & 3;
              if (row < row_valid)
                reinterpret_cast<uint4 *>(blk + (size_t)row * D + h0 + c * 32)[seg] =
                    reinterpret_cast<const uint4 *>(epi)[row * 4 + (seg ^ ((row >> 1) & 3))];
            }
          }
          __syncwarp();
        }
      }
      if (store && r < rows_k) {
        const float lse = (l > 0.f) ? (m_used + __log2f(l)) * 0.69314718055994531f : -INFINITY;
        if (p.drift_rows && p.g.part_group[w.i] == pr.c) {
          // the local unit: its change since the slot was last written
          const float old = p.out_lse[row_off];
          p.drift_rows[((size_t)w.i * p.g.BH + w.bh) * p.g.Lmax + rloc] =
              (lse == old) ? 0.f : fabsf(lse - old);
        }
        p.out_lse[row_off] = lse;
      }
      if (store && p.out_by_slot && p.out_valid && k == 0 && r == 0) p.out_valid[idx] = 1;
     }
    }
    tc_fence_before();
    named_bar_arrive(1, kThreads);
  }
}

}  // namespace attn

// Once per device and kernel: check the register count the setmaxnreg split
// was written for, and opt in to the shared memory the kernel uses.  Done at
// the first launch only, so that later launches (and CUDA graph captures)
// make no attribute calls.
static cudaError_t prepare_attn_kernel(const void *kfn, int smem) {
  static std::mutex mu;
  static std::set<std::pair<int, const void *>> ready;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (ready.count({dev, kfn})) return cudaSuccess;
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, kfn);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != attn::kLaunchRegs) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  ready.insert({dev, kfn});
  return cudaSuccess;
}

// Host launcher (called from the C ABI after validation).
cudaError_t launch_attn_partial(const DevGeom &g, const CUtensorMap &tq, const CUtensorMap &tk,
                                const CUtensorMap &tv, const int *fresh_list, const int *counts,
                                float scale, void *out_O, float *out_lse, int out_by_slot,
                                int state_bf16, unsigned char *out_valid, float *drift_rows,
                                int *dev_status, long long wait_limit_ns, int num_sms,
                                int *work_counter, cudaStream_t stream) {
  attn::Params p;
  p.g = g;
  p.fresh_list = fresh_list;
  p.counts = counts;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.out_O = out_O;
  p.out_lse = out_lse;
  p.out_by_slot = out_by_slot;
  p.out_valid = out_valid;
  p.drift_rows = out_by_slot ? drift_rows : nullptr;
  p.dev_status = dev_status;
  p.wait_limit_ns = wait_limit_ns;
  p.sched = work_counter;
  const long long nqt2 = (g.Lmax + 255) / 256;
  const long long max_units = (long long)g.n_active * g.BH * nqt2;
  if (max_units == 0) return cudaSuccess;
  const int grid = (int)(max_units < num_sms ? max_units : num_sms);
  cudaError_t e = cudaSuccess;
  switch (g.d) {
#define DITANGO_LAUNCH(DD)                                                                       \
  case DD: {                                                                                     \
    const bool gen = g.multi_run || g.token_mask;                                                \
    auto kfn = state_bf16 ? (gen ? attn::attn_partial_kernel<DD, true, true>                     \
                                 : attn::attn_partial_kernel<DD, true, false>)                   \
                          : (gen ? attn::attn_partial_kernel<DD, false, true>                    \
                                 : attn::attn_partial_kernel<DD, false, false>);                 \
    e = prepare_attn_kernel(reinterpret_cast<const void *>(kfn), attn::Cfg<DD>::SMEM);          \
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

// Keys per K/V tile of the kernel for head dimension d (the TMA box height).
int attn_key_tile(int d) {
  return d == 64 ? attn::Cfg<64>::BN : (d == 96 ? attn::Cfg<96>::BN : attn::Cfg<128>::BN);
}

// Read (and optionally clear) this file's check word.
cudaError_t attn_check_status(int *out, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(out, attn::g_attn_check_status, sizeof(int));
  if (e != cudaSuccess || !reset) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(attn::g_attn_check_status, &zero, sizeof(int));
}

}  // namespace ditango
