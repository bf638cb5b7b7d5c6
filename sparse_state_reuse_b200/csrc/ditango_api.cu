// Host side of the C ABI declared in include/ditango.h: argument checks,
// the kernels' geometry, TMA tensor maps and launches.  No device memory is
// allocated here.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"

namespace ditango {
cudaError_t launch_attn_partial(const DevGeom &g, const CUtensorMap &tq, const CUtensorMap &tk,
                                const CUtensorMap &tv, const int *fresh_list, const int *counts,
                                float scale, void *out_O, float *out_lse, int out_by_slot,
                                int state_bf16, unsigned char *out_valid, float *drift_rows,
                                int *dev_status, long long wait_limit_ns, int num_sms,
                                int *work_counter, cudaStream_t stream);
int attn_key_tile(int d);
size_t plan_workspace_bytes(const DevGeom &g);
cudaError_t launch_plan(const DevGeom &g, const float *cache_lse, const unsigned char *cache_valid,
                        int band_k, int target, int anchor, signed char *plan_out, int *fresh_list,
                        int *counts, float *score_out, void *workspace, cudaStream_t stream,
                        const float *drift_rows, float *w_hold, float *age, float *delta,
                        unsigned char *local_ok, int refresh_w, int mass_given);
cudaError_t launch_merge(const DevGeom &g, const signed char *plan, const void *part_O,
                         const float *part_lse, void *cache_O, float *cache_lse,
                         unsigned char *cache_valid, int writeback, int state_bf16, void *out,
                         int out_is_fp32, long long osb, long long osh, long long osn,
                         float *out_lse, float *mass_partials, cudaStream_t stream);
cudaError_t launch_cache_update(const DevGeom &g, const signed char *plan, const void *part_O,
                                const float *part_lse, void *cache_O, float *cache_lse,
                                unsigned char *cache_valid, int state_bf16, int num_sms,
                                cudaStream_t stream);
cudaError_t launch_cache_compose(const DevGeom &fine, const DevGeom &coarse, const void *fine_O,
                                 const float *fine_lse, const unsigned char *fine_valid,
                                 void *coarse_O, float *coarse_lse, unsigned char *coarse_valid,
                                 int state_bf16, cudaStream_t stream);
cudaError_t launch_bounded_wait_selftest(long long limit_ns, int *dev_status,
                                         cudaStream_t stream);
cudaError_t attn_check_status(int *out, bool reset);
cudaError_t merge_check_status(int *out, bool reset);
}  // namespace ditango

using namespace ditango;

namespace {

// An NVTX range over one entry point (shown by profilers; without one
// attached a push/pop costs a few nanoseconds).
struct NvtxRange {
  explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};

// Process-wide limit of every device wait; set from any host thread.
std::atomic<long long> g_wait_limit_ns{1000000000LL};

// Build the kernels' geometry; returns DITANGO_OK or the reason it cannot.
ditango_status make_geom(const ditango_geom *in, DevGeom *out) {
  if (!in) return DITANGO_ERR_INVALID;
  if (in->B < 1 || in->H < 1 || in->N < 1 || in->P < 1 || in->d < 1) return DITANGO_ERR_INVALID;
  if (in->P > kMaxP) return DITANGO_ERR_UNSUPPORTED;
  if (!(in->d == 64 || in->d == 96 || in->d == 128)) return DITANGO_ERR_UNSUPPORTED;
  if ((long long)in->B * in->H > 65535) return DITANGO_ERR_UNSUPPORTED;  // grid.z of the merge
  if (!in->part_off) return DITANGO_ERR_INVALID;
  if (in->part_off[0] != 0 || in->part_off[in->P] != in->N) return DITANGO_ERR_INVALID;
  for (int p = 0; p < in->P; ++p)
    if (in->part_off[p + 1] <= in->part_off[p]) return DITANGO_ERR_INVALID;
  if (in->F < 0 || in->F > kMaxP) return in->F < 0 ? DITANGO_ERR_INVALID : DITANGO_ERR_UNSUPPORTED;
  // frames of the first and the last token of every partition
  int f_lo[kMaxP], f_hi[kMaxP];
  if (in->F > 0) {
    if (!in->frame_off || !in->frame_mask) return DITANGO_ERR_INVALID;
    if (in->frame_off[0] != 0 || in->frame_off[in->F] != in->N) return DITANGO_ERR_INVALID;
    for (int f = 0; f < in->F; ++f)
      if (in->frame_off[f + 1] <= in->frame_off[f]) return DITANGO_ERR_INVALID;
    for (int p = 0, f = 0; p < in->P; ++p) {
      while (in->frame_off[f + 1] <= in->part_off[p]) ++f;
      f_lo[p] = f;
      int e = f;
      while (in->frame_off[e + 1] < in->part_off[p + 1]) ++e;
      f_hi[p] = e;
    }
  }
  DevGeom g;
  std::memset(&g, 0, sizeof(g));
  g.B = in->B;
  g.H = in->H;
  g.N = in->N;
  g.d = in->d;
  g.P = in->P;
  g.BH = in->B * in->H;
  int lmax = 0;
  for (int p = 0; p <= in->P; ++p) g.part_off[p] = in->part_off[p];
  for (int p = 0; p < in->P; ++p) {
    int L = in->part_off[p + 1] - in->part_off[p];
    if (L > lmax) lmax = L;
  }
  g.Lmax = lmax;
  // KV groups: runs of adjacent partitions (one per partition without groups)
  if (in->G < 0 || in->G > in->P) return DITANGO_ERR_INVALID;
  if (in->G == 0) {
    g.G = in->P;
    for (int c = 0; c <= in->P; ++c) g.group_off[c] = c;
  } else {
    if (!in->group_off || in->group_off[0] != 0 || in->group_off[in->G] != in->P)
      return DITANGO_ERR_INVALID;
    for (int c = 0; c < in->G; ++c)
      if (in->group_off[c + 1] <= in->group_off[c]) return DITANGO_ERR_INVALID;
    g.G = in->G;
    for (int c = 0; c <= in->G; ++c) g.group_off[c] = in->group_off[c];
  }
  for (int c = 0; c < g.G; ++c)
    for (int j = g.group_off[c]; j < g.group_off[c + 1]; ++j) g.part_group[j] = (signed char)c;
  // Pair (i, j) is active when some token of partition i may attend some
  // token of partition j.  When a partition straddles frames, an active
  // pair can also hold token pairs the mask forbids: the kernels then mask
  // those logits one by one (token_mask).
  g.F = in->F;
  g.token_mask = 0;
  if (in->F > 0) {
    for (int f = 0; f <= in->F; ++f) g.frame_off[f] = in->frame_off[f];
    for (int f = 0; f < in->F; ++f) {
      unsigned long long a = 0;
      for (int f2 = 0; f2 < in->F; ++f2)
        if (in->frame_mask[f * in->F + f2]) a |= 1ull << f2;
      g.frame_allow[f] = a;
    }
  }
  for (int i = 0; i < in->P; ++i) {
    unsigned long long m = 0;
    for (int j = 0; j < in->P; ++j) {
      if (in->F == 0) {
        m |= 1ull << j;
        continue;
      }
      const unsigned long long kf = bit_range(f_lo[j], f_hi[j] + 1);   // key frames of j
      bool any = false, all = true;
      for (int f = f_lo[i]; f <= f_hi[i]; ++f) {
        const unsigned long long hit = g.frame_allow[f] & kf;
        any = any || hit != 0ull;
        all = all && hit == kf;
      }
      if (any) {
        m |= 1ull << j;
        if (!all) g.token_mask = 1;
      }
    }
    g.pair_mask[i] = m;
  }
  int slot = 0;
  for (int i = 0; i < in->P; ++i) {
    g.row_start[i] = slot;
    unsigned long long m = 0;
    for (int c = 0; c < g.G; ++c)
      if (unit_pairs(g, i, c)) {
        m |= 1ull << c;
        ++slot;
      }
    g.row_mask[i] = m;
  }
  g.row_start[in->P] = slot;
  g.n_active = slot;
  g.multi_run = 0;
  for (int i = 0; i < in->P; ++i)
    for (int c = 0; c < g.G; ++c) {
      const unsigned long long b = unit_pairs(g, i, c);
      if (!b) continue;
      const unsigned long long sh = b >> __builtin_ctzll(b);
      if (sh & (sh + 1ull)) g.multi_run = 1;   // a gap between active partitions
    }
  *out = g;
  return DITANGO_OK;
}

// Fresh-unit count of a plan: max(|band|, floor(budget * active + 1e-9)).
int plan_target(DevGeom *dg, int band_k, double budget) {
  int n_band = 0;
  for (int i = 0; i < dg->P; ++i)
    for (int c = 0; c < dg->G; ++c)
      if (((dg->row_mask[i] >> c) & 1ull) && unit_in_band(*dg, i, c, band_k)) ++n_band;
  int target = (int)std::floor(budget * (double)dg->n_active + 1e-9);
  if (target < n_band) target = n_band;
  if (target > dg->n_active) target = dg->n_active;
  dg->n_band = n_band;
  return target;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool strides_ok(const int64_t s[3]) {
  for (int k = 0; k < 3; ++k)
    if (s[k] <= 0 || ((s[k] * 2) % 16) != 0 || s[k] * 2 >= (1LL << 40)) return false;
  return true;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, []() {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 4-D map over a bf16 [B, H, N, d] tensor (d contiguous), box 64 columns x
// box_rows rows, 128-byte swizzle; columns past d and rows past N read as zero.
bool make_qkv_map(CUtensorMap *m, const void *base, const DevGeom &g, const int64_t s[3],
                  unsigned box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {(cuuint64_t)g.d, (cuuint64_t)g.N, (cuuint64_t)g.H, (cuuint64_t)g.B};
  cuuint64_t strides[3] = {(cuuint64_t)(s[2] * 2), (cuuint64_t)(s[1] * 2), (cuuint64_t)(s[0] * 2)};
  cuuint32_t box[4] = {64, box_rows, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int num_sms_current() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) != cudaSuccess) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return n;
}

ditango_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return DITANGO_OK;
  (void)cudaGetLastError();
  return DITANGO_ERR_CUDA;
}

}  // namespace

extern "C" {

int32_t ditango_version(void) { return 10200; }

const char *ditango_status_string(int32_t s) {
  switch (s) {
    case DITANGO_OK: return "ok";
    case DITANGO_ERR_INVALID: return "invalid argument";
    case DITANGO_ERR_UNSUPPORTED: return "unsupported shape";
    case DITANGO_ERR_CUDA: return "CUDA error";
    case DITANGO_ERR_TIMEOUT: return "device wait timed out";
    case DITANGO_ERR_BOUNDS: return "device input out of range";
    default: return "unknown status";
  }
}

ditango_status ditango_check_geom(const ditango_geom *g) {
  DevGeom dg;
  return make_geom(g, &dg);
}

int64_t ditango_num_active(const ditango_geom *g) {
  DevGeom dg;
  if (make_geom(g, &dg) != DITANGO_OK) return -1;
  return dg.n_active;
}

int64_t ditango_state_rows(const ditango_geom *g) {
  DevGeom dg;
  if (make_geom(g, &dg) != DITANGO_OK) return -1;
  return dg.Lmax;
}

ditango_status ditango_slot_table(const ditango_geom *g, int32_t *slot_out) {
  DevGeom dg;
  ditango_status st = make_geom(g, &dg);
  if (st != DITANGO_OK) return st;
  if (!slot_out) return DITANGO_ERR_INVALID;
  for (int i = 0; i < dg.P; ++i)
    for (int c = 0; c < dg.G; ++c)
      slot_out[i * dg.G + c] = ((dg.row_mask[i] >> c) & 1ull) ? slot_of(dg, i, c) : -1;
  return DITANGO_OK;
}

size_t ditango_plan_workspace_size(const ditango_geom *g) {
  DevGeom dg;
  if (make_geom(g, &dg) != DITANGO_OK) return 0;
  return plan_workspace_bytes(dg);
}

size_t ditango_workspace_size(const ditango_geom *g) { return ditango_plan_workspace_size(g); }

ditango_status ditango_plan(const ditango_geom *g, const float *cache_lse,
                            const uint8_t *cache_valid, int32_t band_k, double budget,
                            int32_t anchor, int8_t *plan, int32_t *fresh_list, int32_t *counts,
                            float *score_out, void *workspace, size_t workspace_bytes,
                            ditango_stream stream) {
  NvtxRange nvtx_range("ditango_plan");
  DevGeom dg;
  ditango_status st = make_geom(g, &dg);
  if (st != DITANGO_OK) return st;
  if (!plan || !fresh_list || !counts) return DITANGO_ERR_INVALID;
  if (!anchor) {
    if (!cache_lse || band_k < 0 || !(budget >= 0.0 && budget <= 1.0)) return DITANGO_ERR_INVALID;
    if (!workspace || workspace_bytes < plan_workspace_bytes(dg)) return DITANGO_ERR_INVALID;
  }
  const int target = plan_target(&dg, band_k, budget);
  return cuda_status(launch_plan(dg, cache_lse, cache_valid, band_k, target, anchor ? 1 : 0,
                                 reinterpret_cast<signed char *>(plan), fresh_list, counts,
                                 score_out, workspace, static_cast<cudaStream_t>(stream), nullptr,
                                 nullptr, nullptr, nullptr, nullptr, 0, 0));
}

ditango_status ditango_plan_from_mass(const ditango_geom *g, float *mass_partials,
                                     size_t mass_bytes, const uint8_t *cache_valid,
                                     int32_t band_k, double budget, int8_t *plan,
                                     int32_t *fresh_list, int32_t *counts, float *score_out,
                                     ditango_stream stream) {
  NvtxRange nvtx_range("ditango_plan_from_mass");
  DevGeom dg;
  ditango_status st = make_geom(g, &dg);
  if (st != DITANGO_OK) return st;
  if (!plan || !fresh_list || !counts || !mass_partials) return DITANGO_ERR_INVALID;
  if (band_k < 0 || !(budget >= 0.0 && budget <= 1.0)) return DITANGO_ERR_INVALID;
  if (mass_bytes < plan_workspace_bytes(dg)) return DITANGO_ERR_INVALID;
  const int target = plan_target(&dg, band_k, budget);
  return cuda_status(launch_plan(dg, nullptr, cache_valid, band_k, target, 0,
                                 reinterpret_cast<signed char *>(plan), fresh_list, counts,
                                 score_out, mass_partials,
                                 static_cast<cudaStream_t>(stream), nullptr, nullptr, nullptr,
                                 nullptr, nullptr, 0, 1));
}

ditango_status ditango_plan_error(const ditango_geom *g, const float *cache_lse,
                                  const uint8_t *cache_valid, int32_t band_k, double budget,
                                  int32_t anchor, int32_t refresh_w,
                                  const ditango_error_state *es, int8_t *plan,
                                  int32_t *fresh_list, int32_t *counts, float *score_out,
                                  void *workspace, size_t workspace_bytes,
                                  ditango_stream stream) {
  NvtxRange nvtx_range("ditango_plan_error");
  DevGeom dg;
  ditango_status st = make_geom(g, &dg);
  if (st != DITANGO_OK) return st;
  if (!plan || !fresh_list || !counts || !es) return DITANGO_ERR_INVALID;
  if (!es->w || !es->age || !es->delta || !es->local_ok) return DITANGO_ERR_INVALID;
  if (!anchor) {
    if (!es->drift_rows || band_k < 0 || !(budget >= 0.0 && budget <= 1.0))
      return DITANGO_ERR_INVALID;
    if (refresh_w && !cache_lse) return DITANGO_ERR_INVALID;
    if (!workspace || workspace_bytes < plan_workspace_bytes(dg)) return DITANGO_ERR_INVALID;
  }
  const int target = plan_target(&dg, band_k, budget);
  return cuda_status(launch_plan(dg, cache_lse, cache_valid, band_k, target, anchor ? 1 : 0,
                                 reinterpret_cast<signed char *>(plan), fresh_list, counts,
                                 score_out, workspace, static_cast<cudaStream_t>(stream),
                                 es->drift_rows, es->w, es->age, es->delta, es->local_ok,
                                 refresh_w ? 1 : 0, 0));
}

ditango_status ditango_attn_partial(const ditango_geom *g, const uint16_t *Q, const uint16_t *K,
                                    const uint16_t *V, const int32_t *fresh_list,
                                    const int32_t *counts, float scale, void *out_O,
                                    float *out_lse, int32_t out_by_slot, int32_t state_bf16,
                                    uint8_t *out_valid, float *drift_rows, int32_t *dev_status,
                                    int32_t *work_counter, ditango_stream stream) {
  NvtxRange nvtx_range("ditango_attn_partial");
  DevGeom dg;
  ditango_status st = make_geom(g, &dg);
  if (st != DITANGO_OK) return st;
  if (!Q || !K || !V || !fresh_list || !counts || !out_O || !out_lse) return DITANGO_ERR_INVALID;
  if (drift_rows && !out_by_slot) return DITANGO_ERR_INVALID;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(out_O))
    return DITANGO_ERR_INVALID;
  if (work_counter && (reinterpret_cast<uintptr_t>(work_counter) & 7u)) return DITANGO_ERR_INVALID;
  // the stride of a dimension of size 1 is never used (frameworks report 0
  // or anything for it): give it the packed value
  int64_t qs[3], ks[3], vs[3];
  for (int k = 0; k < 3; ++k) {
    qs[k] = g->q_strides[k];
    ks[k] = g->k_strides[k];
    vs[k] = g->v_strides[k];
  }
  for (int64_t *s : {qs, ks, vs}) {
    if (dg.N == 1) s[2] = dg.d;
    if (dg.H == 1) s[1] = s[2] * dg.N;
    if (dg.B == 1) s[0] = s[1] * dg.H;
  }
  if (!strides_ok(qs) || !strides_ok(ks) || !strides_ok(vs)) return DITANGO_ERR_INVALID;
  if (!(scale >= 0.f) || !std::isfinite(scale)) return DITANGO_ERR_INVALID;
  if (scale == 0.f) scale = 1.f / std::sqrt((float)dg.d);
  CUtensorMap tq, tk, tv;
  // Q in 128-row tiles, K and V in the kernel's key tiles (96 keys at d = 96, else 128)
  const unsigned bn = (unsigned)attn_key_tile(dg.d);
  if (!make_qkv_map(&tq, Q, dg, qs, 128) || !make_qkv_map(&tk, K, dg, ks, bn) ||
      !make_qkv_map(&tv, V, dg, vs, bn))
    return DITANGO_ERR_CUDA;
  return cuda_status(launch_attn_partial(dg, tq, tk, tv, fresh_list, counts, scale, out_O, out_lse,
                                         out_by_slot ? 1 : 0, state_bf16 ? 1 : 0, out_valid,
                                         drift_rows, dev_status, g_wait_limit_ns.load(),
                                         num_sms_current(), work_counter,
                                         static_cast<cudaStream_t>(stream)));
}

ditango_status ditango_merge(const ditango_geom *g, const int8_t *plan, const void *part_O,
                             const float *part_lse, void *cache_O, float *cache_lse,
                             uint8_t *cache_valid, int32_t writeback, int32_t state_bf16,
                             void *out, int32_t out_is_fp32, const int64_t *out_strides,
                             float *out_lse, float *mass_partials, ditango_stream stream) {
  NvtxRange nvtx_range("ditango_merge");
  DevGeom dg;
  ditango_status st = make_geom(g, &dg);
  if (st != DITANGO_OK) return st;
  if (!plan || !out) return DITANGO_ERR_INVALID;
  if ((part_O == nullptr) != (part_lse == nullptr)) return DITANGO_ERR_INVALID;
  if ((cache_O == nullptr) != (cache_lse == nullptr)) return DITANGO_ERR_INVALID;
  if (part_O == nullptr && cache_O == nullptr) return DITANGO_ERR_INVALID;
  if (writeback && part_O && !cache_O) return DITANGO_ERR_INVALID;
  // the merge moves state rows in 16-byte groups
  if ((part_O && !aligned16(part_O)) || (cache_O && !aligned16(cache_O))) return DITANGO_ERR_INVALID;
  long long osb = (long long)dg.H * dg.N * dg.d, osh = (long long)dg.N * dg.d, osn = dg.d;
  if (out_strides) {
    osb = out_strides[0];
    osh = out_strides[1];
    osn = out_strides[2];
    if (osb <= 0 || osh <= 0 || osn <= 0) return DITANGO_ERR_INVALID;
  }
  const int esz = out_is_fp32 ? 4 : 2;
  if ((osb * esz) % 16 || (osh * esz) % 16 || (osn * esz) % 16 ||
      (reinterpret_cast<uintptr_t>(out) % (out_is_fp32 ? 16 : 8)))
    return DITANGO_ERR_INVALID;
  return cuda_status(launch_merge(dg, reinterpret_cast<const signed char *>(plan), part_O,
                                  part_lse, cache_O, cache_lse, cache_valid,
                                  (writeback && part_O) ? 1 : 0, state_bf16 ? 1 : 0, out,
                                  out_is_fp32 ? 1 : 0, osb, osh, osn, out_lse, mass_partials,
                                  static_cast<cudaStream_t>(stream)));
}

ditango_status ditango_cache_update(const ditango_geom *g, const int8_t *plan,
                                    const void *part_O, const float *part_lse, void *cache_O,
                                    float *cache_lse, uint8_t *cache_valid, int32_t state_bf16,
                                    ditango_stream stream) {
  NvtxRange nvtx_range("ditango_cache_update");
  DevGeom dg;
  ditango_status st = make_geom(g, &dg);
  if (st != DITANGO_OK) return st;
  if (!plan || !part_O || !part_lse || !cache_O || !cache_lse) return DITANGO_ERR_INVALID;
  return cuda_status(launch_cache_update(dg, reinterpret_cast<const signed char *>(plan), part_O,
                                         part_lse, cache_O, cache_lse, cache_valid,
                                         state_bf16 ? 1 : 0, num_sms_current(),
                                         static_cast<cudaStream_t>(stream)));
}

ditango_status ditango_cache_compose(const ditango_geom *fine, const ditango_geom *coarse,
                                     const void *fine_O, const float *fine_lse,
                                     const uint8_t *fine_valid, void *coarse_O,
                                     float *coarse_lse, uint8_t *coarse_valid,
                                     int32_t state_bf16, ditango_stream stream) {
  NvtxRange nvtx_range("ditango_cache_compose");
  DevGeom gf, gc;
  ditango_status st = make_geom(fine, &gf);
  if (st != DITANGO_OK) return st;
  st = make_geom(coarse, &gc);
  if (st != DITANGO_OK) return st;
  // same attention call, only the KV grouping differs
  if (gf.B != gc.B || gf.H != gc.H || gf.N != gc.N || gf.d != gc.d || gf.P != gc.P)
    return DITANGO_ERR_INVALID;
  for (int p = 0; p <= gf.P; ++p)
    if (gf.part_off[p] != gc.part_off[p]) return DITANGO_ERR_INVALID;
  for (int i = 0; i < gf.P; ++i)
    if (gf.pair_mask[i] != gc.pair_mask[i]) return DITANGO_ERR_INVALID;
  // every coarse group boundary is a fine group boundary
  for (int C = 0, c = 0; C <= gc.G; ++C) {
    while (c <= gf.G && gf.group_off[c] < gc.group_off[C]) ++c;
    if (c > gf.G || gf.group_off[c] != gc.group_off[C]) return DITANGO_ERR_INVALID;
  }
  if (!fine_O || !fine_lse || !coarse_O || !coarse_lse) return DITANGO_ERR_INVALID;
  const size_t align = state_bf16 ? 8 : 16;
  if (reinterpret_cast<uintptr_t>(fine_O) % align || reinterpret_cast<uintptr_t>(coarse_O) % align)
    return DITANGO_ERR_INVALID;
  // the two state buffers must not overlap
  const size_t rows = (size_t)gf.BH * gf.Lmax;
  const size_t es = state_bf16 ? 2 : 4;
  const char *f0 = static_cast<const char *>(fine_O), *f1 = f0 + (size_t)gf.n_active * rows * gf.d * es;
  const char *c0 = static_cast<const char *>(coarse_O), *c1 = c0 + (size_t)gc.n_active * rows * gc.d * es;
  if (f0 < c1 && c0 < f1) return DITANGO_ERR_INVALID;
  const float *fl0 = fine_lse, *fl1 = fine_lse + (size_t)gf.n_active * rows;
  const float *cl0 = coarse_lse, *cl1 = coarse_lse + (size_t)gc.n_active * rows;
  if (fl0 < cl1 && cl0 < fl1) return DITANGO_ERR_INVALID;
  return cuda_status(launch_cache_compose(gf, gc, fine_O, fine_lse, fine_valid, coarse_O,
                                          coarse_lse, coarse_valid, state_bf16 ? 1 : 0,
                                          static_cast<cudaStream_t>(stream)));
}

void ditango_set_wait_limit_ns(int64_t ns) { g_wait_limit_ns.store(ns > 0 ? ns : 1); }

int32_t ditango_checked_build(void) {
#ifdef DITANGO_CHECK
  return 1;
#else
  return 0;
#endif
}

ditango_status ditango_check_status(int32_t *status_out, int32_t reset) {
  if (!status_out) return DITANGO_ERR_INVALID;
  int a = 0, m = 0;
  cudaError_t e = attn_check_status(&a, reset != 0);
  if (e == cudaSuccess) e = merge_check_status(&m, reset != 0);
  if (e != cudaSuccess) return cuda_status(e);
  *status_out = a != 0 ? a : m;
  return DITANGO_OK;
}

ditango_status ditango_selftest_bounded_wait(int64_t limit_ns, int32_t *dev_status,
                                             ditango_stream stream) {
  if (!dev_status || limit_ns <= 0) return DITANGO_ERR_INVALID;
  return cuda_status(
      launch_bounded_wait_selftest(limit_ns, dev_status, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free plan.
//
// Some callers cannot allocate device memory at all: code that runs inside a
// memory arena owned by someone else, a serving process whose allocator is
// frozen after start-up, or a host that must never call cudaMalloc between
// denoising steps.  They still pass their own inputs and outputs, but the
// plan's scratch (the mass block sums and their means) lives here, in a fixed device
// array of this library of kNoAllocPlanScratchBytes.  Every GPU that loads
// the library holds that array until the process exits (or until its context
// is destroyed).
//
// The array's host-side name is not a device address: its address is asked
// of the runtime with the device current, and cached per device together
// with the unique ID of the context it belongs to.  A new context on the
// device (after cudaDeviceReset, say) has a new ID, and the address is then
// looked up again instead of reusing one that points into freed memory.
namespace {
constexpr size_t kNoAllocPlanScratchBytes = size_t(4) << 20;  // 4 MiB
constexpr int kNoAllocMaxDevices = 64;

struct NoAllocScratch {
  unsigned long long ctx_id;  // context the address belongs to
  void *ptr;                  // null: not looked up in that context yet
};
std::mutex g_noalloc_mu;
NoAllocScratch g_noalloc_scratch[kNoAllocMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

// Unique ID (for the life of the process) of the calling thread's current
// context; false when no context is current or the driver has no such call.
bool current_context_id(unsigned long long *id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, []() {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}
}  // namespace

static __device__ __align__(256) unsigned char g_plan_scratch[kNoAllocPlanScratchBytes];

extern "C" ditango_status ditango_plan_noalloc(const ditango_geom *g, const float *cache_lse,
                                               const uint8_t *cache_valid, int32_t band_k,
                                               double budget, int32_t anchor, int8_t *plan,
                                               int32_t *fresh_list, int32_t *counts,
                                               float *score_out, ditango_stream stream) {
  NvtxRange nvtx_range("ditango_plan_noalloc");
  DevGeom dg;
  ditango_status st = make_geom(g, &dg);
  if (st != DITANGO_OK) return st;
  if (!plan || !fresh_list || !counts) return DITANGO_ERR_INVALID;
  if (!anchor) {
    if (!cache_lse || band_k < 0 || !(budget >= 0.0 && budget <= 1.0)) return DITANGO_ERR_INVALID;
    if (plan_workspace_bytes(dg) > kNoAllocPlanScratchBytes) return DITANGO_ERR_UNSUPPORTED;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cuda_status(cudaErrorInvalidDevice);
  if (dev < 0 || dev >= kNoAllocMaxDevices) return DITANGO_ERR_UNSUPPORTED;
  void *scratch = nullptr;
  {
    // with this device current: the cached address if it belongs to the
    // current context, else ask the runtime for it (the first ask in a
    // context also makes the primary context current on this thread)
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    NoAllocScratch &e = g_noalloc_scratch[dev];
    unsigned long long id = 0;
    bool have_id = current_context_id(&id);
    if (have_id && e.ptr != nullptr && e.ctx_id == id) {
      scratch = e.ptr;
    } else {
      void *p = nullptr;
      cudaError_t err = cudaGetSymbolAddress(&p, g_plan_scratch);
      if (err != cudaSuccess || p == nullptr)
        return cuda_status(err == cudaSuccess ? cudaErrorUnknown : err);
      if (!have_id) have_id = current_context_id(&id);
      e.ptr = have_id ? p : nullptr;   // without a context ID: look it up every call
      e.ctx_id = have_id ? id : 0;
      scratch = p;
    }
  }
  const int target = plan_target(&dg, band_k, budget);
  return cuda_status(launch_plan(dg, cache_lse, cache_valid, band_k, target, anchor ? 1 : 0,
                                 reinterpret_cast<signed char *>(plan), fresh_list, counts,
                                 score_out, scratch, static_cast<cudaStream_t>(stream), nullptr,
                                 nullptr, nullptr, nullptr, nullptr, 0, 0));
}
