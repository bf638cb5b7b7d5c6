/*
 * ditango.h -- C ABI of the partitioned-attention hot path with selective
 * attention-state reuse, for NVIDIA B200 (sm_100a).
 *
 * What it computes (sources by page title and section):
 *  - "DiTango: Cost-Effective Parallel Diffusion Generation with Selective
 *    Attention State Reuse", technical summary:
 *      Metodologia: the token sequence is split into P context partitions and
 *        attention is computed per (query partition i, KV partition j) pair;
 *        near partitions contribute most (spatial locality).
 *      1. Anchor-Guided Selection Planner: per pair, recompute ("fresh") or
 *        reuse the previous denoising step's attention state, guided by the
 *        partition's importance w; anchor steps recompute everything;
 *        "Strategia per Gruppi": decisions per group of adjacent partitions.
 *      2. State-Centric Parallel Runtime, "Composizione dello Stato": an
 *        attention state is (output, log-sum-exp); states are cached instead
 *        of raw K/V and compose associatively and commutatively;
 *        "Calcolo dello Stato di Gruppo": one state per group;
 *        "Composizione Dinamica dei Gruppi": cached states are merged
 *        recursively into coarser groups to shrink the cache.
 *  - "Efficient-vDiT: Efficient Video Diffusion Transformers With Attention
 *    Tile", abstract: a frame-tile sparse mask whose cost grows linearly
 *    with the number of frames.
 *
 * Conventions shared by every entry point
 *  - Every buffer is allocated by the caller.  "dev" marks device pointers,
 *    "host" host pointers.  The library keeps no pointer after a call
 *    returns and allocates no device memory.
 *  - Every device-side call is asynchronous on `stream` (a cudaStream_t;
 *    NULL is the legacy default stream) and never synchronises the host.
 *  - Arguments are validated before anything is launched: a bad argument
 *    returns DITANGO_ERR_INVALID, a valid but unsupported shape returns
 *    DITANGO_ERR_UNSUPPORTED, a failed launch returns DITANGO_ERR_CUDA.
 *    Device-side failures (a pipeline wait that exceeded its time limit) are
 *    written as a status code into `dev_status` where a call takes one.
 *  - Token order is frame-major; partitions are contiguous token ranges.
 *  - Units: the KV side may be grouped into G runs of adjacent partitions
 *    (ditango_geom.G, group_off).  The unit of planning and of storage is
 *    (query partition i, KV group c); its state is attention of partition
 *    i's rows against every allowed key of the group's partitions.  Without
 *    groups (G = 0) each partition is its own group, G = P and a unit is the
 *    pair (i, j).  A unit is active when some pair (i, j), j in c, is.
 *  - State layout ("state buffer"): O is [n_idx][B*H][Lmax][d], float32 or
 *    (state_bf16 = 1, a compressed cache) bfloat16 bit patterns, and lse is
 *    float32 [n_idx][B*H][Lmax], where Lmax = max partition length
 *    (ditango_state_rows) and the leading index is either the slot of an
 *    active unit (row-major rank of the active units, see ditango_slot_table)
 *    or the position of a unit in the fresh list.  Row r of unit (i, c)
 *    holds query token part_off[i] + r; rows r >= L_i are never written.
 *    O is normalised (sum_k softmax_k v_k) and lse is the natural
 *    log-sum-exp of the scaled logits.
 *  - Plan: int8 [P * G], entry i * G + c; codes 0 skip (masked unit),
 *    1 fresh, 2 reuse.
 */
#ifndef DITANGO_H
#define DITANGO_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DITANGO_OK = 0,
  DITANGO_ERR_INVALID = 1,      /* bad argument (null, negative, inconsistent) */
  DITANGO_ERR_UNSUPPORTED = 2,  /* valid but outside what the kernels handle */
  DITANGO_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed */
  DITANGO_ERR_TIMEOUT = 4,      /* device: a pipeline wait exceeded its limit */
  DITANGO_ERR_BOUNDS = 5        /* device, checked builds: a device-resident input (a count,
                                   a fresh list, a plan code) out of range */
} ditango_status;

enum { DITANGO_PLAN_SKIP = 0, DITANGO_PLAN_FRESH = 1, DITANGO_PLAN_REUSE = 2 };

typedef void *ditango_stream; /* cudaStream_t */

/* Geometry of one attention call; host struct, read during the call only.
 *   B, H     batch and heads; N tokens; d head dim in {64, 96, 128}.
 *   P        partitions, 1 <= P <= 64; part_off host int32 [P+1],
 *            part_off[0] = 0 < part_off[1] < ... < part_off[P] = N.
 *   F        frames of the frame-tile mask, 0 = no mask (all pairs active);
 *            else 1 <= F <= 64, frame_off host int32 [F+1] (same rules as
 *            part_off) and frame_mask host uint8 [F*F], row = query frame,
 *            nonzero = the query frame may attend the key frame.  The mask
 *            applies token by token; pair (i, j) is active when some token of
 *            partition i may attend some token of partition j.  Partitions may
 *            straddle frames: single logits are then masked inside the pair,
 *            and a row that may attend none of a unit's keys gets lse = -inf,
 *            O = 0 for that unit.
 *   q/k/v_strides  element strides of the (b, h, n) dimensions of the bf16
 *            Q, K, V tensors; the d dimension is contiguous.  Strides times 2
 *            bytes must be multiples of 16 and the base pointers 16-byte
 *            aligned (TMA).  The stride of a dimension of size 1 is ignored.
 *   G        KV groups; 0 = one group per partition (group_off ignored).
 *            Else 1 <= G <= P and group_off host int32 [G+1] holds partition
 *            indices, group_off[0] = 0 < ... < group_off[G] = P: group c is
 *            partitions group_off[c] .. group_off[c+1]-1. */
typedef struct {
  int32_t B, H, N, d;
  int32_t P, F;
  const int32_t *part_off;
  const int32_t *frame_off;
  const uint8_t *frame_mask;
  int64_t q_strides[3];
  int64_t k_strides[3];
  int64_t v_strides[3];
  int32_t G;
  const int32_t *group_off;
} ditango_geom;

/* Library version (major * 10000 + minor * 100 + patch). */
int32_t ditango_version(void);

/* Static string for a status code. */
const char *ditango_status_string(int32_t status);

/* Validate a geometry without launching anything. */
ditango_status ditango_check_geom(const ditango_geom *g);

/* Number of active units (= slots): units (i, c) with a pair (i, j), j in c,
 * whose tokens the frame mask lets attend each other (all P*G when F = 0).
 * Returns -1 on a bad geometry. */
int64_t ditango_num_active(const ditango_geom *g);

/* Lmax, rows per (index, b*h) block of a state buffer. -1 on a bad geometry. */
int64_t ditango_state_rows(const ditango_geom *g);

/* Host helper: slot_out host int32 [P*G] receives the slot of each unit,
 * -1 for masked units (row-major rank of the active units). */
ditango_status ditango_slot_table(const ditango_geom *g, int32_t *slot_out);

/* Bytes of device scratch ditango_plan needs; also the size of the mass
 * partials ditango_merge can emit (the same layout: float32 block sums
 * [P][B*H][ceil(Lmax / 128)][G + 1], see ditango_merge). */
size_t ditango_plan_workspace_size(const ditango_geom *g);

/* The same value under its shorter name. */
size_t ditango_workspace_size(const ditango_geom *g);

/* Plan: per unit, fresh or reuse (DiTango, 1. Anchor-Guided Selection
 * Planner and its group strategy; spatial locality from Metodologia).
 *   cache_lse    dev float32 state-buffer lse indexed by slot (the previous
 *                step's cached states); may be NULL when anchor != 0.
 *   cache_valid  dev uint8 [slots] (nonzero = slot holds a state) or NULL
 *                (all valid).  An invalid slot is forced fresh and holds no
 *                mass.
 *   band_k       the band: unit (i, c) is always fresh when some active
 *                pair (i, j), j in c, has |i - j| <= band_k.
 *   budget       fraction of active units to recompute: the fresh count is
 *                max(|band|, floor(budget * active + 1e-9)); the units added
 *                beyond the band are those of largest mass w, ties to the
 *                lower linear index i*G + c.
 *   anchor       nonzero: every active unit fresh (an anchor step).
 * w[i][c] = mean over (b, h, rows r of partition i) of
 *           exp(lse_ic[r]) / sum_{c' active, valid} exp(lse_ic'[r]),
 * computed in float32 with a fixed reduction order (deterministic).
 * Outputs (dev): plan int8 [P*G]; fresh_list int32 [slots] = linear indices
 * i*G + c of the fresh units in row-major order; counts int32 [2] = {fresh,
 * reuse}; score_out float32 [P*G] (w, 0 for masked units) or NULL.
 * workspace: dev, >= ditango_plan_workspace_size bytes. */
ditango_status ditango_plan(const ditango_geom *g, const float *cache_lse,
                            const uint8_t *cache_valid, int32_t band_k, double budget,
                            int32_t anchor, int8_t *plan, int32_t *fresh_list,
                            int32_t *counts, float *score_out, void *workspace,
                            size_t workspace_bytes, ditango_stream stream);

/* Plan from mass partials: ditango_plan with its first stage (the mass
 * score read from the cache) replaced by the block sums a ditango_merge
 * call emitted (its mass_partials argument) -- DiTango, "Anchor Steps":
 * the importance w is refreshed from the states just composed, without
 * reading the cache again.  The partials describe the cache as that merge
 * left it (every state it composed counts as valid); after anything else
 * has changed the cache (states invalidated or written by another call, a
 * composition), plan with ditango_plan instead.  The same selection,
 * outputs and determinism as ditango_plan; given the partials of a merge
 * whose composed states are the cache's valid states, the plan and scores
 * are bit-identical to ditango_plan's on that cache.
 *   mass_partials  dev, written by ditango_merge, mass_bytes >=
 *                  ditango_plan_workspace_size (else INVALID); the part of
 *                  the buffer past the block sums serves as scratch (the
 *                  per-unit means), so the block sums themselves are left
 *                  unchanged.
 *   cache_valid    as for ditango_plan (invalid slots are forced fresh). */
ditango_status ditango_plan_from_mass(const ditango_geom *g, float *mass_partials,
                                     size_t mass_bytes, const uint8_t *cache_valid,
                                     int32_t band_k, double budget, int8_t *plan,
                                     int32_t *fresh_list, int32_t *counts, float *score_out,
                                     ditango_stream stream);

/* Partial attention states of the fresh units (tcgen05 tensor cores, TMA).
 * For each fresh unit (i, c) = fresh_list[f], f < counts[0] (read on the
 * device), and each (b, h): S = Q_i K_c^T * scale over the keys K_c of the
 * active pairs of group c, O = softmax(S) V_c (normalised), lse =
 * logsumexp(S) -- the state of DiTango's "Composizione dello Stato" (one
 * pair, or a whole group: "Calcolo dello Stato di Gruppo").  bf16 inputs, fp32 accumulation and softmax;
 * the probabilities are rounded to bf16 for the P V product.
 *   Q, K, V      dev bf16 (uint16 bit patterns) with the geometry's strides.
 *   scale        logit scale; 0 means 1/sqrt(d).
 *   out_O/out_lse  dev state buffer; index = f (out_by_slot = 0) or the
 *                unit's slot (out_by_slot = 1, e.g. writing the cache in
 *                place).  Must hold counts[0] (resp. all slots) indices.
 *   state_bf16   nonzero: O is stored as bf16 (the normalised fp32 O rounded
 *                to nearest even); lse stays float32.  A compressed cache
 *                halves the cache memory and the merge's read traffic
 *                (DiTango, "Significato e Claim": cache memory is the
 *                method's limitation and cache compression its next step).
 *   out_valid    dev uint8 [slots] or NULL; with out_by_slot = 1 the written
 *                slots are set to 1.
 *   drift_rows   dev float32 [P][B*H][Lmax] or NULL (needs out_by_slot = 1):
 *                for each fresh local unit -- the unit of partition i that
 *                holds partition i, always in the band -- row r receives
 *                |lse_new - lse_old|, lse_old being the slot's lse before
 *                this call overwrites it (equal values, -inf included, give
 *                0): the local state's change that ditango_plan_error reads
 *                (DiTango, "Predizione Online").
 *   dev_status   dev int32 or NULL; set to DITANGO_ERR_TIMEOUT if a pipeline
 *                wait exceeded the limit (the kernel then stops cleanly).
 *   work_counter dev int32 [2], 8-byte aligned, or NULL.  With it, each CTA
 *                of the persistent kernel takes the next work item when it is
 *                ready for one (balanced whatever the items' sizes); without
 *                it, items are dealt in a fixed stride.  Zero it once when it
 *                is allocated: every launch leaves it at zero again.  Launches
 *                that may run at the same time (other streams, concurrent
 *                graph branches) must not share one.
 */
ditango_status ditango_attn_partial(const ditango_geom *g, const uint16_t *Q,
                                    const uint16_t *K, const uint16_t *V,
                                    const int32_t *fresh_list, const int32_t *counts,
                                    float scale, void *out_O, float *out_lse,
                                    int32_t out_by_slot, int32_t state_bf16,
                                    uint8_t *out_valid, float *drift_rows,
                                    int32_t *dev_status, int32_t *work_counter,
                                    ditango_stream stream);

/* Merge: the final output of every token is the log-sum-exp composition of
 * the states of its partition's active units (DiTango, "Composizione dello
 * Stato"): L = log sum_c exp(lse_c), O = sum_c exp(lse_c - L) O_c, with
 * fresh states read from part_O/part_lse (indexed by fresh-list position)
 * and reused ones from cache_O/cache_lse (indexed by slot).  part_O = NULL
 * means the fresh states were already written into the cache slots
 * (ditango_attn_partial with out_by_slot = 1).  The weights
 * exp(lse_c - L) of a row are computed in a fixed order (largest lse first
 * subtracted, a fixed summation tree), shared with ditango_plan's mass
 * score.
 *   plan          dev int8 [P*G] from ditango_plan.
 *   writeback     nonzero: also copy each fresh state into its cache slot
 *                 and mark cache_valid (ignored when part_O is NULL).
 *   state_bf16    format of every state buffer passed (see ditango_attn_partial).
 *   out           dev [B, H, N, d] (element strides out_strides for b, h, n;
 *                 NULL = contiguous), bf16 bits (out_is_fp32 = 0) or float32.
 *   out_lse       dev float32 [B, H, N] or NULL.
 *   mass_partials dev float32 of ditango_plan_workspace_size bytes, or NULL:
 *                 receives, per (query partition i, b*h, block of 128 rows),
 *                 every active unit's sum of its weights over the block's
 *                 rows (0 for a unit the plan skipped) -- the next step's
 *                 importance w before averaging (DiTango, "Anchor Steps":
 *                 refreshed from the states just composed); pass it to
 *                 ditango_plan_from_mass.  Column G is not written.
 * A token whose partition has no active pair gets O = 0, lse = -inf. */
ditango_status ditango_merge(const ditango_geom *g, const int8_t *plan,
                             const void *part_O, const float *part_lse,
                             void *cache_O, float *cache_lse, uint8_t *cache_valid,
                             int32_t writeback, int32_t state_bf16, void *out,
                             int32_t out_is_fp32, const int64_t *out_strides,
                             float *out_lse, float *mass_partials, ditango_stream stream);

/* Cache update: copy the fresh states (indexed by fresh position) into their
 * cache slots and mark them valid -- the write half of an anchor step
 * (DiTango, "Anchor Steps": everything is recomputed and the cache
 * refreshed). */
ditango_status ditango_cache_update(const ditango_geom *g, const int8_t *plan,
                                    const void *part_O, const float *part_lse,
                                    void *cache_O, float *cache_lse,
                                    uint8_t *cache_valid, int32_t state_bf16,
                                    ditango_stream stream);

/* Dynamic group composition (DiTango, "Composizione Dinamica dei Gruppi"):
 * merge the cached states of a fine grouping into the states of a coarser
 * one, with no recomputation: the coarse unit (i, C) gets the log-sum-exp
 * composition of the fine units (i, c), c inside C, that are active.
 *   fine, coarse  geometries identical except for G/group_off, and every
 *                 coarse group boundary a fine group boundary (else INVALID);
 *                 applied repeatedly (groups of 1 -> 2 -> 4 ...) the cache
 *                 halves at every level.
 *   fine_O/fine_lse/fine_valid      dev state buffer of the fine slots
 *                 (fine_valid may be NULL: all valid).
 *   coarse_O/coarse_lse/coarse_valid  dev state buffer of the coarse slots
 *                 (coarse_valid may be NULL); must not overlap the fine one.
 * A coarse slot is valid only if every fine slot it covers is; an invalid
 * one is marked 0 and its rows are not written.  Both buffers use the
 * state format state_bf16 (bf16 results are rounded to nearest even). */
ditango_status ditango_cache_compose(const ditango_geom *fine, const ditango_geom *coarse,
                                     const void *fine_O, const float *fine_lse,
                                     const uint8_t *fine_valid, void *coarse_O,
                                     float *coarse_lse, uint8_t *coarse_valid,
                                     int32_t state_bf16, ditango_stream stream);

/* Error-growth planner state (DiTango, 1. Anchor-Guided Selection Planner:
 * "Modellazione dell'Errore", "Anchor Steps", "Predizione Online").  Device
 * buffers owned by the caller, zeroed once before the first (anchor) step and
 * then carried from step to step by ditango_plan_error. */
typedef struct {
  float *w;                 /* dev float32 [P*G]: importance, refreshed after anchors */
  float *age;               /* dev float32 [slots]: local drift accumulated since each
                               cached state was computed */
  float *delta;             /* dev float32 [P]: last measured local drift (output) */
  uint8_t *local_ok;        /* dev uint8 [P]: the local unit held a state before the
                               last step's attention call */
  const float *drift_rows;  /* dev float32 [P][B*H][Lmax]: written by
                               ditango_attn_partial (drift_rows argument) */
} ditango_error_state;

/* Plan by predicted reuse error.  The same contract as ditango_plan (band,
 * invalid slots, budget, fresh list, counts, workspace) with the ranking
 * score replaced:
 *   delta_i = mean over (b, h, rows of partition i) of drift_rows, when
 *             local_ok[i] (else 0) -- the local state's change in the last
 *             step, standing in for the drift of the partition's remote
 *             states;
 *   age     = 0 for units the previous plan made fresh, age + delta_i for
 *             the units it reused;
 *   score   = w * (age + delta_i): the predicted error of reusing the unit
 *             at this step; the non-band units of largest score fill the
 *             budget (ties to the lower index i*G + c).
 *   plan     in: the previous step's plan (zeros before the first step);
 *            out: this step's plan.
 *   anchor   nonzero: every active unit fresh (an anchor step, "Anchor
 *            Steps"); w, age and delta are left alone.
 *   refresh_w  nonzero (the step after an anchor): w is recomputed from the
 *            cache as in ditango_plan and stored in es->w; otherwise es->w
 *            is used as held.
 *   score_out  dev float32 [P*G] or NULL: the score (0 for masked units).
 * Every call also records es->local_ok for the next step (whether the local
 * unit's slot is valid now, before this step's attention call). */
ditango_status ditango_plan_error(const ditango_geom *g, const float *cache_lse,
                                  const uint8_t *cache_valid, int32_t band_k, double budget,
                                  int32_t anchor, int32_t refresh_w,
                                  const ditango_error_state *es, int8_t *plan,
                                  int32_t *fresh_list, int32_t *counts, float *score_out,
                                  void *workspace, size_t workspace_bytes,
                                  ditango_stream stream);

/* Allocation-free variant of ditango_plan (no counterpart in the papers: it
 * exists for callers, not for the method).  For callers that cannot allocate
 * device memory -- code running inside an arena it does not own, a serving
 * process whose allocator is frozen after start-up, or a host that must not
 * call cudaMalloc between steps -- and so cannot provide ditango_plan's
 * workspace.  Same arguments, meaning and results as ditango_plan without
 * workspace/workspace_bytes; the scratch is a fixed 4 MiB device array inside
 * the library (held by every GPU that loads the library until the process
 * exits).  Returns DITANGO_ERR_UNSUPPORTED when ditango_plan_workspace_size
 * exceeds 4 MiB (anchor plans need no scratch and are never rejected).
 * Allocates nothing itself: no cudaMalloc, cudaFree or allocating library
 * call.  But the CUDA runtime loads the library's device code lazily by
 * default, so the first call on a device (in a context) is what makes the
 * driver load the module and reserve the 4 MiB array; that first load can
 * fail under memory pressure.  A caller whose allocator is frozen should
 * make one call per device at start-up (it must anyway come before any
 * stream capture), or run with CUDA_MODULE_LOADING=EAGER.
 * The array's device address is looked up with cudaGetSymbolAddress, with
 * the device current, on the first call in each context and cached with the
 * context's unique ID; after cudaDeviceReset (a new context) the next call
 * looks it up again.  Every call shares the one array per device and
 * overwrites all of the scratch it reads, so nothing carries over between
 * calls; but calls that overlap on the GPU (other streams, concurrent graph
 * branches) race on it -- order them. */
ditango_status ditango_plan_noalloc(const ditango_geom *g, const float *cache_lse,
                                    const uint8_t *cache_valid, int32_t band_k, double budget,
                                    int32_t anchor, int8_t *plan, int32_t *fresh_list,
                                    int32_t *counts, float *score_out, ditango_stream stream);

/* Time limit, in nanoseconds, of every wait inside the kernels (default
 * 1e9).  Process-wide; read at each launch. */
void ditango_set_wait_limit_ns(int64_t ns);

/* Checked builds.  The library built with -DDITANGO_CHECK
 * (libditango_check.so) validates the device-resident inputs the host cannot
 * see without a synchronisation -- ditango_attn_partial's counts[0] (at most
 * the active units) and fresh list (unit indices in range, active, strictly
 * row-major), and the plan codes ditango_merge reads -- before using them.  A
 * bad attention input makes the kernel compute nothing and record
 * DITANGO_ERR_BOUNDS (also in dev_status when given); a bad plan code is
 * recorded and the unit left out.  The release build skips these checks.
 * ditango_checked_build: 1 in a checked build, 0 otherwise.
 * ditango_check_status: the recorded status (DITANGO_OK if none) into
 * *status_out (host), cleared when reset != 0; synchronises with the device.
 * Always 0 in the release build. */
int32_t ditango_checked_build(void);
ditango_status ditango_check_status(int32_t *status_out, int32_t reset);

/* Failure-detection self-test: launches one block that waits on a barrier
 * nothing will complete, with a limit of limit_ns; the kernel returns and
 * writes DITANGO_ERR_TIMEOUT into dev_status (dev int32).  Exercises the
 * same bounded wait the pipeline kernels use. */
ditango_status ditango_selftest_bounded_wait(int64_t limit_ns, int32_t *dev_status,
                                             ditango_stream stream);

#ifdef __cplusplus
}
#endif
#endif /* DITANGO_H */
