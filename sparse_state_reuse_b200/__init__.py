"""B200 partitioned attention with selective attention-state reuse.

The token sequence is split into P context partitions; for every (query
partition, KV partition) pair -- or, with KV groups, every (query partition,
group of adjacent KV partitions) unit -- the plan either recomputes the
attention state (output, log-sum-exp) or reuses the one cached at the
previous denoising step, and the states of each query partition are composed
by an exact log-sum-exp merge (DiTango: "Cost-Effective Parallel Diffusion
Generation with Selective Attention State Reuse").  A cache can be merged
into coarser groups without recomputation to shrink it.  An optional
frame-tile mask keeps only some frame tiles (Efficient-vDiT: "Efficient Video
Diffusion Transformers With Attention Tile").

All compute runs in libditango.so (CUDA, sm_100a) through its C ABI
(include/ditango.h); this package only marshals arguments.  PyTorch is used
for device memory and streams.
"""
from __future__ import annotations

from ._abi import (  # noqa: F401
    DitangoError, Geometry, PLAN_FRESH, PLAN_REUSE, PLAN_SKIP, LIB_PATH, EXPORTED,
    ditango_version, ditango_check_geom, ditango_num_active, ditango_state_rows,
    ditango_slot_table, ditango_plan_workspace_size, ditango_plan, ditango_attn_partial,
    ditango_merge, ditango_cache_update, ditango_set_wait_limit_ns,
    ditango_selftest_bounded_wait, ditango_plan_noalloc, ditango_cache_compose, status_string,
    ditango_plan_error, error_state, ditango_plan_from_mass, ditango_checked_build,
    ditango_check_status,
)


def check_tensor(t, name, shape, dtypes, contiguous=False):
    """Raise unless t is a tensor of one of `dtypes` with this shape, on a
    CUDA device, its last dimension contiguous (the whole tensor when
    `contiguous`).  The kernels see raw addresses and strides only, so these
    are checked here, before anything is launched."""
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: a torch.Tensor is required, got {type(t).__name__}")
    if t.dtype not in dtypes:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {' or '.join(str(d) for d in dtypes)}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if t.shape[-1] > 1 and t.stride(-1) != 1:
        raise ValueError(f"{name}: the last dimension must be contiguous")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be on a CUDA device, is on {t.device}")


class PartitionedAttention:
    """Device buffers for one geometry and the three-call step.

    The state buffer (O [slots, B*H, Lmax, d] float32, or bfloat16 with
    state_bf16=True, a compressed cache; lse float32 [slots, B*H, Lmax]) is
    the attention-state cache: a step writes its fresh states into their
    slots and the merge reads every active unit from it, so after a step the
    cache holds this step's fresh states and the reused ones.  The merge also
    leaves the next plan's mass score in the workspace, so the next plan does
    not read the cache again; code that writes the cache tensors directly
    must set mass_from_merge = False.  group_off
    (partition offsets of the KV groups) makes the units (query partition,
    KV group); None keeps one group per partition.
    """

    def __init__(self, B, H, N, d, part_off, frame_off=None, frame_mask=None,
                 device="cuda", strides=None, state_bf16=False, group_off=None):
        import torch
        self.B, self.H, self.N, self.d = B, H, N, d
        self.part_off = list(part_off)
        self.frame_off = None if frame_off is None else list(frame_off)
        self.frame_mask = frame_mask
        self.group_off = None if group_off is None else list(group_off)
        self.device = torch.device(device)
        if self.device.type != "cuda":
            raise ValueError(f"the state cache lives on a CUDA device, not {self.device}")
        self.geom = self._geometry(strides)
        self.P = self.geom.P
        self.G = self.geom.G
        self.n_slots = ditango_num_active(self.geom)
        self.Lmax = ditango_state_rows(self.geom)
        BH = B * H
        dev = self.device
        self.state_bf16 = bool(state_bf16)
        self.state_O = torch.empty((self.n_slots, BH, self.Lmax, d),
                                   dtype=torch.bfloat16 if self.state_bf16 else torch.float32,
                                   device=dev)
        self.state_lse = torch.empty((self.n_slots, BH, self.Lmax), dtype=torch.float32, device=dev)
        self.valid = torch.zeros(self.n_slots, dtype=torch.uint8, device=dev)
        self.plan = torch.zeros(self.P * self.G, dtype=torch.int8, device=dev)
        self.fresh_list = torch.zeros(max(self.n_slots, 1), dtype=torch.int32, device=dev)
        self.counts = torch.zeros(2, dtype=torch.int32, device=dev)
        self.score = torch.zeros(self.P * self.G, dtype=torch.float32, device=dev)
        self.ws_bytes = ditango_plan_workspace_size(self.geom)
        self.workspace = torch.empty(max(self.ws_bytes, 16), dtype=torch.uint8, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        # the attention kernel's work counter (each launch leaves it at zero)
        self.work_counter = torch.zeros(2, dtype=torch.int32, device=dev)
        # the workspace holds the mass partials of the last merge, and the
        # cache has not changed since: the next plan need not read the cache
        self.mass_from_merge = False

    def _geometry(self, strides):
        s = strides or (None, None, None)
        return Geometry(self.B, self.H, self.N, self.d, self.part_off, self.frame_off,
                        self.frame_mask, q_strides=s[0], k_strides=s[1], v_strides=s[2],
                        group_off=self.group_off)

    def check_inputs(self, Q, K, V, out=None, out_lse=None):
        """Shapes, dtypes and devices of a step's tensors (raises on a mismatch)."""
        import torch
        qkv = (self.B, self.H, self.N, self.d)
        for name, t in (("Q", Q), ("K", K), ("V", V)):
            check_tensor(t, name, qkv, (torch.bfloat16,))
        if out is not None:
            check_tensor(out, "out", qkv, (torch.float32, torch.bfloat16))
        if out_lse is not None:
            check_tensor(out_lse, "out_lse", (self.B, self.H, self.N), (torch.float32,),
                         contiguous=True)

    def _bind(self, Q, K, V):
        want = tuple(tuple(t.stride()[:3]) for t in (Q, K, V))
        have = (tuple(self.geom.g.q_strides), tuple(self.geom.g.k_strides), tuple(self.geom.g.v_strides))
        if want != have:
            self.geom = self._geometry(want)

    def plan_step(self, band_k=0, budget=1.0, anchor=False, stream=None):
        """The plan of the next attention call.  After a merge (which left the
        mass score of the states it composed in the workspace) the selection
        runs alone; otherwise the mass score is read from the cache."""
        if not anchor and self.mass_from_merge:
            ditango_plan_from_mass(self.geom, self.workspace, self.ws_bytes, self.valid, band_k,
                                   budget, self.plan, self.fresh_list, self.counts, self.score,
                                   stream)
        else:
            ditango_plan(self.geom, None if anchor else self.state_lse, self.valid, band_k, budget,
                         anchor, self.plan, self.fresh_list, self.counts, self.score,
                         self.workspace, self.ws_bytes, stream)
        self.mass_from_merge = False

    def partial(self, Q, K, V, scale=0.0, stream=None, drift_rows=None):
        import torch
        self.check_inputs(Q, K, V)
        if drift_rows is not None:
            check_tensor(drift_rows, "drift_rows", (self.P, self.B * self.H, self.Lmax),
                         (torch.float32,), contiguous=True)
        self._bind(Q, K, V)
        self.mass_from_merge = False
        ditango_attn_partial(self.geom, Q, K, V, self.fresh_list, self.counts, scale,
                             self.state_O, self.state_lse, 1, self.valid, self.status, stream,
                             state_bf16=self.state_bf16, drift_rows=drift_rows,
                             work_counter=self.work_counter)

    def merge(self, out, out_lse=None, stream=None):
        import torch
        qkv = (self.B, self.H, self.N, self.d)
        check_tensor(out, "out", qkv, (torch.float32, torch.bfloat16))
        if out_lse is not None:
            check_tensor(out_lse, "out_lse", (self.B, self.H, self.N), (torch.float32,),
                         contiguous=True)
        ditango_merge(self.geom, self.plan, None, None, self.state_O, self.state_lse, self.valid, 0,
                      out, out.dtype == torch.float32, tuple(out.stride()[:3]), out_lse, stream,
                      state_bf16=self.state_bf16, mass_partials=self.workspace)
        self.mass_from_merge = True

    def step(self, Q, K, V, out, out_lse=None, band_k=0, budget=1.0, anchor=False, scale=0.0,
             stream=None):
        """plan -> partial attention of the fresh units -> merge, on one stream."""
        self.check_inputs(Q, K, V, out, out_lse)
        self.plan_step(band_k, budget, anchor, stream)
        self.partial(Q, K, V, scale, stream)
        self.merge(out, out_lse, stream)

    def compose(self, group_off, stream=None):
        """A new PartitionedAttention with coarser KV groups whose cache is this
        cache's states merged group by group (no attention is recomputed).
        Every boundary of group_off must be one of this object's boundaries.
        The caller may drop this object afterwards to free the finer cache."""
        coarse = PartitionedAttention(self.B, self.H, self.N, self.d, self.part_off, self.frame_off,
                                      self.frame_mask, self.device, None, self.state_bf16,
                                      group_off)
        ditango_cache_compose(self.geom, coarse.geom, self.state_O, self.state_lse, self.valid,
                              coarse.state_O, coarse.state_lse, coarse.valid, self.state_bf16,
                              stream)
        return coarse


class ErrorPlanner:
    """Anchor-guided, error-growth planning of a PartitionedAttention's steps
    (DiTango, 1. Anchor-Guided Selection Planner).

    Step 0 and every anchor_every-th step after it are anchor steps (every
    active unit fresh).  The step after an anchor recomputes the importance w
    from the cache; the others hold it.  Between anchors each unit's
    predicted reuse error w * (age + delta_i) ranks the non-band units under
    the budget, delta_i being the local state's drift that the attention
    call of the previous step measured.  The schedule is host logic; every
    number is computed on the device.
    """

    def __init__(self, pa, band_k, budget, anchor_every):
        import torch
        if anchor_every < 1:
            raise ValueError("anchor_every must be >= 1")
        self.pa = pa
        self.band_k, self.budget, self.anchor_every = band_k, budget, anchor_every
        dev = pa.device
        self.w = torch.zeros(pa.P * pa.G, dtype=torch.float32, device=dev)
        self.age = torch.zeros(max(pa.n_slots, 1), dtype=torch.float32, device=dev)
        self.delta = torch.zeros(pa.P, dtype=torch.float32, device=dev)
        self.local_ok = torch.zeros(pa.P, dtype=torch.uint8, device=dev)
        self.drift_rows = torch.zeros((pa.P, pa.B * pa.H, pa.Lmax), dtype=torch.float32, device=dev)
        self.es = error_state(self.w, self.age, self.delta, self.local_ok, self.drift_rows)
        self.step_index = 0

    def is_anchor(self, s):
        return s % self.anchor_every == 0

    def plan(self, stream=None):
        s = self.step_index
        pa = self.pa
        ditango_plan_error(pa.geom, pa.state_lse, pa.valid, self.band_k, self.budget,
                           self.is_anchor(s), s > 0 and self.is_anchor(s - 1), self.es, pa.plan,
                           pa.fresh_list, pa.counts, pa.score, pa.workspace, pa.ws_bytes, stream)

    def step(self, Q, K, V, out, out_lse=None, scale=0.0, stream=None):
        """plan by predicted error -> attention of the fresh units (measuring the
        local drift) -> merge."""
        self.pa.check_inputs(Q, K, V, out, out_lse)    # before the plan advances the ages
        self.plan(stream)
        self.pa.partial(Q, K, V, scale, stream, drift_rows=self.drift_rows)
        self.pa.merge(out, out_lse, stream)
        self.step_index += 1
