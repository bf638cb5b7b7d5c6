"""Helpers of the GPU parity tests: upload the seeded inputs, run the C-ABI
pipeline, and compare sampled outputs with the oracle in fp64."""
from __future__ import annotations

import numpy as np

from oracle import groups as OG
from oracle import masks as OM
from oracle import step as OS
from oracle.plan import PLAN_FRESH
from workloads import inputs

# spec tolerance against fp64 for bf16 inputs with fp32 accumulation
MAX_ABS = 2e-2
MEAN_ABS = 2e-3


def to_dev(bits: np.ndarray):
    import torch
    t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
    return t.cuda()


def upload(w, prev=False):
    import torch
    Q = to_dev(inputs.full(w, "q"))
    K = to_dev(inputs.full(w, "k", prev=prev))
    V = to_dev(inputs.full(w, "v", prev=prev))
    torch.cuda.synchronize()
    return Q, K, V


def upload_prev(w):
    K = to_dev(inputs.full(w, "k", prev=True))
    V = to_dev(inputs.full(w, "v", prev=True))
    return K, V


def assert_close(got, want, what, max_abs=MAX_ABS, mean_abs=MEAN_ABS):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    fin = np.isfinite(want)
    assert (np.isfinite(got) == fin).all(), f"{what}: finiteness differs"
    err = np.abs(got[fin] - want[fin]) if fin.any() else np.zeros(1)
    assert err.max() <= max_abs and err.mean() <= mean_abs, \
        f"{what}: max abs {err.max():.3e} mean abs {err.mean():.3e}"
    return float(err.max()), float(err.mean())


def slabs(w, b, h, with_prev=True):
    q = inputs.slab_f64(w, "q", b, h)
    k = inputs.slab_f64(w, "k", b, h)
    v = inputs.slab_f64(w, "v", b, h)
    if not with_prev or not w.reuses:
        return q, k, v, k, v
    return q, k, v, inputs.slab_f64(w, "k", b, h, prev=True), inputs.slab_f64(w, "v", b, h, prev=True)


def oracle_rows(w, plan, b, h, i, rows):
    """Final (O, lse) and per-pair states of the given rows of partition i
    (states only without KV groups)."""
    q, k, v, kp, vp = slabs(w, b, h)
    if w.grouped:
        O, lse = OG.step_rows_units(q, k, v, kp, vp, plan, w.part_off(), w.group_off(), i, rows,
                                    w.frame_off(), w.frame_mask())
        return O, lse, None
    return OS.step_rows(q, k, v, kp, vp, plan, w.part_off(), i, rows,
                        w.frame_off(), w.frame_mask())


def unit_masks(w):
    """(active, band) masks over the plan's columns (KV partitions or groups)."""
    A = OM.pair_mask(w.part_off(), w.frame_off(), w.frame_mask())
    go = w.group_off()
    return OG.unit_mask(A, go), OG.unit_band(A, go, w.band_k)


def check_plan_valid(w, plan):
    """Plan properties that hold for any w: skip exactly the masked units,
    band fresh, fresh count = max(|band|, floor(budget*|A|+1e-9))."""
    from oracle.plan import budget_target
    A, band = unit_masks(w)
    plan = np.asarray(plan).reshape(A.shape)
    assert ((plan != 0) == A).all()
    if w.anchor:
        assert (plan[A] == PLAN_FRESH).all()
        return
    assert (plan[band] == PLAN_FRESH).all()
    assert int((plan == PLAN_FRESH).sum()) == budget_target(band.sum(), A.sum(), w.budget)
