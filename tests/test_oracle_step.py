"""Pins for the composed reuse step on the tiny workload.

* a cache built from unchanged K/V makes a reuse step equal the all-fresh
  step (DiTango: reuse is exact when the state has not drifted);
* an all-fresh step over all partitions equals unpartitioned attention, and
  with the frame-tile mask equals dense attention with -inf logits on the
  dropped frame tiles (torch's library attention, fp64);
* a reuse step sits between: its rows differ from fresh only through the
  reused pairs (reported, not gated: the pages print no error values).
"""
import numpy as np
import torch

from oracle import masks, step
from oracle.plan import PLAN_FRESH, PLAN_REUSE, mass_scores, select
from workloads import configs, inputs


def slabs(w, b, h):
    q = inputs.slab_f64(w, "q", b, h)
    k = inputs.slab_f64(w, "k", b, h)
    v = inputs.slab_f64(w, "v", b, h)
    return q, k, v


def sdpa(q, k, v, mask=None):
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x))[None, None]
    m = None if mask is None else torch.from_numpy(mask)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=m)[0, 0].numpy()


def test_inputs_are_bf16_and_reproducible():
    w = configs.TINY
    a = inputs.slab(w, "q", 0, 1)
    b = inputs.slab(w, "q", 0, 1)
    assert (a == b).all() and a.dtype == np.uint16
    f = inputs.bf16_to_f32(a)
    assert (inputs.bf16_bits(f) == a).all()          # bf16 values are fixed points
    assert abs(f.mean()) < 0.05 and abs(f.std() - 1) < 0.05
    kp = inputs.slab_f64(w, "k", 0, 1, prev=True)
    k = inputs.slab_f64(w, "k", 0, 1)
    assert 0.04 < np.std(kp - k) < 0.06


def test_zero_drift_reuse_equals_fresh():
    w = configs.scaled(configs.TINY, drift_sigma=0.0)
    q, k, v = slabs(w, 0, 0)
    kp = inputs.slab_f64(w, "k", 0, 0, prev=True)
    vp = inputs.slab_f64(w, "v", 0, 0, prev=True)
    assert (kp == k).all() and (vp == v).all()
    A = masks.pair_mask(w.part_off())
    plan, _ = select(np.random.default_rng(0).random((w.P, w.P)), A, w.band_k, w.budget)
    assert (plan == PLAN_REUSE).any()
    allfresh = np.where(A, PLAN_FRESH, 0).astype(np.int8)
    for i in range(w.P):
        rows = np.arange(w.part_off()[i], w.part_off()[i + 1])
        O1, l1, _ = step.step_rows(q, k, v, kp, vp, plan, w.part_off(), i, rows)
        O2, l2, _ = step.step_rows(q, k, v, kp, vp, allfresh, w.part_off(), i, rows)
        np.testing.assert_allclose(O1, O2, atol=1e-12)
        np.testing.assert_allclose(l1, l2, atol=1e-12)


def test_all_fresh_equals_unpartitioned_attention():
    w = configs.TINY
    q, k, v = slabs(w, 0, 1)
    A = masks.pair_mask(w.part_off())
    plan = np.where(A, PLAN_FRESH, 0).astype(np.int8)
    ref = sdpa(q, k, v)
    for i in range(w.P):
        rows = np.arange(w.part_off()[i], w.part_off()[i + 1])
        O, _, _ = step.step_rows(q, k, v, k, v, plan, w.part_off(), i, rows)
        np.testing.assert_allclose(O, ref[rows], atol=1e-12)


def test_masked_all_fresh_equals_dense_masked_attention():
    w = configs.scaled(configs.FRAME_TILE, N=8 * 48, H=1, d=32, name="frame_tile_small")
    q, k, v = slabs(w, 0, 0)
    po, fo, fm = w.part_off(), w.frame_off(), w.frame_mask()
    A = masks.pair_mask(po, fo, fm)
    plan = np.where(A, PLAN_FRESH, 0).astype(np.int8)
    allowed = masks.token_allowed(np.arange(w.N), np.arange(w.N), fo, fm)
    ref = sdpa(q, k, v, allowed)
    for i in range(w.P):
        rows = np.arange(po[i], po[i + 1])
        O, _, st = step.step_rows(q, k, v, k, v, plan, po, i, rows, fo, fm)
        assert len(st) == int(A[i].sum()) <= 4
        np.testing.assert_allclose(O, ref[rows], atol=1e-12)


def test_tiny_reuse_step_plan_and_drift_report():
    w = configs.TINY
    po = w.part_off()
    A = masks.pair_mask(po)
    lse = np.stack([
        step.cache_lse_for_slab(*[inputs.slab_f64(w, "q", 0, h)],
                                inputs.slab_f64(w, "k", 0, h, prev=True),
                                inputs.slab_f64(w, "v", 0, h, prev=True), A, po)
        for h in range(w.H)], axis=1)                       # [slots, BH, Lp]
    wts = mass_scores(lse, A, po)
    np.testing.assert_allclose(wts.sum(1), 1.0, atol=1e-12)
    plan, fl = select(wts, A, w.band_k, w.budget)
    assert (plan == PLAN_FRESH).sum() == 12 and (plan == PLAN_REUSE).sum() == 4
    # near partitions hold more mass than far ones on average (locality)
    ii, jj = np.indices((w.P, w.P))
    assert wts[np.abs(ii - jj) == 0].mean() > 0
    # the reused rows drift from fresh by a small amount (reported only)
    q, k, v = slabs(w, 0, 0)
    kp = inputs.slab_f64(w, "k", 0, 0, prev=True)
    vp = inputs.slab_f64(w, "v", 0, 0, prev=True)
    allfresh = np.where(A, PLAN_FRESH, 0).astype(np.int8)
    rows = np.arange(po[0], po[1])
    O1, _, _ = step.step_rows(q, k, v, kp, vp, plan, po, 0, rows)
    O2, _, _ = step.step_rows(q, k, v, kp, vp, allfresh, po, 0, rows)
    drift = np.abs(O1 - O2).max()
    assert 0 < drift < 0.05
