"""The importance w from the merge's mass partials (DiTango, "Anchor Steps":
w is refreshed from the states just composed).

After a merge that emitted its mass partials, the plan made from them must
be bit-identical -- plan, fresh list, counts and float32 scores -- to the
plan that reads the same cache through ditango_plan, and the scores must
equal the oracle's fp64 mass scores of the cached lse within 1e-5 relative.
Checked after the cache-building anchor step and after a reuse step (the
cache then holds this step's fresh states and older reused ones), at full
size and on small cases, with pairs and with KV groups, fp32 and bf16
state caches."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import sparse_state_reuse_b200 as dt
from oracle.plan import mass_scores
from workloads import configs

import gpu_common as G

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)


def plan_both_ways(w, pa):
    """(plan, fresh list, counts, scores) from the merge's partials and from
    the cache, each as host arrays."""
    n = max(pa.n_slots, 1)
    outs = []
    for from_mass in (True, False):
        plan = torch.full((pa.P * pa.G,), -7, dtype=torch.int8, device="cuda")
        fl = torch.full((n,), -7, dtype=torch.int32, device="cuda")
        counts = torch.full((2,), -7, dtype=torch.int32, device="cuda")
        score = torch.full((pa.P * pa.G,), -7.0, dtype=torch.float32, device="cuda")
        if from_mass:
            dt.ditango_plan_from_mass(pa.geom, pa.workspace, pa.ws_bytes, pa.valid, w.band_k,
                                      w.budget, plan, fl, counts, score)
        else:
            ws = torch.empty(pa.ws_bytes, dtype=torch.uint8, device="cuda")
            dt.ditango_plan(pa.geom, pa.state_lse, pa.valid, w.band_k, w.budget, 0, plan, fl,
                            counts, score, ws, pa.ws_bytes)
        torch.cuda.synchronize()
        k = int(counts[0])
        outs.append((plan.cpu().numpy(), fl.cpu().numpy()[:k], counts.cpu().numpy(),
                     score.cpu().numpy()))
    return outs


def check_equal_and_oracle(w, pa, what):
    (p1, f1, c1, s1), (p2, f2, c2, s2) = plan_both_ways(w, pa)
    assert (p1 == p2).all(), f"{what}: plans differ"
    assert (c1 == c2).all() and (f1 == f2).all(), f"{what}: fresh lists differ"
    assert (s1.view(np.uint32) == s2.view(np.uint32)).all(), f"{what}: scores differ in bits"
    A, _ = G.unit_masks(w)
    lse = pa.state_lse.cpu().numpy()
    w_o = mass_scores(lse, A, w.part_off(), valid=pa.valid.cpu().numpy().astype(bool))
    np.testing.assert_allclose(s1.reshape(A.shape)[A], w_o[A], rtol=1e-5, atol=0,
                               err_msg=f"{what}: scores against the oracle")


CASES = [(configs.TINY, False), (configs.DITANGO_REUSE, False), (configs.DITANGO_REUSE, True),
         (configs.LONG_VIDEO, False), (configs.DITANGO_GROUPS, False),
         (configs.scaled(configs.LONG_VIDEO, N=24 * 300, H=3, name="long_video_small"), True)]


@pytest.mark.parametrize("w,sb", CASES, ids=["tiny", "reuse_p32", "reuse_p32_bf16", "long_video",
                                            "groups_p32_g4", "long_video_small_bf16"])
def test_plan_from_merge_mass_equals_plan_from_cache(w, sb):
    Q, K, V = G.upload(w)
    Kp, Vp = G.upload_prev(w)
    pa = dt.PartitionedAttention(w.B, w.H, w.N, w.d, w.part_off(), w.frame_off(), w.frame_mask(),
                                 state_bf16=sb, group_off=w.group_off() if w.grouped else None)
    out = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.bfloat16, device="cuda")
    # anchor step on the previous K/V: every active unit fresh, then merged
    pa.step(Q, Kp, Vp, out, anchor=True)
    del Kp, Vp
    torch.cuda.synchronize()
    assert pa.mass_from_merge
    check_equal_and_oracle(w, pa, "after the anchor step")
    # a reuse step: its plan comes from the anchor merge's partials
    pa.step(Q, K, V, out, band_k=w.band_k, budget=w.budget)
    torch.cuda.synchronize()
    assert pa.status.item() == 0
    check_equal_and_oracle(w, pa, "after a reuse step")


def test_stale_partials_are_not_used_after_a_partial_call():
    """An attention call without a merge changes the cache: the next plan must
    read the cache, not the partials of the merge before it."""
    w = configs.TINY
    Q, K, V = G.upload(w)
    pa = dt.PartitionedAttention(w.B, w.H, w.N, w.d, w.part_off())
    out = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.float32, device="cuda")
    pa.step(Q, K, V, out, anchor=True)
    assert pa.mass_from_merge
    pa.plan_step(anchor=True)
    pa.partial(Q, K, V)
    assert not pa.mass_from_merge
