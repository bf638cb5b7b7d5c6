"""Full-size workloads on the GPU, in the launch configuration the benchmark
times, checked against the oracle on sampled rows (head/tail rows of the
first, a middle and the last partition, including ragged tile tails), plus
the plan kernel at full size on a seeded synthetic cache."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import sparse_state_reuse_b200 as dt
from oracle import groups as OG
from oracle import masks as OM
from oracle.plan import PLAN_FRESH, PLAN_REUSE, mass_scores, select
from workloads import configs, inputs

import gpu_common as G

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)


def sample_rows(w, i, n=24):
    lo, hi = w.part_off()[i], w.part_off()[i + 1]
    L = hi - lo
    picks = list(range(0, min(n, L))) + list(range(max(L - n, 0), L))
    mid = L // 2
    picks += list(range(mid - 4, mid + 4)) + [min(127, L - 1), min(128, L - 1), min(255, L - 1), min(256, L - 1)]
    return lo + np.unique(np.clip(picks, 0, L - 1))


def run_workload(w, out_dtype=torch.float32, state_bf16=False):
    """The benchmark's step on the full-size workload.  Returns the
    PartitionedAttention, the output, its lse and, for a reuse workload, a
    host copy of the cache (lse, valid bits) the plan was computed from."""
    Q, K, V = G.upload(w)
    pa = dt.PartitionedAttention(w.B, w.H, w.N, w.d, w.part_off(), w.frame_off(), w.frame_mask(),
                                 state_bf16=state_bf16,
                                 group_off=w.group_off() if w.grouped else None)
    if w.reuses:
        Kp, Vp = G.upload_prev(w)
        pa.plan_step(anchor=True)
        pa.partial(Q, Kp, Vp)
        del Kp, Vp
    out = torch.empty((w.B, w.H, w.N, w.d), dtype=out_dtype, device="cuda")
    out_lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device="cuda")
    pa.check_inputs(Q, K, V, out, out_lse)
    pa.plan_step(w.band_k, w.budget, w.anchor)
    snap = None
    if w.reuses:
        torch.cuda.synchronize()
        snap = (pa.state_lse.cpu().numpy(), pa.valid.cpu().numpy().astype(bool))
    pa.partial(Q, K, V)
    pa.merge(out, out_lse)
    torch.cuda.synchronize()
    assert pa.status.item() == 0
    return pa, out, out_lse, snap


def check_plan_hard_gate(w, pa, snap):
    """The plan on the workload's real cache (the anchor step's states on the
    previous K/V):
      * the oracle's selection run on the GPU's own float32 scores equals
        the GPU plan and fresh list bit for bit;
      * the GPU scores equal the oracle's fp64 mass scores of the same cached
        lse within 1e-5 relative;
      * the oracle's selection on its own fp64 scores equals the GPU plan,
        except units within 1e-5 relative of the cut (listed; none expected).
    Returns the relative margin at the cut (None when nothing is ranked)."""
    lse, valid = snap
    A, band = G.unit_masks(w)
    C = A.shape[1]
    plan = pa.plan.cpu().numpy().reshape(w.P, C)
    n_fresh = int(pa.counts[0].item())
    fl = pa.fresh_list.cpu().numpy()[:n_fresh]
    score = pa.score.cpu().numpy().reshape(w.P, C)
    valid_pc = np.ones((w.P, C), dtype=bool)
    valid_pc[A] = valid
    plan_s, fl_s = select(score.astype(np.float64), A, w.band_k, w.budget, valid=valid_pc, band=band)
    assert (plan_s == plan).all(), "selection on the GPU's scores differs from the GPU plan"
    assert (fl_s == fl).all(), "fresh list differs"
    w_o = mass_scores(lse, A, w.part_off(), valid=valid)
    np.testing.assert_allclose(score[A], w_o[A], rtol=1e-5, atol=0)
    plan_o, _ = select(w_o, A, w.band_k, w.budget, valid=valid_pc, band=band)
    cand = A & ~band & valid_pc
    sel = cand & (plan_o == PLAN_FRESH)
    rest = cand & (plan_o == PLAN_REUSE)
    if not sel.any() or not rest.any():
        assert (plan_o == plan).all()
        return None
    cut_in, cut_out = w_o[sel].min(), w_o[rest].max()
    margin = (cut_in - cut_out) / cut_in
    near = [(int(i), int(c)) for i, c in zip(*np.nonzero(cand))
            if abs(w_o[i, c] - cut_in) <= 1e-5 * cut_in]
    print(f"{w.name}: {int(sel.sum())} units chosen by mass, relative margin at the cut "
          f"{margin:.3e}, units within 1e-5 of the cut (the cut unit included): {near}")
    diff = plan_o != plan
    for i, c in zip(*np.nonzero(diff)):
        assert abs(w_o[i, c] - cut_in) <= 1e-5 * cut_in, (i, c, w_o[i, c], cut_in)
    return margin


def check_cached_states(w, pa, states, b, h, i, rows):
    """Every active pair's state of these rows as the cache holds it after the
    step -- this step's fresh states and the reused ones -- against the
    oracle's state of the same pair (current K/V when fresh, previous K/V
    when reused).  A wrong state of small weight can hide in the merged
    output; here each is compared on its own."""
    slot = OM.slot_table(OM.pair_mask(w.part_off(), w.frame_off(), w.frame_mask()))
    bh = b * w.H + h
    loc = torch.as_tensor(rows - w.part_off()[i], device="cuda")
    for j, (Oj, lj, code) in states.items():
        s = int(slot[i, j])
        got_O = pa.state_O[s, bh].index_select(0, loc).float().cpu().numpy()
        got_l = pa.state_lse[s, bh].index_select(0, loc).cpu().numpy()
        kind = "fresh" if code == PLAN_FRESH else "reused"
        G.assert_close(got_O, Oj, f"{w.name} cached O of {kind} pair {(i, j)} bh{bh}")
        G.assert_close(got_l, lj, f"{w.name} cached lse of {kind} pair {(i, j)} bh{bh}")


@pytest.mark.parametrize("w,sb", [(configs.FRAME_TILE, False), (configs.DITANGO_REUSE, False),
                                  (configs.LONG_VIDEO, False), (configs.DENSE, False),
                                  (configs.DITANGO_REUSE, True), (configs.LONG_VIDEO, True),
                                  (configs.DITANGO_GROUPS, False)],
                         ids=["frame_tile", "reuse_p32", "long_video", "dense",
                              "reuse_p32_bf16_cache", "long_video_bf16_cache", "groups_p32_g4"])
def test_full_size_sampled_rows(w, sb):
    pa, out, out_lse, snap = run_workload(w, state_bf16=sb)
    plan = pa.plan.cpu().numpy().reshape(w.P, w.G)
    G.check_plan_valid(w, plan)
    counts = pa.counts.cpu().numpy()
    assert counts[0] == int((plan == PLAN_FRESH).sum())
    if snap is not None:
        check_plan_hard_gate(w, pa, snap)
    bhs = sorted({0, w.BH - 1, w.BH // 2})
    parts = sorted({0, w.P // 2, w.P - 1})
    for bh in bhs:
        b, h = divmod(bh, w.H)
        for i in parts:
            rows = sample_rows(w, i)
            Oo, lo, states = G.oracle_rows(w, plan, b, h, i, rows)
            rt = torch.as_tensor(rows, device="cuda")
            G.assert_close(out[b, h].index_select(0, rt).cpu().numpy(), Oo, f"{w.name} out bh{bh} p{i}")
            G.assert_close(out_lse[b, h].index_select(0, rt).cpu().numpy(), lo, f"{w.name} lse bh{bh} p{i}")
            if states is not None:
                check_cached_states(w, pa, states, b, h, i, rows)
    if w.anchor and w.F == 0:
        # all fresh, unmasked: the merged output is unpartitioned attention
        from oracle.attention import dense_attention
        q, k, v, _, _ = G.slabs(w, 0, 0, with_prev=False)
        rows = sample_rows(w, w.P - 1)
        Od, ld = dense_attention(q[rows], k, v)
        G.assert_close(out[0, 0].index_select(0, torch.as_tensor(rows, device="cuda")).cpu().numpy(), Od,
                       "dense equality")


@pytest.mark.parametrize("w,invalid", [(configs.DITANGO_REUSE, ()), (configs.LONG_VIDEO, ()),
                                       (configs.DITANGO_REUSE, (5, 77, 300))],
                         ids=["reuse_p32", "long_video", "reuse_p32_invalid_slots"])
def test_plan_full_size_synthetic_cache(w, invalid):
    g = dt.Geometry(w.B, w.H, w.N, w.d, w.part_off(), w.frame_off(), w.frame_mask())
    A = OM.pair_mask(w.part_off(), w.frame_off(), w.frame_mask())
    pairs = OM.slot_pairs(A)
    lse = inputs.synthetic_cache_lse(w, len(pairs), pairs, seed=w.seed + 500)
    valid = np.ones(len(pairs), dtype=np.uint8)
    valid[list(invalid)] = 0
    lse_d = torch.from_numpy(lse).cuda()
    valid_d = torch.from_numpy(valid).cuda()
    plan = torch.zeros(w.P * w.P, dtype=torch.int8, device="cuda")
    fresh = torch.zeros(len(pairs), dtype=torch.int32, device="cuda")
    counts = torch.zeros(2, dtype=torch.int32, device="cuda")
    score = torch.zeros(w.P * w.P, dtype=torch.float32, device="cuda")
    nws = dt.ditango_plan_workspace_size(g)
    ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
    dt.ditango_plan(g, lse_d, valid_d, w.band_k, w.budget, 0, plan, fresh, counts, score, ws, nws)
    torch.cuda.synchronize()
    w_o = mass_scores(lse, A, w.part_off(), valid=valid.astype(bool))
    valid_pp = np.zeros((w.P, w.P), dtype=bool)
    valid_pp[A] = valid.astype(bool)
    valid_pp[~A] = True
    plan_o, fl_o = select(w_o, A, w.band_k, w.budget, valid=valid_pp)
    got_w = score.cpu().numpy().reshape(w.P, w.P)
    np.testing.assert_allclose(got_w, w_o, rtol=1e-5, atol=1e-9)
    got = plan.cpu().numpy().reshape(w.P, w.P)
    # ties within fp32 resolution may legitimately go either way: locate them
    cand = A & (plan_o != 0)
    diff = got != plan_o
    if diff.any():
        sel = (plan_o == PLAN_FRESH) & cand
        ii, jj = np.indices((w.P, w.P))
        band = A & (np.abs(ii - jj) <= w.band_k)
        extra = sel & ~band & valid_pp
        cut = w_o[extra].min()
        for i, j in zip(*np.nonzero(diff)):
            assert abs(w_o[i, j] - cut) <= 1e-5 * cut, (i, j, w_o[i, j], cut)
    else:
        assert (fresh.cpu().numpy()[:counts[0].item()] == fl_o).all()
    for s in invalid:
        i, j = pairs[s]
        assert got[i, j] == PLAN_FRESH
    assert counts.cpu().numpy()[0] == int((got == PLAN_FRESH).sum())


@pytest.mark.parametrize("sb", [False, True], ids=["fp32_cache", "bf16_cache"])
def test_compose_full_size_sampled_rows(sb):
    """The 32-partition cache (1024 pair states) composed into 8 groups of 4
    KV partitions on the GPU, against the oracle's group states on K/V."""
    w = configs.DITANGO_REUSE
    Q, K, V = G.upload(w)
    pa = dt.PartitionedAttention(w.B, w.H, w.N, w.d, w.part_off(), state_bf16=sb)
    pa.plan_step(anchor=True)
    pa.partial(Q, K, V)
    del Q, K, V
    go = OG.uniform_group_off(w.P, 4)
    coarse = pa.compose(go)
    torch.cuda.synchronize()
    assert pa.status.item() == 0
    assert coarse.n_slots == w.P * 8 and bool(coarse.valid.all())
    del pa
    slot = OM.slot_table(OG.unit_mask(np.ones((w.P, w.P), bool), go))
    for bh in sorted({0, w.BH - 1}):
        b, h = divmod(bh, w.H)
        q, k, v, _, _ = G.slabs(w, b, h, with_prev=False)
        for i in sorted({0, 13, w.P - 1}):
            rows = sample_rows(w, i)
            loc = rows - w.part_off()[i]
            for c in sorted({0, i // 4, 7}):
                Oo, lo = OG.unit_state(q[rows], rows, k, v, w.part_off(), go, c)
                s = int(slot[i, c])
                idx = torch.as_tensor(loc, device="cuda")
                G.assert_close(coarse.state_O[s, bh].index_select(0, idx).float().cpu().numpy(), Oo,
                               f"composed O unit {(i, c)} bh {bh}")
                G.assert_close(coarse.state_lse[s, bh].index_select(0, idx).cpu().numpy(), lo,
                               f"composed lse unit {(i, c)} bh {bh}")
