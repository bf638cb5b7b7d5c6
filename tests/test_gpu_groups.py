"""GPU parity of KV groups (DiTango, "Strategia per Gruppi", "Calcolo dello
Stato di Gruppo", "Composizione Dinamica dei Gruppi") against the fp64
oracle: group states on every row of small ragged and masked cases (a group
whose active partitions form several runs included), a grouped reuse step
with its plan compared exactly, and cache composition -- fine GPU states
merged on the GPU into coarser groups, against the oracle's group states
computed directly from K/V."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import sparse_state_reuse_b200 as dt
from oracle import groups as OG
from oracle import masks as OM
from oracle.plan import PLAN_FRESH, mass_scores, select
from workloads import configs, inputs

import gpu_common as G

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)


def tile_mask(F):
    return [[1 if (abs(f - g) <= 1 or g == 0) else 0 for g in range(F)] for f in range(F)]


RAGGED = [0, 100, 130, 300, 555, 1000]
FRAMES6 = [0, 90, 200, 330, 400, 520, 600]      # ragged frames = partitions


def case(d, part_off, seed):
    return configs.scaled(configs.TINY, N=part_off[-1], d=d, B=2, H=3, P=1, seed=seed, name=f"groups_{d}")


def all_units_partial(geom, Q, K, V, n, Lmax, d, BH, sb):
    plan = torch.zeros(geom.P * geom.G, dtype=torch.int8, device="cuda")
    fresh = torch.full((max(n, 1),), -1, dtype=torch.int32, device="cuda")
    counts = torch.zeros(2, dtype=torch.int32, device="cuda")
    dt.ditango_plan(geom, None, None, 0, 1.0, True, plan, fresh, counts)
    O = torch.full((n, BH, Lmax, d), float("nan"), dtype=torch.bfloat16 if sb else torch.float32,
                   device="cuda")
    lse = torch.full((n, BH, Lmax), float("nan"), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dt.ditango_attn_partial(geom, Q, K, V, fresh, counts, 0.0, O, lse, 0, None, st, state_bf16=sb)
    torch.cuda.synchronize()
    assert st.item() == 0
    return plan.cpu().numpy(), fresh.cpu().numpy(), counts.cpu().numpy(), O.float().cpu().numpy(), \
        lse.cpu().numpy()


@pytest.mark.parametrize("d,part_off,frames,go,sb", [
    (64, RAGGED, None, [0, 2, 3, 5], False),
    (96, RAGGED, None, [0, 5], False),                          # one group: dense attention
    (128, [0, 257, 512, 640, 1024], None, [0, 1, 3, 4], False),
    (96, [0, 130, 300, 555, 1000], ([0, 300, 1000], [[1, 0], [1, 1]]), [0, 2, 4], False),
    (64, FRAMES6, (FRAMES6, tile_mask(6)), [0, 6], False),      # rows 3..5: runs {0} and {f-1..f+1}
    (96, FRAMES6, (FRAMES6, tile_mask(6)), [0, 1, 4, 6], False),
    (128, FRAMES6, (FRAMES6, tile_mask(6)), [0, 3, 6], True),
    (64, RAGGED, None, [0, 2, 3, 5], True),
])
def test_unit_states_every_row(d, part_off, frames, go, sb):
    w = case(d, part_off, 300 + d)
    fo, fm = frames if frames else (None, None)
    geom = dt.Geometry(w.B, w.H, w.N, w.d, part_off, fo, fm, group_off=go)
    Au = OG.unit_mask(OM.pair_mask(part_off, fo, fm), go)
    n, Lmax = int(Au.sum()), int(max(np.diff(part_off)))
    Q, K, V = G.upload(w)
    plan, fresh, counts, O, lse = all_units_partial(geom, Q, K, V, n, Lmax, w.d, w.BH, sb)
    P, Gc = Au.shape
    assert counts.tolist() == [n, 0]
    assert (fresh[:n] == np.nonzero(Au.ravel())[0]).all()
    assert (plan.reshape(P, Gc) == np.where(Au, 1, 0)).all()
    for bh in range(w.BH):
        b, h = divmod(bh, w.H)
        q, k, v, _, _ = G.slabs(w, b, h, with_prev=False)
        for f, u in enumerate(fresh[:n]):
            i, c = divmod(int(u), Gc)
            rows = np.arange(part_off[i], part_off[i + 1])
            Oo, lo = OG.unit_state(q[rows], rows, k, v, part_off, go, c, fo, fm)
            G.assert_close(O[f, bh, :rows.size], Oo, f"O unit {(i, c)} bh {bh}")
            G.assert_close(lse[f, bh, :rows.size], lo, f"lse unit {(i, c)} bh {bh}")


GROUPED_TINY = configs.scaled(configs.TINY, N=2048, P=8, group_size=2, band_k=1, budget=0.5,
                              seed=11, drift_seed=111, name="tiny_groups_p8_g2")


def oracle_unit_cache_lse(w):
    po, go = w.part_off(), w.group_off()
    Au, _ = G.unit_masks(w)
    per = []
    for bh in range(w.BH):
        b, h = divmod(bh, w.H)
        _, l = OG.unit_cache(inputs.slab_f64(w, "q", b, h), inputs.slab_f64(w, "k", b, h, prev=True),
                             inputs.slab_f64(w, "v", b, h, prev=True), Au, po, go,
                             w.frame_off(), w.frame_mask())
        per.append(l)
    return np.stack(per, axis=1), Au


@pytest.mark.parametrize("sb", [False, True], ids=["fp32_cache", "bf16_cache"])
def test_grouped_reuse_step_plan_and_output(sb):
    w = GROUPED_TINY
    assert w.G == 4
    Q, K, V = G.upload(w)
    Kp, Vp = G.upload_prev(w)
    pa = dt.PartitionedAttention(w.B, w.H, w.N, w.d, w.part_off(), state_bf16=sb, group_off=w.group_off())
    pa.plan_step(anchor=True)
    pa.partial(Q, Kp, Vp)
    out = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.float32, device="cuda")
    out_lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device="cuda")
    pa.step(Q, K, V, out, out_lse, band_k=w.band_k, budget=w.budget)
    torch.cuda.synchronize()
    assert pa.status.item() == 0
    lse_o, Au = oracle_unit_cache_lse(w)
    _, band = G.unit_masks(w)
    w_o = mass_scores(lse_o, Au, w.part_off())
    plan_o, fl_o = select(w_o, Au, w.band_k, w.budget, band=band)
    assert int(band.sum()) == 14 and (plan_o == PLAN_FRESH).sum() == 16
    gpu_plan = pa.plan.cpu().numpy().reshape(w.P, w.G)
    assert (gpu_plan == plan_o).all(), (gpu_plan, plan_o)
    assert pa.counts.cpu().numpy().tolist() == [16, 16]
    assert (pa.fresh_list.cpu().numpy()[:16] == fl_o).all()
    np.testing.assert_allclose(pa.score.cpu().numpy().reshape(w.P, w.G), w_o, rtol=1e-4, atol=1e-7)
    o, ol = out.cpu().numpy(), out_lse.cpu().numpy()
    for bh in range(w.BH):
        b, h = divmod(bh, w.H)
        for i in range(w.P):
            rows = np.arange(w.part_off()[i], w.part_off()[i + 1])
            Oo, lo, _ = G.oracle_rows(w, plan_o, b, h, i, rows)
            G.assert_close(o[b, h, rows], Oo, f"out bh {bh} part {i}")
            G.assert_close(ol[b, h, rows], lo, f"out lse bh {bh} part {i}")


@pytest.mark.parametrize("part_off,frames", [(RAGGED, None), (FRAMES6, (FRAMES6, tile_mask(6)))],
                         ids=["ragged", "frame_tile"])
@pytest.mark.parametrize("sb", [False, True], ids=["fp32", "bf16"])
def test_recursive_composition_matches_oracle_group_states(part_off, frames, sb):
    """Pair states built on the GPU, composed on the GPU level by level; each
    level against the oracle's group states computed straight from K/V."""
    d = 96
    w = case(d, part_off, 500)
    fo, fm = frames if frames else (None, None)
    P = len(part_off) - 1
    Q, K, V = G.upload(w)
    pa = dt.PartitionedAttention(w.B, w.H, w.N, w.d, part_off, fo, fm, state_bf16=sb)
    pa.plan_step(anchor=True)
    pa.partial(Q, K, V)
    levels = [[0, 2, 4, P] if P > 4 else [0, 2, P], [0, 4, P] if P > 4 else [0, P], [0, P]]
    cur = pa
    A = OM.pair_mask(part_off, fo, fm)
    for go in levels:
        nxt = cur.compose(go)
        torch.cuda.synchronize()
        assert bool(nxt.valid.all())
        Au = OG.unit_mask(A, go)
        assert nxt.n_slots == int(Au.sum())
        O = nxt.state_O.float().cpu().numpy()
        lse = nxt.state_lse.cpu().numpy()
        for bh in range(w.BH):
            b, h = divmod(bh, w.H)
            q, k, v, _, _ = G.slabs(w, b, h, with_prev=False)
            Oo, lo = OG.unit_cache(q, k, v, Au, part_off, go, fo, fm, Lmax=nxt.Lmax)
            for s, (i, c) in enumerate(OM.slot_pairs(Au)):
                L = part_off[i + 1] - part_off[i]
                G.assert_close(O[s, bh, :L], Oo[s, :L], f"level {go} unit {(i, c)} bh {bh}")
                G.assert_close(lse[s, bh, :L], lo[s, :L], f"level {go} lse {(i, c)} bh {bh}")
        cur = nxt


def test_compose_marks_invalid_and_equals_fresh_group_states():
    """An unwritten fine slot makes its coarse slot invalid (and the plan then
    recomputes it); a composed cache agrees with group states computed fresh
    by the attention kernel to well within the tolerance."""
    d = 64
    w = case(d, RAGGED, 600)
    Q, K, V = G.upload(w)
    pa = dt.PartitionedAttention(w.B, w.H, w.N, w.d, RAGGED)
    pa.plan_step(anchor=True)
    pa.partial(Q, K, V)
    go = [0, 2, 5]
    direct = dt.PartitionedAttention(w.B, w.H, w.N, w.d, RAGGED, group_off=go)
    direct.plan_step(anchor=True)
    direct.partial(Q, K, V)
    comp = pa.compose(go)
    torch.cuda.synchronize()
    for s in range(comp.n_slots):
        i = [i for i in range(5) for _ in range(2)][s]
        L = RAGGED[i + 1] - RAGGED[i]
        G.assert_close(comp.state_O[s, :, :L].cpu().numpy(), direct.state_O[s, :, :L].cpu().numpy(),
                       f"slot {s}", max_abs=1e-2, mean_abs=1e-3)
        G.assert_close(comp.state_lse[s, :, :L].cpu().numpy(), direct.state_lse[s, :, :L].cpu().numpy(),
                       f"lse slot {s}", max_abs=1e-2, mean_abs=1e-3)
    pa.valid[int(OM.slot_table(np.ones((5, 5), bool))[0, 4])] = 0
    comp2 = pa.compose(go)
    torch.cuda.synchronize()
    v = comp2.valid.cpu().numpy()
    assert v.tolist() == [1, 0, 1, 1, 1, 1, 1, 1, 1, 1]     # unit (0, {2,3,4}) only
    # a grouped step on that cache recomputes the invalid unit although it is
    # outside the band and the budget
    out = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.float32, device="cuda")
    comp2.step(Q, K, V, out, band_k=0, budget=0.0)
    torch.cuda.synchronize()
    plan = comp2.plan.cpu().numpy().reshape(5, 2)
    assert plan[0, 1] == PLAN_FRESH
    assert (plan == PLAN_FRESH).sum() == 6
