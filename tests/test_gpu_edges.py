"""Edge cases of the CUDA path against the fp64 oracle: the maximum number of
partitions (P = 64) with ragged lengths down to one token, a single
partition (P = 1), one KV group spanning every partition under the
frame-tile mask (a unit of several runs), and an attention call with no
fresh unit (a no-op that leaves the cache alone)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import sparse_state_reuse_b200 as dt
from oracle import groups as OG
from oracle import masks as OM
from oracle import step as OS
from workloads import configs

import gpu_common as G

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)


def case(N, d, seed):
    return configs.scaled(configs.TINY, N=N, d=d, B=1, H=2, P=1, seed=seed, name=f"edge_{N}_{d}")


def all_fresh_states(w, part_off, fo=None, fm=None, go=None):
    geom = dt.Geometry(w.B, w.H, w.N, w.d, part_off, fo, fm, group_off=go)
    A = OM.pair_mask(part_off, fo, fm)
    Au = OG.unit_mask(A, go) if go is not None else A
    n, Lmax = int(Au.sum()), int(max(np.diff(part_off)))
    Q, K, V = G.upload(w)
    Gc = Au.shape[1]
    plan = torch.zeros((len(part_off) - 1) * Gc, dtype=torch.int8, device="cuda")
    fresh = torch.zeros(n, dtype=torch.int32, device="cuda")
    counts = torch.zeros(2, dtype=torch.int32, device="cuda")
    dt.ditango_plan(geom, None, None, 0, 1.0, True, plan, fresh, counts)
    O = torch.full((n, w.BH, Lmax, w.d), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((n, w.BH, Lmax), float("nan"), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dt.ditango_attn_partial(geom, Q, K, V, fresh, counts, 0.0, O, lse, 0, None, st)
    out = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.float32, device="cuda")
    out_lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device="cuda")
    dt.ditango_merge(geom, plan, O, lse, None, None, None, 0, out, 1, out_lse=out_lse)
    torch.cuda.synchronize()
    assert st.item() == 0
    return Au, fresh.cpu().numpy()[:n], O.cpu().numpy(), lse.cpu().numpy(), out.cpu().numpy(), out_lse.cpu().numpy()


def test_sixty_four_ragged_partitions_down_to_one_token():
    rng = np.random.default_rng(9)
    lens = rng.integers(1, 40, size=64)
    lens[[0, 17, 63]] = 1
    part_off = [0] + np.cumsum(lens).tolist()
    w = case(part_off[-1], 64, 901)
    Au, fresh, O, lse, out, out_lse = all_fresh_states(w, part_off)
    assert len(fresh) == 64 * 64
    for bh in range(w.BH):
        q, k, v, _, _ = G.slabs(w, 0, bh, with_prev=False)
        for f in (0, 1, 63, 64 * 17 + 5, 64 * 63, 64 * 64 - 1):
            i, j = divmod(int(fresh[f]), 64)
            rows = np.arange(part_off[i], part_off[i + 1])
            Oo, lo = OS.pair_state(q[rows], rows, k, v, part_off, j)
            G.assert_close(O[f, bh, :rows.size], Oo, f"O pair {(i, j)}")
            G.assert_close(lse[f, bh, :rows.size], lo, f"lse pair {(i, j)}")
        from oracle.attention import dense_attention
        Od, ld = dense_attention(q, k, v)
        G.assert_close(out[0, bh], Od, "64-way merge = dense")
        G.assert_close(out_lse[0, bh], ld, "64-way merge lse")


def test_single_partition_is_dense_attention():
    w = case(1000, 128, 902)
    Au, fresh, O, lse, out, out_lse = all_fresh_states(w, [0, 1000])
    from oracle.attention import dense_attention
    for bh in range(w.BH):
        q, k, v, _, _ = G.slabs(w, 0, bh, with_prev=False)
        Od, ld = dense_attention(q, k, v)
        G.assert_close(out[0, bh], Od, "P = 1")
        G.assert_close(out_lse[0, bh], ld, "P = 1 lse")


def test_one_group_over_every_partition_with_the_frame_mask():
    """Every row's unit holds frame 0 and its neighbours: up to two runs of
    partitions with a gap between them."""
    fo = [0, 70, 200, 260, 400, 530, 600, 700]
    F = len(fo) - 1
    fm = [[1 if (abs(f - g) <= 1 or g == 0) else 0 for g in range(F)] for f in range(F)]
    w = case(fo[-1], 96, 903)
    Au, fresh, O, lse, out, out_lse = all_fresh_states(w, fo, fo, fm, go=[0, F])
    assert Au.shape == (F, 1) and len(fresh) == F
    for bh in range(w.BH):
        q, k, v, _, _ = G.slabs(w, 0, bh, with_prev=False)
        for f, u in enumerate(fresh):
            i = int(u)
            rows = np.arange(fo[i], fo[i + 1])
            Oo, lo = OG.unit_state(q[rows], rows, k, v, fo, [0, F], 0, fo, fm)
            G.assert_close(O[f, bh, :rows.size], Oo, f"unit row {i}")
            G.assert_close(out[0, bh, rows], Oo, f"merged row {i}")


def test_attention_with_no_fresh_unit_is_a_no_op():
    w = configs.TINY
    Q, K, V = G.upload(w)
    pa = dt.PartitionedAttention(w.B, w.H, w.N, w.d, w.part_off())
    pa.plan_step(anchor=True)
    pa.partial(Q, K, V)
    torch.cuda.synchronize()
    before = (pa.state_O.clone(), pa.state_lse.clone())
    pa.counts.zero_()
    pa.partial(Q, K, V)
    torch.cuda.synchronize()
    assert pa.status.item() == 0
    assert torch.equal(pa.state_O, before[0]) and torch.equal(pa.state_lse, before[1])


def test_mismatched_tensors_are_refused_before_any_launch():
    w = configs.TINY
    Q, K, V = G.upload(w)
    pa = dt.PartitionedAttention(w.B, w.H, w.N, w.d, w.part_off())
    out = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.float32, device="cuda")
    with pytest.raises(ValueError, match="shape"):
        pa.step(Q[:, :, : w.N // 2], K, V, out, anchor=True)
    with pytest.raises(TypeError, match="dtype"):
        pa.step(Q.float(), K, V, out, anchor=True)
    with pytest.raises(ValueError, match="CUDA device"):
        pa.step(Q, K.cpu(), V, out, anchor=True)
    with pytest.raises(TypeError, match="dtype"):
        pa.merge(out.half())
    torch.cuda.synchronize()
    assert pa.status.item() == 0


@pytest.mark.parametrize("band_k,budget", [(0, 0.0), (0, 1.0), (3, 0.0), (0, 0.3125)],
                         ids=["diagonal_only", "budget_all", "band_covers_all", "one_unit_by_mass"])
def test_degenerate_budgets_and_bands(band_k, budget):
    """Budget 0 (only the band is recomputed), budget 1 (everything is), a
    band covering every pair, and a budget one unit above the band: the
    plan equals the oracle's selection on its own fp64 scores of the GPU's
    cache, and the output equals the oracle's composition of that plan."""
    from oracle.plan import mass_scores, select, budget_target
    w = configs.TINY
    Q, K, V = G.upload(w)
    Kp, Vp = G.upload_prev(w)
    pa = dt.PartitionedAttention(w.B, w.H, w.N, w.d, w.part_off())
    pa.plan_step(anchor=True)
    pa.partial(Q, Kp, Vp)
    torch.cuda.synchronize()
    lse = pa.state_lse.cpu().numpy()
    out = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.float32, device="cuda")
    pa.step(Q, K, V, out, band_k=band_k, budget=budget)
    torch.cuda.synchronize()
    assert pa.status.item() == 0
    A = OM.pair_mask(w.part_off())
    plan = pa.plan.cpu().numpy().reshape(w.P, w.P)
    score = pa.score.cpu().numpy().reshape(w.P, w.P)
    plan_s, _ = select(score.astype(np.float64), A, band_k, budget)     # the selection rule, exactly
    assert (plan == plan_s).all(), (plan, plan_s)
    w_o = mass_scores(lse, A, w.part_off())
    np.testing.assert_allclose(score, w_o, rtol=1e-5, atol=1e-9)
    plan_o, _ = select(w_o, A, band_k, budget)                            # and on fp64 scores
    for i, j in zip(*np.nonzero(plan_o != plan)):                          # only ties at the cut
        cut = w_o[(plan_o == 1) & (np.abs(np.subtract.outer(np.arange(w.P), np.arange(w.P))) > band_k)].min()
        assert abs(w_o[i, j] - cut) <= 1e-5 * cut
    n_band = int((np.abs(np.subtract.outer(np.arange(w.P), np.arange(w.P))) <= band_k).sum())
    assert int(pa.counts[0]) == budget_target(n_band, w.P * w.P, budget)
    o = out.cpu().numpy()
    for h in range(w.H):
        for i in range(w.P):
            rows = np.arange(w.part_off()[i], w.part_off()[i + 1])
            Oo, _, _ = G.oracle_rows(w, plan, 0, h, i, rows)
            G.assert_close(o[0, h, rows], Oo, f"out h {h} part {i}")


def test_many_heads_short_sequence():
    """B*H = 3000 slabs of 320 tokens in 3 ragged partitions: thousands of
    small work items and a merge grid of 3000 (b, h) blocks deep."""
    po = [0, 100, 130, 320]
    w = configs.scaled(configs.TINY, N=320, d=64, B=3, H=1000, P=1, seed=909, name="many_heads")
    geom_po = po
    Au, fresh, O, lse, out, out_lse = all_fresh_states(w, geom_po)
    assert len(fresh) == 9
    for bh in (0, 1, 1499, 2998, 2999):
        b, h = divmod(bh, w.H)
        q, k, v, _, _ = G.slabs(w, b, h, with_prev=False)
        from oracle.attention import dense_attention
        Od, ld = dense_attention(q, k, v)
        G.assert_close(out[b, h], Od, f"merged output bh {bh}")
        G.assert_close(out_lse[b, h], ld, f"merged lse bh {bh}")
