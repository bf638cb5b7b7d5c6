"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Small cases are compared element by element (every row of every pair,
ragged partitions and tails included); the full-size workloads are run in
the launch configuration the benchmark times and compared on sampled rows.
Plans are compared exactly; floating point against fp64 within max-abs 2e-2
and mean-abs 2e-3.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import sparse_state_reuse_b200 as dt
from sparse_state_reuse_b200 import _abi
from oracle import masks as OM
from oracle.plan import PLAN_REUSE, mass_scores, select
from oracle import step as OS
from workloads import configs, inputs

import gpu_common as G

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)


def geom_of(w, part_off=None):
    return dt.Geometry(w.B, w.H, w.N, w.d, part_off or w.part_off(), w.frame_off(), w.frame_mask())


def all_pairs_partial(geom, Q, K, V, n, Lmax, d, BH, state_bf16=False):
    P = geom.P
    plan = torch.zeros(P * P, dtype=torch.int8, device="cuda")
    fresh = torch.full((max(n, 1),), -1, dtype=torch.int32, device="cuda")
    counts = torch.zeros(2, dtype=torch.int32, device="cuda")
    dt.ditango_plan(geom, None, None, 0, 1.0, True, plan, fresh, counts)
    O = torch.full((n, BH, Lmax, d), float("nan"), dtype=torch.bfloat16 if state_bf16 else torch.float32,
                   device="cuda")
    lse = torch.full((n, BH, Lmax), float("nan"), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dt.ditango_attn_partial(geom, Q, K, V, fresh, counts, 0.0, O, lse, 0, None, st, state_bf16=state_bf16)
    torch.cuda.synchronize()
    assert st.item() == 0
    return (plan.cpu().numpy(), fresh.cpu().numpy(), counts.cpu().numpy(), O.float().cpu().numpy(),
            lse.cpu().numpy())


# frame-tile mask of 5 frames: each frame attends itself, its neighbours and frame 0
TILE5 = [[1 if (abs(f - g) <= 1 or g == 0) else 0 for g in range(5)] for f in range(5)]


def test_bounded_wait_reports_timeout_and_context_survives():
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dt.ditango_selftest_bounded_wait(2_000_000, st)
    torch.cuda.synchronize()
    assert st.item() == _abi.ERR_TIMEOUT
    x = torch.arange(8, device="cuda", dtype=torch.float32)
    assert float(x.sum()) == 28.0


@pytest.mark.parametrize("d,part_off,frames,sb", [
    (64, None, None, False),                           # the tiny workload's geometry
    (64, [0, 100, 130, 300, 555, 1000], None, False),  # ragged: short and multi-tile partitions
    (96, [0, 100, 130, 300, 555, 1000], None, False),
    (128, [0, 100, 130, 300, 555, 1000], None, False),
    (96, [0, 130, 300, 555, 1000], ([0, 300, 1000], [[1, 0], [1, 1]]), False),  # frame mask
    (128, [0, 257, 512, 640, 1024], None, False),      # 256-row unit boundaries +-1
    (64, [0, 100, 130, 300, 555, 1000], None, True),   # bf16 states (compressed cache)
    (96, [0, 130, 300, 555, 1000], ([0, 300, 1000], [[1, 0], [1, 1]]), True),
    (128, [0, 257, 512, 640, 1024], None, True),
    # partitions that straddle frames: single logits masked by the frame mask
    (96, [0, 130, 400, 555, 1000], ([0, 300, 700, 1000], [[1, 1, 0], [1, 1, 1], [1, 1, 1]]), False),
    (128, [0, 250, 520, 1000], ([0, 200, 400, 600, 800, 1000], TILE5), False),
    (64, [0, 250, 520, 1000], ([0, 200, 400, 600, 800, 1000], TILE5), True),
    (64, [0, 60, 61, 190, 1000], ([0, 45, 90, 135, 180, 1000], TILE5), False),
])
def test_partial_states_every_row(d, part_off, frames, sb):
    if part_off is None:
        w = configs.TINY
        part_off = w.part_off()
    else:
        w = configs.scaled(configs.TINY, N=part_off[-1], d=d, B=2, H=3, P=1, seed=77 + d,
                           name=f"ragged_{d}")
    fo, fm = (frames if frames else (None, None))
    geom = dt.Geometry(w.B, w.H, w.N, w.d, part_off, fo, fm)
    A = OM.pair_mask(part_off, fo, fm)
    n, Lmax = int(A.sum()), max(np.diff(part_off))
    Q, K, V = G.upload(w)
    plan, fresh, counts, O, lse = all_pairs_partial(geom, Q, K, V, n, Lmax, w.d, w.BH, state_bf16=sb)
    P = len(part_off) - 1
    assert counts.tolist() == [n, 0]
    assert (fresh[:n] == np.nonzero(A.ravel())[0]).all()
    assert (plan.reshape(P, P) == np.where(A, 1, 0)).all()
    for bh in range(w.BH):
        b, h = divmod(bh, w.H)
        q, k, v, _, _ = G.slabs(w, b, h, with_prev=False)
        for f, p in enumerate(fresh[:n]):
            i, j = divmod(int(p), P)
            rows = np.arange(part_off[i], part_off[i + 1])
            Oo, lo = OS.pair_state(q[rows], rows, k, v, part_off, j, fo, fm)
            G.assert_close(O[f, bh, :rows.size], Oo, f"O pair {(i, j)} bh {bh}")
            G.assert_close(lse[f, bh, :rows.size], lo, f"lse pair {(i, j)} bh {bh}")


def oracle_cache_lse(w):
    po = w.part_off()
    A = OM.pair_mask(po, w.frame_off(), w.frame_mask())
    per = []
    for bh in range(w.BH):
        b, h = divmod(bh, w.H)
        per.append(OS.cache_lse_for_slab(inputs.slab_f64(w, "q", b, h),
                                         inputs.slab_f64(w, "k", b, h, prev=True),
                                         inputs.slab_f64(w, "v", b, h, prev=True), A, po,
                                         w.frame_off(), w.frame_mask()))
    return np.stack(per, axis=1), A


def build_cache(pa, Q, Kp, Vp):
    pa.plan_step(anchor=True)
    pa.partial(Q, Kp, Vp)


@pytest.mark.parametrize("sb", [False, True], ids=["fp32_cache", "bf16_cache"])
def test_tiny_reuse_step_plan_and_output(sb):
    w = configs.TINY
    Q, K, V = G.upload(w)
    Kp, Vp = G.upload_prev(w)
    pa = dt.PartitionedAttention(w.B, w.H, w.N, w.d, w.part_off(), state_bf16=sb)
    build_cache(pa, Q, Kp, Vp)
    out = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.float32, device="cuda")
    out_lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device="cuda")
    pa.step(Q, K, V, out, out_lse, band_k=w.band_k, budget=w.budget)
    torch.cuda.synchronize()
    assert pa.status.item() == 0
    lse_o, A = oracle_cache_lse(w)
    w_o = mass_scores(lse_o, A, w.part_off())
    plan_o, fl_o = select(w_o, A, w.band_k, w.budget)
    gpu_plan = pa.plan.cpu().numpy().reshape(w.P, w.P)
    assert (gpu_plan == plan_o).all(), (gpu_plan, plan_o)
    counts = pa.counts.cpu().numpy()
    assert counts.tolist() == [12, 4]
    assert (pa.fresh_list.cpu().numpy()[:12] == fl_o).all()
    score = pa.score.cpu().numpy().reshape(w.P, w.P)
    np.testing.assert_allclose(score, w_o, rtol=1e-4, atol=1e-7)
    o = out.cpu().numpy()
    ol = out_lse.cpu().numpy()
    for bh in range(w.BH):
        b, h = divmod(bh, w.H)
        for i in range(w.P):
            rows = np.arange(w.part_off()[i], w.part_off()[i + 1])
            Oo, lo, _ = G.oracle_rows(w, plan_o, b, h, i, rows)
            G.assert_close(o[b, h, rows], Oo, f"out bh {bh} part {i}")
            G.assert_close(ol[b, h, rows], lo, f"out lse bh {bh} part {i}")


@pytest.mark.parametrize("go", [None, [0, 2, 5]], ids=["pairs", "groups"])
def test_reuse_step_with_partitions_straddling_frames(go):
    """A reuse step whose partitions cut across the frames of a frame-tile
    mask (5 partitions over 6 frames): some rows attend none of a pair's keys
    (lse -inf, weight 0 in the merge).  The plan is compared with the
    oracle's selection on the GPU's scores and on its own fp64 scores of the
    GPU's cache; every output row with the oracle's composition."""
    from oracle import groups as OG
    w = configs.scaled(configs.TINY, N=1200, P=5, H=2, d=96, F=6, frame_component=0.5,
                       band_k=0, budget=0.5, seed=91, drift_seed=191, name="straddle")
    po = [0, 150, 410, 700, 990, 1200]
    fo, fm = w.frame_off(), w.frame_mask()
    Q, K, V = G.upload(w)
    Kp, Vp = G.upload_prev(w)
    pa = dt.PartitionedAttention(w.B, w.H, w.N, w.d, po, fo, fm, group_off=go)
    build_cache(pa, Q, Kp, Vp)
    torch.cuda.synchronize()
    lse_cache = pa.state_lse.cpu().numpy()
    out = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.float32, device="cuda")
    out_lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device="cuda")
    pa.step(Q, K, V, out, out_lse, band_k=w.band_k, budget=w.budget)
    torch.cuda.synchronize()
    assert pa.status.item() == 0
    A = OM.pair_mask(po, fo, fm)
    gof = go if go is not None else list(range(w.P + 1))
    Au, band = OG.unit_mask(A, gof), OG.unit_band(A, gof, w.band_k)
    plan = pa.plan.cpu().numpy().reshape(Au.shape)
    score = pa.score.cpu().numpy().reshape(Au.shape)
    sel, _ = select(score.astype(np.float64), Au, w.band_k, w.budget, band=band)
    assert (sel == plan).all()
    w_o = mass_scores(lse_cache, Au, po)
    np.testing.assert_allclose(score[Au], w_o[Au], rtol=1e-5)
    plan_o, _ = select(w_o, Au, w.band_k, w.budget, band=band)
    assert (plan_o == plan).all()
    o, ol = out.cpu().numpy(), out_lse.cpu().numpy()
    for bh in range(w.BH):
        b, h = divmod(bh, w.H)
        q, k, v, kp, vp = G.slabs(w, b, h)
        for i in range(w.P):
            rows = np.arange(po[i], po[i + 1])
            Oo, lo = OG.step_rows_units(q, k, v, kp, vp, plan, po, gof, i, rows, fo, fm)
            G.assert_close(o[b, h, rows], Oo, f"out bh {bh} part {i}")
            G.assert_close(ol[b, h, rows], lo, f"out lse bh {bh} part {i}")


@pytest.mark.parametrize("sb", [False, True], ids=["fp32_states", "bf16_states"])
def test_tiny_compact_partials_merge_writeback_and_cache_update_agree(sb):
    """Three routes to the same step must give bit-identical states and outputs:
    in-place partials, compact partials + merge write-back, compact partials +
    cache update + merge from the cache."""
    w = configs.TINY
    Q, K, V = G.upload(w)
    Kp, Vp = G.upload_prev(w)
    ref = dt.PartitionedAttention(w.B, w.H, w.N, w.d, w.part_off(), state_bf16=sb)
    build_cache(ref, Q, Kp, Vp)
    cache0_O, cache0_l = ref.state_O.clone(), ref.state_lse.clone()
    out_ref = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.float32, device="cuda")
    ref.step(Q, K, V, out_ref, band_k=w.band_k, budget=w.budget)
    g = ref.geom
    nf = 12
    part_O = torch.empty((nf, w.BH, w.Lp, w.d), dtype=torch.bfloat16 if sb else torch.float32, device="cuda")
    part_l = torch.empty((nf, w.BH, w.Lp), dtype=torch.float32, device="cuda")
    for route in ("writeback", "cache_update"):
        cO, cl = cache0_O.clone(), cache0_l.clone()
        valid = torch.ones(ref.n_slots, dtype=torch.uint8, device="cuda")
        plan = torch.zeros(w.P * w.P, dtype=torch.int8, device="cuda")
        fresh = torch.zeros(ref.n_slots, dtype=torch.int32, device="cuda")
        counts = torch.zeros(2, dtype=torch.int32, device="cuda")
        ws = torch.empty(ref.ws_bytes, dtype=torch.uint8, device="cuda")
        dt.ditango_plan(g, cl, valid, w.band_k, w.budget, 0, plan, fresh, counts, None, ws, ref.ws_bytes)
        dt.ditango_attn_partial(g, Q, K, V, fresh, counts, 0.0, part_O, part_l, 0, None, None,
                                state_bf16=sb)
        out = torch.empty_like(out_ref)
        if route == "writeback":
            dt.ditango_merge(g, plan, part_O, part_l, cO, cl, valid, 1, out, 1, state_bf16=sb)
        else:
            dt.ditango_cache_update(g, plan, part_O, part_l, cO, cl, valid, state_bf16=sb)
            dt.ditango_merge(g, plan, None, None, cO, cl, valid, 0, out, 1, state_bf16=sb)
        torch.cuda.synchronize()
        assert torch.equal(plan, ref.plan)
        assert torch.equal(out, out_ref), route
        L = w.Lp
        assert torch.equal(cO[:, :, :L], ref.state_O[:, :, :L]), route
        assert torch.equal(cl[:, :, :L], ref.state_lse[:, :, :L]), route


def test_zero_drift_reuse_is_bitwise_fresh():
    w = configs.TINY
    Q, K, V = G.upload(w)
    pa = dt.PartitionedAttention(w.B, w.H, w.N, w.d, w.part_off())
    build_cache(pa, Q, K, V)                 # cache from the current K/V
    out_r = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.float32, device="cuda")
    pa.step(Q, K, V, out_r, band_k=w.band_k, budget=w.budget)
    assert (pa.plan.cpu().numpy() == PLAN_REUSE).sum() == 4
    out_f = torch.empty_like(out_r)
    pa.step(Q, K, V, out_f, anchor=True)
    torch.cuda.synchronize()
    assert torch.equal(out_r, out_f)


def test_bf16_output_and_strided_output():
    w = configs.TINY
    Q, K, V = G.upload(w)
    pa = dt.PartitionedAttention(w.B, w.H, w.N, w.d, w.part_off())
    o32 = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.float32, device="cuda")
    pa.step(Q, K, V, o32, anchor=True)
    o16 = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.bfloat16, device="cuda")
    pa.merge(o16)
    obnhd = torch.empty((w.B, w.N, w.H, w.d), dtype=torch.float32, device="cuda")
    pa.merge(obnhd.permute(0, 2, 1, 3))
    torch.cuda.synchronize()
    assert torch.equal(o16, o32.to(torch.bfloat16))
    assert torch.equal(obnhd.permute(0, 2, 1, 3), o32)


def test_strided_qkv_inputs():
    """Q/K/V as views of one [B, N, 3, H, d] tensor (head-interleaved layout)."""
    w = configs.TINY
    Q, K, V = G.upload(w)
    qkv = torch.empty((w.B, w.N, 3, w.H, w.d), dtype=torch.bfloat16, device="cuda")
    for t, x in enumerate((Q, K, V)):
        qkv[:, :, t] = x.permute(0, 2, 1, 3)
    Qs, Ks, Vs = (qkv[:, :, t].permute(0, 2, 1, 3) for t in range(3))
    pa = dt.PartitionedAttention(w.B, w.H, w.N, w.d, w.part_off())
    o1 = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.float32, device="cuda")
    pa.step(Q, K, V, o1, anchor=True)
    o2 = torch.empty_like(o1)
    pa.step(Qs, Ks, Vs, o2, anchor=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


def test_step_captured_in_a_cuda_graph_replays_bit_identically():
    """Every call is asynchronous, allocates nothing and never syncs the host,
    so a whole step (plan -> partial -> merge) can be captured in a CUDA graph
    and replayed; replays equal eager steps bit for bit."""
    w = configs.TINY
    Q, K, V = G.upload(w)
    Kp, Vp = G.upload_prev(w)
    pa = dt.PartitionedAttention(w.B, w.H, w.N, w.d, w.part_off())
    build_cache(pa, Q, Kp, Vp)
    cache0 = (pa.state_O.clone(), pa.state_lse.clone(), pa.valid.clone())
    out = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.float32, device="cuda")
    out_lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device="cuda")
    pa.step(Q, K, V, out, out_lse, band_k=w.band_k, budget=w.budget)      # eager reference
    torch.cuda.synchronize()
    ref_out, ref_lse, ref_plan = out.clone(), out_lse.clone(), pa.plan.clone()

    def restore():
        pa.state_O.copy_(cache0[0]); pa.state_lse.copy_(cache0[1]); pa.valid.copy_(cache0[2])
        pa.mass_from_merge = False      # the cache changed behind the object: plan from it

    restore()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):                  # warm-up on a side stream, as capture requires
        pa.step(Q, K, V, out, out_lse, band_k=w.band_k, budget=w.budget)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    restore()
    out.zero_(); out_lse.zero_()
    torch.cuda.synchronize()
    with torch.cuda.graph(graph):
        pa.step(Q, K, V, out, out_lse, band_k=w.band_k, budget=w.budget)
    for _ in range(3):
        restore()
        out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert pa.status.item() == 0
        assert torch.equal(pa.plan, ref_plan)
        assert torch.equal(out, ref_out) and torch.equal(out_lse, ref_lse)


@pytest.mark.parametrize("w", [configs.TINY, configs.scaled(configs.FRAME_TILE, H=3, name="frame_tile_h3"),
                               configs.scaled(configs.LONG_VIDEO, H=2, anchor=True, name="long_video_h2")],
                         ids=["tiny", "frame_tile_h3", "long_video_h2"])
def test_work_counter_gives_the_fixed_order_states_and_returns_to_zero(w):
    """Items taken from the work counter (each CTA the next one when it is
    ready) and items dealt in a fixed stride compute the same states bit for
    bit -- an item's arithmetic does not depend on the CTA that runs it --
    and every launch leaves the counter at zero for the next one."""
    Q, K, V = G.upload(w)
    geom = dt.Geometry(w.B, w.H, w.N, w.d, w.part_off(), w.frame_off(), w.frame_mask())
    A = OM.pair_mask(w.part_off(), w.frame_off(), w.frame_mask())
    n, Lmax = int(A.sum()), w.Lp
    plan = torch.zeros(w.P * w.P, dtype=torch.int8, device="cuda")
    fresh = torch.zeros(n, dtype=torch.int32, device="cuda")
    counts = torch.zeros(2, dtype=torch.int32, device="cuda")
    dt.ditango_plan(geom, None, None, 0, 1.0, True, plan, fresh, counts)
    wc = torch.zeros(2, dtype=torch.int32, device="cuda")
    outs = []
    for counter in (None, wc, wc):
        O = torch.full((n, w.BH, Lmax, w.d), float("nan"), device="cuda")
        lse = torch.full((n, w.BH, Lmax), float("nan"), device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        dt.ditango_attn_partial(geom, Q, K, V, fresh, counts, 0.0, O, lse, 0, None, st,
                                work_counter=counter)
        torch.cuda.synchronize()
        assert st.item() == 0
        assert wc.tolist() == [0, 0]
        outs.append((O, lse))
    for O, lse in outs[1:]:
        assert torch.equal(O, outs[0][0]) and torch.equal(lse, outs[0][1])
