"""The benchmark's algorithmic counts -- the numerators of every roofline
fraction it reports -- against closed forms derived by hand from the
workloads' shapes (equal partitions of length Lp, so a fresh pair costs
4 d B H Lp^2 FLOPs and a merged row reads |A_i| states of (d + 1) * 4 bytes)."""
import numpy as np
import pytest

import bench
from oracle import groups, masks
from workloads import configs


def plan_of(w, fresh_count):
    """A plan with the workload's active units and the first fresh_count of them fresh."""
    A = masks.pair_mask(w.part_off(), w.frame_off(), w.frame_mask())
    if w.grouped:
        A = groups.unit_mask(A, w.group_off())
    plan = np.where(A, 2, 0).astype(np.int8)
    idx = np.nonzero(A.ravel())[0][:fresh_count]
    plan.flat[idx] = 1
    return plan


@pytest.mark.parametrize("w,fresh,tflop", [
    (configs.FRAME_TILE, 28, 4 * 96 * 24 * 3600 ** 2 * 28 / 1e12),       # 3.344
    (configs.DENSE, 256, 4 * 128 * 48 * 2048 ** 2 * 256 / 1e12),          # 26.39
    (configs.DITANGO_REUSE, 256, 4 * 128 * 40 * 2400 ** 2 * 256 / 1e12),  # 30.20
    (configs.LONG_VIDEO, 70, 4 * 96 * 24 * 3600 ** 2 * 70 / 1e12),        # 8.36
    (configs.DITANGO_GROUPS, 64, 4 * 128 * 40 * 2400 ** 2 * 64 * 4 / 1e12),  # 64 units of 4 pairs
])
def test_effective_flops(w, fresh, tflop):
    plan = plan_of(w, fresh)
    got = bench.effective_flops(w, bench.fresh_pairs_of_units(w, plan, bench.pair_mask(w)))
    assert got / 1e12 == pytest.approx(tflop, rel=1e-12)


def test_published_flop_figures_of_the_workloads():
    assert 4 * 96 * 24 * 3600 ** 2 * 28 / 1e12 == pytest.approx(3.344, abs=1e-3)
    assert 4 * 128 * 48 * 2048 ** 2 * 256 / 1e12 == pytest.approx(26.39, abs=1e-2)
    assert 4 * 128 * 40 * 2400 ** 2 * 256 / 1e12 == pytest.approx(30.20, abs=1e-2)


@pytest.mark.parametrize("w,per_row_states,fresh,sob", [
    (configs.FRAME_TILE, None, 28, 4),
    (configs.DENSE, 16, 256, 4),
    (configs.DITANGO_REUSE, 32, 256, 4),
    (configs.DITANGO_REUSE, 32, 256, 2),
    (configs.DITANGO_GROUPS, 8, 64, 4),
])
def test_merge_bytes(w, per_row_states, fresh, sob):
    plan = plan_of(w, fresh)
    A = plan != 0
    got = bench.merge_bytes(w, A, plan == 1, state_o_bytes=sob, mass_partials=False)
    states = int(A.sum()) if per_row_states is None else per_row_states * w.P
    want = states * w.Lp * w.BH * (w.d * sob + 4) + w.BH * w.N * (w.d * 2 + 4)
    assert got == want
    if w is configs.FRAME_TILE:
        assert got / 1e9 == pytest.approx(1.074, abs=1e-3)   # 28 states of 3600 rows, 24 heads
    # the mass partials: one float per KV column per block of 128 rows of each
    # (b*h, partition): ceil(Lp / 128) blocks
    with_mass = bench.merge_bytes(w, A, plan == 1, state_o_bytes=sob)
    assert with_mass - got == w.P * -(-w.Lp // 128) * w.BH * A.shape[1] * 4
