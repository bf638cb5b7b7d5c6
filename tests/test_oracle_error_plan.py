"""Pins for the error-growth planner (oracle.error_plan).

The pages give the ingredients (importance w, temporal growth delta, local
states as the proxy, periodic anchors) but no formula, so the error model's
predictive quality is unpinned.  Pinned here: the rules and what follows from
them --
  * constant drift and fresh ages reduce the planner to the pinned w planner;
  * zero drift (unchanged K/V) measures delta = 0 exactly and leaves every
    non-band choice to the index order;
  * ages accumulate k * delta over k reuses and reset when recomputed;
  * with equal w and equal drift the non-band refreshes rotate oldest-first
    through all units (a closed form derived from the rule);
  * anchors: all fresh every anchor_every steps, ages reset after them, w
    refreshed only then; every other step fills exactly the budget.
"""
import numpy as np
import pytest

from oracle import error_plan as E
from oracle import groups, masks
from oracle.plan import PLAN_FRESH, budget_target, select
from workloads import configs, inputs


def test_local_delta_closed_forms():
    a = np.array([0.5, -1.0, 2.0, -np.inf])
    assert E.local_delta(a, a) == 0.0
    assert E.local_delta(a[:3] + 0.25, a[:3]) == pytest.approx(0.25, abs=1e-15)
    assert E.local_delta([1.0, 2.0], [2.0, 1.0]) == pytest.approx(1.0)
    assert E.local_unit(5, [0, 2, 6, 8]) == 1 and E.local_unit(0, [0, 1, 2]) == 0


def test_age_accumulates_and_resets():
    A = np.ones((2, 2), dtype=bool)
    age = np.zeros(4)
    reuse = np.array([[1, 2], [2, 1]], dtype=np.int8)
    delta = np.array([0.1, 0.3])
    for k in range(1, 6):
        age = E.age_update(age, reuse, A, delta)
        np.testing.assert_allclose(age, [0.0, 0.1 * k, 0.3 * k, 0.0], atol=1e-15)
    age = E.age_update(age, np.ones((2, 2), dtype=np.int8), A, delta)
    assert (age == 0).all()


def test_constant_drift_and_zero_age_is_the_w_planner(rng):
    P = 6
    A = np.ones((P, P), dtype=bool)
    band = groups.unit_band(A, list(range(P + 1)), 1)
    w = rng.random((P, P))
    prev = np.where(A, PLAN_FRESH, 0).astype(np.int8)      # after an anchor: ages reset
    plan, fl, age, score = E.plan_error(w, np.zeros(P * P), prev, np.full(P, 0.02), A, band, 0.5)
    p_w, f_w = select(w, A, 1, 0.5)
    assert (plan == p_w).all() and (fl == f_w).all()
    np.testing.assert_allclose(score, 0.02 * w, rtol=1e-15)


def test_rotation_with_equal_w_and_drift():
    """Equal w and drift: each step refreshes the `extra` oldest non-band
    units, ties by index, so the refreshes sweep the non-band units in index
    order and every one is recomputed within ceil(n / extra) steps."""
    P = 5
    A = np.ones((P, P), dtype=bool)
    band = groups.unit_band(A, list(range(P + 1)), 0)        # the diagonal
    budget = 8 / 25                                          # 5 band + 3 extra
    nonband = [p for p in range(P * P) if not band.flat[p]]  # 20 units
    w = np.full((P, P), 0.2)
    delta = np.full(P, 0.01)
    plan = np.where(A, PLAN_FRESH, 0).astype(np.int8)        # an anchor step
    age = np.zeros(P * P)
    seen = []
    for s in range(1, 8):
        plan, fl, age, _ = E.plan_error(w, age, plan, delta, A, band, budget)
        extra = [int(p) for p in fl if not band.flat[p]]
        assert len(extra) == 3
        seen.append(extra)
    # step k (1..6): all never-refreshed units are the oldest, so the sweep
    # takes nonband[3(k-1) : 3k]; step 7 takes the last two and then the
    # oldest refreshed one, nonband[0] (refreshed at step 1)
    for k in range(1, 7):
        assert seen[k - 1] == nonband[3 * (k - 1):3 * k], k
    assert seen[6] == [nonband[0], nonband[18], nonband[19]]


def tiny_schedule_case(sigma=0.05, groups_size=0, anchor_every=4, budget=0.5, band_k=0):
    w = configs.scaled(configs.TINY, N=768, P=6, d=32, H=2, drift_sigma=sigma, budget=budget,
                       band_k=band_k, group_size=groups_size, seed=21, drift_seed=121,
                       name="tiny_schedule")
    q = [inputs.slab_f64(w, "q", 0, h) for h in range(w.H)]
    return w, q


@pytest.mark.parametrize("gs", [0, 2])
def test_schedule_invariants(gs):
    w, q = tiny_schedule_case(groups_size=gs)
    S = 9
    ks = [inputs.step_slabs(w, "k", 0, h, S) for h in range(w.H)]
    vs = [inputs.step_slabs(w, "v", 0, h, S) for h in range(w.H)]
    A = masks.pair_mask(w.part_off())
    sch = E.Schedule(q, w.part_off(), w.group_off(), A, w.band_k, w.budget, 4)
    Au = sch.Au
    target = budget_target(sch.band.sum(), Au.sum(), w.budget)
    w_seen = []
    for s in range(S + 1):
        k = [inputs.bf16_to_f32(ks[h][s]).astype(np.float64) for h in range(w.H)]
        v = [inputs.bf16_to_f32(vs[h][s]).astype(np.float64) for h in range(w.H)]
        plan, score, O, l = sch.step(s, k, v)
        if s % 4 == 0:
            assert (plan[Au] == PLAN_FRESH).all()
        else:
            assert (plan[sch.band] == PLAN_FRESH).all()
            assert int((plan == PLAN_FRESH).sum()) == target
            if s == 1:
                assert (sch.delta == 0).all()                 # no local state before step 0
            else:
                assert (sch.delta > 0).all()                  # K/V drift every step
            if s % 4 == 1:
                assert (sch.age == 0).all()                   # reset by the anchor
            w_seen.append(sch.w.copy())
        assert sch.valid.all()
    # w changes only at the step after an anchor
    np.testing.assert_array_equal(w_seen[0], w_seen[1])
    np.testing.assert_array_equal(w_seen[1], w_seen[2])
    assert not np.array_equal(w_seen[2], w_seen[3])


def test_zero_drift_measures_zero_and_falls_back_to_index_order():
    w, q = tiny_schedule_case(sigma=0.0)
    k = [inputs.slab_f64(w, "k", 0, h) for h in range(w.H)]
    v = [inputs.slab_f64(w, "v", 0, h) for h in range(w.H)]
    A = masks.pair_mask(w.part_off())
    sch = E.Schedule(q, w.part_off(), w.group_off(), A, w.band_k, w.budget, 100)
    sch.step(0, k, v)
    plan, score, O, l = sch.step(1, k, v)
    assert (sch.delta == 0).all() and (score == 0).all()
    nonband = [p for p in range(w.P * w.P) if not sch.band.flat[p]]
    target = budget_target(sch.band.sum(), sch.Au.sum(), w.budget)
    extra = [p for p in np.nonzero(plan.ravel() == PLAN_FRESH)[0] if not sch.band.flat[p]]
    assert extra == nonband[:target - int(sch.band.sum())]
    # unchanged K/V: the reuse step is exactly the all-fresh result
    ref = E.Schedule(q, w.part_off(), w.group_off(), A, w.band_k, w.budget, 1)
    _, _, O_f, l_f = ref.step(0, k, v)
    np.testing.assert_allclose(O, O_f, atol=1e-12)
    np.testing.assert_allclose(l, l_f, atol=1e-12)


def test_schedule_rows_are_compositions_of_cached_and_fresh_states():
    """Every step's output equals the merge of the unit states the plan says:
    fresh from this step's K/V, reused from the step each state was computed."""
    w, q = tiny_schedule_case(anchor_every=3)
    S = 5
    ks = [inputs.step_slabs(w, "k", 0, h, S) for h in range(w.H)]
    vs = [inputs.step_slabs(w, "v", 0, h, S) for h in range(w.H)]
    A = masks.pair_mask(w.part_off())
    sch = E.Schedule(q, w.part_off(), w.group_off(), A, w.band_k, w.budget, 3)
    born = {}
    for s in range(S + 1):
        k = [inputs.bf16_to_f32(ks[h][s]).astype(np.float64) for h in range(w.H)]
        v = [inputs.bf16_to_f32(vs[h][s]).astype(np.float64) for h in range(w.H)]
        plan, _, O, l = sch.step(s, k, v)
        for (i, c) in sch.slots:
            if plan[i, c] == PLAN_FRESH:
                born[(i, c)] = s
        i = 2
        rows = np.arange(w.part_off()[i], w.part_off()[i + 1])
        for h in range(w.H):
            st = []
            for c in range(sch.Au.shape[1]):
                t = born[(i, c)]
                kt = inputs.bf16_to_f32(ks[h][t]).astype(np.float64)
                vt = inputs.bf16_to_f32(vs[h][t]).astype(np.float64)
                st.append(groups.unit_state(q[h][rows], rows, kt, vt, w.part_off(), w.group_off(), c))
            from oracle.attention import merge_states
            Oe, le = merge_states(st)
            np.testing.assert_allclose(O[h, rows], Oe, atol=1e-12)
            np.testing.assert_allclose(l[h, rows], le, atol=1e-12)
