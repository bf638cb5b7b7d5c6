"""Pins for the oracle's masks, mass scores and fresh/reuse selection.

Pinned against: hand-derived counts of the five workloads
(tests/golden/plan_counts.json), the Efficient-vDiT claim that the kept
frame tiles grow linearly with the number of frames, closed forms of the mass
score (rows sum to one; equal logs give a uniform share), scalar loops, and a
brute-force search over every admissible fresh set on tiny P.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

from oracle import groups, masks
from oracle.plan import PLAN_FRESH, PLAN_REUSE, PLAN_SKIP, budget_target, mass_scores, select
from workloads import configs

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "plan_counts.json")))


def geometry(w):
    return w.part_off(), w.frame_off(), w.frame_mask()


@pytest.mark.parametrize("w", configs.ALL, ids=lambda w: w.name)
def test_golden_counts(w):
    g = GOLD[w.name]
    po, fo, fm = geometry(w)
    A = masks.pair_mask(po, fo, fm)
    P = w.P
    ii, jj = np.indices((P, P))
    band = A & (np.abs(ii - jj) <= w.band_k)
    if w.grouped:
        A = groups.unit_mask(A, w.group_off())
        band = groups.unit_band(masks.pair_mask(po, fo, fm), w.group_off(), w.band_k)
        assert A.shape == (P, g["G"])
    assert int(A.sum()) == g["active"]
    rng = np.random.default_rng(0)
    wts = rng.random(A.shape)
    plan, fl = select(wts, A, w.band_k, w.budget, anchor=w.anchor, band=band if w.grouped else None)
    assert int((plan == PLAN_FRESH).sum()) == g["fresh"] == len(fl)
    assert int((plan == PLAN_REUSE).sum()) == g["reuse"]
    if g["band"] is not None:
        assert int(band.sum()) == g["band"]
        assert budget_target(band.sum(), A.sum(), w.budget) == g["target"]


def test_long_video_reuses_frame_zero_pairs():
    w = configs.LONG_VIDEO
    A = masks.pair_mask(*geometry(w))
    plan, _ = select(np.random.default_rng(1).random((w.P, w.P)), A, w.band_k, w.budget)
    reused = {(int(i), int(j)) for i, j in zip(*np.nonzero(plan == PLAN_REUSE))}
    assert reused == {(f, 0) for f in range(2, w.P)}


@pytest.mark.parametrize("F", [3, 4, 8, 24, 64])
def test_frame_tiles_linear_in_frames(F):
    fl = 7
    fo = [f * fl for f in range(F + 1)]
    fm = [[1 if (abs(f - g) <= 1 or g == 0) else 0 for g in range(F)] for f in range(F)]
    A = masks.pair_mask(fo, fo, fm)
    assert int(A.sum()) == 4 * F - 4
    assert A.sum(axis=1).max() <= 4
    assert A[:, 0].all() and not A[0, 2:].any()   # frame 0 is a global key, not a global query


def test_pair_mask_with_partitions_splitting_frames():
    # 2 frames of 6 tokens, 4 partitions of 3: each partition inside one frame
    fo = [0, 6, 12]
    fm = [[1, 0], [1, 1]]
    po = [0, 3, 6, 9, 12]
    A = masks.pair_mask(po, fo, fm)
    expect = np.array([[1, 1, 0, 0], [1, 1, 0, 0], [1, 1, 1, 1], [1, 1, 1, 1]], dtype=bool)
    assert (A == expect).all()
    # partitions straddling frames: active if any token pair is allowed
    po2 = [0, 5, 12]
    A2 = masks.pair_mask(po2, fo, fm)
    assert A2.all()


def test_slot_table_row_major():
    A = np.array([[1, 0, 1], [0, 0, 0], [1, 1, 1]], dtype=bool)
    s = masks.slot_table(A)
    assert s.tolist() == [[0, -1, 1], [-1, -1, -1], [2, 3, 4]]
    assert masks.slot_pairs(A) == [(0, 0), (0, 2), (2, 0), (2, 1), (2, 2)]


def _lse_array(A, BH, L, rng, scale=3.0):
    n = int(A.sum())
    return rng.standard_normal((n, BH, L)) * scale


def test_mass_rows_sum_to_one_and_match_scalar_loops(rng):
    P, BH, L = 3, 2, 4
    A = np.array([[1, 1, 0], [1, 1, 1], [0, 1, 1]], dtype=bool)
    po = [0, L, 2 * L, 3 * L]
    lse = _lse_array(A, BH, L, rng)
    w = mass_scores(lse, A, po)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, atol=1e-12)
    assert (w[~A] == 0).all()
    slot = masks.slot_table(A)
    for i in range(P):
        for j in range(P):
            if not A[i, j]:
                continue
            acc = 0.0
            for bh in range(BH):
                for r in range(L):
                    den = sum(math.exp(lse[slot[i, jj], bh, r]) for jj in range(P) if A[i, jj])
                    acc += math.exp(lse[slot[i, j], bh, r]) / den
            assert abs(acc / (BH * L) - w[i, j]) < 1e-12


def test_mass_closed_forms():
    P, BH, L = 4, 3, 5
    A = np.ones((P, P), dtype=bool)
    po = [p * L for p in range(P + 1)]
    lse = np.full((P * P, BH, L), 1.7)
    np.testing.assert_allclose(mass_scores(lse, A, po), 0.25, atol=1e-15)
    lse2 = lse.copy()
    lse2[masks.slot_table(A)[1, 3]] = -np.inf     # an empty state holds no mass
    w = mass_scores(lse2, A, po)
    assert w[1, 3] == 0
    np.testing.assert_allclose(w[1, [0, 1, 2]], 1 / 3, atol=1e-15)
    lse3 = lse.copy()
    lse3[masks.slot_table(A)[2, 0]] += math.log(7.0)  # 7x the mass of each other pair
    np.testing.assert_allclose(mass_scores(lse3, A, po)[2, 0], 0.7, atol=1e-12)
    valid = np.ones(P * P, dtype=bool)
    valid[masks.slot_table(A)[1, 3]] = False        # a never-written slot: no mass
    w4 = mass_scores(lse, A, po, valid=valid)
    np.testing.assert_allclose(w4, w, atol=1e-15)


def _brute_force_plan(w, A, band_k, budget):
    """Among all admissible fresh sets of the required size, the one of
    largest total mass (distinct masses make it unique)."""
    P = A.shape[0]
    ii, jj = np.indices((P, P))
    band = A & (np.abs(ii - jj) <= band_k)
    target = budget_target(band.sum(), A.sum(), budget)
    cand = [int(x) for x in np.nonzero((A & ~band).ravel())[0]]
    need = target - int(band.sum())
    best, best_set = -1.0, ()
    for comb in itertools.combinations(cand, max(need, 0)):
        s = sum(w.ravel()[c] for c in comb)
        if s > best:
            best, best_set = s, comb
    fresh = band.copy()
    for c in best_set:
        fresh.flat[c] = True
    return np.where(fresh, 1, np.where(A, 2, 0))


@pytest.mark.parametrize("seed", range(12))
def test_select_equals_brute_force(seed):
    rng = np.random.default_rng(seed)
    P = int(rng.integers(2, 6))
    A = rng.random((P, P)) < 0.8
    np.fill_diagonal(A, True)
    w = rng.random((P, P))
    k = int(rng.integers(0, 2))
    beta = float(rng.choice([0.3, 0.5, 0.75, 0.9]))
    plan, fl = select(w, A, k, beta)
    assert (plan == _brute_force_plan(w, A, k, beta)).all()
    assert (np.nonzero(plan.ravel() == PLAN_FRESH)[0] == fl).all()


def test_select_invariants_and_ties():
    P = 5
    A = np.ones((P, P), dtype=bool)
    A[0, 4] = A[4, 0] = False                       # 23 active pairs
    w = np.full((P, P), 0.1)                        # all tied: index order decides
    plan, fl = select(w, A, 0, 0.6)
    ii, jj = np.indices((P, P))
    band = A & (ii == jj)
    assert (plan[band] == PLAN_FRESH).all()
    assert (plan[~A] == PLAN_SKIP).all()
    target = budget_target(band.sum(), A.sum(), 0.6)
    assert (plan == PLAN_FRESH).sum() == target == 13
    extra = [int(p) for p in fl if not band.flat[p]]
    cand = [p for p in range(P * P) if A.flat[p] and not band.flat[p]]
    assert extra == cand[:target - int(band.sum())]  # lowest linear indices win ties
    # a planted tie between a high and a low index, above every other pair
    w2 = np.full((P, P), 0.1)
    w2[3, 0] = w2[0, 2] = 0.5
    plan2, _ = select(w2, A, 0, 6.5 / 23)           # room for exactly one extra pair
    assert (plan2 == PLAN_FRESH).sum() == 6
    assert plan2[0, 2] == PLAN_FRESH and plan2[3, 0] == PLAN_REUSE


def test_select_anchor_and_invalid_slots():
    P = 4
    A = np.ones((P, P), dtype=bool)
    w = np.random.default_rng(3).random((P, P))
    plan, fl = select(w, A, 0, 0.0, anchor=True)
    assert (plan == PLAN_FRESH).all() and len(fl) == 16
    valid = np.ones((P, P), dtype=bool)
    valid[0, 3] = False
    plan, _ = select(w, A, 0, 0.0, valid=valid)
    assert plan[0, 3] == PLAN_FRESH
    assert (plan == PLAN_FRESH).sum() == P + 1


def test_budget_rounding_reading():
    # floor(budget * active + 1e-9): decimal fractions land on the integer they name
    assert budget_target(0, 10, 0.7) == 7
    assert budget_target(0, 92, 0.40) == 36
    assert budget_target(40, 92, 0.40) == 40


def test_planted_plan_mistakes_are_caught():
    rng = np.random.default_rng(5)
    P = 4
    A = np.ones((P, P), dtype=bool)
    w = rng.random((P, P))
    good = _brute_force_plan(w, A, 1, 0.75)
    plan, _ = select(w, A, 1, 0.75)
    assert (plan == good).all()
    wrong_order = select(-w, A, 1, 0.75)[0]        # ascending instead of descending mass
    assert (wrong_order != good).any()
    wrong_band = select(w, A, 0, 0.75)[0]
    assert (wrong_band != good).any()
