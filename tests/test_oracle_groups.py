"""Pins for the KV-group oracle (oracle.groups).

Pinned against:
  * torch's library attention in fp64 (one group covering every partition is
    unpartitioned attention; with the frame-tile mask, dense attention with the
    dropped frame tiles masked out, the mask built here from frame indices);
  * the pinned pair oracle (a group state is the composition of its pair
    states; one group per partition reduces every unit function to its pair
    form, the plan included);
  * hand-derived unit counts (tests/golden/plan_counts.json) and a closed form
    for the cache size under recursive halving;
  * brute force over every admissible fresh set on tiny unit grids.
"""
import itertools

import numpy as np
import pytest
import torch

from oracle import groups, masks, step
from oracle.attention import merge_states
from oracle.plan import PLAN_FRESH, budget_target, mass_scores, select


def sdpa(q, k, v, mask=None):
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x))[None, None]
    m = None if mask is None else torch.from_numpy(mask)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=m)[0, 0].numpy()


def tile_mask(F):
    return [[1 if (abs(f - g) <= 1 or g == 0) else 0 for g in range(F)] for f in range(F)]


# ragged partitions, each inside one frame (frames of 10 tokens)
PO = [0, 7, 10, 20, 26, 30, 40, 45, 50]
FO = [0, 10, 20, 30, 40, 50]
FM = tile_mask(5)


def frame_allowed(rows, cols):
    """Frame f may attend frames f-1, f, f+1 and 0 (tokens 10 per frame)."""
    fr = np.asarray(rows) // 10
    fc = np.asarray(cols) // 10
    return (np.abs(fr[:, None] - fc[None, :]) <= 1) | (fc[None, :] == 0)


@pytest.fixture
def qkv(rng):
    N, d = 50, 8
    return [rng.standard_normal((N, d)) for _ in range(3)]


def test_one_group_over_everything_is_dense_attention(qkv):
    q, k, v = qkv
    P = len(PO) - 1
    rows = np.arange(PO[3], PO[4])
    O, lse = groups.unit_state(q[rows], rows, k, v, PO, [0, P], 0)
    np.testing.assert_allclose(O, sdpa(q[rows], k, v), atol=1e-12)
    s = q[rows] @ k.T / np.sqrt(q.shape[1])
    np.testing.assert_allclose(lse, np.log(np.exp(s).sum(axis=1)), atol=1e-12)
    # with the frame-tile mask: dense attention with the dropped tiles masked
    Om, _ = groups.unit_state(q[rows], rows, k, v, PO, [0, P], 0, FO, FM)
    np.testing.assert_allclose(Om, sdpa(q[rows], k, v, frame_allowed(rows, np.arange(50))), atol=1e-12)


@pytest.mark.parametrize("goff", [[0, 2, 3, 8], [0, 3, 5, 6, 8], [0, 8]])
def test_group_state_is_composition_of_its_pair_states(qkv, goff):
    q, k, v = qkv
    P = len(PO) - 1
    A = masks.pair_mask(PO, FO, FM)
    Au = groups.unit_mask(A, goff)
    for i in range(P):
        rows = np.arange(PO[i], PO[i + 1])
        for c in range(len(goff) - 1):
            Ou, lu = groups.unit_state(q[rows], rows, k, v, PO, goff, c, FO, FM)
            js = [j for j in range(goff[c], goff[c + 1]) if A[i, j]]
            assert bool(js) == bool(Au[i, c])
            if not js:
                assert np.isneginf(lu).all() and (Ou == 0).all()
                continue
            Op, lp = merge_states([step.pair_state(q[rows], rows, k, v, PO, j, FO, FM) for j in js])
            np.testing.assert_allclose(Ou, Op, atol=1e-12)
            np.testing.assert_allclose(lu, lp, atol=1e-12)


def test_one_group_per_partition_reduces_to_pairs(qkv, rng):
    q, k, v = qkv
    P = len(PO) - 1
    ident = list(range(P + 1))
    A = masks.pair_mask(PO, FO, FM)
    assert (groups.unit_mask(A, ident) == A).all()
    ii, jj = np.indices((P, P))
    assert (groups.unit_band(A, ident, 1) == (A & (np.abs(ii - jj) <= 1))).all()
    w = rng.random((P, P))
    p1, f1 = select(w, A, 1, 0.6)
    p2, f2 = select(w, A, 1, 0.6, band=groups.unit_band(A, ident, 1))
    assert (p1 == p2).all() and (f1 == f2).all()
    kp = k + 0.1 * rng.standard_normal(k.shape)
    vp = v + 0.1 * rng.standard_normal(v.shape)
    rows = np.arange(PO[5], PO[6])
    Ou, lu = groups.step_rows_units(q, k, v, kp, vp, p1, PO, ident, 5, rows, FO, FM)
    Op, lp, _ = step.step_rows(q, k, v, kp, vp, p1, PO, 5, rows, FO, FM)
    np.testing.assert_allclose(Ou, Op, atol=1e-12)
    np.testing.assert_allclose(lu, lp, atol=1e-12)


def test_unit_band_by_hand():
    # 6 partitions, groups {0,1} {2} {3,4,5}, frame-tile mask over 6 frames
    po = list(range(0, 61, 10))
    A = masks.pair_mask(po, po, tile_mask(6))
    goff = [0, 2, 3, 6]
    expect_active = np.array([[1, 0, 0], [1, 1, 0], [1, 1, 1], [1, 1, 1], [1, 0, 1], [1, 0, 1]], dtype=bool)
    expect_band = np.array([[1, 0, 0], [1, 1, 0], [1, 1, 1], [0, 1, 1], [0, 0, 1], [0, 0, 1]], dtype=bool)
    assert (groups.unit_mask(A, goff) == expect_active).all()
    assert (groups.unit_band(A, goff, 1) == expect_band).all()
    # the band counts active pairs only: with (2, 2) masked out and k = 0,
    # unit (2, {2, 3}) is active through (2, 3) but not in the band
    A2 = np.ones((4, 4), dtype=bool)
    A2[2, 2] = False
    assert groups.unit_mask(A2, [0, 2, 4])[2, 1]
    assert groups.unit_band(A2, [0, 2, 4], 0)[1, 0]
    assert not groups.unit_band(A2, [0, 2, 4], 0)[2, 1]
    assert groups.unit_band(A2, [0, 2, 4], 1)[2, 1]


@pytest.mark.parametrize("fine,coarse", [([0, 1, 2, 3, 4, 5, 6, 7, 8], [0, 2, 4, 6, 8]),
                                         ([0, 2, 4, 6, 8], [0, 4, 8]),
                                         ([0, 1, 2, 3, 4, 5, 6, 7, 8], [0, 3, 8]),
                                         ([0, 1, 2, 3, 4, 5, 6, 7, 8], [0, 8])])
@pytest.mark.parametrize("masked", [False, True])
def test_compose_equals_the_coarse_cache_built_directly(qkv, fine, coarse, masked):
    q, k, v = qkv
    fo, fm = (FO, FM) if masked else (None, None)
    A = masks.pair_mask(PO, fo, fm)
    Af, Ac = groups.unit_mask(A, fine), groups.unit_mask(A, coarse)
    Of, lf = groups.unit_cache(q, k, v, Af, PO, fine, fo, fm)
    Oc, lc, vc = groups.compose_cache(Of, lf, np.ones(len(Of), bool), A, fine, coarse, PO)
    Od, ld = groups.unit_cache(q, k, v, Ac, PO, coarse, fo, fm)
    assert vc.all() and Oc.shape == Od.shape
    np.testing.assert_allclose(Oc, Od, atol=1e-12)
    np.testing.assert_allclose(lc, ld, atol=1e-12)


def test_recursive_composition_and_cache_size(qkv):
    q, k, v = qkv
    P = len(PO) - 1
    A = masks.pair_mask(PO)
    levels = [list(range(0, P + 1, s)) for s in (1, 2, 4, 8)]
    O, l = groups.unit_cache(q, k, v, groups.unit_mask(A, levels[0]), PO, levels[0])
    valid = np.ones(len(O), bool)
    for lvl, (a, b) in enumerate(zip(levels, levels[1:])):
        O, l, valid = groups.compose_cache(O, l, valid, A, a, b, PO)
        assert len(O) == P * P >> (lvl + 1)        # each halving halves the cache
    Od, ld = groups.unit_cache(q, k, v, groups.unit_mask(A, levels[-1]), PO, levels[-1])
    np.testing.assert_allclose(O, Od, atol=1e-12)
    np.testing.assert_allclose(l, ld, atol=1e-12)
    # the last level is one group: every row's state is dense attention
    rows = np.arange(PO[2], PO[3])
    np.testing.assert_allclose(O[2, :rows.size], sdpa(q[rows], k, v), atol=1e-12)


def test_compose_validity_and_bad_groupings(qkv):
    q, k, v = qkv
    A = masks.pair_mask(PO)
    fine, coarse = list(range(9)), [0, 2, 4, 6, 8]
    O, l = groups.unit_cache(q, k, v, groups.unit_mask(A, fine), PO, fine)
    valid = np.ones(len(O), bool)
    slot = masks.slot_table(A)
    valid[slot[3, 5]] = False            # fine unit (3, 5) never written
    Oc, lc, vc = groups.compose_cache(O, l, valid, A, fine, coarse, PO)
    sc = masks.slot_table(groups.unit_mask(A, coarse))
    assert not vc[sc[3, 2]] and vc.sum() == len(vc) - 1
    with pytest.raises(ValueError):
        groups.compose_cache(O, l, valid, A, [0, 2, 4, 6, 8], [0, 3, 8], PO)
    with pytest.raises(ValueError):
        groups.unit_mask(A, [0, 4, 4, 8])


def _brute_force_units(w, Au, band, budget):
    target = budget_target(band.sum(), Au.sum(), budget)
    cand = [int(x) for x in np.nonzero((Au & ~band).ravel())[0]]
    need = target - int(band.sum())
    best, best_set = -1.0, ()
    for comb in itertools.combinations(cand, max(need, 0)):
        s = sum(w.ravel()[c] for c in comb)
        if s > best:
            best, best_set = s, comb
    fresh = band.copy()
    for c in best_set:
        fresh.flat[c] = True
    return np.where(fresh, 1, np.where(Au, 2, 0))


@pytest.mark.parametrize("seed", range(10))
def test_unit_select_equals_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    P = int(rng.integers(3, 7))
    cuts = sorted(rng.choice(np.arange(1, P), size=int(rng.integers(1, P)), replace=False).tolist())
    goff = [0] + cuts + [P]
    A = rng.random((P, P)) < 0.8
    np.fill_diagonal(A, True)
    Au = groups.unit_mask(A, goff)
    band = groups.unit_band(A, goff, 0)
    w = rng.random(Au.shape)
    beta = float(rng.choice([0.3, 0.5, 0.75, 0.9]))
    plan, fl = select(w, Au, 0, beta, band=band)
    assert (plan == _brute_force_units(w, Au, band, beta)).all()
    assert (np.nonzero(plan.ravel() == PLAN_FRESH)[0] == fl).all()
    assert (fl < P * Au.shape[1]).all()


def test_unit_mass_scores_closed_forms():
    # 3 partitions of 4 rows, groups {0,1} {2}; equal logs: each unit's share
    # is its number of pairs over the row's pairs only when built from pairs;
    # from unit lse alone, equal unit logs give a uniform share per row.
    po = [0, 4, 8, 12]
    A = masks.pair_mask(po)
    Au = groups.unit_mask(A, [0, 2, 3])
    lse = np.full((int(Au.sum()), 2, 4), 0.3)
    w = mass_scores(lse, Au, po)
    assert w.shape == (3, 2)
    np.testing.assert_allclose(w, 0.5, atol=1e-15)
    # a unit composed of two equal pairs carries log 2 more: share 2/3
    lse2 = lse.copy()
    lse2[masks.slot_table(Au)[:, 0]] += np.log(2.0)
    np.testing.assert_allclose(mass_scores(lse2, Au, po)[:, 0], 2 / 3, atol=1e-12)
