"""Pins for the oracle's attention states and their composition.

Each check ties the oracle to something other than itself: a library
attention routine (torch's scaled_dot_product_attention in fp64 on the CPU),
closed forms, algebraic invariants of the log-sum-exp composition
(associative and commutative, per DiTango "Composizione dello Stato"), and a
scalar pure-Python restatement on tiny inputs.
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import brute, masks


def sdpa(q, k, v, mask=None):
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x))[None, None]
    m = None if mask is None else torch.from_numpy(mask)[None, None]
    out = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=m)
    return out[0, 0].numpy()


@pytest.mark.parametrize("Lq,Lk,d", [(7, 13, 8), (64, 200, 64), (33, 1, 16)])
def test_single_partition_equals_library_attention(rng, Lq, Lk, d):
    q, k, v = (rng.standard_normal((n, d)) for n in (Lq, Lk, Lk))
    O, lse = A.partial_state(q, k, v)
    np.testing.assert_allclose(O, sdpa(q, k, v), rtol=0, atol=1e-12)
    # lse against scipy's logsumexp (a library routine) on the same logits
    from scipy.special import logsumexp
    np.testing.assert_allclose(lse, logsumexp(q @ k.T / math.sqrt(d), axis=1), atol=1e-12)


def test_masked_equals_library_attention_with_mask(rng):
    F, fl, d = 5, 6, 8
    N = F * fl
    frame_off = [f * fl for f in range(F + 1)]
    fm = [[1 if (abs(f - g) <= 1 or g == 0) else 0 for g in range(F)] for f in range(F)]
    q, k, v = (rng.standard_normal((N, d)) for _ in range(3))
    allowed = masks.token_allowed(np.arange(N), np.arange(N), frame_off, fm)
    O, _ = A.partial_state(q, k, v, allowed=allowed)
    np.testing.assert_allclose(O, sdpa(q, k, v, allowed), atol=1e-12)


@pytest.mark.parametrize("cuts", [[0, 40, 41, 100], [0, 1, 2, 3, 100], [0, 100]])
def test_partition_merge_equals_unpartitioned(rng, cuts):
    q = rng.standard_normal((17, 16))
    k = rng.standard_normal((100, 16))
    v = rng.standard_normal((100, 12))
    parts = [A.partial_state(q, k[a:b], v[a:b]) for a, b in zip(cuts[:-1], cuts[1:])]
    O, lse = A.merge_states(parts)
    O1, lse1 = A.dense_attention(q, k, v)
    np.testing.assert_allclose(O, O1, atol=1e-12)
    np.testing.assert_allclose(lse, lse1, atol=1e-12)
    np.testing.assert_allclose(O, sdpa(q, k, v), atol=1e-12)


def test_merge_associative_and_commutative(rng):
    q = rng.standard_normal((9, 8))
    k = rng.standard_normal((60, 8)) * 3
    v = rng.standard_normal((60, 5))
    cuts = [0, 5, 6, 20, 33, 47, 60]
    st = [A.partial_state(q, k[a:b], v[a:b]) for a, b in zip(cuts[:-1], cuts[1:])]
    ref = A.merge_states(st)
    for trial in range(20):
        perm = rng.permutation(len(st))
        pool = [st[p] for p in perm]
        while len(pool) > 1:          # random binary tree
            a = rng.integers(len(pool))
            x = pool.pop(a)
            b = rng.integers(len(pool))
            y = pool.pop(b)
            pool.insert(rng.integers(len(pool) + 1), A.merge_states([x, y]))
        np.testing.assert_allclose(pool[0][0], ref[0], atol=1e-12)
        np.testing.assert_allclose(pool[0][1], ref[1], atol=1e-12)


def test_merge_of_two_is_logaddexp(rng):
    O1, O2 = rng.standard_normal((2, 11, 4))
    l1, l2 = rng.standard_normal((2, 11)) * 5
    O, lse = A.merge_states([(O1, l1), (O2, l2)])
    L = np.logaddexp(l1, l2)
    np.testing.assert_allclose(lse, L, atol=1e-12)
    np.testing.assert_allclose(O, np.exp(l1 - L)[:, None] * O1 + np.exp(l2 - L)[:, None] * O2,
                               atol=1e-12)


def test_closed_forms(rng):
    d = 8
    q = rng.standard_normal((4, d))
    krow = rng.standard_normal(d)
    k = np.tile(krow, (10, 1))              # identical keys: uniform attention
    v = rng.standard_normal((10, 3))
    O, lse = A.partial_state(q, k, v)
    np.testing.assert_allclose(O, np.tile(v.mean(0), (4, 1)), atol=1e-12)
    np.testing.assert_allclose(lse, q @ krow / math.sqrt(d) + math.log(10), atol=1e-12)
    O, lse = A.partial_state(q, k[:1], v[:1])  # one key: its value, its logit
    np.testing.assert_allclose(O, np.tile(v[0], (4, 1)), atol=1e-12)
    np.testing.assert_allclose(lse, q @ krow / math.sqrt(d), atol=1e-12)
    kk = rng.standard_normal((10, d))
    vc = np.full((10, 3), 2.5)               # constant values: output is that constant
    O, _ = A.partial_state(q, kk, vc)
    np.testing.assert_allclose(O, 2.5, atol=1e-12)


def test_dead_rows_and_identity_of_dead_state(rng):
    q = rng.standard_normal((3, 4))
    k = rng.standard_normal((5, 4))
    v = rng.standard_normal((5, 2))
    allowed = np.ones((3, 5), dtype=bool)
    allowed[1] = False
    O, lse = A.partial_state(q, k, v, allowed=allowed)
    assert lse[1] == -np.inf and np.all(O[1] == 0)
    O2, l2 = A.partial_state(q, k, v)
    Om, lm = A.merge_states([(O2, l2), (np.zeros_like(O2), np.full(3, -np.inf))])
    np.testing.assert_allclose(Om, O2, atol=1e-15)
    np.testing.assert_allclose(lm, l2, atol=1e-15)
    Oz, lz = A.merge_states([(np.zeros((2, 2)), np.full(2, -np.inf))])
    assert np.all(lz == -np.inf) and np.all(Oz == 0)


def test_bruteforce_scalar_cross_check(rng):
    d, Lq = 4, 5
    cuts = [0, 3, 4, 9]
    q = rng.standard_normal((Lq, d))
    k = rng.standard_normal((9, d)) * 2
    v = rng.standard_normal((9, 3))
    scale = 1 / math.sqrt(d)
    st = [A.partial_state(q, k[a:b], v[a:b]) for a, b in zip(cuts[:-1], cuts[1:])]
    O, lse = A.merge_states(st)
    for r in range(Lq):
        acc_o, acc_l = [0.0] * 3, -math.inf
        for (a, b), (Oj, lj) in zip(zip(cuts[:-1], cuts[1:]), st):
            o, l = brute.row_attention(q[r].tolist(), k[a:b].tolist(), v[a:b].tolist(), scale)
            assert abs(l - lj[r]) < 1e-12
            assert max(abs(x - y) for x, y in zip(o, Oj[r])) < 1e-12
            acc_o, acc_l = brute.merge_two(acc_o, acc_l, o, l)
        assert abs(acc_l - lse[r]) < 1e-12
        assert max(abs(x - y) for x, y in zip(acc_o, O[r])) < 1e-12
        o_all, l_all = brute.row_attention(q[r].tolist(), k.tolist(), v.tolist(), scale)
        assert abs(l_all - lse[r]) < 1e-12


def test_planted_mistakes_are_caught(rng):
    """A wrong scale, swapped operands or a merge without lse weights fail the pins."""
    q = rng.standard_normal((6, 8))
    k = rng.standard_normal((20, 8))
    v = rng.standard_normal((20, 8))
    good = sdpa(q, k, v)
    assert np.abs(A.partial_state(q, k, v, scale=1 / 8)[0] - good).max() > 1e-3
    assert np.abs(A.partial_state(q, v, k)[0] - good).max() > 1e-3
    o1, l1 = A.partial_state(q, k[:10], v[:10])
    o2, l2 = A.partial_state(q, k[10:], v[10:])
    assert np.abs((o1 + o2) / 2 - good).max() > 1e-3
    assert np.abs(A.merge_states([(o1, l1), (o2, l2)])[0] - good).max() < 1e-12
