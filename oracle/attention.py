"""Attention states and their composition, fp64.

DiTango, "Riepilogo Tecnico" -> Metodologia -> 2. State-Centric Parallel
Runtime -> "Composizione dello Stato": an attention state is the pair
(output, log-sum-exp); states of disjoint key sets compose associatively and
commutatively into the state over their union.

Readings of what the pages leave open:
  * scale: logits are q.k / sqrt(d) unless a scale is given;
  * state form: O is normalised (O = sum_k softmax(s)_k v_k) and
    lse = log sum_k exp(s_k);
  * a row with no admissible key has lse = -inf and O = 0.
"""
from __future__ import annotations

import numpy as np


def partial_state(q, k, v, scale=None, allowed=None):
    """State (O [Lq, d], lse [Lq]) of query rows q against keys k, values v.

    q: [Lq, d], k: [Lk, d], v: [Lk, dv] (fp64).  allowed: optional bool
    [Lq, Lk]; a False entry drops that key for that row (logit -inf).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if scale is None:
        scale = 1.0 / np.sqrt(q.shape[1])
    Lq = q.shape[0]
    if k.shape[0] == 0:
        return np.zeros((Lq, v.shape[1])), np.full(Lq, -np.inf)
    s = (q @ k.T) * scale
    if allowed is not None:
        s = np.where(allowed, s, -np.inf)
    m = s.max(axis=1)
    dead = ~np.isfinite(m)
    m0 = np.where(dead, 0.0, m)
    e = np.exp(s - m0[:, None])          # exp(-inf) = 0 for dropped keys
    l = e.sum(axis=1)
    l1 = np.where(dead, 1.0, l)
    O = (e @ v) / l1[:, None]
    O[dead] = 0.0
    lse = np.where(dead, -np.inf, m0 + np.log(l1))
    return O, lse


def merge_states(states):
    """Compose states [(O_j, lse_j), ...] over disjoint key sets.

    lse = log sum_j exp(lse_j);  O = sum_j exp(lse_j - lse) * O_j.
    """
    states = list(states)
    if not states:
        raise ValueError("merge of zero states")
    lses = np.stack([np.asarray(s[1], dtype=np.float64) for s in states])  # [J, L]
    Os = np.stack([np.asarray(s[0], dtype=np.float64) for s in states])    # [J, L, d]
    M = lses.max(axis=0)
    dead = ~np.isfinite(M)
    M0 = np.where(dead, 0.0, M)
    wts = np.exp(lses - M0[None, :])      # [J, L]
    tot = wts.sum(axis=0)
    tot1 = np.where(dead, 1.0, tot)
    O = np.einsum("jl,jld->ld", wts, Os) / tot1[:, None]
    O[dead] = 0.0
    lse = np.where(dead, -np.inf, M0 + np.log(tot1))
    return O, lse


def dense_attention(q, k, v, scale=None, allowed=None):
    """Unpartitioned softmax(q k^T * scale) v with an optional key mask.

    This is the all-fresh, one-partition special case; it is the same
    definition as partial_state over the whole key set.
    """
    return partial_state(q, k, v, scale=scale, allowed=allowed)
