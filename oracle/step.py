"""One attention call with selective state reuse, composed from the pieces.

DiTango, "Riepilogo Tecnico" -> Metodologia: for each (query partition i,
KV partition j) pair the planner either recomputes the attention state from
the current K/V ("fresh") or reuses the state cached at the previous
denoising step ("reuse"); 2. State-Centric Parallel Runtime,
"Composizione dello Stato": the final output of row r is the composition of
the states of all active pairs of its partition.  Efficient-vDiT, abstract:
pairs the frame-tile mask rules out contribute nothing.

Readings: the cached state of pair (i, j) is the state of the current Q rows
against the previous step's K/V of partition j (only K/V drift between
steps); a fresh state uses the current K/V.
"""
from __future__ import annotations

import numpy as np

from .attention import partial_state, merge_states
from .masks import token_allowed
from .plan import PLAN_FRESH, PLAN_REUSE


def partition_of(token, part_off):
    return int(np.searchsorted(np.asarray(part_off), token, side="right") - 1)


def pair_state(q_rows, rows, k, v, part_off, j, frame_off=None, frame_mask=None, scale=None):
    """State of query rows (global token ids `rows`, values q_rows) against KV partition j."""
    cols = np.arange(part_off[j], part_off[j + 1])
    allowed = None
    if frame_off is not None and frame_mask is not None:
        allowed = token_allowed(rows, cols, frame_off, frame_mask)
    return partial_state(q_rows, k[cols], v[cols], scale=scale, allowed=allowed)


def step_rows(q, k, v, k_prev, v_prev, plan, part_off, i, rows,
              frame_off=None, frame_mask=None, scale=None):
    """Final (O, lse) of the given rows of partition i for one (b, h).

    q, k, v, k_prev, v_prev: [N, d] fp64 slabs; plan: [P, P] codes.
    Returns (O, lse, states) with states = {j: (O_j, lse_j, source)}.
    """
    rows = np.asarray(rows)
    qr = q[rows]
    states = {}
    for j in range(plan.shape[1]):
        code = int(plan[i, j])
        if code == PLAN_FRESH:
            st = pair_state(qr, rows, k, v, part_off, j, frame_off, frame_mask, scale)
        elif code == PLAN_REUSE:
            st = pair_state(qr, rows, k_prev, v_prev, part_off, j, frame_off, frame_mask, scale)
        else:
            continue
        states[j] = (st[0], st[1], code)
    if not states:
        return np.zeros((rows.size, v.shape[1])), np.full(rows.size, -np.inf), states
    O, lse = merge_states([(s[0], s[1]) for s in states.values()])
    return O, lse, states


def cache_lse_for_slab(q, k_prev, v_prev, A, part_off, frame_off=None, frame_mask=None,
                       scale=None, Lmax=None):
    """Cached lse of every active pair for one (b, h): [slots, Lmax] (pad -inf)."""
    P = A.shape[0]
    if Lmax is None:
        Lmax = max(part_off[p + 1] - part_off[p] for p in range(P))
    out = []
    for i in range(P):
        rows = np.arange(part_off[i], part_off[i + 1])
        for j in range(P):
            if not A[i, j]:
                continue
            _, lse = pair_state(q[rows], rows, k_prev, v_prev, part_off, j,
                                frame_off, frame_mask, scale)
            pad = np.full(Lmax, -np.inf)
            pad[:rows.size] = lse
            out.append(pad)
    return np.stack(out)
