"""KV groups: fresh/reuse decisions and cached states per run of adjacent
partitions, and the recursive composition of cached states into coarser groups.

Test infrastructure: plain fp64 NumPy, independent of the CUDA path.

DiTango, "Riepilogo Tecnico" -> Metodologia:
  * 1. Anchor-Guided Selection Planner, "Strategia per Gruppi": spatially
    adjacent partitions are grouped and the fresh/reuse decision is taken per
    group rather than per partition;
  * 2. State-Centric Parallel Runtime, "Calcolo dello Stato di Gruppo": the
    state a group produces is the complete composed state of a query
    partition against the KV of the whole group;
  * "Composizione Dinamica dei Gruppi": under memory pressure the stored
    states are merged recursively into coarser groups, which shrinks the cache
    without recomputing anything;
  * "Composizione dello Stato": states combine associatively and
    commutatively by their output and log-sum-exp.

Readings of what the pages leave open (the plainest that fit the rest):
  * a KV group is a contiguous run of partitions, given by offsets into the
    partition list (group_off[0] = 0 < ... < group_off[G] = P); the query side
    stays one partition, so the unit of decision and of storage is
    (query partition i, KV group c);
  * the state of unit (i, c) is attention of the rows of i against every key
    of the partitions of c that the frame mask allows; unit (i, c) is active
    when some pair (i, j), j in c, is;
  * unit (i, c) is in the distance band when some active pair (i, j) with j
    in c has |i - j| <= k;
  * mass score, budget and ranking are the pair rules of oracle.plan applied
    to units (fresh count max(|band|, floor(budget * |active units|)));
  * the cached state of a coarse unit is the composition of the cached states
    of the fine units it covers, and is valid only when all of them are.
With one group per partition every function here reduces to the pair form.
"""
from __future__ import annotations

import numpy as np

from .attention import partial_state, merge_states
from .masks import token_allowed, slot_pairs
from .plan import PLAN_FRESH, PLAN_REUSE


def uniform_group_off(P, size):
    """Groups of `size` adjacent partitions (the last one may be shorter)."""
    if size <= 0:
        size = 1
    off = list(range(0, P, size)) + [P]
    return off


def check_group_off(group_off, P):
    g = [int(x) for x in group_off]
    if g[0] != 0 or g[-1] != P or any(b <= a for a, b in zip(g, g[1:])):
        raise ValueError("group offsets must rise strictly from 0 to P")
    return g


def unit_mask(A, group_off):
    """A_G [P, G]: unit (i, c) is active when some pair (i, j), j in c, is."""
    A = np.asarray(A, dtype=bool)
    g = check_group_off(group_off, A.shape[1])
    return np.stack([A[:, g[c]:g[c + 1]].any(axis=1) for c in range(len(g) - 1)], axis=1)


def unit_band(A, group_off, band_k):
    """[P, G]: some active pair (i, j) with j in group c has |i - j| <= band_k."""
    A = np.asarray(A, dtype=bool)
    ii, jj = np.indices(A.shape)
    near = A & (np.abs(ii - jj) <= band_k)
    return unit_mask(near, group_off)


def unit_keys(part_off, group_off, c):
    """Global token ids of the keys of KV group c."""
    return np.arange(part_off[group_off[c]], part_off[group_off[c + 1]])


def unit_state(q_rows, rows, k, v, part_off, group_off, c, frame_off=None, frame_mask=None,
               scale=None):
    """State (O, lse) of query rows against every allowed key of KV group c."""
    cols = unit_keys(part_off, group_off, c)
    allowed = None
    if frame_off is not None and frame_mask is not None:
        allowed = token_allowed(rows, cols, frame_off, frame_mask)
    return partial_state(q_rows, k[cols], v[cols], scale=scale, allowed=allowed)


def step_rows_units(q, k, v, k_prev, v_prev, plan_u, part_off, group_off, i, rows,
                    frame_off=None, frame_mask=None, scale=None):
    """Final (O, lse) of rows of partition i for one (b, h) under a unit plan.

    plan_u: [P, G] codes; fresh units use k, v, reused ones k_prev, v_prev
    (the state a cache built at the previous step holds).
    """
    rows = np.asarray(rows)
    qr = q[rows]
    states = []
    for c in range(plan_u.shape[1]):
        code = int(plan_u[i, c])
        if code == PLAN_FRESH:
            states.append(unit_state(qr, rows, k, v, part_off, group_off, c, frame_off, frame_mask, scale))
        elif code == PLAN_REUSE:
            states.append(unit_state(qr, rows, k_prev, v_prev, part_off, group_off, c,
                                     frame_off, frame_mask, scale))
    if not states:
        return np.zeros((rows.size, v.shape[1])), np.full(rows.size, -np.inf)
    return merge_states(states)


def unit_cache(q, k_prev, v_prev, A_units, part_off, group_off, frame_off=None, frame_mask=None,
               scale=None, Lmax=None):
    """Cached states of every active unit for one (b, h).

    Returns O [slots, Lmax, d] and lse [slots, Lmax] in slot order (row-major
    active units); rows past a partition's end hold O = 0, lse = -inf.
    """
    P = A_units.shape[0]
    if Lmax is None:
        Lmax = max(part_off[p + 1] - part_off[p] for p in range(P))
    Os, ls = [], []
    for i, c in slot_pairs(A_units):
        rows = np.arange(part_off[i], part_off[i + 1])
        O, lse = unit_state(q[rows], rows, k_prev, v_prev, part_off, group_off, c,
                            frame_off, frame_mask, scale)
        Op = np.zeros((Lmax, k_prev.shape[1]))
        lp = np.full(Lmax, -np.inf)
        Op[:rows.size] = O
        lp[:rows.size] = lse
        Os.append(Op)
        ls.append(lp)
    return np.stack(Os), np.stack(ls)


def compose_cache(cache_O, cache_lse, valid, A, fine_off, coarse_off, part_off):
    """Merge cached unit states of a fine grouping into a coarser one.

    One (b, h): cache_O [slots_f, Lmax, d], cache_lse [slots_f, Lmax] in fine
    slot order, valid bool [slots_f].
    A: [P, P] pair mask.  Every coarse group must be a union of fine groups.
    Returns (O, lse, valid) in coarse slot order; a coarse state is valid only
    when every fine state it covers is, and rows past a partition's end stay
    O = 0, lse = -inf.
    """
    A = np.asarray(A, dtype=bool)
    P = A.shape[0]
    fo = check_group_off(fine_off, P)
    co = check_group_off(coarse_off, P)
    if not set(co) <= set(fo):
        raise ValueError("every coarse group must be a union of fine groups")
    Af = unit_mask(A, fo)
    Ac = unit_mask(A, co)
    slot_f = {pc: s for s, pc in enumerate(slot_pairs(Af))}
    cache_O = np.asarray(cache_O, dtype=np.float64)
    cache_lse = np.asarray(cache_lse, dtype=np.float64)
    valid = np.asarray(valid, dtype=bool)
    out_O, out_l, out_v = [], [], []
    for i, C in slot_pairs(Ac):
        Li = part_off[i + 1] - part_off[i]
        members = [slot_f[(i, c)] for c in range(len(fo) - 1)
                   if co[C] <= fo[c] and fo[c + 1] <= co[C + 1] and (i, c) in slot_f]
        O = np.zeros(cache_O.shape[1:])
        lse = np.full(cache_lse.shape[1:], -np.inf)
        ok = bool(valid[members].all())
        if ok:
            O_rows, l_rows = merge_states([(cache_O[s, :Li], cache_lse[s, :Li]) for s in members])
            O[:Li] = O_rows
            lse[:Li] = l_rows
        out_O.append(O)
        out_l.append(lse)
        out_v.append(ok)
    return np.stack(out_O), np.stack(out_l), np.array(out_v, dtype=bool)
