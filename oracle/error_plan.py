"""Error-growth planner with anchor scheduling.

Test infrastructure: plain fp64 NumPy, independent of the CUDA path.

DiTango, "Riepilogo Tecnico" -> Metodologia -> 1. Anchor-Guided Selection
Planner:
  * "Modellazione dell'Errore": the error accumulated by reusing an attention
    state from an earlier step is a function of the partition's importance w
    and of the temporal growth of the error, delta;
  * "Anchor Steps": periodic steps recompute every partition, which resets
    the accumulated error and refreshes the importance weights;
  * "Predizione Online": between anchors the planner predicts the growth of
    the error from the change of the local states -- always computed -- as a
    proxy for how the remote states evolve.

Readings (the pages print no formula; these are the plainest that fit):
  * the local state of query partition i is its unit that holds partition i
    itself (the diagonal pair without KV groups); it is in the band, so it is
    fresh at every step;
  * local drift delta_i: the mean over (b, h, rows r of partition i) of
    |lse_loc[r] (this step) - lse_loc[r] (previous step)|, the change of the
    local state's log-sum-exp (equal values, -inf included, change by 0);
    0 when the local state did not exist before the step;
  * age a of a cached state: the local drift accumulated since the state was
    computed -- 0 after a step that computed it, a + delta_i after a step that
    reused it;
  * predicted error of reusing unit (i, c) at the next step:
    w_ic * (a_ic + delta_i), the last measured drift standing in for the next
    step's;
  * selection: the rule of oracle.plan (band and invalid slots fresh, then
    the largest scores up to the budget, float32 ranking, ties to the lower
    index) with the predicted error in place of w;
  * w is computed from the cache (oracle.plan.mass_scores) by the first plan
    after an anchor step and held until the next anchor; step 0 and every
    `anchor_every`-th step after it are anchors.
Parity of the error model's predictive quality is unpinned: the pages give
no formula and no values; the tests pin the rules above and their invariants.
"""
from __future__ import annotations

import numpy as np

from .attention import merge_states
from .groups import unit_band, unit_mask, unit_state
from .masks import slot_pairs, slot_table
from .plan import PLAN_FRESH, mass_scores, select


def local_unit(i, group_off):
    """Column of the unit of query partition i that holds partition i."""
    g = list(group_off)
    for c in range(len(g) - 1):
        if g[c] <= i < g[c + 1]:
            return c
    raise ValueError("partition outside the groups")


def local_delta(lse_new, lse_old):
    """Mean |lse_new - lse_old| over all rows (equal entries, -inf included, give 0)."""
    a = np.asarray(lse_new, dtype=np.float64).ravel()
    b = np.asarray(lse_old, dtype=np.float64).ravel()
    same = a == b
    d = np.zeros(a.shape)
    d[~same] = np.abs(a[~same] - b[~same])
    return float(d.mean()) if d.size else 0.0


def age_update(age, prev_plan, A_units, delta):
    """New age per slot (slot order of A_units) after a step with prev_plan."""
    age = np.asarray(age, dtype=np.float64).copy()
    for s, (i, c) in enumerate(slot_pairs(A_units)):
        age[s] = 0.0 if prev_plan[i, c] == PLAN_FRESH else age[s] + delta[i]
    return age


def error_scores(w, age, delta, A_units):
    """Predicted error [P, G] of reusing each active unit at the next step."""
    score = np.zeros(A_units.shape, dtype=np.float64)
    for s, (i, c) in enumerate(slot_pairs(A_units)):
        score[i, c] = w[i, c] * (age[s] + delta[i])
    return score


def plan_error(w, age, prev_plan, delta, A_units, band, budget, valid=None,
               rank_dtype=np.float32):
    """One non-anchor plan: (plan, fresh_list, new_age, score)."""
    new_age = age_update(age, prev_plan, A_units, delta)
    score = error_scores(w, new_age, delta, A_units)
    plan, fl = select(score, A_units, 0, budget, valid=valid, rank_dtype=rank_dtype, band=band)
    return plan, fl, new_age, score


class Schedule:
    """Multi-step driver: anchor steps, online drift, error-guided reuse.

    q: [BH][N, d] fp64 query slabs (fixed over steps); k_steps/v_steps:
    [S+1][BH][N, d] fp64 K/V per denoising step.  Each call of step(s) plans,
    computes the fresh unit states from step s's K/V (the stale ones stay in
    the cache), records the local drift rows, and returns the merged output of
    every row.
    """

    def __init__(self, q, part_off, group_off, A, band_k, budget, anchor_every,
                 frame_off=None, frame_mask=None):
        self.q = q
        self.BH = len(q)
        self.po = list(part_off)
        self.go = list(group_off)
        self.P = len(self.po) - 1
        self.A = np.asarray(A, dtype=bool)
        self.Au = unit_mask(self.A, self.go)
        self.band = unit_band(self.A, self.go, band_k)
        self.budget = budget
        self.anchor_every = anchor_every
        self.fo, self.fm = frame_off, frame_mask
        self.slots = slot_pairs(self.Au)
        self.slot = slot_table(self.Au)
        self.Lmax = max(np.diff(self.po))
        n = len(self.slots)
        d = q[0].shape[1]
        self.O = np.zeros((n, self.BH, self.Lmax, d))
        self.lse = np.full((n, self.BH, self.Lmax), -np.inf)
        self.valid = np.zeros(n, dtype=bool)
        self.w = np.zeros(self.Au.shape)
        self.age = np.zeros(n)
        self.prev_plan = np.zeros(self.Au.shape, dtype=np.int8)
        self.delta = np.zeros(self.P)
        self.delta_rows = [None] * self.P
        self.local_ok = np.zeros(self.P, dtype=bool)
        self.local_c = [local_unit(i, self.go) for i in range(self.P)]

    def is_anchor(self, s):
        return s % self.anchor_every == 0

    def plan(self, s):
        """Plan of step s; also the planner state it leaves for step s + 1."""
        valid_pp = np.ones(self.Au.shape, dtype=bool)
        valid_pp[self.Au] = self.valid
        if self.is_anchor(s):
            plan = np.where(self.Au, PLAN_FRESH, 0).astype(np.int8)
            score = np.zeros(self.Au.shape)
        else:
            if self.is_anchor(s - 1):
                self.w = mass_scores(self.lse, self.Au, self.po, valid=self.valid)
            self.delta = np.array([self.delta_rows[i] if self.local_ok[i] else 0.0
                                   for i in range(self.P)])
            plan, _, self.age, score = plan_error(self.w, self.age, self.prev_plan, self.delta,
                                                  self.Au, self.band, self.budget, valid=valid_pp)
        self.local_ok = np.array([bool(self.Au[i, self.local_c[i]]) and
                                  bool(self.valid[self.slot[i, self.local_c[i]]])
                                  for i in range(self.P)])
        return plan, score

    def step(self, s, k, v, plan_override=None):
        """k, v: [BH][N, d] of step s.  Returns (plan, score, O [BH][N, d], lse [BH][N]).

        plan_override: execute this plan instead of the one planned (the
        planner state still advances from the planned scores and the
        executed plan), so that a run of another implementation can be
        followed step by step; the plan the oracle made itself is kept in
        self.planned."""
        plan, score = self.plan(s)
        self.planned = plan          # the oracle's own plan, before any override
        if plan_override is not None:
            plan = np.asarray(plan_override, dtype=np.int8).reshape(self.Au.shape)
        N, d = self.q[0].shape
        out_O = np.zeros((self.BH, N, d))
        out_l = np.full((self.BH, N), -np.inf)
        for i in range(self.P):
            rows = np.arange(self.po[i], self.po[i + 1])
            L = rows.size
            drift = []
            for c in range(self.Au.shape[1]):
                if plan[i, c] != PLAN_FRESH:
                    continue
                sl = self.slot[i, c]
                for bh in range(self.BH):
                    O, l = unit_state(self.q[bh][rows], rows, k[bh], v[bh], self.po, self.go, c,
                                      self.fo, self.fm)
                    if c == self.local_c[i]:
                        drift.append((l, self.lse[sl, bh, :L].copy()))
                    self.O[sl, bh, :L] = O
                    self.lse[sl, bh, :L] = l
                self.valid[sl] = True
            if drift:
                self.delta_rows[i] = local_delta(np.concatenate([a for a, _ in drift]),
                                                 np.concatenate([b for _, b in drift]))
            for bh in range(self.BH):
                states = [(self.O[self.slot[i, c], bh, :L], self.lse[self.slot[i, c], bh, :L])
                          for c in range(self.Au.shape[1]) if plan[i, c] != 0]
                if states:
                    out_O[bh, rows], out_l[bh, rows] = merge_states(states)
        self.prev_plan = plan
        return plan, score, out_O, out_l
