"""Fresh-versus-reuse plan over (query partition, KV partition) pairs.

DiTango, "Riepilogo Tecnico" -> Metodologia:
  * spatial locality: partitions close to the query's contribute far more
    than distant ones -> the pairs within a distance band are always fresh;
  * 1. Anchor-Guided Selection Planner, "Modellazione dell'Errore": the error
    of reusing a stale attention state grows with the partition's importance
    w -> outside the band, the pairs with the largest w are recomputed first;
  * "Anchor Steps": periodic steps recompute every partition (all fresh) and
    refresh w.

Readings of what the pages leave open (the plainest ones that fit the rest):
  * w[i][j] = mean over (batch, head, row r of partition i) of the share of
    row r's softmax denominator that partition j holds in the cached states:
    exp(lse_ij[r] - LSE_i[r]), LSE_i[r] = log sum_{j active} exp(lse_ij[r]);
  * the number of fresh pairs is max(|band|, floor(budget * |active| + 1e-9));
    the band is fresh even above the budget; the budget fills with the
    highest-w active pairs outside the band;
  * equal w: the lower linear index i * P + j is taken first;
  * a pair whose cache slot was never written is fresh regardless of budget
    and holds no mass;
  * one plan per (i, j), shared by every batch entry and head;
  * the ranking decision is taken on w rounded to float32 (the precision the
    CUDA path holds w in).
"""
from __future__ import annotations

import math

import numpy as np

PLAN_SKIP, PLAN_FRESH, PLAN_REUSE = 0, 1, 2


def mass_scores(cache_lse, A, part_off, valid=None):
    """w [P, C] (fp64) from cached log-sum-exps.

    A: [P, C] active mask, one row per query partition and one column per KV
    partition (C = P) or per KV group (see oracle.groups).
    cache_lse: [slots, BH, Lmax] array indexed by slot (row-major rank of the
    active entry); row r of entry (i, j) is cache_lse[slot(i,j), :, r] for
    r < L_i.  Inactive entries get w = 0.  valid: optional bool [slots]; a
    slot that was never written holds no state and therefore no mass.
    """
    A = np.asarray(A, dtype=bool)
    P = A.shape[0]
    lse_all = np.asarray(cache_lse)
    if valid is not None:
        lse_all = np.where(np.asarray(valid, dtype=bool)[:, None, None], lse_all, -np.inf)
    w = np.zeros(A.shape, dtype=np.float64)
    slot = 0
    for i in range(P):
        js = np.nonzero(A[i])[0]
        if js.size == 0:
            continue
        Li = part_off[i + 1] - part_off[i]
        lse = lse_all[slot:slot + js.size, :, :Li].astype(np.float64)  # [J, BH, Li]
        slot += js.size
        M = lse.max(axis=0)
        dead = ~np.isfinite(M)
        M0 = np.where(dead, 0.0, M)
        share = np.exp(lse - M0[None])                  # [J, BH, Li]
        tot = share.sum(axis=0)
        share = share / np.where(dead, 1.0, tot)[None]
        share[:, dead] = 0.0
        w[i, js] = share.reshape(js.size, -1).mean(axis=1)
    return w


def budget_target(n_band, n_active, budget):
    return max(int(n_band), int(math.floor(float(budget) * int(n_active) + 1e-9)))


def select(w, A, band_k, budget, anchor=False, valid=None, rank_dtype=np.float32, band=None):
    """Plan int8 [P, C] in {0 skip, 1 fresh, 2 reuse} and the fresh list.

    The fresh list holds the linear indices i * C + j of the fresh entries
    in row-major order.  The band is |i - j| <= band_k on a square A; a
    caller with KV groups passes its own band mask (oracle.groups.unit_band).
    """
    A = np.asarray(A, dtype=bool)
    P, C = A.shape
    ii, jj = np.meshgrid(np.arange(P), np.arange(C), indexing="ij")
    fresh = np.zeros((P, C), dtype=bool)
    if anchor:
        fresh[:] = A
    else:
        if band is None:
            band = A & (np.abs(ii - jj) <= band_k)
        else:
            band = A & np.asarray(band, dtype=bool)
        fresh |= band
        if valid is not None:
            fresh |= A & ~np.asarray(valid, dtype=bool)
        target = budget_target(band.sum(), A.sum(), budget)
        need = target - int(fresh.sum())
        if need > 0:
            cand = np.nonzero((A & ~fresh).ravel())[0]
            key = np.asarray(w, dtype=np.float64).ravel()[cand].astype(rank_dtype)
            order = sorted(range(cand.size), key=lambda t: (-float(key[t]), int(cand[t])))
            for t in order[:need]:
                fresh.flat[cand[t]] = True
    plan = np.where(fresh, PLAN_FRESH, np.where(A, PLAN_REUSE, PLAN_SKIP)).astype(np.int8)
    fresh_list = np.nonzero(fresh.ravel())[0].astype(np.int32)
    return plan, fresh_list
