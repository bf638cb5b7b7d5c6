"""Context partitions, the frame-tile mask and the active-pair slot table.

Efficient-vDiT, abstract: 3D attention maps of video show a tile-style
repeating pattern, and a sparse 3D attention that keeps only some frame tiles
costs time linear in the number of frames.  Here the kept tiles are given by a
frame mask M[f][g] (query frame f may attend key frame g); the workloads use
g in {f-1, f, f+1, 0}.

DiTango, Problematica / Metodologia: the sequence is split into contiguous
context partitions; attention is computed per (query partition, KV partition)
pair.  A pair (i, j) is active when some token of partition i may attend some
token of partition j.  Active pairs are numbered row-major ("slots").
"""
from __future__ import annotations

import numpy as np


def frame_of(tokens, frame_off):
    """Frame index of each token (frame_off: [F+1] increasing offsets)."""
    return np.searchsorted(np.asarray(frame_off), np.asarray(tokens), side="right") - 1


def token_allowed(rows, cols, frame_off=None, frame_mask=None):
    """bool [len(rows), len(cols)]: may query token r attend key token c."""
    rows = np.asarray(rows)
    cols = np.asarray(cols)
    if frame_off is None or frame_mask is None:
        return np.ones((rows.size, cols.size), dtype=bool)
    fm = np.asarray(frame_mask, dtype=bool)
    fr = frame_of(rows, frame_off)
    fc = frame_of(cols, frame_off)
    return fm[fr[:, None], fc[None, :]]


def pair_mask(part_off, frame_off=None, frame_mask=None):
    """A[i][j]: some token of partition i may attend some token of partition j."""
    P = len(part_off) - 1
    if frame_off is None or frame_mask is None:
        return np.ones((P, P), dtype=bool)
    A = np.zeros((P, P), dtype=bool)
    fm = np.asarray(frame_mask, dtype=bool)
    frames = [np.unique(frame_of(np.arange(part_off[p], part_off[p + 1]), frame_off))
              for p in range(P)]
    for i in range(P):
        for j in range(P):
            A[i, j] = bool(fm[np.ix_(frames[i], frames[j])].any())
    return A


def slot_table(A):
    """int [P, P]: row-major rank of each active pair, -1 where inactive."""
    A = np.asarray(A, dtype=bool)
    slot = np.full(A.shape, -1, dtype=np.int64)
    slot[A] = np.arange(int(A.sum()))
    return slot


def slot_pairs(A):
    """List of (i, j) in slot order."""
    ii, jj = np.nonzero(np.asarray(A, dtype=bool))
    return list(zip(ii.tolist(), jj.tolist()))
