"""Seeded sweep of the C ABI's host-side geometry logic (no GPU needed).

Random valid geometries -- ragged partitions, frames holding one or more
partitions or partitions cut across frames, arbitrary frame masks, optional
KV groups -- must give the
oracle's active units, slot table and state rows; random geometries with one
rule broken must be refused with the status that rule carries (invalid
argument, or a valid but unsupported shape)."""
import numpy as np
import pytest

import sparse_state_reuse_b200 as dt
from oracle import groups, masks


def random_offsets(rng, total, parts):
    cuts = np.sort(rng.choice(np.arange(1, total), size=parts - 1, replace=False))
    return [0] + [int(c) for c in cuts] + [total]


def random_geometry(rng):
    """(kwargs of dt.Geometry, frames-or-None, group_off-or-None) of a valid geometry."""
    F = int(rng.integers(0, 6))
    if F:
        frame_len = rng.integers(8, 40, size=F)
        frame_off = [0] + np.cumsum(frame_len).astype(int).tolist()
        if rng.random() < 0.5:
            # each frame split into 1..3 partitions: every partition inside one frame
            part_off = [0]
            for f in range(F):
                n = int(rng.integers(1, min(3, frame_len[f]) + 1))
                sub = random_offsets(rng, int(frame_len[f]), n)
                part_off += [frame_off[f] + s for s in sub[1:]]
        else:
            # partitions cut anywhere: some straddle frame boundaries
            N = frame_off[-1]
            P = int(rng.integers(1, min(N, 12) + 1))
            part_off = random_offsets(rng, N, P) if P > 1 else [0, N]
        mask = (rng.random((F, F)) < 0.6).astype(int)
        frames = (frame_off, mask.tolist())
    else:
        N = int(rng.integers(4, 300))
        P = int(rng.integers(1, min(N, 64) + 1))
        part_off = random_offsets(rng, N, P) if P > 1 else [0, N]
        frames = None
    P = len(part_off) - 1
    go = None
    if rng.random() < 0.5 and P > 1:
        G = int(rng.integers(1, P + 1))
        go = random_offsets(rng, P, G) if G > 1 else [0, P]
    kw = dict(B=int(rng.integers(1, 3)), H=int(rng.integers(1, 4)), N=part_off[-1],
              d=int(rng.choice([64, 96, 128])), part_off=part_off)
    return kw, frames, go


def make(kw, frames, go):
    fo, fm = frames if frames else (None, None)
    return dt.Geometry(kw["B"], kw["H"], kw["N"], kw["d"], kw["part_off"], fo, fm, group_off=go)


@pytest.mark.parametrize("seed", range(12))
def test_valid_geometries_match_the_oracle(seed):
    rng = np.random.default_rng(7000 + seed)
    for _ in range(25):
        kw, frames, go = random_geometry(rng)
        g = make(kw, frames, go)
        assert dt.ditango_check_geom(g) == 0, (kw, frames, go)
        fo, fm = frames if frames else (None, None)
        A = masks.pair_mask(kw["part_off"], fo, fm)
        Au = groups.unit_mask(A, go) if go is not None else A
        assert dt.ditango_num_active(g) == int(Au.sum())
        assert (np.array(dt.ditango_slot_table(g)).reshape(Au.shape) == masks.slot_table(Au)).all()
        assert dt.ditango_state_rows(g) == max(np.diff(kw["part_off"]))


INVALID, UNSUPPORTED = 1, 2


def broken(rng, kw, frames, go):
    """One rule broken at random: (kwargs, frames, group_off, expected status)."""
    kw = dict(kw)
    po = list(kw["part_off"])
    P = len(po) - 1
    choice = int(rng.integers(0, 8))
    if choice == 0 and P > 1:                     # an empty partition
        k = int(rng.integers(1, P))
        po[k] = po[k - 1]
        kw["part_off"] = po
        return kw, frames, go, INVALID
    if choice == 1:                               # offsets that do not end at N
        kw["N"] = po[-1] + 1
        return kw, frames, go, INVALID
    if choice == 2:                               # a head dim without a kernel
        kw["d"] = int(rng.choice([32, 80, 256]))
        return kw, frames, go, UNSUPPORTED
    if choice == 3 and P > 1:                     # groups that do not end at P
        return kw, frames, [0, P - 1], INVALID
    if choice == 4 and P > 2:                     # groups that do not rise
        return kw, frames, [0, 2, 1, P], INVALID
    if choice == 5 and frames and len(frames[0]) > 2:
        # frame offsets that do not rise
        fo = list(frames[0])
        fo[1] = fo[2]
        return kw, (fo, frames[1]), go, INVALID
    if choice == 6:
        kw["B"] = 0
        return kw, frames, go, INVALID
    # B*H beyond the merge's grid: unsupported
    kw["B"], kw["H"] = 256, 257
    return kw, frames, go, UNSUPPORTED


@pytest.mark.parametrize("seed", range(8))
def test_broken_geometries_are_refused_with_their_status(seed):
    rng = np.random.default_rng(9000 + seed)
    for _ in range(25):
        kw, frames, go, status = broken(rng, *random_geometry(rng))
        g = make(kw, frames, go)
        assert dt.ditango_check_geom(g) == status, (kw, frames, go)
        with pytest.raises(dt.DitangoError) as e:     # the C call returns -1
            dt.ditango_num_active(g)
        assert e.value.status == status
