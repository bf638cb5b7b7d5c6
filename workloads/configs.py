"""The five synthetic workloads the hot path is tested and measured on.

Each workload is shaped like one of the settings the source pages discuss:
a DiTango context-partitioned video DiT attention call (DiTango,
"Riepilogo Tecnico" -> "Metodologia") and an Efficient-vDiT frame-tile sparse
3D attention over 720p latent frames of 45 x 80 patches (Efficient-vDiT,
abstract).  The models, weights and prompt suites of the pages are not
available, so seeded N(0, 1) tensors of the same shapes stand in for them.

This module holds geometry and seeds only; none of the method's arithmetic.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    P: int                      # context partitions, equal length N // P
    F: int = 0                  # latent frames (0: no frame-tile mask)
    band_k: int = 0             # |i - j| <= band_k is always fresh
    budget: float = 1.0         # recompute budget, fraction of active pairs
    anchor: bool = True         # all active pairs fresh (no reuse)
    drift_sigma: float = 0.0    # previous-step K/V = K/V + sigma * N(0, 1)
    frame_component: float = 0.0  # per-frame shared component amplitude
    group_size: int = 0         # partitions per KV group (0: one group per partition)
    seed: int = 0
    drift_seed: int = 0
    description: str = ""

    @property
    def BH(self) -> int:
        return self.B * self.H

    @property
    def Lp(self) -> int:
        return self.N // self.P

    def part_off(self) -> List[int]:
        return [p * self.Lp for p in range(self.P + 1)]

    def frame_off(self) -> Optional[List[int]]:
        if self.F == 0:
            return None
        fl = self.N // self.F
        return [f * fl for f in range(self.F + 1)]

    def frame_mask(self) -> Optional[List[List[int]]]:
        """Frame-tile mask: frame f attends to frames f-1, f, f+1 and frame 0."""
        if self.F == 0:
            return None
        F = self.F
        return [[1 if (abs(f - g) <= 1 or g == 0) else 0 for g in range(F)]
                for f in range(F)]

    @property
    def G(self) -> int:
        """KV groups (columns of the plan)."""
        return len(self.group_off()) - 1

    def group_off(self) -> List[int]:
        """Partition offsets of the KV groups: runs of group_size adjacent partitions."""
        s = self.group_size if self.group_size > 0 else 1
        return list(range(0, self.P, s)) + [self.P]

    @property
    def grouped(self) -> bool:
        return self.group_size > 1

    @property
    def reuses(self) -> bool:
        return not self.anchor


TINY = Workload(
    name="tiny_reuse_p4", B=1, H=2, N=1024, d=64, P=4,
    band_k=1, budget=0.75, anchor=False, drift_sigma=0.05,
    seed=1, drift_seed=101,
    description="tiny oracle case: 1024 tokens in 4 partitions, band 1, 75% budget")

FRAME_TILE = Workload(
    name="frame_tile_8x3600", B=1, H=24, N=28800, d=96, P=8, F=8,
    anchor=True, frame_component=0.5, seed=2,
    description="29-frame 720p latent (8 x 45 x 80 tokens), frame-tile mask, all fresh")

DITANGO_REUSE = Workload(
    name="ditango_reuse_p32", B=1, H=40, N=76800, d=128, P=32,
    band_k=2, budget=0.25, anchor=False, drift_sigma=0.03,
    seed=3, drift_seed=103,
    description="76800 tokens in 32 partitions of 2400, band 2 + top mass to 25%")

LONG_VIDEO = Workload(
    name="long_video_24x3600", B=1, H=24, N=86400, d=96, P=24, F=24,
    band_k=1, budget=0.40, anchor=False, drift_sigma=0.03, frame_component=0.5,
    seed=4, drift_seed=104,
    description="24 latent frames x 3600 tokens, frame-tile mask, 40% budget reuse")

DENSE = Workload(
    name="dense_p16", B=2, H=24, N=32768, d=128, P=16,
    anchor=True, seed=5,
    description="all-fresh dense case, 16-way merge, equals unpartitioned attention")

DITANGO_GROUPS = Workload(
    name="ditango_groups_p32_g4", B=1, H=40, N=76800, d=128, P=32,
    band_k=2, budget=0.25, anchor=False, drift_sigma=0.03, group_size=4,
    seed=3, drift_seed=103,
    description="the 32-partition reuse case with decisions and cached states per group of "
                "4 adjacent KV partitions (8 groups): a 4x smaller cache")

ALL = [TINY, FRAME_TILE, DITANGO_REUSE, LONG_VIDEO, DENSE, DITANGO_GROUPS]
BY_NAME = {w.name: w for w in ALL}


def scaled(w: Workload, **kw) -> Workload:
    """A copy of a workload with some fields replaced (smaller parity cases)."""
    d = dict(w.__dict__)
    d.update(kw)
    return Workload(**d)
