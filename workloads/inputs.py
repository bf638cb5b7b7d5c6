"""Seeded synthetic inputs shared by the oracle tests and the CUDA path.

Every (tensor, b, h) slab [N, d] is drawn from its own PCG64 stream, keyed by
(seed, tensor id, b, h), so any slab can be regenerated on its own: the
oracle checks sampled rows of the full-size workloads without materialising
the whole tensor.  Values are N(0, 1) in float32, optionally plus a per-frame
shared component (amplitude * one N(0, 1) vector per (tensor, b, h, frame)),
then rounded to bfloat16 (round to nearest, ties to even).  The previous
denoising step's K/V are bf16(current + sigma * N(0, 1)) from a separate
stream keyed by the drift seed.  A multi-step sequence (denoising steps
s = 0, 1, ...) keeps Q fixed and lets K/V walk: step s adds
sigma * (e_1 + ... + e_s) to the workload's tensor in float32, one N(0, 1)
stream per (drift seed, tensor, b, h, step), then rounds to bf16.

Nothing here computes attention, plans or merges.
"""
from __future__ import annotations

from concurrent.futures import ThreadPoolExecutor
import os

import numpy as np

from .configs import Workload

TENSOR_ID = {"q": 11, "k": 12, "v": 13}


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


def _fresh_f32(w: Workload, which: str, b: int, h: int) -> np.ndarray:
    tid = TENSOR_ID[which]
    x = _rng(w.seed, tid, b, h).standard_normal((w.N, w.d), dtype=np.float32)
    if w.frame_component and w.F:
        s = _rng(w.seed, tid, b, h, 7).standard_normal((w.F, w.d), dtype=np.float32)
        fl = w.N // w.F
        x = x.reshape(w.F, fl, w.d)
        x += np.float32(w.frame_component) * s[:, None, :]
        x = x.reshape(w.N, w.d)
    return x


def slab(w: Workload, which: str, b: int, h: int) -> np.ndarray:
    """bf16 bits [N, d] of Q, K or V for one (b, h)."""
    return bf16_bits(_fresh_f32(w, which, b, h))


def prev_slab(w: Workload, which: str, b: int, h: int) -> np.ndarray:
    """bf16 bits [N, d] of the previous step's K or V for one (b, h)."""
    assert which in ("k", "v")
    cur = bf16_to_f32(slab(w, which, b, h))
    eps = _rng(w.drift_seed, TENSOR_ID[which], b, h).standard_normal(
        (w.N, w.d), dtype=np.float32)
    return bf16_bits(cur + np.float32(w.drift_sigma) * eps)


def slab_f64(w: Workload, which: str, b: int, h: int, prev: bool = False) -> np.ndarray:
    bits = prev_slab(w, which, b, h) if prev else slab(w, which, b, h)
    return bf16_to_f32(bits).astype(np.float64)


def step_slabs(w: Workload, which: str, b: int, h: int, steps: int):
    """bf16 bits [N, d] of K or V at denoising steps 0..steps of the walk."""
    assert which in ("k", "v")
    x = bf16_to_f32(slab(w, which, b, h))
    out = [bf16_bits(x)]
    acc = np.zeros_like(x)
    for s in range(1, steps + 1):
        acc += _rng(w.drift_seed, TENSOR_ID[which], b, h, 1000 + s).standard_normal(
            (w.N, w.d), dtype=np.float32)
        out.append(bf16_bits(x + np.float32(w.drift_sigma) * acc))
    return out


def step_full(w: Workload, which: str, steps: int, threads: int = 0):
    """bf16 bits [steps + 1, B, H, N, d] of K or V along the walk."""
    out = np.empty((steps + 1, w.B, w.H, w.N, w.d), dtype=np.uint16)

    def work(bh):
        b, h = divmod(bh, w.H)
        for s, x in enumerate(step_slabs(w, which, b, h, steps)):
            out[s, b, h] = x

    threads = threads or min(16, os.cpu_count() or 1)
    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(work, range(w.BH)))
    return out


def full(w: Workload, which: str, prev: bool = False, threads: int = 0) -> np.ndarray:
    """bf16 bits [B, H, N, d] of a whole tensor (slabs drawn in parallel)."""
    out = np.empty((w.B, w.H, w.N, w.d), dtype=np.uint16)
    fn = prev_slab if prev else slab

    def work(bh):
        b, h = divmod(bh, w.H)
        out[b, h] = fn(w, which, b, h)

    threads = threads or min(16, os.cpu_count() or 1)
    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(work, range(w.BH)))
    return out


def synthetic_cache_lse(w: Workload, n_slots: int, slot_pairs, seed: int,
                        decay: float = 0.35, noise: float = 0.5) -> np.ndarray:
    """A cache log-sum-exp array [slots, B*H, Lp] (float32) with DiTango-like
    structure: lse_ij[r] = c[r] - decay * |i - j| + noise * N(0, 1).
    Used to drive the plan at full size without computing attention."""
    rng = _rng(seed, 99)
    Lp = w.Lp
    base = np.float32(np.log(Lp)) + rng.standard_normal((w.BH, Lp), dtype=np.float32)
    out = np.empty((n_slots, w.BH, Lp), dtype=np.float32)
    for s, (i, j) in enumerate(slot_pairs):
        out[s] = base - np.float32(decay * abs(i - j)) + np.float32(noise) * \
            rng.standard_normal((w.BH, Lp), dtype=np.float32)
    return out
