"""ctypes binding of libditango.so (include/ditango.h).

Argument marshalling only: every step of the hot path runs in the library's
CUDA kernels.  Device buffers may be passed as torch tensors (their
data_ptr is used), as integer addresses, or as None for optional ones.  A
non-OK status raises DitangoError.  The library must exist: there is no
fallback of any kind.
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# DITANGO_LIBRARY selects another build of the same ABI, e.g. the checked
# build libditango_check.so
LIB_PATH = os.environ.get("DITANGO_LIBRARY") or os.path.join(_HERE, "libditango.so")

OK, ERR_INVALID, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_BOUNDS = 0, 1, 2, 3, 4, 5
PLAN_SKIP, PLAN_FRESH, PLAN_REUSE = 0, 1, 2


class DitangoError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn}: {status_string(status)} (status {status})")


class ditango_geom(C.Structure):
    _fields_ = [
        ("B", C.c_int32), ("H", C.c_int32), ("N", C.c_int32), ("d", C.c_int32),
        ("P", C.c_int32), ("F", C.c_int32),
        ("part_off", C.POINTER(C.c_int32)),
        ("frame_off", C.POINTER(C.c_int32)),
        ("frame_mask", C.POINTER(C.c_uint8)),
        ("q_strides", C.c_int64 * 3),
        ("k_strides", C.c_int64 * 3),
        ("v_strides", C.c_int64 * 3),
        ("G", C.c_int32),
        ("group_off", C.POINTER(C.c_int32)),
    ]


class ditango_error_state(C.Structure):
    _fields_ = [
        ("w", C.c_void_p), ("age", C.c_void_p), ("delta", C.c_void_p),
        ("local_ok", C.c_void_p), ("drift_rows", C.c_void_p),
    ]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python sparse_state_reuse_b200/build.py` "
            "(nvcc, sm_100a). There is no CPU fallback.")
    return C.CDLL(LIB_PATH)


_lib = _load()
_P = C.c_void_p
_G = C.POINTER(ditango_geom)
_SIGS = {
    "ditango_version": (C.c_int32, []),
    "ditango_status_string": (C.c_char_p, [C.c_int32]),
    "ditango_check_geom": (C.c_int, [_G]),
    "ditango_num_active": (C.c_int64, [_G]),
    "ditango_state_rows": (C.c_int64, [_G]),
    "ditango_slot_table": (C.c_int, [_G, _P]),
    "ditango_plan_workspace_size": (C.c_size_t, [_G]),
    "ditango_workspace_size": (C.c_size_t, [_G]),
    "ditango_plan": (C.c_int, [_G, _P, _P, C.c_int32, C.c_double, C.c_int32, _P, _P, _P, _P, _P,
                               C.c_size_t, _P]),
    "ditango_attn_partial": (C.c_int, [_G, _P, _P, _P, _P, _P, C.c_float, _P, _P, C.c_int32,
                                       C.c_int32, _P, _P, _P, _P, _P]),
    "ditango_plan_error": (C.c_int, [_G, _P, _P, C.c_int32, C.c_double, C.c_int32, C.c_int32,
                                     C.POINTER(ditango_error_state), _P, _P, _P, _P, _P,
                                     C.c_size_t, _P]),
    "ditango_plan_from_mass": (C.c_int, [_G, _P, C.c_size_t, _P, C.c_int32, C.c_double, _P, _P,
                                         _P, _P, _P]),
    "ditango_merge": (C.c_int, [_G, _P, _P, _P, _P, _P, _P, C.c_int32, C.c_int32, _P, C.c_int32,
                                _P, _P, _P, _P]),
    "ditango_cache_update": (C.c_int, [_G, _P, _P, _P, _P, _P, _P, C.c_int32, _P]),
    "ditango_plan_noalloc": (C.c_int, [_G, _P, _P, C.c_int32, C.c_double, C.c_int32, _P, _P, _P,
                                       _P, _P]),
    "ditango_cache_compose": (C.c_int, [_G, _G, _P, _P, _P, _P, _P, _P, C.c_int32, _P]),
    "ditango_set_wait_limit_ns": (None, [C.c_int64]),
    "ditango_checked_build": (C.c_int32, []),
    "ditango_check_status": (C.c_int, [_P, C.c_int32]),
    "ditango_selftest_bounded_wait": (C.c_int, [C.c_int64, _P, _P]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args

EXPORTED = tuple(_SIGS)


def status_string(s: int) -> str:
    return _lib.ditango_status_string(int(s)).decode()


def _ptr(x):
    """Device address of a tensor (or an address given as an int)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if getattr(x, "is_cuda", True) is False:
        # a host tensor's address would be dereferenced by a kernel
        raise ValueError(f"a CUDA tensor is required here, got one on {x.device}")
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(fn, st):
    if st != OK:
        raise DitangoError(fn, st)


class Geometry:
    """Owns the host arrays a ditango_geom points to.

    group_off: partition offsets of the KV groups (None: one group per
    partition); G, the number of plan columns, is len(group_off) - 1.
    """

    def __init__(self, B, H, N, d, part_off, frame_off=None, frame_mask=None,
                 q_strides=None, k_strides=None, v_strides=None, group_off=None):
        P = len(part_off) - 1
        F = 0 if frame_off is None else len(frame_off) - 1
        self._part = (C.c_int32 * (P + 1))(*[int(x) for x in part_off])
        self._groups = None
        if group_off is not None:
            self._groups = (C.c_int32 * len(group_off))(*[int(x) for x in group_off])
        self._frame = None
        self._fmask = None
        if F:
            self._frame = (C.c_int32 * (F + 1))(*[int(x) for x in frame_off])
            flat = [int(bool(v)) for row in frame_mask for v in row]
            self._fmask = (C.c_uint8 * (F * F))(*flat)
        contig = (H * N * d, N * d, d)
        g = ditango_geom()
        g.B, g.H, g.N, g.d, g.P, g.F = B, H, N, d, P, F
        g.part_off = C.cast(self._part, C.POINTER(C.c_int32))
        g.frame_off = C.cast(self._frame, C.POINTER(C.c_int32)) if F else None
        g.frame_mask = C.cast(self._fmask, C.POINTER(C.c_uint8)) if F else None
        g.G = 0 if group_off is None else len(group_off) - 1
        g.group_off = C.cast(self._groups, C.POINTER(C.c_int32)) if group_off is not None else None
        for name, s in (("q_strides", q_strides), ("k_strides", k_strides), ("v_strides", v_strides)):
            getattr(g, name)[:] = list(s if s is not None else contig)
        self.g = g
        self.B, self.H, self.N, self.d, self.P, self.F = B, H, N, d, P, F
        self.group_off = None if group_off is None else [int(x) for x in group_off]
        self.G = P if group_off is None else len(group_off) - 1

    @property
    def ref(self):
        return C.byref(self.g)

    @property
    def BH(self):
        return self.B * self.H


def ditango_version() -> int:
    return _lib.ditango_version()


def ditango_check_geom(geom: Geometry) -> int:
    return _lib.ditango_check_geom(geom.ref)


def ditango_num_active(geom: Geometry) -> int:
    n = _lib.ditango_num_active(geom.ref)
    if n < 0:
        raise DitangoError("ditango_num_active", ditango_check_geom(geom))
    return n


def ditango_state_rows(geom: Geometry) -> int:
    n = _lib.ditango_state_rows(geom.ref)
    if n < 0:
        raise DitangoError("ditango_state_rows", ditango_check_geom(geom))
    return n


def ditango_slot_table(geom: Geometry):
    out = (C.c_int32 * (geom.P * geom.G))()
    _check("ditango_slot_table", _lib.ditango_slot_table(geom.ref, C.cast(out, C.c_void_p)))
    return [[out[i * geom.G + c] for c in range(geom.G)] for i in range(geom.P)]


def ditango_plan_workspace_size(geom: Geometry) -> int:
    return _lib.ditango_plan_workspace_size(geom.ref)


def ditango_plan(geom, cache_lse, cache_valid, band_k, budget, anchor, plan, fresh_list, counts,
                 score_out=None, workspace=None, workspace_bytes=0, stream=None):
    _check("ditango_plan", _lib.ditango_plan(
        geom.ref, _ptr(cache_lse), _ptr(cache_valid), int(band_k), float(budget), int(bool(anchor)),
        _ptr(plan), _ptr(fresh_list), _ptr(counts), _ptr(score_out), _ptr(workspace),
        int(workspace_bytes), _stream(stream)))


def ditango_attn_partial(geom, Q, K, V, fresh_list, counts, scale, out_O, out_lse,
                         out_by_slot=0, out_valid=None, dev_status=None, stream=None,
                         state_bf16=0, drift_rows=None, work_counter=None):
    _check("ditango_attn_partial", _lib.ditango_attn_partial(
        geom.ref, _ptr(Q), _ptr(K), _ptr(V), _ptr(fresh_list), _ptr(counts), float(scale),
        _ptr(out_O), _ptr(out_lse), int(out_by_slot), int(bool(state_bf16)), _ptr(out_valid),
        _ptr(drift_rows), _ptr(dev_status), _ptr(work_counter), _stream(stream)))


def error_state(w, age, delta, local_ok, drift_rows):
    """A ditango_error_state over five device buffers (tensors or addresses)."""
    return ditango_error_state(_ptr(w), _ptr(age), _ptr(delta), _ptr(local_ok), _ptr(drift_rows))


def ditango_plan_error(geom, cache_lse, cache_valid, band_k, budget, anchor, refresh_w, es, plan,
                       fresh_list, counts, score_out=None, workspace=None, workspace_bytes=0,
                       stream=None):
    _check("ditango_plan_error", _lib.ditango_plan_error(
        geom.ref, _ptr(cache_lse), _ptr(cache_valid), int(band_k), float(budget),
        int(bool(anchor)), int(bool(refresh_w)), C.byref(es), _ptr(plan), _ptr(fresh_list),
        _ptr(counts), _ptr(score_out), _ptr(workspace), int(workspace_bytes), _stream(stream)))


def ditango_plan_from_mass(geom, mass_partials, mass_bytes, cache_valid, band_k, budget, plan,
                           fresh_list, counts, score_out=None, stream=None):
    """ditango_plan with the mass score taken from a merge's mass partials."""
    _check("ditango_plan_from_mass", _lib.ditango_plan_from_mass(
        geom.ref, _ptr(mass_partials), int(mass_bytes), _ptr(cache_valid), int(band_k),
        float(budget), _ptr(plan), _ptr(fresh_list), _ptr(counts), _ptr(score_out),
        _stream(stream)))


def ditango_merge(geom, plan, part_O, part_lse, cache_O, cache_lse, cache_valid, writeback,
                  out, out_is_fp32, out_strides=None, out_lse=None, stream=None, state_bf16=0,
                  mass_partials=None):
    strides = None
    if out_strides is not None:
        strides = (C.c_int64 * 3)(*[int(s) for s in out_strides])
    _check("ditango_merge", _lib.ditango_merge(
        geom.ref, _ptr(plan), _ptr(part_O), _ptr(part_lse), _ptr(cache_O), _ptr(cache_lse),
        _ptr(cache_valid), int(bool(writeback)), int(bool(state_bf16)), _ptr(out),
        int(bool(out_is_fp32)),
        C.cast(strides, C.c_void_p) if strides is not None else None, _ptr(out_lse),
        _ptr(mass_partials), _stream(stream)))


def ditango_cache_update(geom, plan, part_O, part_lse, cache_O, cache_lse, cache_valid,
                         stream=None, state_bf16=0):
    _check("ditango_cache_update", _lib.ditango_cache_update(
        geom.ref, _ptr(plan), _ptr(part_O), _ptr(part_lse), _ptr(cache_O), _ptr(cache_lse),
        _ptr(cache_valid), int(bool(state_bf16)), _stream(stream)))


def ditango_cache_compose(fine, coarse, fine_O, fine_lse, fine_valid, coarse_O, coarse_lse,
                          coarse_valid, state_bf16=0, stream=None):
    _check("ditango_cache_compose", _lib.ditango_cache_compose(
        fine.ref, coarse.ref, _ptr(fine_O), _ptr(fine_lse), _ptr(fine_valid), _ptr(coarse_O),
        _ptr(coarse_lse), _ptr(coarse_valid), int(bool(state_bf16)), _stream(stream)))


def ditango_checked_build() -> bool:
    return bool(_lib.ditango_checked_build())


def ditango_check_status(reset=False) -> int:
    """Status recorded by a checked build's device-side input checks (0: none)."""
    out = C.c_int32(0)
    _check("ditango_check_status", _lib.ditango_check_status(C.byref(out), int(bool(reset))))
    return out.value


def ditango_set_wait_limit_ns(ns: int) -> None:
    _lib.ditango_set_wait_limit_ns(int(ns))


def ditango_selftest_bounded_wait(limit_ns, dev_status, stream=None):
    _check("ditango_selftest_bounded_wait", _lib.ditango_selftest_bounded_wait(
        int(limit_ns), _ptr(dev_status), _stream(stream)))


def ditango_plan_noalloc(geom, cache_lse, cache_valid, band_k, budget, anchor, plan, fresh_list,
                         counts, score_out=None, stream=None):
    """ditango_plan with the library's own fixed scratch (allocates nothing)."""
    _check("ditango_plan_noalloc", _lib.ditango_plan_noalloc(
        geom.ref, _ptr(cache_lse), _ptr(cache_valid), int(band_k), float(budget), int(bool(anchor)),
        _ptr(plan), _ptr(fresh_list), _ptr(counts), _ptr(score_out), _stream(stream)))
