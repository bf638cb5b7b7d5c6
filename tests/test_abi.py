"""The C ABI library loads without a GPU, exports every declared entry point,
and its host-side logic (argument checks, active pairs, slot numbering)
agrees with the oracle.  No compute call is made here."""
import os
import re

import numpy as np
import pytest

import sparse_state_reuse_b200 as dt
from oracle import groups, masks
from workloads import configs

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "ditango.h")


def declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ditango_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    import ctypes
    lib = ctypes.CDLL(dt.LIB_PATH)
    names = declared()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(dt.EXPORTED)


def test_checked_build_exports_the_same_abi():
    """libditango_check.so (built with -DDITANGO_CHECK) exports every declared
    symbol too, and says it is the checked build; the release library says
    it is not.  No GPU needed: neither call touches the device."""
    import ctypes
    import subprocess
    import sys
    path = os.path.join(os.path.dirname(dt.LIB_PATH), "libditango_check.so")
    if not os.path.exists(path):
        subprocess.run([sys.executable, os.path.join(os.path.dirname(dt.LIB_PATH), "build.py"),
                        "--check"], check=True, capture_output=True)
    lib = ctypes.CDLL(path)
    for n in declared():
        assert hasattr(lib, n), n
    lib.ditango_checked_build.restype = ctypes.c_int32
    assert lib.ditango_checked_build() == 1
    assert not dt.ditango_checked_build()


def test_version_and_status_strings():
    assert dt.ditango_version() >= 10000
    assert dt.status_string(0) == "ok"
    assert "timed out" in dt.status_string(4)
    assert "out of range" in dt.status_string(5)


@pytest.mark.parametrize("w", configs.ALL, ids=lambda w: w.name)
def test_active_pairs_and_slots_match_oracle(w):
    go = w.group_off() if w.grouped else None
    g = dt.Geometry(w.B, w.H, w.N, w.d, w.part_off(), w.frame_off(), w.frame_mask(), group_off=go)
    A = masks.pair_mask(w.part_off(), w.frame_off(), w.frame_mask())
    if go is not None:
        A = groups.unit_mask(A, go)
    assert dt.ditango_check_geom(g) == 0
    assert dt.ditango_num_active(g) == int(A.sum())
    assert dt.ditango_state_rows(g) == w.Lp
    assert (np.array(dt.ditango_slot_table(g)) == masks.slot_table(A)).all()


def test_ragged_partitions_within_frames():
    po = [0, 100, 130, 300, 555, 1000]
    fo = [0, 300, 1000]
    fm = [[1, 0], [1, 1]]
    g = dt.Geometry(2, 3, 1000, 64, po, fo, fm)
    A = masks.pair_mask(po, fo, fm)
    assert dt.ditango_num_active(g) == int(A.sum())
    assert (np.array(dt.ditango_slot_table(g)) == masks.slot_table(A)).all()
    assert dt.ditango_state_rows(g) == 445


def test_partitions_straddling_frames():
    """Partitions cut across frame boundaries: a pair is active when any of
    its token pairs is allowed (the kernels then mask single logits)."""
    fo = [0, 50, 100, 150, 200]
    fm = [[1, 0, 0, 1], [1, 1, 0, 0], [0, 1, 1, 0], [0, 0, 1, 1]]
    po = [0, 30, 75, 140, 170, 200]
    g = dt.Geometry(1, 2, 200, 64, po, fo, fm)
    A = masks.pair_mask(po, fo, fm)
    assert dt.ditango_num_active(g) == int(A.sum())
    assert (np.array(dt.ditango_slot_table(g)) == masks.slot_table(A)).all()
    go = [0, 2, 5]
    g = dt.Geometry(1, 2, 200, 64, po, fo, fm, group_off=go)
    Au = groups.unit_mask(A, go)
    assert (np.array(dt.ditango_slot_table(g)) == masks.slot_table(Au)).all()


@pytest.mark.parametrize("kw,status", [
    (dict(part_off=[0, 10, 10, 64]), 1),          # empty partition
    (dict(part_off=[0, 32, 63]), 1),              # does not end at N
    (dict(d=80), 2),                              # head dim without a kernel
    (dict(part_off=list(range(0, 65 * 2, 2))[:66] + [130]), 2),  # P > 64
    (dict(frame_off=[0, 40, 64], frame_mask=[[1, 1], [1, 1]]), 0),  # partition straddling frames
    (dict(frame_off=[0, 40, 63], frame_mask=[[1, 1], [1, 1]]), 1),  # frames not ending at N
    (dict(B=0), 1),
])
def test_geometry_validation(kw, status):
    args = dict(B=1, H=2, N=64, d=64, part_off=[0, 32, 64], frame_off=None, frame_mask=None)
    args.update(kw)
    if args["part_off"][-1] != args["N"] and status == 2 and len(args["part_off"]) > 65:
        args["N"] = args["part_off"][-1]
    g = dt.Geometry(**args)
    assert dt.ditango_check_geom(g) == status


def test_calls_reject_bad_arguments_before_launching():
    g = dt.Geometry(1, 2, 64, 64, [0, 32, 64])
    with pytest.raises(dt.DitangoError) as e:
        dt.ditango_plan(g, None, None, 1, 0.5, 0, None, None, None, stream=0)
    assert e.value.status == 1
    with pytest.raises(dt.DitangoError):
        dt.ditango_plan(g, 16, None, 1, 1.5, 0, 16, 16, 16, None, 16, 10**6, stream=0)  # budget > 1
    with pytest.raises(dt.DitangoError):
        dt.ditango_attn_partial(g, 16, 16, 8, 16, 16, 0.0, 16, 16, stream=0)  # misaligned V
    with pytest.raises(dt.DitangoError):
        dt.ditango_merge(g, 16, None, None, None, None, None, 0, 16, 1, stream=0)  # no sources
    with pytest.raises(dt.DitangoError):
        dt.ditango_selftest_bounded_wait(0, 16, stream=0)
    assert dt.ditango_plan_workspace_size(g) > 0


@pytest.mark.parametrize("go", [[0, 1, 3, 6, 24], [0, 24], [0, 2, 4, 8, 16, 24], list(range(25))])
def test_unit_slots_match_oracle(go):
    w = configs.LONG_VIDEO
    g = dt.Geometry(w.B, w.H, w.N, w.d, w.part_off(), w.frame_off(), w.frame_mask(), group_off=go)
    Au = groups.unit_mask(masks.pair_mask(w.part_off(), w.frame_off(), w.frame_mask()), go)
    assert dt.ditango_num_active(g) == int(Au.sum())
    assert (np.array(dt.ditango_slot_table(g)) == masks.slot_table(Au)).all()


@pytest.mark.parametrize("go,status", [([0, 2, 2, 4], 1), ([0, 2, 3], 1), ([1, 4], 1), ([0, 4], 0),
                                       ([0, 1, 2, 3, 4], 0)])
def test_group_validation(go, status):
    g = dt.Geometry(1, 2, 64, 64, [0, 16, 32, 48, 64], group_off=go)
    assert dt.ditango_check_geom(g) == status


def test_compose_rejects_bad_groupings_before_launching():
    po = [0, 16, 32, 48, 64]
    fine = dt.Geometry(1, 2, 64, 64, po, group_off=[0, 2, 4])
    with pytest.raises(dt.DitangoError) as e:   # [0, 1, 4] is not a coarsening of [0, 2, 4]
        dt.ditango_cache_compose(fine, dt.Geometry(1, 2, 64, 64, po, group_off=[0, 1, 4]),
                                 16, 16, None, 4096, 4096, None, stream=0)
    assert e.value.status == 1
    with pytest.raises(dt.DitangoError):        # a different attention call
        dt.ditango_cache_compose(fine, dt.Geometry(1, 3, 64, 64, po, group_off=[0, 4]),
                                 16, 16, None, 4096, 4096, None, stream=0)
    with pytest.raises(dt.DitangoError):        # overlapping state buffers
        dt.ditango_cache_compose(fine, dt.Geometry(1, 2, 64, 64, po, group_off=[0, 4]),
                                 16, 16, None, 16, 16, None, stream=0)


def test_error_plan_rejects_bad_arguments_before_launching():
    g = dt.Geometry(1, 2, 64, 64, [0, 32, 64])
    es = dt.error_state(16, 16, 16, 16, None)          # no drift rows
    with pytest.raises(dt.DitangoError) as e:
        dt.ditango_plan_error(g, 16, None, 0, 0.5, 0, 0, es, 16, 16, 16, None, 16, 10**6, stream=0)
    assert e.value.status == 1
    es2 = dt.error_state(None, 16, 16, 16, 16)         # no w buffer
    with pytest.raises(dt.DitangoError):
        dt.ditango_plan_error(g, 16, None, 0, 0.5, 1, 0, es2, 16, 16, 16, stream=0)
    with pytest.raises(dt.DitangoError):               # drift rows need out_by_slot
        dt.ditango_attn_partial(g, 16, 16, 16, 16, 16, 0.0, 16, 16, 0, drift_rows=16, stream=0)


def test_size_one_dimensions_may_have_any_stride():
    """B = 1 with a 0 batch stride (numpy/torch broadcast views) passes the
    argument checks: only the CUDA stage can fail here (no GPU)."""
    g = dt.Geometry(1, 2, 64, 64, [0, 32, 64], q_strides=(0, 4096, 64), k_strides=(0, 4096, 64),
                    v_strides=(0, 4096, 64))
    with pytest.raises(dt.DitangoError) as e:
        dt.ditango_attn_partial(g, 4096, 4096, 4096, 4096, 4096, 0.0, 4096, 4096, 1, stream=0)
    assert e.value.status != 1
    g2 = dt.Geometry(2, 2, 64, 64, [0, 32, 64], q_strides=(0, 4096, 64))   # B = 2: a real stride
    with pytest.raises(dt.DitangoError) as e:
        dt.ditango_attn_partial(g2, 4096, 4096, 4096, 4096, 4096, 0.0, 4096, 4096, 1, stream=0)
    assert e.value.status == 1


def test_plain_c_program_uses_the_abi(tmp_path):
    """The boundary is a C ABI: a C program built with gcc against
    include/ditango.h and linked to libditango.so runs its host-side calls."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc") or shutil.which("cc")
    if gcc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(__file__))
    exe = str(tmp_path / "abi_host")
    libdir = os.path.dirname(dt.LIB_PATH)
    r = subprocess.run([gcc, "-std=c99", "-O1", "-Wall", "-Werror", "-I", os.path.join(root, "include"),
                        os.path.join(root, "tests", "c", "abi_host.c"), "-L", libdir, "-lditango",
                        "-Wl,-rpath," + libdir, "-o", exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stdout + run.stderr
    out = dict(line.split() for line in run.stdout.splitlines())
    assert out["fails"] == "0" and out["active_pairs"] == "28"
    assert int(out["version"]) == dt.ditango_version()
