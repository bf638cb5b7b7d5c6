"""The allocation-free plan entry point, for callers that cannot allocate
device memory (an arena they do not own, an allocator frozen after start-up,
a host that must not call cudaMalloc between steps).

ditango_plan_noalloc keeps its scratch in the library's own fixed device
array instead of a caller workspace.  Its results must equal ditango_plan's,
here on two calls in a row with different caches (the array keeps the last
call's contents, which must not leak into the next), and it must refuse a
geometry whose scratch would not fit.  This file is collected last.
"""
import ctypes
import os
import shutil
import subprocess

import pytest

torch = pytest.importorskip("torch")

import sparse_state_reuse_b200 as dt
from oracle import groups as OG
from oracle import masks as OM
from workloads import configs, inputs

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)


def _buffers(P, n, G=None):
    dev = "cuda"
    G = P if G is None else G
    return (torch.full((P * G,), -7, dtype=torch.int8, device=dev),
            torch.full((n,), -7, dtype=torch.int32, device=dev),
            torch.full((2,), -7, dtype=torch.int32, device=dev),
            torch.full((P * G,), -7.0, dtype=torch.float32, device=dev))


@pytest.mark.parametrize("w", [configs.DITANGO_REUSE, configs.LONG_VIDEO, configs.DITANGO_GROUPS],
                         ids=lambda w: w.name)
def test_noalloc_plan_equals_plan_on_two_calls(w):
    lib = ctypes.CDLL(dt.LIB_PATH)
    assert hasattr(lib, "ditango_plan_noalloc")
    go = w.group_off() if w.grouped else None
    g = dt.Geometry(w.B, w.H, w.N, w.d, w.part_off(), w.frame_off(), w.frame_mask(), group_off=go)
    A = OM.pair_mask(w.part_off(), w.frame_off(), w.frame_mask())
    if go is not None:
        A = OG.unit_mask(A, go)
    pairs = OM.slot_pairs(A)
    n = len(pairs)
    nws = dt.ditango_plan_workspace_size(g)
    ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
    valid = torch.ones(n, dtype=torch.uint8, device="cuda")
    for call, seed in enumerate((11, 12)):
        lse = torch.from_numpy(inputs.synthetic_cache_lse(w, n, pairs, seed=seed + w.seed)).cuda()
        if call == 1:
            valid[3] = 0                      # a different cache state on the second call
        ref = _buffers(w.P, n, g.G)
        dt.ditango_plan(g, lse, valid, w.band_k, w.budget, 0, *ref, ws, nws)
        got = _buffers(w.P, n, g.G)
        dt.ditango_plan_noalloc(g, lse, valid, w.band_k, w.budget, 0, *got)
        torch.cuda.synchronize()
        assert torch.equal(ref[0], got[0]), f"plan differs on call {call}"
        assert torch.equal(ref[2], got[2]), f"counts differ on call {call}"
        k = int(ref[2][0])
        assert torch.equal(ref[1][:k], got[1][:k]), f"fresh list differs on call {call}"
        assert torch.equal(ref[3], got[3]), f"scores differ on call {call}"


def test_noalloc_anchor_plan_and_size_limit():
    w = configs.TINY
    g = dt.Geometry(w.B, w.H, w.N, w.d, w.part_off())
    got = _buffers(w.P, 16)
    dt.ditango_plan_noalloc(g, None, None, 0, 1.0, 1, *got)
    torch.cuda.synchronize()
    assert (got[0].cpu().numpy() == dt.PLAN_FRESH).all() and got[2].tolist() == [16, 0]
    # 64 partitions x 64 x 4 B per chunk of 1024 rows: > 4 MiB of scratch
    big = dt.Geometry(1, 1024, 64 * 1024, 64, [p * 1024 for p in range(65)])
    assert dt.ditango_plan_workspace_size(big) > (4 << 20)
    lse = torch.empty(1, dtype=torch.float32, device="cuda")
    bufs = _buffers(64, 64 * 64)
    with pytest.raises(dt.DitangoError) as e:
        dt.ditango_plan_noalloc(big, lse, None, 1, 0.5, 0, *bufs)
    assert e.value.status == 2


def test_noalloc_call_takes_no_device_memory():
    """After a first call on the device (which loads the library's device
    code, the array included), further calls change no free-memory count."""
    w = configs.DITANGO_REUSE
    g = dt.Geometry(w.B, w.H, w.N, w.d, w.part_off())
    pairs = OM.slot_pairs(OM.pair_mask(w.part_off()))
    n = len(pairs)
    lse = torch.from_numpy(inputs.synthetic_cache_lse(w, n, pairs, seed=w.seed + 31)).cuda()
    bufs = _buffers(w.P, n)
    dt.ditango_plan_noalloc(g, lse, None, w.band_k, w.budget, 0, *bufs)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        dt.ditango_plan_noalloc(g, lse, None, w.band_k, w.budget, 0, *bufs)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, (free0, free1)


def test_noalloc_after_device_reset(tmp_path):
    """A plain C program plans with both entry points, resets the device and
    plans again, three times: the allocation-free plan must look its array
    up again in every new context and keep matching ditango_plan."""
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    exe = str(tmp_path / "noalloc_reset")
    libdir = os.path.dirname(dt.LIB_PATH)
    r = subprocess.run([nvcc, "-O1", "-Wno-deprecated-gpu-targets", "-I", os.path.join(ROOT, "include"),
                        os.path.join(ROOT, "tests", "c", "noalloc_reset.c"), "-L", libdir, "-lditango",
                        "-Xlinker", "-rpath=" + libdir, "-o", exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    assert run.stdout.count("equal") == 3, run.stdout
