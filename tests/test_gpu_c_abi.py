"""A whole step through the C ABI from plain C on the GPU (tests/c/abi_device.c:
CUDA runtime memory, no Python in the compute path), checked against the fp64
oracle on the same seeded inputs: the anchor step of the tiny workload equals
unpartitioned attention."""
import os
import shutil
import subprocess

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import sparse_state_reuse_b200 as dt
from oracle.attention import dense_attention
from workloads import configs, inputs

import gpu_common as G

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_c_program_runs_a_step_that_matches_the_oracle(tmp_path):
    w = configs.TINY
    assert (w.B, w.H, w.N, w.d, w.P) == (1, 2, 1024, 64, 4)
    for t in "qkv":
        inputs.full(w, t).tofile(str(tmp_path / f"{t}.bin"))
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    exe = str(tmp_path / "abi_device")
    libdir = os.path.dirname(dt.LIB_PATH)
    r = subprocess.run([nvcc, "-O1", "-Wno-deprecated-gpu-targets", "-I", os.path.join(ROOT, "include"),
                        os.path.join(ROOT, "tests", "c", "abi_device.c"), "-L", libdir, "-lditango",
                        "-Xlinker", "-rpath=" + libdir, "-o", exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([exe, str(tmp_path)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    out = np.fromfile(str(tmp_path / "out.bin"), dtype=np.float32).reshape(w.B, w.H, w.N, w.d)
    lse = np.fromfile(str(tmp_path / "lse.bin"), dtype=np.float32).reshape(w.B, w.H, w.N)
    for h in range(w.H):
        q, k, v, _, _ = G.slabs(w, 0, h, with_prev=False)
        Od, ld = dense_attention(q, k, v)
        G.assert_close(out[0, h], Od, f"C step head {h}")
        G.assert_close(lse[0, h], ld, f"C step lse head {h}")
