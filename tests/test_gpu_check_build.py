"""The checked build (libditango_check.so, -DDITANGO_CHECK) on the GPU.

It validates the device-resident inputs the host cannot see without a
synchronisation before using them: ditango_attn_partial's count and fresh
list, and the plan codes the merge reads.  Each case here corrupts one of
them; the checks turn it into DITANGO_ERR_BOUNDS before any memory is
touched through it (nothing is computed), the outputs stay as they were, and
the context stays usable.  Runs in a child process that loads the checked
library through DITANGO_LIBRARY."""
import os
import subprocess
import sys
import textwrap

import pytest

torch = pytest.importorskip("torch")

import sparse_state_reuse_b200 as dt

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent("""
    import numpy as np, torch
    import sparse_state_reuse_b200 as dt
    from workloads import configs, inputs
    assert dt.ditango_checked_build()
    w = configs.TINY
    up = lambda b: torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).cuda()
    Q, K, V = (up(inputs.full(w, t)) for t in "qkv")
    pa = dt.PartitionedAttention(w.B, w.H, w.N, w.d, w.part_off())
    out = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.float32, device="cuda")
    pa.step(Q, K, V, out, anchor=True)               # a valid step: nothing recorded
    torch.cuda.synchronize()
    assert pa.status.item() == 0 and dt.ditango_check_status() == 0
    ref = out.clone()
    n = pa.n_slots
    cases = {
        "count beyond the active units": lambda fl, c: c.copy_(torch.tensor([n + 3, 0])),
        "unit index out of range": lambda fl, c: fl.__setitem__(5, w.P * w.P + 7),
        "list not row-major": lambda fl, c: fl.__setitem__(slice(2, 4), fl[2:4].flip(0).clone()),
    }
    for name, corrupt in cases.items():
        plan = torch.zeros(w.P * w.P, dtype=torch.int8, device="cuda")
        fl = torch.zeros(n, dtype=torch.int32, device="cuda")
        counts = torch.zeros(2, dtype=torch.int32, device="cuda")
        dt.ditango_plan(pa.geom, None, None, 0, 1.0, 1, plan, fl, counts)
        corrupt(fl, counts)
        O = torch.full((n, w.BH, w.Lp, w.d), float("nan"), device="cuda")
        lse = torch.full((n, w.BH, w.Lp), float("nan"), device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        wc = torch.zeros(2, dtype=torch.int32, device="cuda")
        dt.ditango_attn_partial(pa.geom, Q, K, V, fl, counts, 0.0, O, lse, 0, None, st,
                                work_counter=wc)
        torch.cuda.synchronize()
        assert st.item() == dt._abi.ERR_BOUNDS, (name, st.item())
        assert dt.ditango_check_status(reset=True) == dt._abi.ERR_BOUNDS, name
        assert torch.isnan(O).all() and torch.isnan(lse).all(), name   # nothing written
        assert wc.tolist() == [0, 0], name
        print("caught:", name)
    # a plan code outside {0, 1, 2} on an active unit: recorded by the merge
    bad = pa.plan.clone()
    bad[1] = 7
    out2 = torch.empty_like(out)
    dt.ditango_merge(pa.geom, bad, None, None, pa.state_O, pa.state_lse, pa.valid, 0, out2, 1)
    torch.cuda.synchronize()
    assert dt.ditango_check_status(reset=True) == dt._abi.ERR_BOUNDS
    print("caught: plan code 7")
    # the context is intact: a valid step gives the same output as before
    pa.step(Q, K, V, out, anchor=True)
    torch.cuda.synchronize()
    assert pa.status.item() == 0 and dt.ditango_check_status() == 0
    assert torch.equal(out, ref)
    print("checked build ok")
""")


def test_checked_build_turns_bad_device_inputs_into_a_status():
    lib = os.path.join(ROOT, "sparse_state_reuse_b200", "libditango_check.so")
    if not os.path.exists(lib):
        sys.path.insert(0, os.path.join(ROOT, "sparse_state_reuse_b200"))
        import build as B
        B.build(check=True)
    env = dict(os.environ, DITANGO_LIBRARY=lib, PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", CHILD], capture_output=True, text=True, env=env,
                       cwd=ROOT, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.count("caught:") == 4 and "checked build ok" in r.stdout, r.stdout


def test_release_build_reports_no_checks():
    assert not dt.ditango_checked_build()
    assert dt.ditango_check_status() == 0
