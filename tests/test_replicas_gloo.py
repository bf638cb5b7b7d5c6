"""Multi-process host logic of the replica benchmark, on CPU with gloo.

Each rank runs an independent replica of the step; the slowest rank sets the
step time (max over ranks) and the whole-job value is world x per-replica
work / that time.  Replicas derive identical workloads and plans from the
seeds, so their work is the same."""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from oracle import masks
        from oracle.plan import select
        from workloads import configs, inputs
        per_rank_ms = [3.0, 7.5][rank]
        m = bench.max_over_ranks(per_rank_ms, "cpu", dist)
        w = configs.LONG_VIDEO
        A = masks.pair_mask(w.part_off(), w.frame_off(), w.frame_mask())
        plan, fl = select(np.zeros((w.P, w.P)), A, w.band_k, w.budget)
        flops = bench.effective_flops(w, plan == 1)
        digest = int(inputs.slab(configs.TINY, "q", 0, rank % 2)[:4].sum())
        q.put((rank, m, flops, fl.tolist(), digest))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_identical_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, m0, f0, l0, _), (r1, m1, f1, l1, _) = res
    assert m0 == m1 == 7.5                       # slowest replica sets the time
    assert f0 == f1 and l0 == l1                 # identical replicas
    import bench
    assert bench.aggregate_tflops(2, f0, 7.5) == pytest.approx(2 * f0 / 7.5e-3 / 1e12)
