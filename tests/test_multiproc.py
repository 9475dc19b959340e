"""World-size-2 checks of the multi-rank bench plumbing on CPU (gloo).

Each rank runs its own batch (weak scaling, no data-path collective); the job
time is the maximum over ranks and the job throughput counts every rank's
tokens.  Here two gloo ranks run the oracle's routing on their own seeded
batches and exercise the same helpers bench.py uses.
"""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from tests.conftest import ROOT


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import sys

    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from oracle import oracle as O
        from sparse_mixture_experts_stable_b200 import inputs as I

        cfg = I.full_layer_bf16(seed=bench.rank_seed(rank), T=256, H=64, E=16, F=8, k=4, F_shared=8)
        s = O.router_logits(cfg["x"].double().numpy(), cfg["w_router"].double().numpy().T,
                            cfg["router_bias"].double().numpy())
        _, sel, _, counts, _ = O.route(s, 4)
        fake_ms = 10.0 + 5.0 * rank
        mx = bench.max_over_ranks(fake_ms, world, device="cpu")
        thr = bench.job_throughput(256, 3, world, mx)
        q.put((rank, sel.tobytes(), int(counts.sum()), mx, thr))
    finally:
        dist.destroy_process_group()


def test_two_rank_weak_scaling_plumbing():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=240) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, sel0, c0, mx0, thr0), (r1, sel1, c1, mx1, thr1) = res
    assert sel0 != sel1  # each rank routes its own batch
    assert c0 == c1 == 256 * 4
    assert mx0 == mx1 == 15.0  # the slowest rank decides
    assert thr0 == thr1 == 256 * 3 * 2 / 0.015
