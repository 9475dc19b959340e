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


def _ep_worker(rank, world, port, q):
    import sys

    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import oracle as O
        from sparse_mixture_experts_stable_b200 import ep

        # one global batch, split over the ranks (uneven); every rank draws the same numbers
        tokens = [37, 52]
        E, k, cf = 8, 2, 0.75
        T = sum(tokens)
        rng = np.random.default_rng(4)
        s = rng.standard_normal((T, E))
        _, sel_all, _, _, _ = O.route(s, k)
        C = O.capacity(T, k, E, cf)
        base_tok = ep.token_bases(tokens)[rank]
        sel = sel_all[base_tok:base_tok + tokens[rank]]
        epr = ep.partition(E, world)
        # host side of the step: counts exchange and handle exchange
        counts = torch.from_numpy(np.bincount(sel.ravel(), minlength=E).astype(np.int32))
        counts_all = ep.gather_counts(counts)
        handles = ep.exchange_handles((rank, b"h%d" % rank))
        # the expert-parallel reading: this rank's assignment to e takes slot
        # sum_{q < rank} count_q[e] + (its rank among this rank's assignments to e)
        rank_base = counts_all[:rank].sum(0).numpy()
        local = O.dispatch(sel, E, sel.size)["slot"]  # capacity never binds: the local running count
        ep_slot = np.where(local + rank_base[sel] < C, local + rank_base[sel], -1)
        want = O.dispatch(sel_all, E, C)["slot"][base_tok:base_tok + tokens[rank]]
        q.put((rank, epr, counts_all.numpy().tobytes(), [h[1] for h in handles],
               bool(np.array_equal(ep_slot, want)), int((want < 0).sum())))
    finally:
        dist.destroy_process_group()


def test_two_rank_expert_parallel_host_logic():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ep_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=240) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, epr0, ca0, h0, ok0, drop0), (r1, epr1, ca1, h1, ok1, drop1) = res
    assert epr0 == epr1 == 4
    assert ca0 == ca1  # every rank sees the same (R, E) counts
    assert h0 == h1 == [b"h0", b"h1"]
    assert ok0 and ok1  # per-rank slots from the exchanged counts == the one-batch greedy loop
    assert drop0 + drop1 > 0  # the capacity binds somewhere


def test_expert_parallel_partition_rules():
    from sparse_mixture_experts_stable_b200 import ep
    # Module 7 page, expert-parallel payload: 2048 tokens, hidden 7168, top-8, bf16 -> 448 MiB round trip
    assert ep.payload_bytes(2048, 7168, 8, 2) == 448 * 2 ** 20
    assert ep.payload_bytes(2048, 7168, 8, 2, include_return=False) == 224 * 2 ** 20
    assert ep.partition(256, 8) == 32
    assert ep.token_bases([5, 0, 7]) == [0, 5, 5]
    for E, R in [(10, 4), (8, 0), (128, 128)]:
        try:
            ep.partition(E, R)
        except ValueError:
            continue
        raise AssertionError((E, R))
