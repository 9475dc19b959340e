"""Expert parallelism: R ranks, one GPU each, E / R experts per rank.

The layer over the R ranks is the layer over the whole batch with the tokens in
rank order (capacity C from the global T, greedy position priority across
ranks; ``include/moe.h``, "Expert parallelism").  One step on rank r:

    moe_route (local tokens)                  -> selected, gates, counts
    all-gather of the counts                  -> counts_all (R, E)
    moe_ep_plan                               -> slot base per expert, global used
    moe_ep_dispatch                           -> kept rows written into the owner
                                                 ranks' expert-major buffers
    barrier
    moe_expert_ffn on the local experts       -> this rank's ybuf
    barrier
    moe_ep_combine                            -> y, each kept row read from its
                                                 owner rank's ybuf

Two drivers run that sequence with the same library calls:

* ``EPGroup``: ranks in separate processes (``torch.distributed``, NCCL for the
  counts and the barriers); the other ranks' buffers are mapped once with
  ``moe_ipc_export`` / ``moe_ipc_import``, so the row exchange is the gather and
  combine kernels reading and writing peer memory.
* ``run_ranks_on_one_device``: every rank's buffers on one GPU in one process;
  each phase runs for all ranks, rank after rank, in stream order before the
  next phase starts (no kernel ever waits for another).  The pointer tables
  then hold the other ranks' buffers on the same device.

The host-side pieces (``partition``, ``token_bases``, ``gather_counts``,
``exchange_handles``) work with any process-group backend.
"""
from __future__ import annotations

from typing import List, Optional, Sequence

import torch
import torch.distributed as dist

from . import binding as B


def partition(E: int, R: int) -> int:
    """Experts per rank; E must be a multiple of R (rank r owns [r E/R, (r+1) E/R))."""
    if R < 1 or E < 1 or E % R != 0:
        raise ValueError(f"{E} experts cannot be split evenly over {R} ranks")
    if R > 64:
        raise ValueError("at most 64 ranks")
    return E // R


def payload_bytes(tokens: int, hidden: int, k: int, bytes_per_value: int, include_return: bool = True) -> int:
    """Activation bytes an expert-parallel step moves with no drops (Module 7 page,
    expert-parallel payload): T*k rows of ``hidden`` values out, and as many back."""
    for v in (tokens, hidden, k, bytes_per_value):
        if int(v) < 1:
            raise ValueError("sizes must be positive")
    one_way = int(tokens) * int(hidden) * int(k) * int(bytes_per_value)
    return one_way * (2 if include_return else 1)


def token_bases(tokens_per_rank: Sequence[int]) -> List[int]:
    """Global index of every rank's first token (tokens in rank order)."""
    out, acc = [], 0
    for t in tokens_per_rank:
        out.append(acc)
        acc += int(t)
    return out


def gather_counts(counts: torch.Tensor, group=None) -> torch.Tensor:
    """(R, E) int32: row q = rank q's pre-drop counts."""
    R = dist.get_world_size(group)
    parts = [torch.empty_like(counts) for _ in range(R)]
    dist.all_gather(parts, counts.contiguous(), group=group)
    return torch.stack(parts).to(torch.int32)


def exchange_handles(local, group=None) -> list:
    """Every rank's ``local`` object (e.g. IPC handles and offsets), in rank order."""
    out = [None] * dist.get_world_size(group)
    dist.all_gather_object(out, local, group=group)
    return out


def _expert_ffn(kind: str, xbuf, used, w: dict, ybuf):
    return B.moe_expert_ffn(kind, xbuf, used, w["w1"], b1=w.get("b1"), w2=w.get("w2"), b2=w.get("b2"),
                            w3=w.get("w3"), ybuf=ybuf)


def _out_features(kind: str, w: dict) -> int:
    return w["w1"].shape[1] if kind == "linear" else w["w2"].shape[1]


class EPGroup:
    """Expert-parallel layer over the ranks of ``group`` (one process per GPU).

    ``weights`` holds this rank's experts only (E / R of them, the library's
    (out, in) layout).  Buffers are allocated once; the other ranks' buffers
    are mapped into this process at construction.
    """

    def __init__(self, T_local: int, D: int, E: int, k: int, C: int, kind: str, weights: dict,
                 dtype=torch.bfloat16, group=None, device=None):
        self.group = group
        self.rank = dist.get_rank(group)
        self.R = dist.get_world_size(group)
        self.epr = partition(E, self.R)
        self.T, self.D, self.E, self.k, self.C, self.kind = T_local, D, E, k, C, kind
        self.weights = weights
        self.device = device or torch.device("cuda", torch.cuda.current_device())
        self.Dout = _out_features(kind, weights)
        self.xbuf = torch.empty(self.epr, C, D, dtype=dtype, device=self.device)
        self.ybuf = torch.empty(self.epr, C, self.Dout, dtype=dtype, device=self.device)
        self.flag = torch.zeros(1, dtype=torch.float32, device=self.device)
        info = exchange_handles((T_local, B.moe_ipc_export(self.xbuf), B.moe_ipc_export(self.ybuf)), group)
        self.token_base = token_bases([i[0] for i in info])[self.rank]
        self.mappings: List[int] = []
        self.xbuf_ranks, self.ybuf_ranks = [], []
        for q, (_, (hx, ox), (hy, oy)) in enumerate(info):
            if q == self.rank:
                self.xbuf_ranks.append(self.xbuf.data_ptr())
                self.ybuf_ranks.append(self.ybuf.data_ptr())
                continue
            mx, my = B.moe_ipc_import(hx), B.moe_ipc_import(hy)
            self.mappings += [mx, my]
            self.xbuf_ranks.append(mx + ox)
            self.ybuf_ranks.append(my + oy)

    def barrier(self):
        dist.all_reduce(self.flag, group=self.group)

    def forward(self, x: torch.Tensor, w_router: torch.Tensor, logit_bias: Optional[torch.Tensor] = None,
                base_kind: str = "input", base: Optional[torch.Tensor] = None,
                dev_status: Optional[torch.Tensor] = None) -> dict:
        r = B.moe_route(x, self.k, w_router=w_router, logit_bias=logit_bias, dev_status=dev_status)
        counts_all = gather_counts(r["counts"], self.group)
        plan = B.moe_ep_plan(counts_all, self.rank, self.C)
        d = B.moe_ep_dispatch(r["selected"], self.E, self.C, plan["rank_base"], self.token_base, x,
                              self.xbuf_ranks, dev_status=dev_status)
        self.barrier()
        lo = self.rank * self.epr
        _expert_ffn(self.kind, self.xbuf, plan["used"][lo:lo + self.epr], self.weights, self.ybuf)
        self.barrier()
        b = x if base_kind == "input" else base
        y = B.moe_ep_combine(self.ybuf_ranks, r["selected"], d["slot"], r["gates_f32"], self.E, self.C, self.Dout,
                             x.dtype, base_kind=base_kind, base=b, dev_status=dev_status)
        return dict(y=y, route=r, plan=plan, dispatch=d)

    def close(self):
        for m in self.mappings:
            B.moe_ipc_close(m)
        self.mappings = []


def run_ranks_on_one_device(xs: Sequence[torch.Tensor], E: int, k: int, C: int, kind: str, w_router: torch.Tensor,
                            weights: Sequence[dict], logit_bias: Optional[torch.Tensor] = None,
                            base_kind: str = "input", bases: Optional[Sequence[torch.Tensor]] = None,
                            dev_status: Optional[torch.Tensor] = None) -> dict:
    """The expert-parallel step for R = len(xs) ranks whose buffers all live on one GPU.

    ``weights[q]`` holds rank q's E / R experts.  Returns per-rank lists of the
    outputs (y, route, plan, dispatch) and the expert-major buffers.
    """
    R = len(xs)
    epr = partition(E, R)
    dev = xs[0].device
    D = xs[0].shape[1]
    Dout = _out_features(kind, weights[0])
    xbufs = [torch.empty(epr, C, D, dtype=xs[0].dtype, device=dev) for _ in range(R)]
    ybufs = [torch.empty(epr, C, Dout, dtype=xs[0].dtype, device=dev) for _ in range(R)]
    bases_tok = token_bases([x.shape[0] for x in xs])
    routes = [B.moe_route(x, k, w_router=w_router, logit_bias=logit_bias, dev_status=dev_status) for x in xs]
    counts_all = torch.stack([r["counts"] for r in routes])
    plans = [B.moe_ep_plan(counts_all, q, C) for q in range(R)]
    disp = [B.moe_ep_dispatch(routes[q]["selected"], E, C, plans[q]["rank_base"], bases_tok[q], xs[q], xbufs,
                              dev_status=dev_status) for q in range(R)]
    for q in range(R):
        _expert_ffn(kind, xbufs[q], plans[q]["used"][q * epr:(q + 1) * epr], weights[q], ybufs[q])
    ys = []
    for q in range(R):
        b = xs[q] if base_kind == "input" else (bases[q] if bases is not None else None)
        ys.append(B.moe_ep_combine(ybufs, routes[q]["selected"], disp[q]["slot"], routes[q]["gates_f32"], E, C, Dout,
                                   xs[q].dtype, base_kind=base_kind, base=b, dev_status=dev_status))
    return dict(y=ys, route=routes, plan=plans, dispatch=disp, xbuf=xbufs, ybuf=ybufs, counts_all=counts_all)
