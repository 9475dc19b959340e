"""moe_dispatch (slot scan + gather) on the GPU against the oracle's greedy loop.

Every output is an integer or a copied row, so the comparison is exact.
"""
import numpy as np
import pytest
import torch

import sparse_mixture_experts_stable_b200 as moe
from oracle import oracle as O
from sparse_mixture_experts_stable_b200 import inputs as I
from tests.gpu_util import DEV, check_dispatch, cpu, cpu64

pytestmark = pytest.mark.gpu


def _random_selection(rng, T, E, k):
    return np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int64)


@pytest.mark.parametrize("T,E,k,C", [
    (1, 1, 1, 1), (2, 4, 2, 1), (1500, 256, 8, 47), (1500, 256, 8, 0), (1500, 256, 8, 10000),
    (5000, 64, 1, 50), (2049, 8, 2, 300), (777, 1000, 3, 2), (3000, 33, 33, 100),
])
def test_dispatch_random(T, E, k, C):
    rng = np.random.default_rng(T + E + k + C)
    sel = _random_selection(rng, T, E, k)
    D = 72
    x = torch.randn(T, D, device=DEV, dtype=torch.bfloat16)
    g = moe.moe_dispatch(torch.from_numpy(sel).to(DEV), E, C, x=x)
    o = O.dispatch(sel, E, C)
    check_dispatch(o, g, E, C, f"T={T} E={E} k={k} C={C}")
    # gathered rows are exact copies
    if C > 0:
        xb, xs = cpu64(g["xbuf"]), cpu64(x)
        for e in range(E):
            u = o["used"][e]
            if u:
                np.testing.assert_array_equal(xb[e, :u], xs[o["token_of_slot"][e, :u]])


def test_dispatch_duplicate_indices():
    # a given index tensor may repeat an expert within a token: each copy takes a slot
    sel = np.array([[0, 0], [0, 1], [1, 1]], dtype=np.int64)
    g = moe.moe_dispatch(torch.from_numpy(sel).to(DEV), 2, 3)
    check_dispatch(O.dispatch(sel, 2, 3), g, 2, 3, "duplicates")


def test_dispatch_zipf_top1_full_size():
    cfg = I.dispatch_top1_bf16(seed=0)  # T=32768, E=64, C=512
    C = moe.moe_capacity(cfg["T"], 1, cfg["E"], cfg["capacity_factor"])
    assert C == 512
    idx = cfg["expert_idx"].view(-1, 1)
    x = cfg["x"].to(DEV)
    g = moe.moe_dispatch(idx.to(DEV), cfg["E"], C, x=x)
    o = O.dispatch(idx.numpy(), cfg["E"], C)
    check_dispatch(o, g, cfg["E"], C, "zipf top-1")
    assert o["overflow"].sum() > 0  # the skew forces drops
    # exclusive running count form (top-1): the slot is the number of earlier tokens on the expert
    flat = idx.numpy().ravel()
    onehot = np.eye(cfg["E"], dtype=np.int64)[flat]
    pos = ((np.cumsum(onehot, 0) - onehot) * onehot).sum(1)
    np.testing.assert_array_equal(cpu(g["slot"]).ravel(), np.where(pos < C, pos, -1))
    xb, xs = g["xbuf"], x
    tos = torch.from_numpy(o["token_of_slot"]).to(DEV).long()
    for e in range(cfg["E"]):
        u = int(o["used"][e])
        assert torch.equal(xb[e, :u], xs[tos[e, :u]])


def test_dispatch_full_layer_routing():
    cfg = I.full_layer_bf16(seed=0, T=16384, H=2048, E=256, F=8, F_shared=8)
    x, w = cfg["x"].to(DEV), cfg["w_router"].to(DEV)
    bias = cfg["router_bias"].to(DEV)
    r = moe.moe_route(x, 8, w_router=w, logit_bias=bias)
    C = moe.moe_capacity(16384, 8, 256, 1.25)
    g = moe.moe_dispatch(r["selected"], 256, C)
    s64 = O.router_logits(cpu64(x), cpu64(w).T, cpu64(cfg["router_bias"]))
    _, sel, _, _, _ = O.route(s64, 8)
    np.testing.assert_array_equal(cpu(r["selected"]), sel)
    o = O.dispatch(sel, 256, C)
    check_dispatch(o, g, 256, C, "full layer routing")
    assert o["overflow"].sum() > 0


def test_dispatch_reports_bad_index():
    sel = np.array([[0, 5], [-1, 1], [1, 0]], dtype=np.int64)
    st = moe.new_status()
    g = moe.moe_dispatch(torch.from_numpy(sel).to(DEV), 2, 4, dev_status=st)
    assert moe.moe_read_status(st) == moe.binding.MOE_ERR_BAD_INDEX
    o = O.dispatch(sel, 2, 4)
    assert o["bad_index"]
    check_dispatch(o, g, 2, 4, "bad index")


def test_dispatch_is_deterministic():
    rng = np.random.default_rng(5)
    sel = torch.from_numpy(_random_selection(rng, 20000, 128, 4)).to(DEV)
    a = moe.moe_dispatch(sel, 128, 400)
    b = moe.moe_dispatch(sel, 128, 400)
    for key in ("slot", "kept", "used", "overflow", "drops", "token_of_slot"):
        assert torch.equal(a[key], b[key]), key
