"""Expert parallelism (moe_ep_plan / moe_ep_dispatch / moe_ep_combine) on one GPU.

R ranks are run in one process with every rank's buffers on the same device
(``ep.run_ranks_on_one_device``: each phase for all ranks in stream order, no
kernel waits for another), so the kernels write into and read from "other
ranks'" buffers through the same pointer tables a multi-GPU group uses.  The
expert-parallel layer must equal the one-device layer over the concatenated
batch: integer outputs and moved rows bit for bit, and y bit for bit too,
since every expert sees the same rows in the same slots and the combine adds
the same terms in the same order.  A second process on the same GPU maps a
buffer through moe_ipc_export / moe_ipc_import and combines from it.
"""
import os
import subprocess
import sys
import tempfile

import numpy as np
import pytest
import torch

import sparse_mixture_experts_stable_b200 as moe
from oracle import oracle as O
from sparse_mixture_experts_stable_b200 import ep
from tests.conftest import ROOT
from tests.gpu_util import DEV, cpu

pytestmark = pytest.mark.gpu


def _weights(kind, E, D, F, g, dtype):
    def rnd(*s, scale):
        return (torch.randn(*s, generator=g) * scale).to(dtype).to(DEV)
    if kind == "swiglu":
        return {"w1": rnd(E, F, D, scale=D ** -0.5), "w3": rnd(E, F, D, scale=D ** -0.5),
                "w2": rnd(E, D, F, scale=F ** -0.5)}
    if kind == "gelu_mlp":
        return {"w1": rnd(E, F, D, scale=D ** -0.5), "b1": rnd(E, F, scale=0.1), "w2": rnd(E, D, F, scale=F ** -0.5),
                "b2": rnd(E, D, scale=0.1)}
    return {"w1": rnd(E, D, D, scale=D ** -0.5)}


def _slice(w, lo, hi):
    return {n: t[lo:hi].contiguous() for n, t in w.items()}


@pytest.mark.parametrize("kind,dtype,tokens,D,F,E,k,cf", [
    ("swiglu", torch.bfloat16, [256, 256], 256, 128, 16, 4, 1.0),
    ("swiglu", torch.bfloat16, [200, 313, 96, 257], 128, 64, 32, 2, 0.75),  # uneven ranks, drops
    ("linear", torch.float32, [100, 157], 64, 0, 8, 2, 1.25),
    ("gelu_mlp", torch.float32, [64, 64, 64, 64], 64, 96, 8, 2, 0.5),
])
def test_ep_equals_one_device_layer(kind, dtype, tokens, D, F, E, k, cf):
    R = len(tokens)
    epr = E // R
    T = sum(tokens)
    C = moe.moe_capacity(T, k, E, cf)
    g = torch.Generator().manual_seed(T + E)
    x = torch.randn(T, D, generator=g).to(dtype).to(DEV)
    w_router = (torch.randn(E, D, generator=g) * D ** -0.5).to(dtype).to(DEV)
    w = _weights(kind, E, D, F, g, dtype)
    xs = list(torch.split(x, tokens))
    xs = [t.contiguous() for t in xs]
    st = moe.new_status()
    out = ep.run_ranks_on_one_device(xs, E, k, C, kind, w_router, [_slice(w, q * epr, (q + 1) * epr)
                                                                    for q in range(R)], dev_status=st)
    assert moe.moe_read_status(st) == 0

    # the one-device layer over the concatenated batch
    r = moe.moe_route(x, k, w_router=w_router)
    d = moe.moe_dispatch(r["selected"], E, C, x=x)
    yb = moe.moe_expert_ffn(kind, d["xbuf"], d["used"], w["w1"], b1=w.get("b1"), w2=w.get("w2"), b2=w.get("b2"),
                            w3=w.get("w3"))
    y = moe.moe_combine(yb, r["selected"], d["slot"], r["gates_f32"], base_kind="input", base=x)

    cat = lambda key, part: torch.cat([o[key] for o in out[part]])  # noqa: E731
    assert torch.equal(cat("selected", "route"), r["selected"])
    assert torch.equal(cat("slot", "dispatch"), d["slot"])
    assert torch.equal(cat("kept", "dispatch"), d["kept"])
    assert torch.equal(cat("drops", "dispatch"), d["drops"])
    for q in range(R):
        assert torch.equal(out["plan"][q]["used"], d["used"])
        assert torch.equal(out["plan"][q]["overflow"], d["overflow"])
        assert torch.equal(out["plan"][q]["counts_total"], r["counts"])
    if cf < 1.0:
        assert int(d["overflow"].sum()) > 0
    # token_of_slot: each rank holds exactly the slots its tokens took
    merged = torch.stack([o["token_of_slot"] for o in out["dispatch"]]).max(0).values
    assert torch.equal(merged, d["token_of_slot"])
    # moved rows and expert outputs, expert by expert
    used = cpu(d["used"])
    for e in range(E):
        q, el, u = e // epr, e % epr, int(used[e])
        assert torch.equal(out["xbuf"][q][el, :u], d["xbuf"][e, :u])
        assert torch.equal(out["ybuf"][q][el, :u], yb[e, :u])
    assert torch.equal(torch.cat(out["y"]), y)
    # integer parts against the oracle's greedy loop on the whole batch
    disp = O.dispatch(cpu(r["selected"]), E, C)
    np.testing.assert_array_equal(cpu(cat("slot", "dispatch")), disp["slot"])


def test_ep_full_layer_shape_four_ranks():
    # the full-layer shape (H = 2048, E = 256, k = 8, F = 512, cf = 1.25) split over 4 ranks of 2048 tokens
    R, Tr, H, E, F, k = 4, 2048, 2048, 256, 512, 8
    T = R * Tr
    C = moe.moe_capacity(T, k, E, 1.25)
    g = torch.Generator().manual_seed(11)
    x = (torch.randint(-8, 9, (T, H), generator=g).float() / 8).to(torch.bfloat16).to(DEV)
    w_router = (torch.randint(-8, 9, (E, H), generator=g).float() / 128).to(torch.bfloat16).to(DEV)
    w = _weights("swiglu", E, H, F, g, torch.bfloat16)
    xs = [t.contiguous() for t in torch.split(x, Tr)]
    out = ep.run_ranks_on_one_device(xs, E, k, C, "swiglu", w_router,
                                     [_slice(w, q * (E // R), (q + 1) * (E // R)) for q in range(R)])
    r = moe.moe_route(x, k, w_router=w_router)
    d = moe.moe_dispatch(r["selected"], E, C, x=x)
    yb = moe.moe_expert_ffn("swiglu", d["xbuf"], d["used"], w["w1"], w2=w["w2"], w3=w["w3"])
    y = moe.moe_combine(yb, r["selected"], d["slot"], r["gates_f32"], base_kind="input", base=x)
    assert torch.equal(torch.cat([o["slot"] for o in out["dispatch"]]), d["slot"])
    assert torch.equal(torch.cat(out["y"]), y)


_CHILD = r"""
import sys, torch
sys.path.insert(0, sys.argv[1])
import sparse_mixture_experts_stable_b200 as moe
d = torch.load(sys.argv[2])
m = moe.moe_ipc_import(d["handle"])
sel, slot, gates = d["selected"].cuda(), d["slot"].cuda(), d["gates"].cuda()
E, C, N = d["E"], d["C"], d["N"]
y = moe.moe_ep_combine([m + d["offset"]], sel, slot, gates, E, C, N, torch.bfloat16)
torch.cuda.synchronize()
moe.moe_ipc_close(m)
torch.save(y.cpu(), sys.argv[3])
"""


def test_ipc_mapping_in_a_second_process():
    # A second process maps this process's expert output buffer and combines from it.
    E, C, N, T, k = 4, 32, 128, 60, 2
    g = torch.Generator().manual_seed(5)
    pad = torch.empty(3 * 1024, dtype=torch.uint8, device=DEV)  # the buffer need not start its allocation
    ybuf = torch.randn(E, C, N, generator=g).to(torch.bfloat16).to(DEV)
    lg = torch.randn(T, E, generator=g).to(DEV)
    r = moe.moe_route(lg, k)
    d = moe.moe_dispatch(r["selected"], E, C)
    want = moe.moe_combine(ybuf, r["selected"], d["slot"], r["gates_f32"])
    handle, offset = moe.moe_ipc_export(ybuf)
    torch.cuda.synchronize()
    with tempfile.TemporaryDirectory() as tmp:
        inp, outp = os.path.join(tmp, "in.pt"), os.path.join(tmp, "out.pt")
        torch.save(dict(handle=handle, offset=offset, selected=r["selected"].cpu(), slot=d["slot"].cpu(),
                        gates=r["gates_f32"].cpu(), E=E, C=C, N=N), inp)
        res = subprocess.run([sys.executable, "-c", _CHILD, ROOT, inp, outp], capture_output=True, text=True,
                             timeout=240)
        assert res.returncode == 0, res.stderr[-2000:]
        got = torch.load(outp)
    assert torch.equal(got, want.cpu())
    del pad


def test_ep_with_zero_capacity_keeps_every_row_as_its_base():
    # C = 0 (the numpy-layer page, section 3 edge checks): every assignment is dropped on every rank and y = x
    E, k, D, F = 8, 2, 64, 64
    g = torch.Generator().manual_seed(9)
    xs = [torch.randn(t, D, generator=g).to(torch.bfloat16).to(DEV) for t in (40, 24)]
    w_router = (torch.randn(E, D, generator=g) * D ** -0.5).to(torch.bfloat16).to(DEV)
    w = _weights("swiglu", E, D, F, g, torch.bfloat16)
    out = ep.run_ranks_on_one_device(xs, E, k, 0, "swiglu", w_router, [_slice(w, q * 4, (q + 1) * 4) for q in range(2)])
    for q in range(2):
        assert (out["dispatch"][q]["slot"] == -1).all()
        assert (out["plan"][q]["used"] == 0).all()
        assert torch.equal(out["y"][q], xs[q])
