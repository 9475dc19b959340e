"""Whole-layer forward passes on the GPU against the oracle, per workload.

Small sizes compare every output; the stated full sizes compare every integer
output and the routing floats on all tokens, and the layer output on sampled
tokens that the oracle computes one by one.
"""
import math

import numpy as np
import pytest
import torch

import sparse_mixture_experts_stable_b200 as moe
from oracle import oracle as O
from sparse_mixture_experts_stable_b200 import inputs as I
from sparse_mixture_experts_stable_b200.inputs import pages_layout
from sparse_mixture_experts_stable_b200.layer import SwiGLUMoE
from tests.gpu_util import (BF16_ATOL, BF16_RTOL, DEV, F32_ATOL, F32_RTOL, assert_close, assert_close_mag,
                            assert_within_bf16_ulp, check_dispatch, cpu, cpu64)

pytestmark = pytest.mark.gpu


def test_tiny_gelu_fp32_layer():
    cfg = I.tiny_gelu_fp32(seed=0)
    T, D, E, F, k = cfg["T"], cfg["D"], cfg["E"], cfg["F"], cfg["k"]
    C = moe.moe_capacity(T, k, E, cfg["capacity_factor"])
    assert C == 160
    dv = {n: cfg[n].to(DEV) for n in ("x", "w_router", "w1", "b1", "w2", "b2")}
    st = moe.new_status()
    r = moe.moe_route(dv["x"], k, w_router=dv["w_router"], dev_status=st)
    d = moe.moe_dispatch(r["selected"], E, C, x=dv["x"], dev_status=st)
    ybuf = moe.moe_expert_ffn("gelu_mlp", d["xbuf"], d["used"], dv["w1"], b1=dv["b1"], w2=dv["w2"], b2=dv["b2"],
                              dev_status=st)
    y = moe.moe_combine(ybuf, r["selected"], d["slot"], r["gates_f32"], base_kind="input", base=dv["x"],
                        dev_status=st)
    f, P, aux = moe.moe_aux_stats(r["counts"], r["prob_sum"], T, k, True, 0.01)
    assert moe.moe_read_status(st) == 0

    x64 = cpu64(cfg["x"])
    s = O.router_logits(x64, cpu64(cfg["w_router"]).T)
    w = dict(w1=pages_layout(cfg["w1"]), b1=cpu64(cfg["b1"]), w2=pages_layout(cfg["w2"]), b2=cpu64(cfg["b2"]))
    o = O.forward("gelu_mlp", x64, s, k, C, w, base_kind="input")
    np.testing.assert_array_equal(cpu(r["selected"]), o["selected"])
    check_dispatch(o, d, E, C, "tiny")
    wabs = {n: np.abs(v) for n, v in w.items()}
    mag = O.layer_rows("gelu_mlp", np.abs(x64), o["selected"], o["kept"], o["gates"], wabs, base_kind="input")
    assert_close_mag(cpu64(y), o["y"], mag, F32_RTOL, F32_ATOL, "tiny y")
    assert_close(cpu64(f), o["f"], F32_RTOL, 0, "f")
    assert_close(cpu64(P), o["P"], F32_RTOL, F32_ATOL, "P")
    assert math.isclose(float(aux[0]), o["aux"], rel_tol=F32_RTOL)
    assert math.isclose(float(aux[1]), 0.01 * o["aux"], rel_tol=F32_RTOL)
    # dropped assignments leave only the residual
    full = np.flatnonzero(o["drops"] == k)
    np.testing.assert_array_equal(cpu64(y)[full], x64[full])


@pytest.mark.parametrize("full_size", [False, True])
def test_dispatch_combine_top1_linear_bf16(full_size):
    cfg = I.dispatch_top1_bf16(seed=0) if full_size else I.dispatch_top1_bf16(seed=4, T=3000, D=256, E=16)
    T, D, E = cfg["T"], cfg["D"], cfg["E"]
    C = moe.moe_capacity(T, 1, E, cfg["capacity_factor"])
    idx = cfg["expert_idx"].view(T, 1).to(DEV)
    x, w, gate = cfg["x"].to(DEV), cfg["w"].to(DEV), cfg["gate"].view(T, 1).to(DEV)
    st = moe.new_status()
    d = moe.moe_dispatch(idx, E, C, x=x, dev_status=st)
    ybuf = moe.moe_expert_ffn("linear", d["xbuf"], d["used"], w, dev_status=st)
    y = moe.moe_combine(ybuf, idx, d["slot"], gate, base_kind="zero", dev_status=st)
    assert moe.moe_read_status(st) == 0
    o = O.dispatch(cpu(idx), E, C)
    check_dispatch(o, d, E, C, "top-1")
    yc = cpu64(y)
    dropped = ~o["kept"][:, 0]
    assert dropped.any()
    assert (yc[dropped] == 0).all()  # dropped tokens give all-zero rows
    rng = np.random.default_rng(0)
    kept_t = np.flatnonzero(~dropped)
    sample = np.sort(rng.choice(kept_t, min(160, len(kept_t)), replace=False)) if full_size else kept_t
    want = O.layer_rows("linear", cpu64(x), cpu(idx), o["kept"], cpu64(gate),
                        {"w1": pages_layout(cfg["w"])}, base_kind="zero", tokens=sample)
    assert_close(yc[sample], want, BF16_RTOL, BF16_ATOL, "top-1 y")


def _expert_weights64(cfg, e, prefix="w"):
    """One expert's SwiGLU weights in the pages' x @ W layout (float64)."""
    sl = slice(e, e + 1)
    return {"w1": pages_layout(cfg[prefix + "_gate"][sl]), "w3": pages_layout(cfg[prefix + "_up"][sl]),
            "w2": pages_layout(cfg[prefix + "_down"][sl])}


def _check_swiglu_layer(cfg, out, sel, kept, gates, token_of_slot, used, tokens, experts):
    """Compare the GPU's expert outputs and layer output with the oracle.

    ``experts``: every kept row of these experts is compared in the expert-major
    output buffer.  ``tokens``: y of these tokens is compared; the oracle forms
    each kept (token, expert) output and combines them with the gates and the
    shared-expert row.  The oracle converts each expert's weights once.
    """
    x64 = cpu64(cfg["x"])
    k = sel.shape[1]
    H = x64.shape[1]
    ybuf = out["ybuf"]
    pairs = {}  # expert -> list of (position in tokens, j)
    for i, t in enumerate(tokens):
        for j in range(k):
            if kept[t, j]:
                pairs.setdefault(int(sel[t, j]), []).append((i, j))
    u = np.zeros((len(tokens), k, H))
    for e in sorted(set(pairs) | set(int(e) for e in experts)):
        w = _expert_weights64(cfg, e)
        if e in experts and used[e]:
            rows = token_of_slot[e, :used[e]]
            want = O.expert_rows("swiglu", x64, rows, np.zeros(len(rows), np.int64), w)
            assert_close(cpu64(ybuf[e, :used[e]]), want, BF16_RTOL, BF16_ATOL, f"ybuf rows of expert {e}")
        if e in pairs:
            ij = pairs[e]
            toks = np.array([tokens[i] for i, _ in ij], np.int64)
            rows = O.expert_rows("swiglu", x64, toks, np.zeros(len(toks), np.int64), w)
            for (i, j), r in zip(ij, rows):
                u[i, j] = r
    shared = O.expert_rows("swiglu", x64, tokens, np.zeros(len(tokens), np.int64), _expert_weights64(cfg, 0, "s"))
    local = np.tile(np.arange(k), (len(tokens), 1))
    want_y = O.combine_precomputed(u, local, kept[tokens], gates[tokens], base=shared)
    assert_close(cpu64(out["y"])[tokens], want_y, BF16_RTOL, BF16_ATOL, "swiglu y")
    return want_y


def _unit_scale(cfg):
    """Expert weights rescaled so that gate/up pre-activations and expert outputs are O(1):
    then |y| is about 1 and the stated atol would catch one missing expert term."""
    c = dict(cfg)
    xs = float(cfg["x"].float().std())
    H, F = cfg["H"], cfg["F"]
    for pre, f_in in (("w", F), ("s", cfg["F_shared"])):
        for n in ("_gate", "_up"):
            t = cfg[pre + n].float()
            c[pre + n] = (t * (H ** -0.5 / xs / float(t.std()))).to(torch.bfloat16)
        t = cfg[pre + "_down"].float()
        c[pre + "_down"] = (t * (f_in ** -0.5 / float(t.std()))).to(torch.bfloat16)
    return c


@pytest.mark.parametrize("full_size,gathered,unit", [(False, False, False), (False, True, False),
                                                     (True, False, False), (True, True, False),
                                                     (True, False, True)])
def test_full_swiglu_layer_bf16(full_size, gathered, unit):
    if full_size:
        cfg = I.full_layer_bf16(seed=0)
    else:
        cfg = I.full_layer_bf16(seed=7, T=2048, H=512, E=32, F=256, k=8, F_shared=256)
    if unit:
        cfg = _unit_scale(cfg)
    T, H, E, F, k = cfg["T"], cfg["H"], cfg["E"], cfg["F"], cfg["k"]
    layer = SwiGLUMoE(T, H, E, F, k, cfg["capacity_factor"], F_shared=cfg["F_shared"], aux_coef=cfg["aux_coef"],
                      gathered=gathered)
    C = layer.C
    dv = {n: cfg[n].to(DEV) for n in ("x", "w_router", "router_bias", "w_gate", "w_up", "w_down", "s_gate", "s_up",
                                       "s_down")}
    out = layer.forward(dv["x"], dv["w_router"], dv["router_bias"], dv["w_gate"], dv["w_up"], dv["w_down"],
                        dv["s_gate"], dv["s_up"], dv["s_down"])
    assert moe.moe_read_status(layer.status) == 0

    x64 = cpu64(cfg["x"])
    s = O.router_logits(x64, cpu64(cfg["w_router"]).T, cpu64(cfg["router_bias"]))
    probs, sel, gates, counts, psum = O.route(s, k)
    np.testing.assert_array_equal(cpu(out["selected"]), sel)
    np.testing.assert_array_equal(cpu(out["counts"]), counts)
    assert_close(cpu64(out["gates_f32"]), gates, F32_RTOL, F32_ATOL, "gates")
    o = O.dispatch(sel, E, C)
    check_dispatch(o, out, E, C, "swiglu layer")
    fo, Po, auxo = O.aux(counts, psum, T, k)
    assert_within_bf16_ulp(cpu64(out["f"]), fo, "f")
    assert_within_bf16_ulp(cpu64(out["P"]), Po, "P")
    assert math.isclose(float(out["aux"][0]), auxo, rel_tol=1e-5)
    assert math.isclose(float(out["aux"][1]), cfg["aux_coef"] * auxo, rel_tol=1e-5)

    rng = np.random.default_rng(1)
    if full_size:
        tokens = np.sort(rng.choice(T, 512, replace=False))
        # every token with a dropped assignment among the first ones, and the fullest and emptiest experts
        tokens = np.unique(np.concatenate([tokens, np.flatnonzero(o["drops"] > 0)[:32]]))
        order = np.argsort(o["used"], kind="stable")
        experts = np.unique(np.concatenate([order[-4:], order[:4], rng.choice(E, 8, replace=False)]))
        assert len(experts) >= 16
    else:
        tokens, experts = np.arange(0, T, 3), np.arange(E)
    out["ybuf"] = layer.ybuf
    want = _check_swiglu_layer(cfg, out, sel, o["kept"], gates, o["token_of_slot"], o["used"], tokens, experts)
    if unit:
        # at unit scale the output is O(1): one expert term (gate ~ 1/k of an O(1) row) exceeds the tolerance
        assert float(np.abs(want).mean()) > 0.3


def test_full_layer_is_deterministic():
    cfg = I.full_layer_bf16(seed=9, T=1024, H=256, E=16, F=128, k=4, F_shared=128)
    layer = SwiGLUMoE(cfg["T"], cfg["H"], cfg["E"], cfg["F"], cfg["k"], cfg["capacity_factor"], F_shared=128)
    dv = {n: cfg[n].to(DEV) for n in ("x", "w_router", "router_bias", "w_gate", "w_up", "w_down", "s_gate", "s_up",
                                       "s_down")}
    args = [dv[n] for n in ("x", "w_router", "router_bias", "w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down")]
    y1 = layer.forward(*args)["y"].clone()
    y2 = layer.forward(*args)["y"].clone()
    assert torch.equal(y1, y2)
