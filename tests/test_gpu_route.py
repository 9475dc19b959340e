"""moe_route / moe_aux_stats on the GPU against the fp64 oracle.

Integer outputs (selected experts, counts) must match bit for bit: the inputs
are dyadic, so every fp32 score is exact and the tie rule decides alone.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import sparse_mixture_experts_stable_b200 as moe
from oracle import oracle as O
from sparse_mixture_experts_stable_b200 import inputs as I
from tests.conftest import GOLDEN
from tests.gpu_util import DEV, F32_ATOL, F32_RTOL, assert_close, assert_within_bf16_ulp, cpu, cpu64

pytestmark = pytest.mark.gpu


def _check_route(r, s64, k, what, logits_exact=True):
    probs, sel, gates, counts, psum = O.route(s64, k)
    if "logits" in r and logits_exact:
        np.testing.assert_array_equal(cpu64(r["logits"]), s64, err_msg=what + " logits")
    np.testing.assert_array_equal(cpu(r["selected"]), sel, err_msg=what + " selected")
    np.testing.assert_array_equal(cpu(r["counts"]), counts, err_msg=what + " counts")
    assert_close(cpu64(r["gates_f32"]), gates, F32_RTOL, F32_ATOL, what + " gates_f32")
    if r["gates"].dtype == torch.bfloat16:
        assert_within_bf16_ulp(cpu64(r["gates"]), gates, what + " gates bf16")
    assert_close(cpu64(r["prob_sum"]), psum, F32_RTOL, F32_ATOL * s64.shape[0], what + " prob_sum")
    return probs, sel, gates, counts, psum


def test_router_page_examples_on_gpu():
    g = json.load(open(os.path.join(GOLDEN, "router_load_statistics_examples.json")))
    tol = 0.5 * 10 ** -g["print_decimals"]
    for ex in g["examples"]:
        x = torch.tensor(ex["x"], dtype=torch.float32, device=DEV)
        w = torch.tensor(ex["w_router"], dtype=torch.float32, device=DEV)  # (D, E) as on the page
        k = ex["k"]
        T, E = x.shape[0], w.shape[1]
        r = moe.moe_route(x, k, w_router=w, layout="DE")
        assert cpu(r["selected"]).tolist() == ex["selected_experts"]
        np.testing.assert_allclose(cpu64(r["gates_f32"]), ex["selected_weights"], rtol=0, atol=1e-7)
        f, P, aux = moe.moe_aux_stats(r["counts"], r["prob_sum"], T, k)
        np.testing.assert_allclose(cpu64(f), ex["token_fraction"], rtol=0, atol=0)
        np.testing.assert_allclose(cpu64(P), ex["probability_mass"], rtol=0, atol=tol)
        # page form of the combine: expert_outputs (T, E, Dout) seen as ybuf[e, t] with slot t
        u = torch.tensor(ex["expert_outputs"], dtype=torch.float32, device=DEV)
        ybuf = u.transpose(0, 1).contiguous()  # (E, C=T, Dout)
        slot = torch.arange(T, device=DEV).view(T, 1).expand(T, k).contiguous()
        base = torch.tensor(ex["shared_output"], dtype=torch.float32, device=DEV)
        y = moe.moe_combine(ybuf, r["selected"], slot, r["gates_f32"], base_kind="tensor", base=base)
        np.testing.assert_allclose(cpu64(y), ex["output"], rtol=0, atol=1e-6)


@pytest.mark.parametrize("layout", ["ED", "DE"])
def test_router_bf16_ties_small(layout):
    # several 128-row tiles plus a ragged tail; tie columns and all-zero rows
    cfg = I.router_bf16(seed=1, T=3000, D=512, E=256, k=8)
    x = cfg["x"].to(DEV)
    w_ed = cfg["w_router"].to(DEV)
    w = w_ed if layout == "ED" else w_ed.t().contiguous()
    r = moe.moe_route(x, 8, w_router=w, layout=layout, want_logits=True)
    s64 = O.router_logits(cpu64(x), cpu64(w_ed).T)
    _, sel, _, _, _ = _check_route(r, s64, 8, f"router bf16 {layout}")
    # all-zero rows tie across every expert: the lowest indices win
    assert (sel[::64] == np.arange(8)).all()


def test_router_bf16_full_size():
    cfg = I.router_bf16(seed=0)  # T=65536, D=2048, E=256, k=8
    x = cfg["x"].to(DEV)
    w = cfg["w_router"].to(DEV)
    r = moe.moe_route(x, 8, w_router=w, layout="ED", want_logits=True)
    s64 = O.router_logits(cpu64(x), cpu64(w).T)
    probs, sel, gates, counts, psum = _check_route(r, s64, 8, "router bf16 full")
    f, P, aux = moe.moe_aux_stats(r["counts"], r["prob_sum"], cfg["T"], 8, out_dtype=torch.bfloat16)
    fo, Po, auxo = O.aux(counts, psum, cfg["T"], 8)
    assert_within_bf16_ulp(cpu64(f), fo, "f")
    assert_within_bf16_ulp(cpu64(P), Po, "P")
    assert math.isclose(float(aux[0]), auxo, rel_tol=1e-5)
    assert math.isclose(float(cpu64(f).sum()), 8.0, rel_tol=1e-2)


def test_router_fp32_tiny_exact_scores():
    cfg = I.tiny_gelu_fp32(seed=0)
    x, w = cfg["x"].to(DEV), cfg["w_router"].to(DEV)
    # precondition for exact fp32 scores: every partial sum is a multiple of
    # 2^-18 below 2^6 in magnitude
    bound = (np.abs(cpu64(x)) @ np.abs(cpu64(w)).T).max()
    assert bound < 64
    r = moe.moe_route(x, cfg["k"], w_router=w, layout="ED", want_logits=True)
    s64 = O.router_logits(cpu64(x), cpu64(w).T)
    _check_route(r, s64, cfg["k"], "router fp32")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_given_logits(dtype):
    cfg = I.fwd_bwd_fp32(seed=3, T=8192, D=8, E=64, k=2)
    lg = cfg["logits"].to(dtype).to(DEV)
    bias = torch.linspace(-0.5, 0.5, 64, device=DEV)
    r = moe.moe_route(lg, 2, logit_bias=bias, want_logits=True)
    s64 = cpu64(lg) + cpu64(bias).astype(np.float32).astype(np.float64)
    s32 = (cpu64(lg).astype(np.float32) + cpu64(bias).astype(np.float32)).astype(np.float64)
    _check_route(r, s32, 2, f"given logits {dtype}")
    assert np.abs(s64 - s32).max() < 1e-6


@pytest.mark.parametrize("E,k", [(1, 1), (8, 8), (3, 2), (64, 64), (1000, 5)])
def test_route_edge_shapes(E, k):
    rng = np.random.default_rng(E * 100 + k)
    T = 777
    lg = torch.tensor(rng.integers(-3, 4, size=(T, E)).astype(np.float32), device=DEV)
    r = moe.moe_route(lg, k)
    _check_route(r, cpu64(lg), k, f"E={E} k={k}")


def test_route_flags_nonfinite_logits():
    lg = torch.randn(100, 16, device=DEV)
    lg[37, 5] = float("nan")
    st = moe.new_status()
    r = moe.moe_route(lg, 2, dev_status=st)
    assert moe.moe_read_status(st) == moe.binding.MOE_ERR_NONFINITE
    ok = np.ones(100, bool)
    ok[37] = False
    _, sel, _, _, _ = O.route(cpu64(lg)[ok], 2)
    np.testing.assert_array_equal(cpu(r["selected"])[ok], sel)


def test_route_is_deterministic():
    cfg = I.router_bf16(seed=2, T=5000, D=256, E=256, k=8, zero_row_every=0)
    x, w = cfg["x"].to(DEV), cfg["w_router"].to(DEV)
    a = moe.moe_route(x, 8, w_router=w)
    b = moe.moe_route(x, 8, w_router=w)
    for key in ("selected", "gates_f32", "counts", "prob_sum"):
        assert torch.equal(a[key], b[key]), key
