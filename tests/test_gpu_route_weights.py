"""moe_route with a bf16 router weight (tensor-core scores, then the top-k
kernel) against the fp64 oracle over expert counts that are not multiples of
32, k from 1 to 16, a logit bias, the Module 7 variants, and no logits output.

Inputs are dyadic (integers times 2^-6, sums below 2^6), so every fp32 score is
exact whatever the accumulation order: selections and counts must match bit for
bit, ties included (the lower expert index wins).
"""
import math

import numpy as np
import pytest
import torch

import sparse_mixture_experts_stable_b200 as moe
from oracle import oracle as O
from sparse_mixture_experts_stable_b200 import inputs as I
from tests.gpu_util import DEV, F32_ATOL, F32_RTOL, assert_close, assert_within_bf16_ulp, cpu, cpu64

pytestmark = pytest.mark.gpu


def _dyadic_router(seed, T, D, E, ties=True):
    cfg = I.router_bf16(seed=seed, T=T, D=D, E=E, k=1, tie_columns=4 if (ties and E >= 8) else 0,
                        zero_row_every=37)
    return cfg["x"].to(DEV), cfg["w_router"].to(DEV)


def _check(r, s64, k, what):
    probs, sel, gates, counts, psum = O.route(s64, k)
    np.testing.assert_array_equal(cpu(r["selected"]), sel, err_msg=what + " selected")
    np.testing.assert_array_equal(cpu(r["counts"]), counts, err_msg=what + " counts")
    assert_close(cpu64(r["gates_f32"]), gates, F32_RTOL, F32_ATOL, what + " gates_f32")
    assert_within_bf16_ulp(cpu64(r["gates"]), gates, what + " gates bf16")
    assert_close(cpu64(r["prob_sum"]), psum, F32_RTOL, F32_ATOL * s64.shape[0], what + " prob_sum")


@pytest.mark.parametrize("E,k", [(256, 8), (256, 1), (64, 2), (40, 8), (8, 8), (1, 1), (200, 5), (256, 16), (320, 8)])
def test_router_weights_match_oracle(E, k):
    # T spans several 128-token tiles and ends in a ragged tile
    T, D = 1000, 256
    x, w = _dyadic_router(7 + E + k, T, D, E)
    r = moe.moe_route(x, k, w_router=w, want_logits=True, want_z_loss=True)
    s64 = O.router_logits(cpu64(x), cpu64(w).T)
    np.testing.assert_array_equal(cpu64(r["logits"]), s64)
    _check(r, s64, k, f"weights E={E} k={k}")
    assert math.isclose(float(r["z_loss"][0]), O.z_loss(s64), rel_tol=1e-5)


def test_router_without_logits_output_and_with_bias():
    T, D, E, k = 777, 192, 96, 4
    x, w = _dyadic_router(11, T, D, E)
    bias = torch.tensor((np.arange(E) % 7 - 3) / 16.0, dtype=torch.float32, device=DEV)
    r = moe.moe_route(x, k, w_router=w, logit_bias=bias)  # no logits requested
    s64 = O.router_logits(cpu64(x), cpu64(w).T, cpu64(bias))
    _check(r, s64, k, "with logit bias")
    r2 = moe.moe_route(x, k, w_router=w, logit_bias=bias, want_logits=True)
    np.testing.assert_array_equal(cpu64(r2["logits"]), s64)
    for key in ("selected", "counts", "gates_f32", "prob_sum"):
        assert torch.equal(r[key], r2[key]), key


@pytest.mark.parametrize("scoring", ["softmax", "sigmoid"])
@pytest.mark.parametrize("with_bias", [False, True])
def test_router_weight_variants(scoring, with_bias):
    T, D, E, k = 1500, 512, 64, 4
    cfg = I.router_spread_bf16(seed=21 + with_bias, T=T, D=D, E=E)
    x, w = cfg["x"].to(DEV), cfg["w_router"].to(DEV)
    sb = torch.tensor((np.arange(E) % 5 - 2) / 64.0, dtype=torch.float32, device=DEV) if with_bias else None
    r = moe.moe_route(x, k, w_router=w, scoring=scoring, selection_bias=sb, want_logits=True, want_z_loss=True)
    s64 = O.router_logits(cpu64(x), cpu64(w).T)
    np.testing.assert_array_equal(cpu64(r["logits"]), s64)
    sb64 = None if sb is None else cpu64(sb)
    clean, sel, gates, counts = O.route_variant(s64, k, scoring, sb64)
    gsel = cpu(r["selected"])
    # with a selection bias the ranking is on fp32 clean scores: near-ties are
    # decided within fp32 resolution, so those tokens are only checked for validity
    key = clean + sb64[None, :] if sb64 is not None else s64
    srt = -np.sort(-key, axis=1)
    sure = (srt[:, k - 1] - srt[:, k]) > 1e-5
    assert sure.mean() > 0.9
    np.testing.assert_array_equal(gsel[sure], sel[sure])
    assert_close(cpu64(r["gates_f32"])[sure], gates[sure], F32_RTOL, F32_ATOL, "gates")
    picked = np.take_along_axis(key, gsel, 1)
    assert (picked >= srt[:, k - 1:k] - 1e-5).all()
    assert all(len(set(row)) == k for row in gsel.tolist())
    np.testing.assert_array_equal(cpu(r["counts"]), np.bincount(gsel.ravel(), minlength=E))
    assert_close(cpu64(r["prob_sum"]), clean.sum(0), F32_RTOL, F32_ATOL * T, "prob_sum")
    assert math.isclose(float(r["z_loss"][0]), O.z_loss(s64), rel_tol=1e-5)


def test_weights_and_given_logits_paths_agree():
    T, D, E, k = 2000, 256, 128, 8
    x, w = _dyadic_router(41, T, D, E)
    a = moe.moe_route(x, k, w_router=w, want_logits=True)
    b = moe.moe_route(a["logits"], k)
    for key in ("selected", "counts"):
        assert torch.equal(a[key], b[key]), key
    assert_close(cpu64(a["gates_f32"]), cpu64(b["gates_f32"]), F32_RTOL, F32_ATOL, "gates")
    assert_close(cpu64(a["prob_sum"]), cpu64(b["prob_sum"]), F32_RTOL, F32_ATOL * T, "prob_sum")
