"""moe_route_ex (sigmoid scoring, selection-only bias, z-loss) and
moe_renormalize_kept_gates on the GPU, against the page's pinned values and the oracle.

The ranking with a selection bias is decided on fp32 clean scores on the GPU and
fp64 in the oracle; tokens whose k-th and (k+1)-th oracle keys are closer than
fp32 can resolve are ambiguous, so for them only the validity of the GPU's
choice is checked.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import sparse_mixture_experts_stable_b200 as moe
from oracle import oracle as O
from tests.conftest import GOLDEN
from tests.gpu_util import DEV, F32_ATOL, F32_RTOL, assert_close, cpu, cpu64

pytestmark = pytest.mark.gpu


def test_module7_sigmoid_router_on_gpu():
    g = json.load(open(os.path.join(GOLDEN, "module7_router_variants.json")))
    lg = torch.tensor([g["logits"]], dtype=torch.float32, device=DEV)
    r = moe.moe_route(lg, g["top_k"], scoring="sigmoid")
    assert cpu(r["selected"])[0].tolist() == g["selected"]
    assert_close(cpu64(r["gates_f32"])[0], g["gates"], F32_RTOL, F32_ATOL, "sigmoid gates")
    assert_close(cpu64(r["prob_sum"]), g["scores"], F32_RTOL, F32_ATOL, "sigmoid scores")
    bias = torch.tensor(g["bias"], dtype=torch.float32, device=DEV)
    rb = moe.moe_route(lg, g["top_k"], scoring="sigmoid", selection_bias=bias)
    assert cpu(rb["selected"])[0].tolist() == g["selected_with_bias"]
    assert_close(cpu64(rb["gates_f32"])[0], g["gates_with_bias"], F32_RTOL, F32_ATOL, "sigmoid gates with bias")


def _key_margin(clean, s, sel_bias, k):
    key = clean + sel_bias[None, :] if sel_bias is not None else s
    srt = -np.sort(-key, axis=1)
    return srt[:, k - 1] - srt[:, k]


@pytest.mark.parametrize("scoring", ["softmax", "sigmoid"])
@pytest.mark.parametrize("with_bias", [False, True])
def test_route_variants_match_oracle(scoring, with_bias):
    rng = np.random.default_rng(31 + with_bias)
    T, E, k = 3000, 64, 4
    s = rng.standard_normal((T, E)).astype(np.float32)
    sb = (rng.standard_normal(E) * 0.05).astype(np.float32) if with_bias else None
    r = moe.moe_route(torch.from_numpy(s).to(DEV), k, scoring=scoring,
                      selection_bias=None if sb is None else torch.from_numpy(sb).to(DEV), want_z_loss=True)
    clean, sel, gates, counts = O.route_variant(s.astype(np.float64), k, scoring,
                                                None if sb is None else sb.astype(np.float64))
    gsel = cpu(r["selected"])
    sure = _key_margin(clean, s.astype(np.float64), None if sb is None else sb.astype(np.float64), k) > 1e-5
    assert sure.mean() > 0.95
    np.testing.assert_array_equal(gsel[sure], sel[sure])
    assert_close(cpu64(r["gates_f32"])[sure], gates[sure], F32_RTOL, F32_ATOL, "gates")
    # counts are those of the GPU's own selection; prob_sum is the clean-score sum
    np.testing.assert_array_equal(cpu(r["counts"]), np.bincount(gsel.ravel(), minlength=E))
    assert_close(cpu64(r["prob_sum"]), clean.sum(0), F32_RTOL, F32_ATOL * T, "prob_sum")
    assert math.isclose(float(r["z_loss"][0]), O.z_loss(s), rel_tol=1e-5)
    # every selection is a valid top-k within fp32 resolution of the oracle keys
    key = clean + sb[None, :] if sb is not None else s.astype(np.float64)
    kth = -np.sort(-key, axis=1)[:, k - 1]
    picked = np.take_along_axis(key, gsel, 1)
    assert (picked >= kth[:, None] - 1e-5).all()
    assert all(len(set(row)) == k for row in gsel.tolist())


def test_renormalize_kept_gates_matches_oracle():
    rng = np.random.default_rng(41)
    T, E, k, C = 2000, 32, 4, 150
    s = rng.standard_normal((T, E))
    _, sel, gates, _, _ = O.route(s, k)
    d = O.dispatch(sel, E, C)
    want = O.renormalize_kept(gates, d["kept"])
    got = moe.moe_renormalize_kept_gates(torch.from_numpy(gates.astype(np.float32)).to(DEV),
                                         torch.from_numpy(d["slot"]).to(DEV))
    assert_close(cpu64(got), want, F32_RTOL, F32_ATOL, "renormalised gates")
    full = d["drops"] == k
    assert (cpu64(got)[full] == 0).all()
