"""The one-kernel bf16 router (scores on tcgen05, softmax, top-k, gates) on the GPU.

moe_route takes this path for bf16 activations with a router weight, softmax
scoring, no selection bias or z-loss, E = 256 and k <= 8 (the E = 128 cases
below exercise the two-kernel path that every other shape takes).  Each CTA
owns a run of tokens balanced in 32-row units and walks it in tiles of up to
128 rows, so the cases below cover runs shorter than one box, runs ending
inside a tile, several tiles per CTA, K not a multiple of 64, a logit bias and
the fp32 logits output.  Inputs are dyadic, so every score is exact in fp32 and
the integer outputs must equal the oracle's bit for bit.
"""
import numpy as np
import pytest
import torch

import sparse_mixture_experts_stable_b200 as moe
from oracle import oracle as O
from sparse_mixture_experts_stable_b200 import inputs as I
from tests.gpu_util import DEV, F32_ATOL, F32_RTOL, assert_close, assert_within_bf16_ulp, cpu, cpu64

pytestmark = pytest.mark.gpu


def _dyadic_bias(E, seed):
    rng = np.random.default_rng(seed)
    return torch.tensor(np.round(rng.normal(0.0, 0.5, E) * 1024) / 1024, dtype=torch.float32)


@pytest.mark.parametrize("T,D,E,k", [
    (1, 64, 256, 8), (31, 64, 128, 2), (33, 128, 256, 1), (129, 200, 256, 8), (4733, 256, 128, 4),
    (20000, 128, 256, 8), (40000, 64, 256, 6),
])
@pytest.mark.parametrize("with_bias", [False, True])
def test_fused_router_matches_oracle(T, D, E, k, with_bias):
    cfg = I.router_bf16(seed=T % 97, T=T, D=D, E=E, k=k)
    x, w = cfg["x"].to(DEV), cfg["w_router"].to(DEV)
    bias = _dyadic_bias(E, T).to(DEV) if with_bias else None
    st = moe.new_status()
    r = moe.moe_route(x, k, w_router=w, layout="ED", logit_bias=bias, want_logits=True, dev_status=st)
    assert moe.moe_read_status(st) == 0
    s64 = O.router_logits(cpu64(x), cpu64(w).T, None if bias is None else cpu64(bias))
    probs, sel, gates, counts, psum = O.route(s64, k)
    np.testing.assert_array_equal(cpu64(r["logits"]), s64)
    np.testing.assert_array_equal(cpu(r["selected"]), sel)
    np.testing.assert_array_equal(cpu(r["counts"]), counts)
    assert_close(cpu64(r["gates_f32"]), gates, F32_RTOL, F32_ATOL, "gates_f32")
    assert_within_bf16_ulp(cpu64(r["gates"]), gates, "gates bf16")
    assert_close(cpu64(r["prob_sum"]), psum, F32_RTOL, F32_ATOL * T, "prob_sum")


def test_fused_router_heavy_ties():
    # integer scores from a short contraction: most rows hold long runs of equal scores, spread over all
    # four column quarters of the epilogue, so the merge must keep every tie in index order
    rng = np.random.default_rng(44)
    T, D, E, k = 2500, 16, 256, 8
    x = torch.tensor(rng.integers(-1, 2, size=(T, D)), dtype=torch.bfloat16)
    w = torch.tensor(rng.integers(-1, 2, size=(E, D)), dtype=torch.bfloat16)
    r = moe.moe_route(x.to(DEV), k, w_router=w.to(DEV))
    s64 = O.router_logits(cpu64(x), cpu64(w).T)
    _, sel, _, counts, _ = O.route(s64, k)
    np.testing.assert_array_equal(cpu(r["selected"]), sel)
    np.testing.assert_array_equal(cpu(r["counts"]), counts)


def test_fused_router_without_logits_output_and_strided_x():
    # x as a column slice of a wider matrix (row stride 2*D), no logits requested
    T, D, E, k = 3001, 256, 256, 8
    cfg = I.router_bf16(seed=5, T=T, D=2 * D, E=E, k=k)
    xw = cfg["x"].to(DEV)
    x = xw[:, :D]
    w = cfg["w_router"][:, :D].contiguous().to(DEV)
    r = moe.moe_route(x, k, w_router=w)
    s64 = O.router_logits(cpu64(x), cpu64(w).T)
    _, sel, gates, counts, _ = O.route(s64, k)
    np.testing.assert_array_equal(cpu(r["selected"]), sel)
    np.testing.assert_array_equal(cpu(r["counts"]), counts)
    assert_close(cpu64(r["gates_f32"]), gates, F32_RTOL, F32_ATOL, "gates_f32")


def test_fused_router_flags_nonfinite_rows():
    T, D, E, k = 500, 64, 256, 8
    cfg = I.router_bf16(seed=6, T=T, D=D, E=E, k=k)
    x = cfg["x"].clone()
    x[123, 7] = float("inf")
    st = moe.new_status()
    r = moe.moe_route(x.to(DEV), k, w_router=cfg["w_router"].to(DEV), dev_status=st)
    assert moe.moe_read_status(st) == moe.binding.MOE_ERR_NONFINITE
    ok = np.ones(T, bool)
    ok[123] = False
    s64 = O.router_logits(cpu64(x)[ok], cpu64(cfg["w_router"]).T)
    _, sel, _, _, _ = O.route(s64, k)
    np.testing.assert_array_equal(cpu(r["selected"])[ok], sel)
    # the flagged token's experts are still valid indices
    assert ((cpu(r["selected"]) >= 0) & (cpu(r["selected"]) < E)).all()
