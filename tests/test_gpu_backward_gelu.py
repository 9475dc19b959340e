"""moe_backward_gelu (fp32 GELU-MLP experts, split-tf32 products) against the
fp64 oracle backward.

The forward runs on the GPU (route, dispatch, GELU experts); the oracle
recomputes everything in fp64 from the same fp32 inputs.  Integer routing is
exact.  Each gradient is a sum of terms; the fp32 tolerance is applied to the
magnitude of those terms, estimated by the oracle backward on absolute values
(|x|, |W|, |b|, |dy|).  For the GELU factors that estimate stays within a
factor of about two of the true term magnitudes (gelu(|z|) >= |gelu(z)|/2 and
gelu'(|z|) >= 0.44 max|gelu'|), which is far inside the margin between the
fp32 tolerance and the split-tf32 rounding (about 2^-22 relative).
"""
import numpy as np
import pytest
import torch

import sparse_mixture_experts_stable_b200 as moe
from oracle import oracle as O
from sparse_mixture_experts_stable_b200 import inputs as I
from sparse_mixture_experts_stable_b200.inputs import pages_layout
from tests.gpu_util import DEV, F32_ATOL, F32_RTOL, assert_close_mag, check_dispatch, cpu, cpu64

pytestmark = pytest.mark.gpu


def _run_and_compare(x, w_router, w1, b1, w2, b2, dy, k, cf, residual, aux):
    T, D = x.shape
    E, F, _ = w1.shape
    C = moe.moe_capacity(T, k, E, cf)
    xd, dyd = x.to(DEV), dy.to(DEV)
    w1d, b1d, w2d, b2d = w1.to(DEV), b1.to(DEV), w2.to(DEV), b2.to(DEV)
    st = moe.new_status()
    r = moe.moe_route(xd, k, w_router=w_router.to(DEV), want_logits=True, dev_status=st)
    d = moe.moe_dispatch(r["selected"], E, C, x=xd, dev_status=st)
    ybuf = moe.moe_expert_ffn("gelu_mlp", d["xbuf"], d["used"], w1d, b1=b1d, w2=w2d, b2=b2d, dev_status=st)
    dx, dw1, db1, dw2, db2, dl, dg = moe.moe_backward_gelu(
        dyd, r["logits"], r["selected"], r["gates_f32"], d["slot"], d["used"], d["xbuf"], ybuf, w1d, b1d, w2d, C,
        use_residual=residual, aux_coef=aux, counts=r["counts"], dev_status=st)
    assert moe.moe_read_status(st) == 0

    s64 = cpu64(r["logits"])
    x64, dy64 = cpu64(x), cpu64(dy)
    W = {"w1": pages_layout(w1), "b1": cpu64(b1), "w2": pages_layout(w2), "b2": cpu64(b2)}
    o = O.forward("gelu_mlp", x64, s64, k, C, W, base_kind="input" if residual else "zero")
    np.testing.assert_array_equal(cpu(r["selected"]), o["selected"])
    check_dispatch(o, d, E, C, "fwd")
    sel, kept, g = o["selected"], o["kept"], o["gates"]
    if cf < 1.0:
        assert (~kept).any()
    want = O.backward_gelu(dy64, x64, s64, sel, kept, g, W["w1"], W["b1"], W["w2"], W["b2"], use_residual=residual,
                           aux_coef=aux, counts=o["counts"])
    mag = O.backward_gelu(np.abs(dy64), np.abs(x64), s64, sel, kept, g, np.abs(W["w1"]), np.abs(W["b1"]),
                          np.abs(W["w2"]), np.abs(W["b2"]), use_residual=residual, aux_coef=0.0,
                          counts=o["counts"])
    wdx, wdW1, wdb1, wdW2, wdb2, wdl, wdg = want
    mdx, mdW1, mdb1, mdW2, mdb2, _, mdg = mag
    assert_close_mag(cpu64(dg), wdg, mdg, F32_RTOL, F32_ATOL, "dgate")
    assert (cpu64(dg)[~kept] == 0).all()
    assert_close_mag(cpu64(dx), wdx, mdx, F32_RTOL, F32_ATOL, "dx")
    # the oracle's weight gradients are in the x@W layout: (E, D, F) and (E, F, N)
    assert_close_mag(cpu64(dw1), wdW1.transpose(0, 2, 1), mdW1.transpose(0, 2, 1), F32_RTOL, F32_ATOL, "dw1")
    assert_close_mag(cpu64(dw2), wdW2.transpose(0, 2, 1), mdW2.transpose(0, 2, 1), F32_RTOL, F32_ATOL, "dw2")
    assert_close_mag(cpu64(db1), wdb1, mdb1, F32_RTOL, F32_ATOL, "db1")
    assert_close_mag(cpu64(db2), wdb2, mdb2, F32_RTOL, F32_ATOL, "db2")
    # dlogits = g_i (dgate_i - sum_j g_j dgate_j) (+ aux): bound from the magnitudes of its operands
    scale = np.zeros_like(wdl)
    gm = (g * mdg).sum(1)
    for j in range(k):
        np.add.at(scale, (np.arange(T), sel[:, j]), g[:, j] * (mdg[:, j] + gm))
    assert_close_mag(cpu64(dl), wdl, scale, F32_RTOL, F32_ATOL, "dlogits")
    # an expert that received no token has exactly zero weight and bias gradients
    for e in np.flatnonzero(o["used"] == 0):
        assert (cpu64(dw1)[e] == 0).all() and (cpu64(db2)[e] == 0).all()


def test_backward_gelu_tiny_layer():
    # the tiny fp32 GELU layer (T=512, D=64, E=8, F=256, k=2, cf=1.25) with a residual base
    cfg = I.tiny_gelu_fp32(seed=1)
    dy = torch.randn(cfg["T"], cfg["D"], generator=torch.Generator().manual_seed(7))
    _run_and_compare(cfg["x"], cfg["w_router"], cfg["w1"], cfg["b1"], cfg["w2"], cfg["b2"], dy, cfg["k"],
                     cfg["capacity_factor"], True, 0.0)


@pytest.mark.parametrize("T,D,F,E,k,cf,residual,aux", [
    (517, 72, 40, 5, 3, 0.8, False, 0.2),    # ragged sizes, drops, aux term
    (300, 128, 160, 6, 2, 1.5, True, 0.0),   # several K tiles in every product
    (64, 32, 8, 3, 1, 2.0, True, 0.0),       # top-1, tiny F
    (300, 160, 256, 4, 2, 1.2, True, 0.0),   # dW1 through TMA stores with a last column tile past D
])
def test_backward_gelu_matches_oracle(T, D, F, E, k, cf, residual, aux):
    g = torch.Generator().manual_seed(T + D + F)

    def rnd(*shape, scale=1.0):
        return torch.randn(*shape, generator=g) * scale

    # weights scaled so that z = x W1^T + b1 is about N(0, 1): GELU well away from linear
    x = rnd(T, D)
    w_router = rnd(E, D, scale=D ** -0.5)
    w1, b1 = rnd(E, F, D, scale=D ** -0.5), rnd(E, F, scale=0.3)
    w2, b2 = rnd(E, D, F, scale=F ** -0.5), rnd(E, D, scale=0.3)
    dy = rnd(T, D)
    _run_and_compare(x, w_router, w1, b1, w2, b2, dy, k, cf, residual, aux)


def test_backward_gelu_with_nothing_kept():
    T, D, F, E, k = 40, 32, 16, 2, 1
    g = torch.Generator().manual_seed(4)
    lg = torch.randn(T, E, generator=g).to(DEV)
    dy = torch.randn(T, D, generator=g).to(DEV)
    w1, b1 = torch.randn(E, F, D, generator=g).to(DEV), torch.randn(E, F, generator=g).to(DEV)
    w2 = torch.randn(E, D, F, generator=g).to(DEV)
    r = moe.moe_route(lg, k)
    d = moe.moe_dispatch(r["selected"], E, 0)
    empty_x = torch.empty(E, 0, D, device=DEV)
    dx, dw1, db1, dw2, db2, dl, dg = moe.moe_backward_gelu(dy, lg, r["selected"], r["gates_f32"], d["slot"],
                                                           d["used"], empty_x, empty_x, w1, b1, w2, 0,
                                                           use_residual=True)
    assert torch.equal(dx, dy)
    for t in (dw1, db1, dw2, db2, dl, dg):
        assert (t == 0).all()
