"""moe_backward (fp32 linear experts) on the GPU against the oracle's closed forms.

Every output is a sum of terms; the fp32 tolerance is applied to the magnitude
of those terms (the oracle's closed forms evaluated on absolute values), and
for dlogits = g_i (dgate_i - sum_j g_j dgate_j) to the magnitudes of its operands.
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


def _run(cfg, aux_coef, residual=True):
    T, D, E, k = cfg["T"], cfg["D"], cfg["E"], cfg["k"]
    C = moe.moe_capacity(T, k, E, cfg["capacity_factor"])
    lg, x, w, dy = (cfg[n].to(DEV) for n in ("logits", "x", "w", "dy"))
    st = moe.new_status()
    r = moe.moe_route(lg, k, dev_status=st)
    d = moe.moe_dispatch(r["selected"], E, C, x=x, dev_status=st)
    ybuf = moe.moe_expert_ffn("linear", d["xbuf"], d["used"], w, dev_status=st)
    y = moe.moe_combine(ybuf, r["selected"], d["slot"], r["gates_f32"], base_kind="input" if residual else "zero",
                        base=x if residual else None, dev_status=st)
    dx, dW, dl, dg = moe.moe_backward(dy, x, lg, r["selected"], r["gates_f32"], d["slot"], d["used"],
                                      d["token_of_slot"], d["xbuf"], ybuf, w, C, use_residual=residual,
                                      aux_coef=aux_coef, counts=r["counts"], dev_status=st)
    assert moe.moe_read_status(st) == 0
    return C, r, d, y, dx, dW, dl, dg


def _compare(cfg, C, r, d, y, dx, dW, dl, dg, aux_coef, residual=True):
    T, E, k = cfg["T"], cfg["E"], cfg["k"]
    s = cpu64(cfg["logits"])
    x64, dy64 = cpu64(cfg["x"]), cpu64(cfg["dy"])
    W = pages_layout(cfg["w"])
    base = "input" if residual else "zero"
    o = O.forward("linear", x64, s, k, C, {"w1": W}, base_kind=base)
    np.testing.assert_array_equal(cpu(r["selected"]), o["selected"])
    check_dispatch(o, d, E, C, "fwd")
    sel, kept, g = o["selected"], o["kept"], o["gates"]
    # magnitudes of the summed terms: the same closed forms on absolute values
    y_mag = O.layer_rows("linear", np.abs(x64), sel, kept, g, {"w1": np.abs(W)}, base_kind=base)
    assert_close_mag(cpu64(y), o["y"], y_mag, F32_RTOL, F32_ATOL, "y")
    dx_o, dW_o, dl_o, dg_o = O.backward_linear(dy64, x64, s, sel, kept, g, W, use_residual=residual,
                                               aux_coef=aux_coef, normalize_by_k=True, counts=o["counts"])
    dx_m, dW_m, _, dg_m = O.backward_linear(np.abs(dy64), np.abs(x64), s, sel, kept, g, np.abs(W),
                                            use_residual=residual, aux_coef=0.0, counts=o["counts"])
    assert_close_mag(cpu64(dg), dg_o, dg_m, F32_RTOL, F32_ATOL, "dgate")
    assert_close_mag(cpu64(dx), dx_o, dx_m, F32_RTOL, F32_ATOL, "dx")
    assert_close_mag(cpu64(dW).transpose(0, 2, 1), dW_o, dW_m, F32_RTOL, F32_ATOL, "dW")
    # dlogits = g_i (dgate_i - sum_j g_j dgate_j): bound from the magnitudes of its operands
    scale = np.zeros_like(dl_o)
    gm = (g * dg_m).sum(1)
    for j in range(k):
        np.add.at(scale, (np.arange(T), sel[:, j]), g[:, j] * (dg_m[:, j] + gm))
    assert_close_mag(cpu64(dl), dl_o, scale, F32_RTOL, F32_ATOL, "dlogits")
    # unselected experts get exactly zero without the aux term
    if aux_coef == 0.0:
        mask = np.ones_like(dl_o, bool)
        mask[np.arange(T)[:, None], sel] = False
        assert (cpu64(dl)[mask] == 0).all()


@pytest.mark.parametrize("aux_coef,residual", [(0.0, True), (0.37, True), (0.0, False)])
def test_backward_small(aux_coef, residual):
    cfg = I.fwd_bwd_fp32(seed=2, T=700, D=256, E=16, k=2)
    res = _run(cfg, aux_coef, residual)
    _compare(cfg, *res, aux_coef=aux_coef, residual=residual)


def test_backward_full_size():
    cfg = I.fwd_bwd_fp32(seed=0)  # T=8192, D=1024, E=64, k=2, C=256
    res = _run(cfg, 0.0)
    assert res[0] == 256
    _compare(cfg, *res, aux_coef=0.0)


def test_backward_top1_logit_gradient_is_zero():
    cfg = I.fwd_bwd_fp32(seed=5, T=300, D=64, E=8, k=1)
    _, _, _, _, _, _, dl, _ = _run(cfg, 0.0)
    assert torch.count_nonzero(dl) == 0
