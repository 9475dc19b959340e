"""moe_backward (fp32 linear experts) on the GPU against the oracle's closed forms.

dlogits is a difference of similar terms, so its bound scales with the terms
it is formed from: |err| <= atol + rtol * gate_i * (|dgate_i| + sum_j gate_j |dgate_j|)
(the fp32 tolerance applied to the operands of the subtraction).
"""
import numpy as np
import pytest
import torch

import sparse_mixture_experts_stable_b200 as moe
from oracle import oracle as O
from sparse_mixture_experts_stable_b200 import inputs as I
from sparse_mixture_experts_stable_b200.inputs import pages_layout
from tests.gpu_util import DEV, F32_ATOL, F32_RTOL, assert_close, check_dispatch, cpu, cpu64

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
    o = O.forward("linear", x64, s, k, C, {"w1": W}, base_kind="input" if residual else "zero")
    np.testing.assert_array_equal(cpu(r["selected"]), o["selected"])
    check_dispatch(o, d, E, C, "fwd")
    assert_close(cpu64(y), o["y"], F32_RTOL, F32_ATOL, "y")
    dx_o, dW_o, dl_o, dg_o = O.backward_linear(dy64, x64, s, o["selected"], o["kept"], o["gates"], W,
                                               use_residual=residual, aux_coef=aux_coef, normalize_by_k=True,
                                               counts=o["counts"])
    assert_close(cpu64(dg), dg_o, F32_RTOL, F32_ATOL, "dgate")
    assert_close(cpu64(dx), dx_o, F32_RTOL, F32_ATOL, "dx")
    assert_close(cpu64(dW).transpose(0, 2, 1), dW_o, F32_RTOL, F32_ATOL, "dW")
    # dlogits: bound from the magnitude of the terms it is formed from
    g = o["gates"]
    scale = np.zeros_like(dl_o)
    gabs = (g * np.abs(dg_o)).sum(1)
    for j in range(k):
        np.add.at(scale, (np.arange(T), o["selected"][:, j]), g[:, j] * (np.abs(dg_o[:, j]) + gabs))
    err = np.abs(cpu64(dl) - dl_o)
    bound = F32_ATOL + F32_RTOL * np.maximum(scale, np.abs(dl_o))
    assert (err <= bound).all(), f"dlogits: {(err > bound).sum()} elements, worst {np.max(err - bound)}"
    # unselected experts get exactly zero without the aux term
    if aux_coef == 0.0:
        mask = np.ones_like(dl_o, bool)
        mask[np.arange(T)[:, None], o["selected"]] = False
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
