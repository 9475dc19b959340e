"""The full-layer training step at its full size, checked on sampled outputs.

Workload: T=16384 tokens, hidden 2048, 256 SwiGLU experts (intermediate 512),
top-8, capacity factor 1.25, aux coefficient 0.001, upstream dy ~ 0.1 N(0,1);
the forward keeps the gate/up pre-activations, then moe_backward_swiglu and
moe_router_backward run, exactly the step the benchmark times.

The oracle cannot run the whole backward at this size in seconds, so each
sampled output comes from a small oracle problem that has the same value:

* a token's dgate, its selected logit gradients and its expert input gradient
  depend only on its own k experts: the oracle runs that token alone with the
  k selected experts (their logits in selection order, so the same ranking);
* the auxiliary-loss part of dlogits depends on the token's whole probability
  row, the global counts and 1/T^2: the oracle runs the sampled tokens with
  every assignment dropped (so only that term remains) and the coefficient
  scaled by (S/T)^2, which makes its 1/S^2 factor equal the layer's 1/T^2;
* an expert's weight gradients are sums over its kept rows of products that
  are linear in gate * dy: the oracle runs that expert's kept rows as a
  one-expert top-1 layer (gate 1) with upstream rows gate * dy.

Tolerance: the stated bf16 one (rtol 2e-2, atol 2e-2) for outputs of unit
size; gradients scale with dy, so the atol is taken relative to each sampled
tensor's root mean square.  dlogits, a difference of similar terms, gets the
rtol on the magnitude of those terms, as the fp32 tests do, and so do the
weight gradients (besides the atol), sums over an expert's kept rows that can
cancel: their magnitude is the sum over the rows of the absolute one-row
gradients, which the oracle gives row by row.
"""
import numpy as np
import pytest
import torch

import sparse_mixture_experts_stable_b200 as moe
from oracle import oracle as O
from sparse_mixture_experts_stable_b200 import inputs as I
from sparse_mixture_experts_stable_b200.inputs import pages_layout
from sparse_mixture_experts_stable_b200.layer import SwiGLUMoE
from tests.gpu_util import BF16_ATOL, BF16_RTOL, DEV, F32_RTOL, cpu, cpu64

pytestmark = pytest.mark.gpu


def _close_rms(got, want, what):
    """|got - want| <= rtol |want| + atol * rms(want), the stated bf16 rtol and atol."""
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    rms = float(np.sqrt(np.mean(want ** 2)))
    assert rms > 0, what
    err = np.abs(got - want)
    bound = BF16_RTOL * np.abs(want) + BF16_ATOL * rms
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {err.size} outside; worst at {i}: got {got[i]!r} "
                             f"want {want[i]!r} (rms {rms:.3e})")


def _close_mag(got, want, mag, what):
    """|got - want| <= rtol * max(|want|, mag) + atol * rms(want): the stated rtol on the magnitude of the
    summed terms (rows that cancel) and the stated atol at unit scale (a gradient near a zero of the SwiGLU
    derivative moves with the bf16 rounding of the saved pre-activation, not with its own size)."""
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    assert got.shape == want.shape == mag.shape, what
    err = np.abs(got - want)
    bound = BF16_RTOL * np.maximum(np.abs(want), mag) + BF16_ATOL * float(np.sqrt(np.mean(want ** 2)))
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {err.size} outside; worst at {i}: got {got[i]!r} "
                             f"want {want[i]!r} magnitude {mag[i]!r}")


def _weights64(cfg, experts):
    idx = torch.as_tensor(np.asarray(experts, np.int64))
    return pages_layout(cfg["w_gate"][idx]), pages_layout(cfg["w_up"][idx]), pages_layout(cfg["w_down"][idx])


def test_full_layer_training_step_sampled():
    cfg = I.full_layer_bf16(seed=0)
    T, H, E, F, k = cfg["T"], cfg["H"], cfg["E"], cfg["F"], cfg["k"]
    aux_coef = cfg["aux_coef"]
    dv = {n: cfg[n].to(DEV) for n in ("x", "w_router", "router_bias", "w_gate", "w_up", "w_down")}
    dy = (torch.randn(T, H, generator=torch.Generator().manual_seed(1)) * 0.1).to(torch.bfloat16)
    layer = SwiGLUMoE(T, H, E, F, k, cfg["capacity_factor"], F_shared=0, aux_coef=aux_coef, device=DEV,
                      save_for_backward=True)
    layer.route_out["logits"] = torch.empty(T, E, dtype=torch.float32, device=DEV)
    o = layer.forward(dv["x"], dv["w_router"], dv["router_bias"], dv["w_gate"], dv["w_up"], dv["w_down"])
    dxe, dwg, dwu, dwd, dl, dg = moe.moe_backward_swiglu(
        dy.to(DEV), layer.route_out["logits"], o["selected"], o["gates_f32"], o["slot"], o["used"], o["xbuf"],
        layer.ybuf, dv["w_gate"], dv["w_up"], dv["w_down"], layer.C, aux_coef=aux_coef, counts=o["counts"],
        dev_status=layer.status, saved_ab=layer.saved_ab)
    dxr, _, _ = moe.moe_router_backward(dv["x"], dv["w_router"], dl, dev_status=layer.status)
    assert moe.moe_read_status(layer.status) == 0

    x64, dy64 = cpu64(cfg["x"]), cpu64(dy)
    wr_de = cpu64(cfg["w_router"]).T
    s = O.router_logits(x64, wr_de, cpu64(cfg["router_bias"]))
    np.testing.assert_array_equal(cpu64(layer.route_out["logits"]), s)  # dyadic inputs: exact scores
    _, sel, gates, counts, _ = O.route(s, k)
    np.testing.assert_array_equal(cpu(o["selected"]), sel)
    disp = O.dispatch(sel, E, layer.C)
    kept = disp["kept"]
    assert (~kept).any()

    # ---- per-token outputs on a sample (tokens with drops included) ----
    rng = np.random.default_rng(11)
    S = np.unique(np.concatenate([rng.choice(T, 56, replace=False), np.flatnonzero(disp["drops"] > 0)[:8]]))
    n = len(S)
    want_dg = np.zeros((n, k))
    want_dl = np.zeros((n, E))
    want_dx = np.zeros((n, H))
    mag_dl = np.zeros((n, E))
    for i, t in enumerate(S):
        wg, wu, wd = _weights64(cfg, sel[t])
        sub = O.backward_swiglu(dy64[t:t + 1], x64[t:t + 1], s[t:t + 1, sel[t]], np.arange(k)[None],
                                kept[t:t + 1], gates[t:t + 1], wg, wu, wd)
        want_dx[i], want_dg[i] = sub[0][0], sub[5][0]
        want_dl[i, sel[t]] = sub[4][0]
        g, dgt = gates[t], np.abs(sub[5][0])
        mag_dl[i, sel[t]] = g * (dgt + np.dot(g, dgt))
    # the auxiliary-loss term of dlogits: every assignment dropped, coefficient scaled by (n/T)^2
    one = np.zeros((E, 1, 1))
    aux_part = O.backward_swiglu(np.zeros((n, 1)), np.zeros((n, 1)), s[S], sel[S], np.zeros((n, k), bool),
                                 gates[S], one, one, one, aux_coef=aux_coef * (n / T) ** 2, counts=counts)[4]
    assert np.abs(aux_part).max() > 0
    want_dl += aux_part

    _close_rms(cpu64(dg)[S], want_dg, "dgate")
    assert (cpu64(dg)[S][~kept[S]] == 0).all()
    got_dl = cpu64(dl)[S]
    rms_dg = float(np.sqrt(np.mean(want_dg ** 2)))
    gsel = np.zeros((n, E))
    for i, t in enumerate(S):
        gsel[i, sel[t]] = gates[t]
    bound = F32_RTOL * np.abs(aux_part) + 1e-9 + BF16_RTOL * (mag_dl + 2.0 * gsel * rms_dg)
    err = np.abs(got_dl - want_dl)
    assert (err <= bound).all(), f"dlogits: {int((err > bound).sum())} outside, worst {float((err - bound).max())}"
    _close_rms(cpu64(dxe)[S], want_dx, "dx (experts)")
    want_dxr = O.router_backward(x64[S], wr_de, want_dl)[0]
    _close_rms(cpu64(dxr)[S], want_dxr, "dx (router)")

    # ---- weight gradients of three experts: the fullest, a median one and the emptiest in use ----
    used = disp["used"]
    order = np.argsort(used, kind="stable")
    nz = order[used[order] > 0]
    for e in (int(nz[-1]), int(nz[len(nz) // 2]), int(nz[0])):
        rows = disp["token_of_slot"][e, :used[e]]
        jj = np.array([int(np.flatnonzero(sel[t] == e)[0]) for t in rows])
        g = gates[rows, jj]
        wg, wu, wd = _weights64(cfg, [e])
        m = len(rows)
        def one_expert(r_idx):
            n = len(r_idx)
            return O.backward_swiglu(g[r_idx, None] * dy64[rows[r_idx]], x64[rows[r_idx]], np.zeros((n, 1)),
                                     np.zeros((n, 1), np.int64), np.ones((n, 1), bool), np.ones((n, 1)), wg, wu, wd)

        sub = one_expert(np.arange(m))
        mag = [np.zeros_like(sub[1][0]), np.zeros_like(sub[2][0]), np.zeros_like(sub[3][0])]
        for i in range(m):  # the magnitude of each summed term: one kept row at a time
            one = one_expert(np.array([i]))
            for q, w_i in zip(mag, (1, 2, 3)):
                q += np.abs(one[w_i][0])
        _close_mag(cpu64(dwg[e]), sub[1][0].T, mag[0].T, f"dw_gate[{e}] ({m} rows)")
        _close_mag(cpu64(dwu[e]), sub[2][0].T, mag[1].T, f"dw_up[{e}]")
        _close_mag(cpu64(dwd[e]), sub[3][0].T, mag[2].T, f"dw_down[{e}]")
    # an expert with no kept row has a zero gradient
    for e in np.flatnonzero(used == 0)[:4]:
        assert (cpu64(dwg[e]) == 0).all() and (cpu64(dwd[e]) == 0).all()
