"""moe_backward_swiglu (bf16 SwiGLU experts) and moe_router_backward against the
fp64 oracle backward.

The forward runs on the GPU (route on given logits, dispatch, SwiGLU experts);
the oracle recomputes everything in fp64 from the same bf16 inputs.  Integer
routing is exact; the gradients carry bf16 roundings of the forward output, of
the scaled upstream rows and of h, da, db, so they are held to the bf16
tolerance, scaled by the largest magnitude of each gradient tensor.
"""
import numpy as np
import pytest
import torch

import sparse_mixture_experts_stable_b200 as moe
from oracle import oracle as O
from sparse_mixture_experts_stable_b200.inputs import pages_layout
from tests.gpu_util import BF16_RTOL, DEV, F32_ATOL, F32_RTOL, assert_close, assert_close_mag, cpu, cpu64

pytestmark = pytest.mark.gpu


def _close(got, want, what):
    scale = float(np.abs(want).max()) if want.size else 1.0
    assert_close(got, want, BF16_RTOL, BF16_RTOL * scale, what)


@pytest.mark.parametrize("T,H,F,E,k,cf,residual,aux", [
    (300, 128, 96, 6, 2, 0.8, False, 0.0),   # capacity binds: drops
    (517, 64, 48, 4, 3, 1.5, True, 0.1),     # ragged token count, residual, aux term
    (64, 72, 40, 3, 1, 2.0, False, 0.0),     # top-1; H, F not multiples of 64
    (400, 128, 128, 6, 2, 1.0, True, 0.0),   # H, F multiples of 64: weights read MN-major, no transposed copies
    (333, 256, 64, 5, 3, 0.7, False, 0.05),  # the same with drops and the aux term
    (260, 192, 256, 4, 2, 1.2, False, 0.0),  # F a multiple of 128: dW gate and up from one split-output GEMM
    (300, 320, 128, 4, 2, 1.2, False, 0.0),  # H = 320: the weight gradients' last column tile extends past H
])
@pytest.mark.parametrize("saved", [False, True])
def test_backward_swiglu_matches_oracle(T, H, F, E, k, cf, residual, aux, saved):
    g = torch.Generator().manual_seed(T + H)

    def rnd(*shape, scale=1.0):
        return (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16)

    x = rnd(T, H)
    lg = torch.randn(T, E, generator=g)
    wg, wu, wd = rnd(E, F, H, scale=H ** -0.5), rnd(E, F, H, scale=H ** -0.5), rnd(E, H, F, scale=F ** -0.5)
    dy = rnd(T, H)
    C = moe.moe_capacity(T, k, E, cf)

    xd, lgd, dyd = x.to(DEV), lg.to(DEV), dy.to(DEV)
    wgd, wud, wdd = wg.to(DEV), wu.to(DEV), wd.to(DEV)
    r = moe.moe_route(lgd, k)
    d = moe.moe_dispatch(r["selected"], E, C, x=xd)
    st = moe.new_status()
    saved_ab = None
    if saved:  # the forward keeps [a | b] (bf16) and the backward skips recomputing them
        ybuf, saved_ab = moe.moe_expert_ffn_save(d["xbuf"], d["used"], wgd, wdd, wud, dev_status=st)
        ref = moe.moe_expert_ffn("swiglu", d["xbuf"], d["used"], wgd, w2=wdd, w3=wud, dev_status=st)
        used_h = cpu(d["used"])
        for e in range(E):  # the same expert outputs as without saving
            assert torch.equal(ybuf[e, :int(used_h[e])], ref[e, :int(used_h[e])])
        # the saved pre-activations are x W^T rounded to bf16
        e0 = int(np.argmax(used_h))
        a_ref = (d["xbuf"][e0, :int(used_h[e0])].float() @ wgd[e0].float().T)
        np.testing.assert_allclose(cpu64(saved_ab[e0, :int(used_h[e0]), :F]), cpu64(a_ref), rtol=2e-2,
                                   atol=2e-2 * float(a_ref.abs().max()))
    else:
        ybuf = moe.moe_expert_ffn("swiglu", d["xbuf"], d["used"], wgd, w2=wdd, w3=wud, dev_status=st)
    dx, dwg, dwu, dwd, dl, dg = moe.moe_backward_swiglu(
        dyd, lgd, r["selected"], r["gates_f32"], d["slot"], d["used"], d["xbuf"], ybuf, wgd, wud, wdd, C,
        use_residual=residual, aux_coef=aux, counts=r["counts"], dev_status=st, saved_ab=saved_ab)
    assert moe.moe_read_status(st) == 0

    s64 = cpu64(lg)
    probs, sel, gates, counts, _ = O.route(s64, k)
    np.testing.assert_array_equal(cpu(r["selected"]), sel)
    disp = O.dispatch(sel, E, C)
    kept = disp["kept"]
    if cf < 1.0:
        assert (~kept).any()
    want = O.backward_swiglu(cpu64(dy), cpu64(x), s64, sel, kept, gates, pages_layout(wg), pages_layout(wu),
                             pages_layout(wd), use_residual=residual, aux_coef=aux, counts=counts)
    wdx, wdWg, wdWu, wdWd, wdl, wdg = want
    _close(cpu64(dg), wdg, "dgate")
    assert (cpu64(dg)[~kept] == 0).all()
    _close(cpu64(dl), wdl, "dlogits")
    _close(cpu64(dx), wdx, "dx")
    # the oracle's weight gradients are in the x@W layout: (E, D, F) and (E, F, N)
    _close(cpu64(dwg), wdWg.transpose(0, 2, 1), "dw_gate")
    _close(cpu64(dwu), wdWu.transpose(0, 2, 1), "dw_up")
    _close(cpu64(dwd), wdWd.transpose(0, 2, 1), "dw_down")
    # an expert that received no token has an exactly zero gradient
    for e in np.flatnonzero(disp["used"] == 0):
        assert (cpu64(dwg)[e] == 0).all() and (cpu64(dwd)[e] == 0).all()


def test_backward_swiglu_with_nothing_kept():
    T, H, F, E, k = 50, 64, 32, 2, 1
    g = torch.Generator().manual_seed(3)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16).to(DEV)
    lg = torch.randn(T, E, generator=g).to(DEV)
    dy = torch.randn(T, H, generator=g).to(torch.bfloat16).to(DEV)
    w = [torch.randn(*s, generator=g).to(torch.bfloat16).to(DEV) for s in ((E, F, H), (E, F, H), (E, H, F))]
    r = moe.moe_route(lg, k)
    d = moe.moe_dispatch(r["selected"], E, 0)
    ybuf = torch.empty(E, 0, H, dtype=torch.bfloat16, device=DEV)
    xbuf = torch.empty(E, 0, H, dtype=torch.bfloat16, device=DEV)
    dx, dwg, dwu, dwd, dl, dg = moe.moe_backward_swiglu(dy, lg, r["selected"], r["gates_f32"], d["slot"], d["used"],
                                                        xbuf, ybuf, *w, 0, use_residual=True)
    assert torch.equal(dx, dy)
    assert (dwg == 0).all() and (dwu == 0).all() and (dwd == 0).all()
    assert (dl == 0).all() and (dg == 0).all()


@pytest.mark.parametrize("dtype,layout,T,E", [(torch.bfloat16, "ED", 700, 40), (torch.bfloat16, "DE", 700, 40),
                                              (torch.float32, "ED", 700, 40),
                                              (torch.bfloat16, "ED", 4096, 40),   # token reduction split 8 ways
                                              (torch.float32, "DE", 4100, 40),    # split 4 ways
                                              # bf16 with E a multiple of 64: dlogits in three bf16 parts on the
                                              # bf16 tensor cores (one group at T = 700, four at T = 4096)
                                              (torch.bfloat16, "ED", 700, 64), (torch.bfloat16, "DE", 4096, 128),
                                              (torch.bfloat16, "ED", 4096, 256)])
def test_router_backward_matches_oracle(dtype, layout, T, E):
    # s = x W (+ b): dx = dlogits W^T, dW = x^T dlogits, db = column sums (fp32 accuracy)
    D = 192
    g = torch.Generator().manual_seed(5 + (layout == "DE"))
    x = torch.randn(T, D, generator=g).to(dtype)
    w_ed = (torch.randn(E, D, generator=g) * 0.1).to(dtype)
    dl = torch.randn(T, E, generator=g)
    w = w_ed if layout == "ED" else w_ed.t().contiguous()
    dx, dw, db = moe.moe_router_backward(x.to(DEV), w.to(DEV), dl.to(DEV), layout=layout)
    wdx, wdw, wdb = O.router_backward(cpu64(x), cpu64(w_ed).T, cpu64(dl))  # oracle weight is (D, E)
    mdx, mdw, mdb = O.router_backward(np.abs(cpu64(x)), np.abs(cpu64(w_ed)).T, np.abs(cpu64(dl)))
    assert_close_mag(cpu64(dx), wdx, mdx, F32_RTOL, F32_ATOL, "dx_router")
    got_dw = cpu64(dw) if layout == "DE" else cpu64(dw).T
    assert_close_mag(got_dw, wdw, mdw, F32_RTOL, F32_ATOL, "dw_router")
    assert_close_mag(cpu64(db), wdb, mdb, F32_RTOL, F32_ATOL, "db_router")
