"""moe_expert_ffn (grouped expert GEMMs) on the GPU against the fp64 oracle.

Shapes are chosen to cover several 128-row tiles, ragged row counts per expert
(including empty and single-row experts), partial N tiles and K tails.
"""
import numpy as np
import pytest
import torch

import sparse_mixture_experts_stable_b200 as moe
from oracle import oracle as O
from sparse_mixture_experts_stable_b200.inputs import pages_layout
from tests.gpu_util import BF16_ATOL, BF16_RTOL, DEV, F32_ATOL, F32_RTOL, assert_close, assert_close_mag, cpu64

pytestmark = pytest.mark.gpu


def _case(kind, dtype, E, C, D, F, Dout, used, seed):
    g = torch.Generator().manual_seed(seed)

    def rnd(*shape, scale=1.0):
        return (torch.randn(*shape, generator=g) * scale).to(dtype)

    xbuf = rnd(E, C, D)
    w = {}
    if kind == "linear":
        w["w1"] = rnd(E, Dout, D, scale=D ** -0.5)
    elif kind == "gelu_mlp":
        w["w1"] = rnd(E, F, D, scale=D ** -0.5)
        w["b1"] = rnd(E, F, scale=0.5)
        w["w2"] = rnd(E, Dout, F, scale=F ** -0.5)
        w["b2"] = rnd(E, Dout, scale=0.5)
    else:
        w["w1"] = rnd(E, F, D, scale=D ** -0.5)
        w["w3"] = rnd(E, F, D, scale=D ** -0.5)
        w["w2"] = rnd(E, Dout, F, scale=F ** -0.5)
    used_t = torch.tensor(used, dtype=torch.int32)
    return xbuf, w, used_t


def _oracle(kind, xbuf, w, used, absolute=False):
    """Oracle expert outputs per expert; with absolute=True, the same evaluated on |inputs|
    (the magnitude of the summed terms)."""
    E, C, D = xbuf.shape
    f = np.abs if absolute else (lambda a: a)
    pw = {}
    for name, t in w.items():
        pw[name] = f(pages_layout(t) if t.dim() == 3 else t.to(torch.float64).numpy())
    out = []
    for e in range(E):
        u = int(used[e])
        rows = f(cpu64(xbuf[e, :u])) if u else np.zeros((0, D))
        if u:
            out.append(O.expert_rows(kind, rows, np.arange(u), np.full(u, e), pw))
        else:
            out.append(None)
    return out


@pytest.mark.parametrize("kind", ["linear", "swiglu", "gelu_mlp"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_expert_ffn_small(kind, dtype):
    E, C, D, F, Dout = 5, 300, 192, 160, 288
    used = [300, 0, 129, 1, 257]
    xbuf, w, used_t = _case(kind, dtype, E, C, D, F, Dout, used, seed=["linear", "swiglu", "gelu_mlp"].index(kind) * 2 + (dtype == torch.bfloat16))
    dev = {k_: v.to(DEV) for k_, v in w.items()}
    ybuf = torch.full((E, C, Dout), float("nan"), dtype=dtype, device=DEV)
    st = moe.new_status()
    moe.moe_expert_ffn(kind, xbuf.to(DEV), used_t.to(DEV), dev["w1"], b1=dev.get("b1"), w2=dev.get("w2"),
                       b2=dev.get("b2"), w3=dev.get("w3"), ybuf=ybuf, dev_status=st)
    assert moe.moe_read_status(st) == 0
    want = _oracle(kind, xbuf, w, used)
    mag = _oracle(kind, xbuf, w, used, absolute=True)
    yb = cpu64(ybuf)
    for e in range(E):
        u = used[e]
        if u and dtype == torch.bfloat16:
            assert_close(yb[e, :u], want[e], BF16_RTOL, BF16_ATOL, f"{kind} {dtype} expert {e}")
        elif u:
            assert_close_mag(yb[e, :u], want[e], mag[e], F32_RTOL, F32_ATOL, f"{kind} {dtype} expert {e}")
        # rows past used[e] are not written
        assert np.isnan(yb[e, u:]).all()


def test_expert_ffn_bf16_all_rows_no_used():
    # used == NULL: every one of the C rows, one expert (the shared-expert form)
    E, C, D, F, Dout = 1, 1000, 256, 512, 256
    xbuf, w, _ = _case("swiglu", torch.bfloat16, E, C, D, F, Dout, [C], seed=11)
    ybuf = moe.moe_expert_ffn("swiglu", xbuf.to(DEV), None, w["w1"].to(DEV), w2=w["w2"].to(DEV),
                              w3=w["w3"].to(DEV))
    want = _oracle("swiglu", xbuf, w, [C])
    assert_close(cpu64(ybuf)[0], want[0], BF16_RTOL, BF16_ATOL, "shared swiglu")


def test_expert_ffn_bf16_many_experts_tile_scheduler():
    # 64 experts with random occupancy over a long K: exercises the persistent
    # tile walk (more tiles than SMs) and the 4-stage ring wrap-around
    E, C, D, Dout = 64, 256, 1024, 512
    rng = np.random.default_rng(3)
    used = rng.integers(0, C + 1, E).tolist()
    used[0], used[1] = 0, C
    xbuf, w, used_t = _case("linear", torch.bfloat16, E, C, D, 0, Dout, used, seed=12)
    ybuf = moe.moe_expert_ffn("linear", xbuf.to(DEV), used_t.to(DEV), w["w1"].to(DEV))
    yb = cpu64(ybuf)
    for e in rng.choice(E, 8, replace=False).tolist() + [1]:
        u = used[e]
        if not u:
            continue
        want = O.expert_rows("linear", cpu64(xbuf[e, :u]), np.arange(u), np.full(u, e),
                             {"w1": pages_layout(w["w1"])})
        assert_close(yb[e, :u], want, BF16_RTOL, BF16_ATOL, f"expert {e}")


def test_expert_ffn_deterministic():
    E, C, D, F, Dout = 8, 200, 256, 256, 256
    xbuf, w, used_t = _case("swiglu", torch.bfloat16, E, C, D, F, Dout, [200, 3, 150, 0, 64, 129, 128, 127], 5)
    args = (xbuf.to(DEV), used_t.to(DEV), w["w1"].to(DEV))
    kw = dict(w2=w["w2"].to(DEV), w3=w["w3"].to(DEV))
    a = moe.moe_expert_ffn("swiglu", *args, ybuf=torch.zeros(E, C, Dout, dtype=torch.bfloat16, device=DEV), **kw)
    b = moe.moe_expert_ffn("swiglu", *args, ybuf=torch.zeros(E, C, Dout, dtype=torch.bfloat16, device=DEV), **kw)
    assert torch.equal(a, b)


def test_transpose_weights_roundtrip():
    src = torch.randn(3, 40, 24, device=DEV).to(torch.bfloat16)
    dst = moe.moe_transpose_weights(src)
    assert torch.equal(dst, src.transpose(1, 2))
    src32 = torch.randn(2, 33, 65, device=DEV)
    assert torch.equal(moe.moe_transpose_weights(src32), src32.transpose(1, 2))


def test_swiglu_gate_up_elementwise_error():
    """The routed SwiGLU gate/up epilogue element by element.

    With F == Dout and every down-projection matrix the identity, each output
    element is h = silu(a) * b itself (one product with 1.0, accumulated in fp32
    and rounded to bf16 again: exact).  The epilogue computes the sigmoid as
    1/2 + tanh(a/2)/2 with the hardware tanh approximation, whose absolute error
    is below 2^-11, so |sigmoid error| < 2^-12 and the bound per element is the
    bf16 rounding of h, plus that error times |a * b|, plus the fp32 sums of a and
    b (any order: at most D * 2^-24 * sum |x w| each) carried through
    silu(a) * b (|silu'| < 1.1).  Pre-activations reach |a| ~ 9, where the
    cancellation in 1 + tanh(a/2) matters most.
    """
    E, C, D, F = 3, 300, 256, 256
    used = [300, 77, 0]
    g = torch.Generator().manual_seed(29)
    xbuf = torch.randn(E, C, D, generator=g).to(torch.bfloat16)
    wg = (torch.randn(E, F, D, generator=g) * 3.0 * D ** -0.5).to(torch.bfloat16)
    wu = (torch.randn(E, F, D, generator=g) * D ** -0.5).to(torch.bfloat16)
    eye = torch.eye(F).to(torch.bfloat16).expand(E, F, F).contiguous()
    ybuf = torch.full((E, C, F), float("nan"), dtype=torch.bfloat16, device=DEV)
    st = moe.new_status()
    moe.moe_expert_ffn("swiglu", xbuf.to(DEV), torch.tensor(used, dtype=torch.int32).to(DEV), wg.to(DEV),
                       w2=eye.to(DEV), w3=wu.to(DEV), ybuf=ybuf, dev_status=st)
    assert moe.moe_read_status(st) == 0
    w = {"w1": wg, "w2": eye, "w3": wu}
    want = _oracle("swiglu", xbuf, w, used)
    yb = cpu64(ybuf)
    n_neg = 0
    for e in range(E):
        u = used[e]
        assert np.isnan(yb[e, u:]).all()
        if not u:
            continue
        rows = cpu64(xbuf[e, :u])
        a = rows @ cpu64(wg[e]).T  # magnitudes for the bound only
        b = rows @ cpu64(wu[e]).T
        da = D * 2.0 ** -24 * (np.abs(rows) @ np.abs(cpu64(wg[e])).T)
        db = D * 2.0 ** -24 * (np.abs(rows) @ np.abs(cpu64(wu[e])).T)
        silu = a / (1.0 + np.exp(-a))
        n_neg += int((a < -4).sum())
        bound = (2.0 ** -8 * np.abs(want[e]) + 2.0 ** -11 * np.abs(a * b) + 1.1 * da * np.abs(b)
                 + np.abs(silu) * db + 1e-30)
        err = np.abs(yb[e, :u] - want[e])
        bad = err > bound
        assert not bad.any(), (e, int(bad.sum()), float((err / bound).max()))
    assert n_neg > 1000  # the strongly negative range was exercised
