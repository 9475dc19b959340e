"""moe_expert_ffn_gathered: SwiGLU experts reading their rows from x through
token_of_slot, against the gather + moe_expert_ffn path and the fp64 oracle.

The two paths run different gate/up kernels (the gathered one fills its token
tiles with cp.async, 128 tokens per tile; the other takes 256-token tiles
through TMA and a faster SiLU exponential), so they agree to the bf16
tolerance, not bit for bit.

Shapes cover ragged experts (empty, one row, exactly one tile, full C), a K
tail (D not a multiple of 64), several tiles per expert and the full-layer
size; an index outside [0, T) must be reported and read as a zero row.
"""
import numpy as np
import pytest
import torch

import sparse_mixture_experts_stable_b200 as moe
from oracle import oracle as O
from sparse_mixture_experts_stable_b200 import inputs as I
from sparse_mixture_experts_stable_b200.inputs import pages_layout
from tests.gpu_util import BF16_ATOL, BF16_RTOL, DEV, assert_close, cpu64

pytestmark = pytest.mark.gpu


def _weights(E, D, F, Dout, seed):
    g = torch.Generator().manual_seed(seed)

    def rnd(*shape, scale):
        return (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16)

    return rnd(E, F, D, scale=D ** -0.5), rnd(E, F, D, scale=D ** -0.5), rnd(E, Dout, F, scale=F ** -0.5)


def _route_tokens(T, E, k, seed):
    """Random distinct experts per token (a stand-in for the router's selection)."""
    rng = np.random.default_rng(seed)
    sel = np.argsort(rng.random((T, E)), axis=1)[:, :k]
    return torch.from_numpy(sel.astype(np.int64))


@pytest.mark.parametrize("T,D,E,k,cf", [(700, 192, 6, 2, 1.0), (1000, 200, 4, 3, 0.6), (64, 64, 8, 8, 2.0)])
def test_gathered_matches_gather_then_ffn(T, D, E, k, cf):
    F, Dout = 160, 96
    x = torch.randn(T, D, generator=torch.Generator().manual_seed(T)).to(torch.bfloat16).to(DEV)
    wg, wu, wd = (w.to(DEV) for w in _weights(E, D, F, Dout, seed=D))
    C = moe.moe_capacity(T, k, E, cf)
    sel = _route_tokens(T, E, k, seed=E).to(DEV)
    d = moe.moe_dispatch(sel, E, C, x=x)
    st = moe.new_status()
    ref = torch.full((E, C, Dout), float("nan"), dtype=torch.bfloat16, device=DEV)
    moe.moe_expert_ffn("swiglu", d["xbuf"], d["used"], wg, w2=wd, w3=wu, ybuf=ref, dev_status=st)
    got = torch.full((E, C, Dout), float("nan"), dtype=torch.bfloat16, device=DEV)
    moe.moe_expert_ffn_gathered(x, d["token_of_slot"], d["used"], wg, wd, wu, ybuf=got, dev_status=st)
    assert moe.moe_read_status(st) == 0
    used = d["used"].cpu().tolist()
    for e in range(E):
        u = used[e]
        assert_close(cpu64(got[e, :u]), cpu64(ref[e, :u]), BF16_RTOL, BF16_ATOL, f"expert {e}")
        # rows past used stay untouched
        assert torch.isnan(got[e, u:].float()).all()
    # against the oracle on the rows the dispatch chose
    pw = {"w1": pages_layout(wg.cpu()), "w3": pages_layout(wu.cpu()), "w2": pages_layout(wd.cpu())}
    tos = d["token_of_slot"].cpu().numpy()
    x64 = cpu64(x)
    for e in range(E):
        u = used[e]
        if u:
            want = O.expert_rows("swiglu", x64[tos[e, :u]], np.arange(u), np.full(u, e), pw)
            assert_close(cpu64(got[e, :u]), want, BF16_RTOL, BF16_ATOL, f"expert {e} vs oracle")


def test_gathered_reports_index_outside_x():
    T, D, E, C, F, Dout = 100, 128, 2, 40, 64, 64
    x = torch.randn(T, D).to(torch.bfloat16).to(DEV)
    wg, wu, wd = (w.to(DEV) for w in _weights(E, D, F, Dout, seed=5))
    tos = torch.arange(E * C, dtype=torch.int32).view(E, C) % T
    tos[1, 3] = T + 7  # outside x
    used = torch.tensor([C, 10], dtype=torch.int32)
    st = moe.new_status()
    got = moe.moe_expert_ffn_gathered(x, tos.to(DEV), used.to(DEV), wg, wd, wu, dev_status=st)
    assert moe.moe_read_status(st) == moe.binding.MOE_ERR_BAD_INDEX
    # the bad slot computed on a zero row: SwiGLU without biases gives exactly 0
    assert (got[1, 3].float() == 0).all()
    assert (got[1, 2].float() != 0).any()


def test_gathered_full_layer_size_sampled():
    cfg = I.full_layer_bf16(seed=4)
    T, H, E, F, k = cfg["T"], cfg["H"], cfg["E"], cfg["F"], cfg["k"]
    x = cfg["x"].to(DEV)
    r = moe.moe_route(x, k, w_router=cfg["w_router"].to(DEV), logit_bias=cfg["router_bias"].to(DEV))
    C = moe.moe_capacity(T, k, E, cfg["capacity_factor"])
    d = moe.moe_dispatch(r["selected"], E, C, x=x)
    wg, wu, wd = cfg["w_gate"].to(DEV), cfg["w_up"].to(DEV), cfg["w_down"].to(DEV)
    st = moe.new_status()
    ref = moe.moe_expert_ffn("swiglu", d["xbuf"], d["used"], wg, w2=wd, w3=wu, dev_status=st)
    got = moe.moe_expert_ffn_gathered(x, d["token_of_slot"], d["used"], wg, wd, wu, dev_status=st)
    assert moe.moe_read_status(st) == 0
    used = d["used"].cpu().tolist()
    for e in range(E):
        assert_close(cpu64(got[e, :used[e]]), cpu64(ref[e, :used[e]]), BF16_RTOL, BF16_ATOL, f"expert {e}")
