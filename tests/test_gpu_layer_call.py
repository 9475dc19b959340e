"""moe_swiglu_layer_forward: the whole layer in one C call, device or host buffers.

The call chains the same kernels as the layer built from the individual entry
points (SwiGLUMoE), so its output must be bitwise identical to that layer's,
with x and y in device memory or in pinned host memory (copies done inside the
library), and over consecutive batches that alternate between two workspaces
on separate copy streams.  A small case is also compared with the oracle.
"""
import math

import numpy as np
import pytest
import torch

import sparse_mixture_experts_stable_b200 as moe
from oracle import oracle as O
from sparse_mixture_experts_stable_b200 import inputs as I
from sparse_mixture_experts_stable_b200.inputs import pages_layout
from sparse_mixture_experts_stable_b200.layer import SwiGLULayer, SwiGLUMoE
from tests.gpu_util import BF16_ATOL, BF16_RTOL, DEV, assert_close, cpu64

pytestmark = pytest.mark.gpu

NAMES = ("x", "w_router", "router_bias", "w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down")


def _layers(cfg, shared=True, n_workspaces=1):
    dv = {n: cfg[n].to(DEV) for n in NAMES}
    T, H, E, F, k = cfg["T"], cfg["H"], cfg["E"], cfg["F"], cfg["k"]
    sh = (dv["s_gate"], dv["s_up"], dv["s_down"]) if shared else (None, None, None)
    ref = SwiGLUMoE(T, H, E, F, k, cfg["capacity_factor"], F_shared=cfg["F_shared"] if shared else 0,
                    aux_coef=cfg["aux_coef"])
    call = SwiGLULayer(T, H, E, F, k, cfg["capacity_factor"], dv["w_router"], dv["router_bias"], dv["w_gate"],
                       dv["w_up"], dv["w_down"], *sh, aux_coef=cfg["aux_coef"], n_workspaces=n_workspaces)
    return dv, ref, call


@pytest.mark.parametrize("shared", [True, False])
def test_layer_call_equals_entry_point_chain_device_buffers(shared):
    cfg = I.full_layer_bf16(seed=4, T=3000, H=512, E=32, F=256, k=8, F_shared=256)
    dv, ref, call = _layers(cfg, shared)
    args = [dv[n] for n in NAMES[:6]] + ([dv[n] for n in NAMES[6:]] if shared else [])
    want = ref.forward(*args)
    y = torch.empty_like(dv["x"])
    aux = torch.empty(2, dtype=torch.float32, device=DEV)
    call.forward(dv["x"], y, aux)
    assert moe.moe_read_status(call.status) == 0
    assert torch.equal(y, want["y"])
    assert torch.equal(aux, want["aux"])


def test_layer_call_host_buffers_two_workspaces():
    cfg = I.full_layer_bf16(seed=5, T=2048, H=256, E=16, F=128, k=4, F_shared=128)
    dv, ref, call = _layers(cfg, True, n_workspaces=2)
    g = torch.Generator().manual_seed(9)
    xs = [(torch.randint(-8, 9, (cfg["T"], cfg["H"]), generator=g).float() / 8).to(torch.bfloat16) for _ in range(4)]
    x_host = [x.pin_memory() for x in xs]
    y_host = [torch.empty_like(x).pin_memory() for x in xs]
    aux_host = [torch.empty(2, dtype=torch.float32).pin_memory() for _ in xs]
    side, cin, cout = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    for i in range(4):
        call.forward(x_host[i], y_host[i], aux_host[i], slot=i % 2, side_stream=side, copy_in_stream=cin,
                     copy_out_stream=cout)
    torch.cuda.synchronize()
    assert moe.moe_read_status(call.status) == 0
    w = [dv[n] for n in NAMES[1:]]
    for i in range(4):
        want = ref.forward(xs[i].to(DEV), *w)
        assert torch.equal(y_host[i], want["y"].cpu()), i
        assert torch.equal(aux_host[i], want["aux"].cpu()), i


def test_layer_call_matches_oracle_small():
    cfg = I.full_layer_bf16(seed=6, T=700, H=128, E=8, F=64, k=2, F_shared=64)
    dv, _, call = _layers(cfg, True)
    y = torch.empty(cfg["T"], cfg["H"], dtype=torch.bfloat16).pin_memory()
    aux = torch.empty(2, dtype=torch.float32).pin_memory()
    call.forward(cfg["x"].pin_memory(), y, aux)
    torch.cuda.synchronize()
    x64 = cpu64(cfg["x"])
    s = O.router_logits(x64, cpu64(cfg["w_router"]).T, cpu64(cfg["router_bias"]))
    o = O.forward("swiglu", x64, s, cfg["k"], call.C,
                  {"w1": pages_layout(cfg["w_gate"]), "w3": pages_layout(cfg["w_up"]),
                   "w2": pages_layout(cfg["w_down"])}, base_kind="tensor",
                  base=O.expert_rows("swiglu", x64, np.arange(cfg["T"]), np.zeros(cfg["T"], np.int64),
                                     {"w1": pages_layout(cfg["s_gate"]), "w3": pages_layout(cfg["s_up"]),
                                      "w2": pages_layout(cfg["s_down"])}))
    assert_close(cpu64(y), o["y"], BF16_RTOL, BF16_ATOL, "layer call y")
    assert math.isclose(float(aux[0]), o["aux"], rel_tol=1e-5)


def test_layer_call_rejects_small_workspace():
    cfg = I.full_layer_bf16(seed=7, T=256, H=128, E=8, F=64, k=2, F_shared=0)
    dv, _, call = _layers(cfg, False)
    y = torch.empty_like(dv["x"])
    small = torch.empty(1024, dtype=torch.uint8, device=DEV)
    with pytest.raises(moe.MoeError) as e:
        moe.moe_swiglu_layer_forward(call.desc, dv["x"], y, None, small)
    assert e.value.code == moe.binding.MOE_ERR_WORKSPACE
