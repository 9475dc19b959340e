"""C-ABI checks that need no GPU: the library loads, exports every entry point
that include/moe.h declares, and its host-side logic (capacity, argument
validation, workspace sizing) behaves as documented.  No kernel is launched."""
import ctypes
import os
import re

import numpy as np
import pytest

import sparse_mixture_experts_stable_b200 as moe
from oracle import oracle as O
from sparse_mixture_experts_stable_b200 import binding as B
from tests.conftest import ROOT


def _declared():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"^MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", txt, flags=re.M)
    return names


def test_library_exports_every_declared_symbol():
    L = moe.lib()
    declared = _declared()
    assert len(declared) >= 16
    for name in declared:
        assert hasattr(L, name), name
    assert sorted(declared) == sorted(B.EXPORTED)


def test_version_and_status_strings():
    assert moe.lib().moe_version() >= 100
    for code in range(8):
        assert moe.status_string(code)
    assert moe.status_string(99) == "unknown status"


@pytest.mark.parametrize("seed", range(3))
def test_capacity_matches_oracle(seed):
    rng = np.random.default_rng(seed)
    for _ in range(300):
        E = int(rng.integers(1, 300))
        k = int(rng.integers(1, E + 1))
        T = int(rng.integers(1, 100000))
        cf = float(rng.choice([0.5, 1.0, 1.25, 2.0, 0.1, 3.7, float(rng.uniform(0.01, 4))]))
        assert moe.moe_capacity(T, k, E, cf) == O.capacity(T, k, E, cf)
    assert moe.moe_capacity(16384, 8, 256, 1.25) == 640


def test_capacity_rejects_bad_arguments():
    for args in [(8, 2, 4, 0.0), (8, 2, 4, -1.0), (8, 2, 4, float("nan")), (8, 5, 4, 1.0), (0, 1, 4, 1.0),
                 (8, 0, 4, 1.0)]:
        with pytest.raises(moe.MoeError) as ei:
            moe.moe_capacity(*args)
        assert ei.value.code == B.MOE_ERR_INVALID_ARG


def test_host_validation_before_any_launch():
    L = moe.lib()
    nul = None
    # k > E
    rc = L.moe_route(ctypes.c_void_p(16), 0, 4, 0, 2, nul, 1, 2, nul, 3, nul, ctypes.c_void_p(16), nul, nul,
                     ctypes.c_void_p(16), ctypes.c_void_p(16), nul, ctypes.c_void_p(16), 1 << 20, nul)
    assert rc == B.MOE_ERR_INVALID_ARG
    # k beyond this build's limit
    rc = L.moe_route(ctypes.c_void_p(16), 0, 4, 0, 200, nul, 1, 200, nul, 100, nul, ctypes.c_void_p(16), nul, nul,
                     ctypes.c_void_p(16), ctypes.c_void_p(16), nul, ctypes.c_void_p(16), 1 << 20, nul)
    assert rc == B.MOE_ERR_UNSUPPORTED
    # missing workspace
    rc = L.moe_route(ctypes.c_void_p(16), 0, 4, 0, 2, nul, 1, 2, nul, 1, nul, ctypes.c_void_p(16), nul, nul,
                     ctypes.c_void_p(16), ctypes.c_void_p(16), nul, nul, 0, nul)
    assert rc == B.MOE_ERR_WORKSPACE
    # dispatch: NULL outputs, negative capacity
    p = ctypes.c_void_p(16)
    rc = L.moe_dispatch(p, 4, 1, 2, 2, nul, 0, 0, 0, nul, p, p, p, p, p, nul, nul, p, 1 << 20, nul)
    assert rc == B.MOE_ERR_INVALID_ARG
    rc = L.moe_dispatch(p, 4, 1, 2, -1, nul, 0, 0, 0, p, p, p, p, p, p, nul, nul, p, 1 << 20, nul)
    assert rc == B.MOE_ERR_INVALID_ARG
    # backward: only fp32 linear experts in this build
    rc = L.moe_backward(1, 0, *([p] * 11), 4, 1, 2, 2, 8, 8, 1, ctypes.c_float(0), 1, p, p, p, p, p, nul, p,
                        1 << 30, nul)
    assert rc == B.MOE_ERR_UNSUPPORTED
    # combine: residual base without a base tensor
    rc = L.moe_combine(p, p, p, nul, 0, 4, 1, 2, 2, 8, 1, nul, 8, p, 8, 0, nul, nul)
    assert rc == B.MOE_ERR_INVALID_ARG


def test_workspace_sizes():
    assert moe.binding.moe_dispatch_workspace_size(16384, 8, 256) >= 32 * 256 * 4
    assert moe.binding.moe_route_workspace_size(65536, 2048, 256, B.MOE_BF16, True, "DE") > 65536 * 256 * 4
    assert moe.binding.moe_expert_ffn_workspace_size("linear", B.MOE_BF16, 8, 16, 64, 32, 64) == 0
    assert moe.binding.moe_expert_ffn_workspace_size("swiglu", B.MOE_BF16, 256, 640, 2048, 512, 2048) >= 256 * 640 * 512 * 2
    # fp32 adds the split-tf32 operands: hi and lo of rows and weights, K rounded up to 32
    assert moe.binding.moe_expert_ffn_workspace_size("linear", B.MOE_F32, 8, 16, 64, 0, 48) >= 2 * 4 * (8 * 16 * 64 + 8 * 48 * 64)
    assert moe.binding.moe_backward_workspace_size(64, 256, 1024, 1024) >= 2 * 64 * 256 * 1024 * 4
    # GELU backward: dybuf, z, dh, dxbuf (fp32) plus the split operands
    E, C, D, F = 8, 160, 64, 256
    assert moe.binding.moe_backward_gelu_workspace_size(E, C, D, F, D) >= 4 * E * C * (D + 2 * F + D)
    assert moe.binding.moe_backward_gelu_workspace_size(E, 0, D, F, D) > 0


def test_backward_gelu_host_checks():
    L = moe.lib()
    p, nul = ctypes.c_void_p(16), None

    def call(dtype, T=8, k=2, E=4, C=4, D=16, F=16, Dout=16, residual=0, ws_bytes=1 << 30):
        return L.moe_backward_gelu(dtype, p, p, p, p, p, p, p, p, p, p, p, T, k, E, C, D, F, Dout, residual, 0.0, 1,
                                   nul, p, p, p, p, p, p, p, nul, p, ws_bytes, nul)

    assert call(B.MOE_BF16) == B.MOE_ERR_UNSUPPORTED        # fp32 only
    assert call(B.MOE_F32, k=5) == B.MOE_ERR_INVALID_ARG     # k > E
    assert call(B.MOE_F32, residual=1, Dout=8) == B.MOE_ERR_INVALID_ARG  # residual needs Dout == D
    assert call(B.MOE_F32, ws_bytes=64) == B.MOE_ERR_WORKSPACE


def test_expert_parallel_host_checks():
    L = moe.lib()
    p, nul = ctypes.c_void_p(16), None
    tab2 = (ctypes.c_void_p * 2)(16, 32)
    # E not a multiple of the rank count
    rc = L.moe_ep_dispatch(p, 8, 2, 6, 4, p, 0, nul, 0, 0, 0, tab2, 4, p, p, p, nul, nul, p, 1 << 20, nul)
    assert rc == B.MOE_ERR_INVALID_ARG
    # more ranks than the peer-pointer table holds
    rc = L.moe_ep_dispatch(p, 8, 2, 128, 4, p, 0, nul, 0, 0, 0, tab2, 128, p, p, p, nul, nul, p, 1 << 20, nul)
    assert rc == B.MOE_ERR_UNSUPPORTED
    # a NULL entry in the table when rows are moved
    bad = (ctypes.c_void_p * 2)(16, 0)
    rc = L.moe_ep_dispatch(p, 8, 2, 4, 4, p, 0, p, 1, 8, 8, bad, 2, p, p, p, nul, nul, p, 1 << 20, nul)
    assert rc == B.MOE_ERR_INVALID_ARG
    # combine: rank out of range for the plan, missing table
    assert L.moe_ep_plan(p, 2, 2, 4, 4, p, nul, nul, nul, nul) == B.MOE_ERR_INVALID_ARG
    rc = L.moe_ep_combine(nul, 2, p, p, nul, 0, 8, 2, 4, 4, 8, 0, nul, 0, p, 8, 1, nul, nul)
    assert rc == B.MOE_ERR_INVALID_ARG
    # IPC calls reject NULL arguments before touching the driver
    assert L.moe_ipc_export(nul, nul, nul) == B.MOE_ERR_INVALID_ARG
    assert L.moe_ipc_import(nul, nul) == B.MOE_ERR_INVALID_ARG
    assert L.moe_ipc_close(nul) == B.MOE_ERR_INVALID_ARG


def test_expert_ffn_with_zero_capacity_touches_nothing():
    # C = 0: nothing is read or written, so NULL buffers are accepted and no kernel is launched
    L = moe.lib()
    nul = None
    for kind in (0, 1, 2):
        for dtype in (B.MOE_F32, B.MOE_BF16):
            rc = L.moe_expert_ffn(kind, dtype, nul, nul, 4, 0, 64, 32, 64, nul, nul, nul, nul, nul, nul, nul, nul, 0,
                                  nul)
            assert rc == B.MOE_OK, (kind, dtype)
    assert L.moe_expert_ffn_save(nul, nul, 4, 0, 64, 32, 64, nul, nul, nul, nul, nul, nul, nul, 0, nul) == B.MOE_OK
    # with rows to compute the buffers are required
    rc = L.moe_expert_ffn(2, B.MOE_BF16, nul, nul, 4, 8, 64, 32, 64, nul, nul, nul, nul, nul, nul, nul, nul, 0, nul)
    assert rc == B.MOE_ERR_INVALID_ARG


def test_wait_probe_host_checks():
    L = moe.lib()
    p, nul = ctypes.c_void_p(16), None
    assert L.moe_wait_probe(nul, 1000, p, nul) == B.MOE_ERR_INVALID_ARG
    assert L.moe_wait_probe(p, 0, p, nul) == B.MOE_ERR_INVALID_ARG
    assert L.moe_wait_probe(p, 5_000_000_000, p, nul) == B.MOE_ERR_INVALID_ARG  # above the library's wait bound
