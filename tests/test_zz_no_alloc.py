"""The workspace-free dispatch entry point, checked on the GPU.

moe_dispatch_static serves callers that may not allocate device memory, such as
code that a host framework hands only input and output pointers; its slot-scan
state is a fixed device array inside the library instead of a caller
workspace.  Two calls in a row (different shapes and selections) must each
match moe_dispatch exactly and the oracle's greedy loop, so state left by one
call never leaks into the next; and a call whose outputs are all provided must
leave the device's memory use unchanged.  This file is collected last on
purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import oracle as O
from sparse_mixture_experts_stable_b200 import binding as B
from tests.gpu_util import check_dispatch, cpu64

pytestmark = pytest.mark.gpu

KEYS = ("slot", "kept", "used", "overflow", "drops", "token_of_slot", "xbuf")


def _selection(seed, T, E, k):
    rng = np.random.default_rng(seed)
    return np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int64)


def _outputs(T, k, E, C, D, dtype):
    dev = "cuda"
    return dict(slot=torch.empty(T, k, dtype=torch.int64, device=dev),
                kept=torch.empty(T, k, dtype=torch.uint8, device=dev),
                used=torch.empty(E, dtype=torch.int32, device=dev),
                overflow=torch.empty(E, dtype=torch.int32, device=dev),
                drops=torch.empty(T, dtype=torch.int32, device=dev),
                token_of_slot=torch.empty(E, C, dtype=torch.int32, device=dev),
                xbuf=torch.empty(E, C, D, dtype=dtype, device=dev))


def test_static_dispatch_matches_workspace_dispatch_and_oracle_twice():
    cases = [(5000, 256, 8, 100, 1), (3001, 64, 2, 70, 2)]
    got_all, ref_all = [], []
    for T, E, k, C, seed in cases:
        sel = _selection(seed, T, E, k)
        x = torch.randn(T, 136, device="cuda").to(torch.bfloat16)
        st = B.new_status()
        got_all.append(B.moe_dispatch_static(torch.from_numpy(sel).cuda(), E, C, x=x, dev_status=st))
        assert B.moe_read_status(st) == 0
        ref_all.append((sel, E, C, x))
    for got, (sel, E, C, x) in zip(got_all, ref_all):
        ref = B.moe_dispatch(torch.from_numpy(sel).cuda(), E, C, x=x)
        torch.cuda.synchronize()
        for key in KEYS[:-1]:
            assert torch.equal(got[key], ref[key]), key
        o = O.dispatch(sel, E, C)
        check_dispatch(o, got, E, C, f"static dispatch E={E} C={C}")
        xb, xs = cpu64(got["xbuf"]), cpu64(x)
        for e in range(E):
            u = int(o["used"][e])
            if u:
                np.testing.assert_array_equal(xb[e, :u], xs[o["token_of_slot"][e, :u]])


def test_static_dispatch_allocates_no_device_memory():
    T, E, k, C, D = 4000, 128, 4, 150, 64
    x = torch.randn(T, D, device="cuda").to(torch.bfloat16)
    sels = [torch.from_numpy(_selection(s, T, E, k)).cuda() for s in (5, 6)]
    out = _outputs(T, k, E, C, D, x.dtype)
    st = B.new_status()
    # the first call on the device looks up the array's address and loads the kernels
    B.moe_dispatch_static(sels[0], E, C, x=x, out=out, dev_status=st)
    torch.cuda.synchronize()
    alloc0, reserved0 = torch.cuda.memory_allocated(), torch.cuda.memory_reserved()
    free0, _ = torch.cuda.mem_get_info()
    got = B.moe_dispatch_static(sels[1], E, C, x=x, out=out, dev_status=st)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == alloc0
    assert torch.cuda.memory_reserved() == reserved0
    assert free1 >= free0, (free0, free1)
    assert all(got[key] is out[key] for key in KEYS)
    assert B.moe_read_status(st) == 0
    check_dispatch(O.dispatch(sels[1].cpu().numpy(), E, C), got, E, C, "static dispatch, preallocated outputs")


def test_static_dispatch_rejects_problems_beyond_its_array():
    L = B.lib()
    limit = L.moe_dispatch_static_max_state_bytes()
    assert limit == 4 << 20
    p = ctypes.c_void_p(16)
    # E = 256 and T = 600000 need more look-back state than the array holds
    rc = L.moe_dispatch_static(p, 600000, 1, 256, 10, None, 0, 0, 0, p, p, p, p, p, p, None, None, None)
    assert rc == B.MOE_ERR_UNSUPPORTED
