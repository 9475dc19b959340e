"""The workspace-free dispatch entry point against the regular one.

moe_dispatch_static serves callers that may not allocate device memory, such as
code that a host framework hands only input and output pointers; its slot-scan
state is a fixed device array inside the library instead of a caller
workspace.  Two calls in a row (different shapes and selections) must each
match moe_dispatch exactly, so state left by one call never leaks into the next.
This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from sparse_mixture_experts_stable_b200 import binding as B

pytestmark = pytest.mark.gpu

KEYS = ("slot", "kept", "used", "overflow", "drops", "token_of_slot", "xbuf")


def _selection(seed, T, E, k):
    rng = np.random.default_rng(seed)
    return torch.from_numpy(np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int64)).cuda()


def test_static_dispatch_matches_workspace_dispatch_twice():
    cases = [(5000, 256, 8, 100, 1), (3001, 64, 2, 70, 2)]
    got_all, ref_all = [], []
    for T, E, k, C, seed in cases:
        sel = _selection(seed, T, E, k)
        x = torch.randn(T, 136, device="cuda").to(torch.bfloat16)
        st = B.new_status()
        got_all.append(B.moe_dispatch_static(sel, E, C, x=x, dev_status=st))  # through the C ABI
        assert B.moe_read_status(st) == 0
        ref_all.append((sel, E, C, x))
    for got, (sel, E, C, x) in zip(got_all, ref_all):
        ref = B.moe_dispatch(sel, E, C, x=x)
        torch.cuda.synchronize()
        for key in KEYS[:-1]:
            assert torch.equal(got[key], ref[key]), key
        used = ref["used"].cpu().numpy()
        for e in range(E):
            u = int(used[e])
            assert torch.equal(got["xbuf"][e, :u], ref["xbuf"][e, :u])


def test_static_dispatch_rejects_problems_beyond_its_array():
    L = B.lib()
    limit = L.moe_dispatch_static_max_state_bytes()
    assert limit == 4 << 20
    p = ctypes.c_void_p(16)
    # E = 256 and T = 600000 need more look-back state than the array holds
    rc = L.moe_dispatch_static(p, 600000, 1, 256, 10, None, 0, 0, 0, p, p, p, p, p, p, None, None, None)
    assert rc == B.MOE_ERR_UNSUPPORTED
