"""moe_combine on the GPU against the oracle's expert-major combine."""
import numpy as np
import pytest
import torch

import sparse_mixture_experts_stable_b200 as moe
from oracle import oracle as O
from tests.gpu_util import BF16_ATOL, BF16_RTOL, DEV, F32_ATOL, F32_RTOL, assert_close, assert_close_mag, cpu64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("base_kind", ["zero", "input", "tensor"])
@pytest.mark.parametrize("N", [1024, 100])
def test_combine_matches_oracle(dtype, base_kind, N):
    rng = np.random.default_rng(N)
    T, E, k = 1000, 16, 4
    C = 200
    sel = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int64)
    d = O.dispatch(sel, E, C)
    gates = rng.uniform(0, 1, (T, k)).astype(np.float32)
    ybuf = torch.randn(E, C, N).to(dtype)
    base = torch.randn(T, N).to(dtype) if base_kind != "zero" else None
    y = moe.moe_combine(ybuf.to(DEV), torch.from_numpy(sel).to(DEV), torch.from_numpy(d["slot"]).to(DEV),
                        torch.from_numpy(gates).to(DEV), base_kind=base_kind,
                        base=None if base is None else base.to(DEV))
    want = O.combine_slots(cpu64(ybuf), sel, d["slot"], d["kept"], gates,
                           base=None if base is None else cpu64(base))
    if dtype == torch.float32:
        mag = O.combine_slots(np.abs(cpu64(ybuf)), sel, d["slot"], d["kept"], gates,
                              base=None if base is None else np.abs(cpu64(base)))
        assert_close_mag(cpu64(y), want, mag, F32_RTOL, F32_ATOL, f"combine {dtype} {base_kind}")
    else:
        assert_close(cpu64(y), want, BF16_RTOL, BF16_ATOL, f"combine {dtype} {base_kind}")
    # fully dropped tokens give exactly the base row
    full = np.flatnonzero(d["drops"] == k)
    if len(full):
        exp = np.zeros((len(full), N)) if base is None else cpu64(base)[full]
        np.testing.assert_array_equal(cpu64(y)[full], exp)


def test_combine_bf16_gates_and_determinism():
    rng = np.random.default_rng(1)
    T, E, k, C, N = 3000, 64, 8, 400, 512
    sel = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int64)
    d = O.dispatch(sel, E, C)
    g = torch.from_numpy(rng.uniform(0, 1, (T, k)).astype(np.float32)).to(torch.bfloat16)
    ybuf = torch.randn(E, C, N).to(torch.bfloat16).to(DEV)
    args = (ybuf, torch.from_numpy(sel).to(DEV), torch.from_numpy(d["slot"]).to(DEV), g.to(DEV))
    y1 = moe.moe_combine(*args)
    y2 = moe.moe_combine(*args)
    assert torch.equal(y1, y2)
    want = O.combine_slots(cpu64(ybuf), sel, d["slot"], d["kept"], cpu64(g))
    assert_close(cpu64(y1), want, BF16_RTOL, BF16_ATOL, "bf16 gates")
