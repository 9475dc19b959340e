"""Helpers shared by the GPU parity tests (comparison with the fp64 oracle)."""
import numpy as np
import torch

# Tolerances stated for the floating-point outputs: fp32 paths and bf16 expert GEMMs.
F32_RTOL, F32_ATOL = 1e-5, 1e-6
BF16_RTOL, BF16_ATOL = 2e-2, 2e-2

DEV = "cuda"


def cpu64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def cpu(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def assert_close(got, want, rtol, atol, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    err = np.abs(got - want)
    bound = atol + rtol * np.abs(want)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {err.size} elements outside rtol={rtol} atol={atol}; "
                             f"worst at {i}: got {got[i]!r} want {want[i]!r}")


def bf16_round(a: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


def check_dispatch(o, gpu, E, C, what=""):
    """Compare every integer output of moe_dispatch with the oracle's dispatch dict ``o``."""
    np.testing.assert_array_equal(cpu(gpu["slot"]), o["slot"], err_msg=what + " slot")
    np.testing.assert_array_equal(cpu(gpu["kept"]).astype(bool), o["kept"], err_msg=what + " kept")
    np.testing.assert_array_equal(cpu(gpu["used"]), o["used"], err_msg=what + " used")
    np.testing.assert_array_equal(cpu(gpu["overflow"]), o["overflow"], err_msg=what + " overflow")
    np.testing.assert_array_equal(cpu(gpu["drops"]), o["drops"], err_msg=what + " drops")
    if C > 0:
        np.testing.assert_array_equal(cpu(gpu["token_of_slot"]), o["token_of_slot"], err_msg=what + " token_of_slot")
