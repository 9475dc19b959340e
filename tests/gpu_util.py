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


def assert_close_mag(got, want, mag, rtol, atol, what=""):
    """|got - want| <= atol + rtol * max(|want|, mag).

    ``mag`` is the magnitude of the terms summed into each output (the oracle
    evaluated on the absolute values of its inputs).  Any fp32 summation of
    those terms, in any order, has an error proportional to it; applying rtol
    to |want| alone would demand more than fp32 can give where terms cancel.
    """
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    mag = np.broadcast_to(np.asarray(mag, dtype=np.float64), want.shape)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    err = np.abs(got - want)
    bound = atol + rtol * np.maximum(np.abs(want), mag)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {err.size} elements outside rtol={rtol}*magnitude "
                             f"atol={atol}; worst at {i}: got {got[i]!r} want {want[i]!r} magnitude {mag[i]!r}")


def bf16_ulp(a: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |a| (8 significant bits)."""
    a = np.abs(np.asarray(a, dtype=np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def assert_within_bf16_ulp(got_bf16, want_f64, what=""):
    """A bf16 output may differ from the oracle value rounded to bf16 by one bf16 ulp
    (the fp32 result and the fp64 value can straddle a rounding boundary)."""
    want = bf16_round(want_f64)
    got = np.asarray(got_bf16, dtype=np.float64)
    err = np.abs(got - want)
    ulp = bf16_ulp(np.maximum(np.abs(np.asarray(want_f64, dtype=np.float64)), np.abs(want)))
    bad = err > ulp * 1.0000001
    if bad.any():
        i = np.unravel_index(np.argmax(err), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} elements more than one bf16 ulp away; "
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
