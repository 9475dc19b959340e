"""Seeded synthetic inputs shaped like the pages' MoE workloads.

This module only draws random numbers and arranges them in the library's
storage layouts; it contains none of the layer's arithmetic.  The tests, the
benchmark, the smoke check and the CPU oracle all take their inputs from here,
so the CUDA path and the oracle always see identical values.

Storage conventions (what the C-ABI expects):
  * activations ``x``: (T, D) row-major, fp32 or bf16;
  * router weight: (E, D), the (out, in) layout of ``nn.Linear(D, E)``;
    ``w_router_de`` gives the same values as the (D, E) matrix of the router
    page;
  * expert weights: (E, N_out, K_in) per matrix, the (out, in) layout of
    ``nn.Linear``; the oracle receives them transposed to the pages' x @ W form
    (E, K_in, N_out) via :func:`pages_layout`.

Every generator takes a ``seed`` and optional size overrides, so the parity
tests can run the same recipe at sizes the oracle finishes in seconds.
All draws use ``numpy.random.default_rng(seed)`` (PCG64).
"""
from __future__ import annotations

import numpy as np
import torch


def _round_to(a: np.ndarray, step_log2: int) -> np.ndarray:
    """Round to the nearest multiple of 2**-step_log2 (dyadic grid)."""
    s = float(2 ** step_log2)
    return np.round(a * s) / s


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def _f32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))


def pages_layout(w_out_in: torch.Tensor) -> np.ndarray:
    """(E, N_out, K_in) storage -> float64 (E, K_in, N_out) for the x @ W formulas."""
    return w_out_in.to(torch.float64).transpose(-1, -2).contiguous().numpy()


def as_f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()


def tiny_gelu_fp32(seed: int = 0, T: int = 512, D: int = 64, E: int = 8, F: int = 256,
                   k: int = 2, capacity_factor: float = 1.25) -> dict:
    """Tiny top-2 layer with two-layer GELU experts, fp32.

    x ~ N(0,1) rounded to multiples of 2^-8 and clipped to [-6, 6]; router and
    expert weights and biases ~ N(0, 0.02) rounded to multiples of 2^-10.  On
    this grid every partial sum of the router dot product is exact in fp32
    (the tests check the bound), so the routing decision is exact.
    """
    rng = np.random.default_rng(seed)
    x = np.clip(_round_to(rng.standard_normal((T, D)), 8), -6.0, 6.0)
    w_router = _round_to(rng.normal(0.0, 0.02, (E, D)), 10)
    w1 = _round_to(rng.normal(0.0, 0.02, (E, F, D)), 10)
    b1 = _round_to(rng.normal(0.0, 0.02, (E, F)), 10)
    w2 = _round_to(rng.normal(0.0, 0.02, (E, D, F)), 10)
    b2 = _round_to(rng.normal(0.0, 0.02, (E, D)), 10)
    return dict(name="tiny_gelu_fp32", T=T, D=D, E=E, F=F, k=k, capacity_factor=capacity_factor,
                x=_f32(x), w_router=_f32(w_router), w1=_f32(w1), b1=_f32(b1), w2=_f32(w2),
                b2=_f32(b2))


def router_bf16(seed: int = 0, T: int = 65536, D: int = 2048, E: int = 256, k: int = 8,
                tie_columns: int = 16, zero_row_every: int = 64) -> dict:
    """Router-only workload with load statistics, bf16 storage.

    x and the router weight are integers in [-4, 4] times 2^-6, so every score
    is a multiple of 2^-12 bounded by 8 in magnitude and exact in fp32.  To
    force exact ties, the last ``tie_columns`` router columns repeat the first
    ones, and every ``zero_row_every``-th token row of x is zero (all E scores
    tie).
    """
    rng = np.random.default_rng(seed)
    x = rng.integers(-4, 5, size=(T, D)).astype(np.float32) / 64.0
    if zero_row_every:
        x[::zero_row_every] = 0.0
    w = rng.integers(-4, 5, size=(E, D)).astype(np.float32) / 64.0
    if tie_columns and E >= 2 * tie_columns:
        w[E - tie_columns:] = w[:tie_columns]
    return dict(name="router_bf16", T=T, D=D, E=E, k=k, x=_bf16(x), w_router=_bf16(w))


def zipf_expert_ids(rng: np.random.Generator, T: int, E: int, s: float = 1.1) -> np.ndarray:
    """Truncated Zipf(s) over E experts: P(rank r) proportional to r^-s, expert = r - 1."""
    r = np.arange(1, E + 1, dtype=np.float64)
    p = r ** (-s)
    p /= p.sum()
    return rng.choice(E, size=T, p=p).astype(np.int64)


def dispatch_top1_bf16(seed: int = 0, T: int = 32768, D: int = 1024, E: int = 64,
                       capacity_factor: float = 1.0) -> dict:
    """Capacity-limited top-1 dispatch/combine with linear experts, bf16.

    expert_idx ~ truncated Zipf(1.1) over E (forces overflow), gate ~ U(0,1)
    stored bf16, x ~ N(0,1) bf16, expert weights ~ N(0, 0.02) bf16 stored
    (E, D_out, D_in).
    """
    rng = np.random.default_rng(seed)
    idx = zipf_expert_ids(rng, T, E)
    gate = rng.uniform(0.0, 1.0, T)
    x = rng.standard_normal((T, D), dtype=np.float32)
    w = rng.standard_normal((E, D, D), dtype=np.float32) * np.float32(0.02)
    return dict(name="dispatch_top1_bf16", T=T, D=D, E=E, k=1, capacity_factor=capacity_factor,
                expert_idx=torch.from_numpy(idx), gate=_bf16(gate), x=_bf16(x), w=_bf16(w))


def full_layer_bf16(seed: int = 0, T: int = 16384, H: int = 2048, E: int = 256, F: int = 512,
                    k: int = 8, capacity_factor: float = 1.25, F_shared: int = 512,
                    aux_coef: float = 0.001) -> dict:
    """Full layer: router + SwiGLU routed experts + one always-on shared expert, bf16.

    Dyadic realisation of "logits ~ N(0,1) with a per-expert skew N(0, 0.5)":
    x = a/8 with a uniform in the integers [-8, 8]; router weight = b * 2^-7 with
    b uniform in [-8, 8] (scores are multiples of 2^-10, |s| < 2^7, exact in
    fp32, standard deviation about 1.06); router bias ~ N(0, 0.5) rounded to
    2^-10.  Expert weights ~ N(0, 0.02) bf16: gate/up (E, F, H), down (E, H, F);
    shared expert gate/up (F_shared, H), down (H, F_shared).
    """
    rng = np.random.default_rng(seed)
    x = rng.integers(-8, 9, size=(T, H)).astype(np.float32) / 8.0
    w_router = rng.integers(-8, 9, size=(E, H)).astype(np.float32) / 128.0
    bias = _round_to(rng.normal(0.0, 0.5, E), 10)

    def normal(shape):
        return rng.standard_normal(shape, dtype=np.float32) * np.float32(0.02)

    w_gate = normal((E, F, H))
    w_up = normal((E, F, H))
    w_down = normal((E, H, F))
    s_gate = normal((F_shared, H))
    s_up = normal((F_shared, H))
    s_down = normal((H, F_shared))
    return dict(name="full_layer_bf16", T=T, H=H, D=H, E=E, F=F, k=k,
                capacity_factor=capacity_factor, F_shared=F_shared, aux_coef=aux_coef,
                x=_bf16(x), w_router=_bf16(w_router), router_bias=_f32(bias),
                w_gate=_bf16(w_gate), w_up=_bf16(w_up), w_down=_bf16(w_down),
                s_gate=_bf16(s_gate[None]), s_up=_bf16(s_up[None]), s_down=_bf16(s_down[None]))


def router_spread_bf16(seed: int = 0, T: int = 1500, D: int = 512, E: int = 64) -> dict:
    """Router inputs with the full layer's score spread (std about 0.5 at D = 512).

    Same recipe as the router part of full_layer_bf16: x = a/8, router weight
    b * 2^-7 with a, b uniform in the integers [-8, 8], so every score is a
    multiple of 2^-10 below 2^6 in magnitude for D <= 512 and exact in fp32.
    """
    rng = np.random.default_rng(seed)
    x = rng.integers(-8, 9, size=(T, D)).astype(np.float32) / 8.0
    w_router = rng.integers(-8, 9, size=(E, D)).astype(np.float32) / 128.0
    return dict(name="router_spread_bf16", T=T, D=D, E=E, x=_bf16(x), w_router=_bf16(w_router))


def fwd_bwd_fp32(seed: int = 0, T: int = 8192, D: int = 1024, E: int = 64, k: int = 2,
                 capacity_factor: float = 1.0) -> dict:
    """Forward + backward of a top-2 linear-expert layer with residual, fp32.

    Router logits (given) ~ N(0,1), x ~ N(0,1), W ~ N(0, 0.02) stored
    (E, D_out, D_in), upstream gradient dy ~ N(0,1).
    """
    rng = np.random.default_rng(seed)
    logits = rng.standard_normal((T, E), dtype=np.float32)
    x = rng.standard_normal((T, D), dtype=np.float32)
    w = rng.standard_normal((E, D, D), dtype=np.float32) * np.float32(0.02)
    dy = rng.standard_normal((T, D), dtype=np.float32)
    return dict(name="fwd_bwd_fp32", T=T, D=D, E=E, k=k, capacity_factor=capacity_factor,
                logits=_f32(logits), x=_f32(x), w=_f32(w), dy=_f32(dy))


CONFIGS = {
    "tiny_gelu_fp32": tiny_gelu_fp32,
    "router_bf16": router_bf16,
    "dispatch_top1_bf16": dispatch_top1_bf16,
    "full_layer_bf16": full_layer_bf16,
    "fwd_bwd_fp32": fwd_bwd_fp32,
}
