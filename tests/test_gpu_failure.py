"""Failure detection on the GPU without a fault: a bounded device wait whose
flag nothing sets must give up, record MOE_ERR_TIMEOUT in the status word that
the host reads, and leave the context usable for the next call."""
import time

import numpy as np
import pytest
import torch

import sparse_mixture_experts_stable_b200 as moe
from oracle import oracle as O
from sparse_mixture_experts_stable_b200 import binding as B
from tests.gpu_util import DEV, cpu, cpu64

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_the_context_stays_usable():
    flag = torch.zeros(1, dtype=torch.int32, device=DEV)
    st = moe.new_status()
    t0 = time.perf_counter()
    B.moe_wait_probe(flag, 200_000_000, st)  # 0.2 s
    assert moe.moe_read_status(st) == B.MOE_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 5.0
    # a flag that is set ends the wait at once, with no error
    flag.fill_(1)
    st2 = moe.new_status()
    B.moe_wait_probe(flag, 200_000_000, st2)
    assert moe.moe_read_status(st2) == B.MOE_OK
    # the next library call works and gives the oracle's routing
    lg = torch.randn(64, 8, generator=torch.Generator().manual_seed(1)).to(DEV)
    r = moe.moe_route(lg, 2, dev_status=st2)
    assert moe.moe_read_status(st2) == B.MOE_OK
    _, sel, _, _, _ = O.route(cpu64(lg), 2)
    np.testing.assert_array_equal(cpu(r["selected"]), sel)
