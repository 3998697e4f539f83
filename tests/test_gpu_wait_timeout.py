"""The bounded pipeline waits of the tensor-core kernels give up cleanly.

With the wait limit lowered to a few nanoseconds (moe_debug_set_wait_limit_ns,
a test hook), the grouped GEMMs' waits for their TMA copies and MMAs run out:
the kernel must set MOE_DEVERR_TIMEOUT, drain what it has in flight, free its
tensor memory and return; with the default limit restored the next call must
give the same bits as a clean run. Nothing faults, traps or hangs: the waits
are bounded by construction and the drain waits keep their own limit."""
import time

import numpy as np
import pytest
import torch

from dropless_top_mixture_b200.workloads import adversarial_logits
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu


def _moe():
    from dropless_top_mixture_b200 import moe
    return moe


def _problem(T=300, d=256, F=256, E=5, k=2, seed=7):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, d, generator=g).to(torch.bfloat16)
    W1 = (torch.randn(E, F, d, generator=g) * d ** -0.5).to(torch.bfloat16)
    W3 = (torch.randn(E, F, d, generator=g) * d ** -0.5).to(torch.bfloat16)
    W2 = (torch.randn(E, d, F, generator=g) * F ** -0.5).to(torch.bfloat16)
    lg = adversarial_logits(T, E, "normal", seed=seed).numpy()
    idx, _, _ = O.route(lg, k)
    meta = O.routing_metadata(idx, E)
    Xe = torch.from_numpy(O.dispatch(x.double().numpy(), meta["slot"])).to(torch.bfloat16)
    return Xe, W1, W3, W2, torch.from_numpy(meta["offsets"])


def test_grouped_gemm_wait_timeout_sets_status_and_recovers():
    moe = _moe()
    Xe, W1, W3, W2, offs = (t.cuda() for t in _problem())
    assert moe.moe_get_status(clear=True) == 0
    H0, Y0 = moe.moe_grouped_swiglu(Xe, W1, W3, W2, offs)
    torch.cuda.synchronize()
    assert moe.moe_get_status() == 0
    H1 = torch.full_like(H0, 3.0)
    Y1 = torch.full_like(Y0, 3.0)
    try:
        moe.moe_debug_set_wait_limit_ns(4)
        t0 = time.monotonic()
        moe.moe_grouped_swiglu(Xe, W1, W3, W2, offs, H=H1, Ye=Y1)
        torch.cuda.synchronize()
        took = time.monotonic() - t0
    finally:
        moe.moe_debug_set_wait_limit_ns(0)
    st = moe.moe_get_status(clear=True)
    assert st & moe.MOE_DEVERR_TIMEOUT, st
    assert took < 5.0, took  # the kernels returned (each drain wait is bounded by 0.1 s)
    # the default limit is back: the same call gives the clean run's bits
    H2, Y2 = moe.moe_grouped_swiglu(Xe, W1, W3, W2, offs)
    torch.cuda.synchronize()
    assert moe.moe_get_status() == 0
    assert torch.equal(H2, H0) and torch.equal(Y2, Y0)
