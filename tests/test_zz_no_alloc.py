"""moe_route_noalloc — the route step for callers that cannot allocate
device memory — called through the C ABI and compared with moe_route, which
takes a caller workspace. Two different batches are routed back to back so
the second call runs on scratch the first one left behind.

This file is collected last on purpose: it passes alone in a fresh process
and after every other test."""
import ctypes

import numpy as np
import pytest
import torch

from dropless_top_mixture_b200.workloads import adversarial_logits
from tests._util import gate_tolerance

pytestmark = pytest.mark.gpu


def _outputs(T, E, k, dev, with_logits=False):
    from dropless_top_mixture_b200 import moe
    i32 = dict(dtype=torch.int32, device=dev)
    r = moe.Route(idx=torch.full((T, k), -7, **i32),
                  gate=torch.full((T, k), -7.0, dtype=torch.float32, device=dev),
                  counts=torch.full((E,), -7, **i32), offsets=torch.full((E + 1,), -7, **i32),
                  slot=torch.full((T, k), -7, **i32), tile_offsets=torch.full((E + 1,), -7, **i32))
    if with_logits:
        r.logits = torch.full((T, E), -7.0, dtype=torch.float32, device=dev)
    return r


def _call_noalloc(lib, r, k, logits=None, x=None, Wr=None, dtype=0):
    p = lambda t: None if t is None else t.data_ptr()
    if logits is not None:
        T, E = logits.shape
        d = 0
    else:
        T, d = x.shape
        E = Wr.shape[0]
    stream = torch.cuda.current_stream().cuda_stream
    return lib.moe_route_noalloc(p(logits), p(x), p(Wr), dtype, T, d, E, k, 0, p(r.logits),
                                 p(r.idx), p(r.gate), p(r.counts), p(r.offsets), p(r.slot),
                                 p(r.tile_offsets), ctypes.c_void_p(stream))


def _same(a, b, lg, k):
    for name in ("idx", "counts", "offsets", "slot", "tile_offsets"):
        assert torch.equal(getattr(a, name).cpu(), getattr(b, name).cpu()), name
    ga = a.gate.cpu().double().numpy()
    gb = b.gate.cpu().double().numpy()
    tol = gate_tolerance(lg, a.idx.cpu().numpy(), False)
    assert np.all(np.abs(ga - gb) <= tol * np.abs(gb))


def test_noalloc_route_matches_workspace_route_twice():
    from dropless_top_mixture_b200 import moe
    lib = moe.lib
    dev = torch.device("cuda", 0)
    # call 1: logits given (a sweep-shaped batch)
    T1, E1, k1 = 4096, 128, 4
    lg1 = adversarial_logits(T1, E1, "normal", seed=101)
    a1 = _outputs(T1, E1, k1, dev)
    assert _call_noalloc(lib, a1, k1, logits=lg1.to(dev)) == moe.MOE_OK
    ref1 = moe.moe_route(k1, logits=lg1.to(dev))
    torch.cuda.synchronize()
    _same(a1, ref1, lg1.numpy(), k1)
    # call 2, straight after: a different shape, logits computed from x and Wr,
    # on the scratch the first call left behind
    T2, d2, E2, k2 = 3000, 256, 64, 8
    g = torch.Generator().manual_seed(102)
    x2 = torch.randn(T2, d2, generator=g).to(torch.bfloat16).to(dev)
    Wr2 = (torch.randn(E2, d2, generator=g) * 0.02).to(torch.bfloat16).to(dev)
    a2 = _outputs(T2, E2, k2, dev, with_logits=True)
    assert _call_noalloc(lib, a2, k2, x=x2, Wr=Wr2, dtype=moe.MOE_BF16) == moe.MOE_OK
    ref2 = moe.moe_route(k2, x=x2, Wr=Wr2, keep_logits=True)
    torch.cuda.synchronize()
    assert torch.equal(a2.logits.cpu(), ref2.logits.cpu())
    _same(a2, ref2, ref2.logits.cpu().numpy(), k2)
    # and the first batch again, to see nothing of call 2 leaks into call 3
    a3 = _outputs(T1, E1, k1, dev)
    assert _call_noalloc(lib, a3, k1, logits=lg1.to(dev)) == moe.MOE_OK
    torch.cuda.synchronize()
    _same(a3, ref1, lg1.numpy(), k1)
    assert moe.moe_get_status() == 0


def test_noalloc_route_rejects_sizes_beyond_its_scratch():
    from dropless_top_mixture_b200 import moe
    lib = moe.lib
    dev = torch.device("cuda", 0)
    T, E, k = 200_000, 256, 2   # chunk counts alone need 25.6 MB > 8 MiB
    assert lib.moe_route_workspace_size(T, E, 0) > (8 << 20)
    lg = torch.zeros((T, E), dtype=torch.float32, device=dev)
    r = _outputs(T, E, k, dev)
    assert _call_noalloc(lib, r, k, logits=lg) == moe.MOE_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert (r.idx == -7).all() and (r.counts == -7).all()  # nothing launched
