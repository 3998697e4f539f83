"""moe_layer_fwd_host: the layer from and to pinned host memory in token
slices with overlapped copies. The layer is token-wise, so every token's
output, expert choice and gate must equal the single device-resident call's
bit for bit, whatever the slicing; the slot of each slice must be a
permutation of that slice's expert rows."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from dropless_top_mixture_b200.workloads import WORKLOADS, make_inputs
from tests._util import assert_close_layer, np64

pytestmark = pytest.mark.gpu


def _moe():
    from dropless_top_mixture_b200 import moe
    return moe


def _problem(T, d, F, E, k, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, d, generator=g).to(dtype)
    W1 = (torch.randn(E, F, d, generator=g) * d ** -0.5).to(dtype)
    W3 = (torch.randn(E, F, d, generator=g) * d ** -0.5).to(dtype)
    W2 = (torch.randn(E, d, F, generator=g) * F ** -0.5).to(dtype)
    Wr = (torch.randn(E, d, generator=g) * d ** -0.5).to(dtype)
    lg = torch.randn(T, E, generator=g)
    return x, W1, W3, W2, Wr, lg


def _slice_bounds(T, chunks):
    """Token slices of the host pipeline: equal for one or two slices; from
    three on, the first and the last are half the size of the others."""
    if chunks < 3:
        return [T * i // chunks for i in range(chunks + 1)]
    w2 = 2 * (chunks - 1)
    return [0] + [T * (2 * i - 1) // w2 for i in range(1, chunks)] + [T]


def _check_slices(slot, T, k, chunks):
    b = _slice_bounds(T, chunks)
    for t0, t1 in zip(b[:-1], b[1:]):
        if t1 <= t0:
            continue
        s = slot[t0:t1].reshape(-1)
        assert np.array_equal(np.sort(s), np.arange(s.size))


@pytest.mark.parametrize("T,d,F,E,k,dtype,chunks,router", [
    (1000, 256, 256, 8, 2, torch.bfloat16, 1, False),
    (1000, 256, 256, 8, 2, torch.bfloat16, 3, False),
    (1333, 512, 384, 16, 4, torch.bfloat16, 7, True),
    (300, 128, 128, 5, 2, torch.float32, 4, True),
    (17, 256, 128, 4, 2, torch.bfloat16, 16, False),   # slices of 2 tokens, the last of 1
])
def test_host_pipeline_matches_device_call(T, d, F, E, k, dtype, chunks, router):
    moe = _moe()
    x, W1, W3, W2, Wr, lg = _problem(T, d, F, E, k, dtype, seed=T + chunks)
    dev = "cuda"
    W1d, W3d, W2d = W1.to(dev), W3.to(dev), W2.to(dev)
    kw = dict(Wr=Wr.to(dev)) if router else dict(logits=lg.to(dev))
    ref = moe.moe_layer_fwd(x.to(dev), k, W1d, W3d, W2d, **kw)
    hl = moe.HostLayer(T, d, E, F, k, dtype, dev, logits_given=not router, chunks=chunks)
    xh = x.pin_memory()
    lh = None if router else lg.pin_memory()
    out = hl(xh, W1d, W3d, W2d, logits_host=lh, Wr=kw.get("Wr"))
    torch.cuda.current_stream().synchronize()
    assert moe.moe_get_status() == 0
    assert torch.equal(out, ref.out.cpu())
    assert torch.equal(hl.res.idx.cpu(), ref.idx.cpu())
    assert torch.equal(hl.res.gate.cpu(), ref.gate.cpu())
    _check_slices(hl.res.slot.cpu().numpy(), T, k, chunks)
    # and against the oracle on a few tokens
    if not router:
        toks = np.arange(0, T, max(1, T // 6))
        idx, gate, _ = O.route(lg.numpy(), k)
        want = O.moe_layer_tokens(x, toks, idx, gate, W1, W3, W2)
        assert_close_layer(np64(out[torch.as_tensor(toks)]), want, "host pipeline vs oracle")


def test_host_pipeline_repeated_calls_reuse_buffers():
    """Two calls in a row on new inputs: the second call's copy-in must not
    overtake the first call's compute (the staging buffers are shared)."""
    moe = _moe()
    T, d, F, E, k = 2048, 512, 512, 8, 2
    dev = "cuda"
    outs = []
    hl = moe.HostLayer(T, d, E, F, k, torch.bfloat16, dev, logits_given=True, chunks=4)
    problems = [_problem(T, d, F, E, k, torch.bfloat16, seed=s) for s in (1, 2)]
    W1, W3, W2 = (t.to(dev) for t in problems[0][1:4])
    hosts = [(p[0].pin_memory(), p[5].pin_memory()) for p in problems]
    for xh, lh in hosts:
        outs.append(hl(xh, W1, W3, W2, logits_host=lh))
    torch.cuda.current_stream().synchronize()
    for (xh, lh), o in zip(hosts, outs):
        ref = moe.moe_layer_fwd(xh.to(dev), k, W1, W3, W2, logits=lh.to(dev))
        assert torch.equal(o, ref.out.cpu())


def test_host_pipeline_rejects_bad_arguments():
    moe = _moe()
    hl = moe.HostLayer(64, 128, 4, 128, 2, torch.bfloat16, "cuda", logits_given=True, chunks=2)
    W = torch.zeros(4, 128, 128, dtype=torch.bfloat16, device="cuda")
    xh = torch.zeros(64, 128, dtype=torch.bfloat16).pin_memory()
    with pytest.raises(ValueError):
        hl(xh, W, W, W)                      # logits missing
    with pytest.raises(ValueError):
        moe.HostLayer(64, 128, 4, 128, 2, torch.bfloat16, "cuda", logits_given=True, chunks=65)


@pytest.mark.slow
def test_host_pipeline_full_size():
    """The 64-expert top-8 OLMoE-shaped workload (T=16384, d=2048, F=1024)
    in 8 slices: bit-identical to the device-resident call."""
    moe = _moe()
    wl = WORKLOADS["olmoe_1b7b"]
    inp = make_inputs(wl, "cuda")
    ref = moe.moe_layer_fwd(inp["x"], wl.k, inp["W1"], inp["W3"], inp["W2"], Wr=inp["Wr"])
    hl = moe.HostLayer(wl.T, wl.d, wl.E, wl.F, wl.k, wl.torch_dtype, "cuda",
                       logits_given=False, chunks=8)
    out = hl(inp["x"].cpu().pin_memory(), inp["W1"], inp["W3"], inp["W2"], Wr=inp["Wr"])
    torch.cuda.current_stream().synchronize()
    assert moe.moe_get_status() == 0
    assert torch.equal(out, ref.out.cpu())
    assert torch.equal(hl.res.idx.cpu(), ref.idx.cpu())


@pytest.mark.parametrize("chunks", [1, 3, 5])
def test_mxfp8_host_pipeline_matches_device_call(chunks):
    moe = _moe()
    T, d, F, E, k = 700, 256, 256, 8, 2
    x, W1, W3, W2, Wr, lg = _problem(T, d, F, E, k, torch.bfloat16, seed=31 + chunks)
    dev = "cuda"
    w = moe.mxfp8_quantize_weights(W1.to(dev), W3.to(dev), W2.to(dev))
    ref = moe.moe_layer_fwd_mxfp8(x.to(dev), k, w, logits=lg.to(dev))
    hl = moe.HostLayerMxfp8(T, d, E, F, k, dev, logits_given=True, chunks=chunks)
    out = hl(x.pin_memory(), w, logits_host=lg.pin_memory())
    torch.cuda.current_stream().synchronize()
    assert moe.moe_get_status() == 0
    assert torch.equal(out, ref.out.cpu())
    assert torch.equal(hl.res.idx.cpu(), ref.idx.cpu())
    _check_slices(hl.res.slot.cpu().numpy(), T, k, chunks)
