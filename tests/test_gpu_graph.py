"""The library's entry points are stream-ordered launches with no host
synchronisation and no allocation, so a whole layer step can be captured in
a CUDA graph and replayed. Replays must give the same bits as eager calls on
the same inputs, also after new inputs are copied into the captured buffers
(the graph reads the live buffers, not the values seen at capture)."""
import pytest
import torch

from dropless_top_mixture_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def _moe():
    from dropless_top_mixture_b200 import moe
    return moe


def _capture(fn):
    """Warm fn on a side stream, then capture one call into a graph."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def _same(a, b, what):
    assert torch.equal(a, b), what


@pytest.mark.parametrize("router", [True, False])
def test_layer_fwd_graph_replay_matches_eager(router):
    moe = _moe()
    w = WORKLOADS["olmoe_1b7b"].scaled(name="graph", T=700, d=256, E=16, k=4, F=256)
    inp = make_inputs(w, "cuda")
    x = inp["x"].clone()
    lg = None if router else torch.randn((w.T, w.E), device="cuda")
    kw = dict(Wr=inp["Wr"]) if router else dict(logits=lg)
    out = moe.moe_layer_fwd(x, w.k, inp["W1"], inp["W3"], inp["W2"], **kw)
    g = _capture(lambda: moe.moe_layer_fwd(x, w.k, inp["W1"], inp["W3"], inp["W2"], out=out, **kw))
    for seed in (1, 2):
        gen = torch.Generator(device="cuda").manual_seed(seed)
        x.copy_(torch.randn(x.shape, device="cuda", generator=gen).to(x.dtype))
        if lg is not None:
            lg.copy_(torch.randn(lg.shape, device="cuda", generator=gen))
        g.replay()
        torch.cuda.synchronize()
        ref = moe.moe_layer_fwd(x, w.k, inp["W1"], inp["W3"], inp["W2"], **kw)
        torch.cuda.synchronize()
        for f in ("out", "idx", "gate", "slot", "counts", "offsets"):
            _same(getattr(out, f), getattr(ref, f), f"{f} after replay {seed}")
    assert moe.moe_get_status() == 0


def test_layer_fwd_mxfp8_graph_replay_matches_eager():
    moe = _moe()
    w = WORKLOADS["mxfp8_e128"].scaled(name="graph_mx", T=300, d=256, E=8, k=2, F=256)
    inp = make_inputs(w, "cuda")
    mw = moe.mxfp8_quantize_weights(inp["W1"], inp["W3"], inp["W2"])
    x = inp["x"].clone()
    lg = inp["logits"].clone()
    out = moe.moe_layer_fwd_mxfp8(x, w.k, mw, logits=lg)
    g = _capture(lambda: moe.moe_layer_fwd_mxfp8(x, w.k, mw, logits=lg, out=out))
    gen = torch.Generator(device="cuda").manual_seed(3)
    x.copy_(torch.randn(x.shape, device="cuda", generator=gen).to(x.dtype))
    lg.copy_(torch.randn(lg.shape, device="cuda", generator=gen))
    g.replay()
    torch.cuda.synchronize()
    ref = moe.moe_layer_fwd_mxfp8(x, w.k, mw, logits=lg)
    torch.cuda.synchronize()
    for f in ("out", "idx", "slot"):
        _same(getattr(out, f), getattr(ref, f), f)
    assert moe.moe_get_status() == 0


def test_layer_bwd_graph_replay_matches_eager():
    moe = _moe()
    w = WORKLOADS["olmoe_1b7b"].scaled(name="graph_bwd", T=400, d=256, E=8, k=2, F=256,
                                       backward=True)
    inp = make_inputs(w, "cuda")
    W1, W3, W2, Wr = inp["W1"], inp["W3"], inp["W2"], inp["Wr"]
    x, dOut = inp["x"].clone(), inp["dOut"].clone()
    fwd = moe.moe_layer_fwd(x, w.k, W1, W3, W2, Wr=Wr, save=True)
    grads = moe.moe_layer_bwd(fwd, dOut, w.k, W1, W3, W2, router=True, x=x, Wr=Wr,
                              aux_coef=0.01)

    def step():
        moe.moe_layer_fwd(x, w.k, W1, W3, W2, Wr=Wr, save=True, out=fwd)
        moe.moe_layer_bwd(fwd, dOut, w.k, W1, W3, W2, out=grads, router=True, x=x, Wr=Wr,
                          aux_coef=0.01)

    g = _capture(step)
    gen = torch.Generator(device="cuda").manual_seed(4)
    dOut.copy_(torch.randn(dOut.shape, device="cuda", generator=gen).to(dOut.dtype))
    g.replay()
    torch.cuda.synchronize()
    f2 = moe.moe_layer_fwd(x, w.k, W1, W3, W2, Wr=Wr, save=True)
    r2 = moe.moe_layer_bwd(f2, dOut, w.k, W1, W3, W2, router=True, x=x, Wr=Wr, aux_coef=0.01)
    torch.cuda.synchronize()
    for f in ("dx", "dW1", "dW3", "dW2", "dlogits", "dWr"):
        _same(getattr(grads, f), getattr(r2, f), f)
    assert moe.moe_get_status() == 0
