"""Backward of the expert layer on the GPU against the oracle: the grouped
SwiGLU backward (dH with the pairwise SwiGLU-backward epilogue, dX, and the
variable-K weight gradients) and the whole-layer backward, on small shapes
with ragged expert segments and empty experts, then the fine-grained
workload at full size on sampled tokens and experts."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from dropless_top_mixture_b200.workloads import WORKLOADS, adversarial_logits, make_inputs
from tests._util import assert_close_layer, assert_close_scaled, np64, router_logits_checked

pytestmark = pytest.mark.gpu


def _moe():
    from dropless_top_mixture_b200 import moe
    return moe


def _problem(T, d, F, E, k, seed, skew=True):
    g = torch.Generator().manual_seed(seed)
    bf = torch.bfloat16
    x = torch.randn(T, d, generator=g).to(bf)
    W1 = (torch.randn(E, F, d, generator=g) * d ** -0.5).to(bf)
    W3 = (torch.randn(E, F, d, generator=g) * d ** -0.5).to(bf)
    W2 = (torch.randn(E, d, F, generator=g) * F ** -0.5).to(bf)
    dOut = torch.randn(T, d, generator=g).to(bf)
    lg = adversarial_logits(T, E, "normal", seed=seed).numpy()
    if skew and E >= 4:
        lg[:, 1] -= 40.0   # expert 1 empty
        lg[:, 0] += 3.0    # expert 0 heavy
    return x, W1, W3, W2, dOut, lg


def _check_grads(g, ref, E, what=""):
    assert_close_scaled(np64(g.dW1), ref["dW1"], what + "dW1")
    assert_close_scaled(np64(g.dW3), ref["dW3"], what + "dW3")
    assert_close_scaled(np64(g.dW2), ref["dW2"], what + "dW2")
    counts = np.diff(ref["offsets"])
    for e in range(E):
        if counts[e] == 0:
            assert (g.dW1[e] == 0).all() and (g.dW2[e] == 0).all() and (g.dW3[e] == 0).all()
        else:
            assert_close_scaled(np64(g.dW1[e]), ref["dW1"][e], f"{what}dW1[{e}]")
            assert_close_scaled(np64(g.dW2[e]), ref["dW2"][e], f"{what}dW2[{e}]")


@pytest.mark.parametrize("T,d,F,E,k", [(300, 256, 256, 6, 2), (97, 512, 256, 4, 3),
                                       (700, 256, 512, 16, 4), (33, 256, 256, 5, 2)])
def test_layer_backward_small(T, d, F, E, k):
    moe = _moe()
    x, W1, W3, W2, dOut, lg = _problem(T, d, F, E, k, seed=T + d + F + E)
    dev = "cuda"
    W = [w.to(dev) for w in (W1, W3, W2)]
    fwd = moe.moe_layer_fwd(x.to(dev), k, *W, logits=torch.from_numpy(lg).to(dev), save=True)
    g = moe.moe_layer_bwd(fwd, dOut.to(dev), k, *W)
    torch.cuda.synchronize()
    assert moe.moe_get_status() == 0
    ref = O.moe_layer_bwd(x, dOut, k, W1, W3, W2, lg)
    assert np.array_equal(fwd.offsets.cpu().numpy(), ref["offsets"])
    assert_close_scaled(np64(g.dx), ref["dx"], "dx")
    _check_grads(g, ref, E)


@pytest.mark.parametrize("counts", [[1, 63, 64, 65, 128, 129, 0, 300],
                                    [1, 63, 64, 65, 128, 129, 0, 300, 512, 257]])
def test_expert_backward_ragged_segments(counts):
    """Counts 1, 63, 64, 65, 128, 129, 0 and large experts: K slabs that end
    inside, at, and just past a 64-row boundary; averaging under 128 rows
    per expert (weight gradients in the store-bound form) and over it."""
    moe = _moe()
    d, F = 256, 256
    E = len(counts)
    R = sum(counts)
    g = torch.Generator().manual_seed(77)
    bf = torch.bfloat16
    Xe = torch.randn(R, d, generator=g).to(bf)
    dYe = torch.randn(R, d, generator=g).to(bf)
    W1 = (torch.randn(E, F, d, generator=g) * d ** -0.5).to(bf)
    W3 = (torch.randn(E, F, d, generator=g) * d ** -0.5).to(bf)
    W2 = (torch.randn(E, d, F, generator=g) * F ** -0.5).to(bf)
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    # forward pre-activations from the GPU gate/up (they are inputs to the
    # backward, not compared here); the oracle recomputes its own in fp64
    dev = "cuda"
    H, A, B = moe.moe_grouped_gate_up_save(Xe.to(dev), W1.to(dev), W3.to(dev),
                                           torch.from_numpy(offs).to(dev))
    gr = moe.moe_grouped_swiglu_bwd(Xe.to(dev), A, B, H, dYe.to(dev), W1.to(dev), W3.to(dev),
                                    W2.to(dev), torch.from_numpy(offs).to(dev))
    torch.cuda.synchronize()
    assert moe.moe_get_status() == 0
    dXe, dW1, dW3, dW2 = O.expert_ffn_bwd(np64(Xe), offs, np64(W1), np64(W3), np64(W2), np64(dYe))
    assert_close_scaled(np64(gr.dXe), dXe, "dXe")
    ref = dict(dW1=dW1, dW3=dW3, dW2=dW2, offsets=offs)
    _check_grads(gr, ref, E)


def test_backward_deterministic():
    moe = _moe()
    T, d, F, E, k = 400, 256, 256, 8, 2
    x, W1, W3, W2, dOut, lg = _problem(T, d, F, E, k, seed=5)
    W = [w.cuda() for w in (W1, W3, W2)]
    fwd = moe.moe_layer_fwd(x.cuda(), k, *W, logits=torch.from_numpy(lg).cuda(), save=True)
    a = moe.moe_layer_bwd(fwd, dOut.cuda(), k, *W)
    b = moe.moe_layer_bwd(fwd, dOut.cuda(), k, *W)
    for n in ("dx", "dW1", "dW3", "dW2"):
        assert torch.equal(getattr(a, n), getattr(b, n)), n


@pytest.mark.slow
def test_fine_grained_backward_full_size_sampled():
    """T=4096, d=7168, E=384, k=8, F=2048 (34 GB of expert weights): dx on
    sampled tokens, dW1/dW3/dW2 on sampled experts."""
    moe = _moe()
    w = WORKLOADS["fine_grained_e384"]
    inp = make_inputs(w, "cuda")
    fwd = moe.moe_layer_fwd(inp["x"], w.k, inp["W1"], inp["W3"], inp["W2"],
                            logits=inp["logits"], save=True)
    g = moe.moe_layer_bwd(fwd, inp["dOut"], w.k, inp["W1"], inp["W3"], inp["W2"])
    torch.cuda.synchronize()
    assert moe.moe_get_status() == 0
    counts = fwd.counts.cpu().numpy()
    rng = np.random.default_rng(1)
    toks = np.sort(rng.choice(w.T, size=16, replace=False))
    experts = [int(np.argmax(counts)), int(np.argmin(counts))] + list(rng.choice(w.E, 2, replace=False))
    ref = O.moe_layer_bwd_sampled(inp["x"].cpu(), inp["dOut"].cpu(), w.k, inp["W1"], inp["W3"],
                                  inp["W2"], inp["logits"].cpu().numpy(), toks, experts)
    assert np.array_equal(fwd.offsets.cpu().numpy(), ref["offsets"])
    assert_close_layer(np64(g.dx[torch.as_tensor(toks, device="cuda")]), ref["dx"], "dx")
    for e in experts:
        r1, r3, r2 = ref["dW"][e]
        assert_close_scaled(np64(g.dW1[e]), r1, f"dW1[{e}]")
        assert_close_scaled(np64(g.dW3[e]), r3, f"dW3[{e}]")
        assert_close_scaled(np64(g.dW2[e]), r2, f"dW2[{e}]")


@pytest.mark.parametrize("renorm", [False, True])
@pytest.mark.parametrize("router_from_x", [True, False])
def test_layer_backward_with_router(renorm, router_from_x):
    """The whole training backward of the layer: expert path, the gates
    through the softmax (and renorm) with the load-balancing term, and the
    router GEMM backward (dx += dlogits Wr, dWr) when the logits come from
    x and Wr; against the oracle at the layer tolerance."""
    moe = _moe()
    T, d, F, E, k = 384, 256, 256, 8, 2
    x, W1, W3, W2, dOut, lg = _problem(T, d, F, E, k, seed=77, skew=False)
    g = torch.Generator().manual_seed(78)
    Wr = (torch.randn(E, d, generator=g) * 0.05).to(torch.bfloat16)
    dev = "cuda"
    W = [w.to(dev) for w in (W1, W3, W2)]
    kw = dict(Wr=Wr.to(dev)) if router_from_x else dict(logits=torch.from_numpy(lg).to(dev))
    fwd = moe.moe_layer_fwd(x.to(dev), k, *W, renorm=renorm, save=True, **kw)
    gr = moe.moe_layer_bwd(fwd, dOut.to(dev), k, *W, router=True, x=x.to(dev),
                           Wr=kw.get("Wr"), aux_coef=0.01)
    torch.cuda.synchronize()
    assert moe.moe_get_status() == 0
    if router_from_x:  # route both sides on the GPU's logits (checked against the oracle's)
        lg = router_logits_checked(fwd.logits.cpu().numpy(), x, Wr)
    ref = O.moe_layer(x, k, W1, W3, W2, logits=lg, renorm=renorm)
    idx = ref["idx"]
    assert np.array_equal(gr.dgate.shape, (T, k))
    assert np.array_equal(fwd.idx.cpu().numpy(), idx)
    logits = ref["logits"]
    # expert path with the gates held constant (its own oracle), plus the
    # router path
    eb = O.moe_layer_bwd(x, dOut, k, W1, W3, W2, logits) if not renorm else None
    Y = ref["Ye"][ref["slot"]]
    dg = O.gate_grad(np64(dOut), Y)
    dlog = O.router_grad(logits, idx, dg, renorm=renorm, aux_coef=0.01)
    assert_close_layer(np64(gr.dgate), dg, "dgate", max_abs=2e-2 * np.abs(dg).max())
    assert_close_layer(np64(gr.dlogits), dlog, "dlogits", max_abs=2e-2 * np.abs(dlog).max())
    if router_from_x:
        gx, gW = O.router_linear_grad(dlog, x, Wr)
        assert_close_layer(np64(gr.dWr), gW, "dWr", max_abs=2e-2 * np.abs(gW).max())
        if eb is not None:
            want = eb["dx"] + gx
            assert_close_scaled(np64(gr.dx), want, "dx (experts + router)")
    elif eb is not None:
        assert gr.dWr is None
        assert_close_scaled(np64(gr.dx), eb["dx"], "dx (experts only)")
