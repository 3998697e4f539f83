"""Router backward and load-balancing loss (§8(f) f2) on the GPU against the
oracle: gate gradients, the softmax / renorm backward with the aux term,
the router GEMM backward, and the aux loss itself; small ragged shapes,
a whole-layer chain, and the OLMoE-shaped workload at full size."""
import math

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from dropless_top_mixture_b200.workloads import WORKLOADS, make_inputs
from tests._util import assert_close_layer, np64, rel_l2, router_logits_checked

pytestmark = pytest.mark.gpu

U32 = 2.0 ** -24   # fp32 unit roundoff


def _moe():
    from dropless_top_mixture_b200 import moe
    return moe


def _routing(T, E, k, seed, renorm=False):
    lg = np.random.default_rng(seed).normal(size=(T, E)).astype(np.float32)
    idx, gate, _ = O.route(lg, k, renorm)
    meta = O.routing_metadata(idx, E)
    return lg, idx, meta


def _dev(a, dtype=None):
    t = torch.as_tensor(np.ascontiguousarray(a)).cuda()
    return t if dtype is None else t.to(dtype)


def _check_dlogits(got, ref, what):
    # fp32 softmax (expf <= 2 ulp), an fp32 dot product per gate and sums of
    # E terms: relative error of order (d + E) * 2^-24 of the magnitudes
    scale = float(np.abs(ref).max())
    err = float(np.abs(got - ref).max())
    assert err <= 1e-5 * scale + 1e-12, f"{what}: max-abs {err:.3e} (scale {scale:.3e})"
    assert rel_l2(got, ref) <= 1e-5, f"{what}: rel-L2 {rel_l2(got, ref):.3e}"


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("renorm", [False, True])
@pytest.mark.parametrize("aux_coef", [0.0, 0.01])
@pytest.mark.parametrize("T,d,E,k", [(300, 256, 16, 4), (77, 136, 40, 3), (5, 64, 4, 2),
                                     (129, 512, 64, 8)])
def test_router_bwd_matches_oracle(dtype, renorm, aux_coef, T, d, E, k):
    """Same Ye rows and dOut on both sides, so this checks the kernel's
    arithmetic: the gate dot products, the softmax Jacobian, the renorm
    backward and the aux-loss term."""
    moe = _moe()
    lg, idx, meta = _routing(T, E, k, seed=T + E, renorm=renorm)
    R = T * k
    g = torch.Generator().manual_seed(T * 7 + d)
    Ye = torch.randn(R, d, generator=g).to(dtype)
    dOut = torch.randn(T, d, generator=g).to(dtype)
    r = moe.moe_router_bwd(dOut.cuda(), Ye.cuda(), _dev(meta["slot"]), _dev(idx), _dev(lg),
                           _dev(meta["counts"]), renorm=renorm, aux_coef=aux_coef)
    assert moe.moe_get_status() == 0
    Y = np64(Ye)[meta["slot"]]                       # [T, k, d]
    dg_ref = O.gate_grad(np64(dOut), Y)
    # fp32 dot products of d terms: |err| <= gamma_d * sum |dOut * Ye| (x2)
    bound = 2 * d * U32 * np.einsum("td,tjd->tj", np.abs(np64(dOut)), np.abs(Y))
    assert np.all(np.abs(np64(r.dgate) - dg_ref) <= bound + 1e-30)
    ref = O.router_grad(lg, idx, dg_ref, renorm=renorm, aux_coef=aux_coef)
    _check_dlogits(np64(r.dlogits), ref, "dlogits")


def test_router_bwd_aux_only_and_bad_index():
    """dOut = 0 leaves only the aux-loss gradient; an out-of-range slot is
    flagged and skipped, not used as an address."""
    moe = _moe()
    T, d, E, k = 200, 128, 8, 2
    lg, idx, meta = _routing(T, E, k, seed=3)
    Ye = torch.randn(T * k, d, dtype=torch.bfloat16)
    r = moe.moe_router_bwd(torch.zeros(T, d, dtype=torch.bfloat16).cuda(), Ye.cuda(),
                           _dev(meta["slot"]), _dev(idx), _dev(lg), _dev(meta["counts"]),
                           aux_coef=0.5)
    assert np.all(np64(r.dgate) == 0.0)
    ref = O.router_grad(lg, idx, np.zeros((T, k)), aux_coef=0.5)
    _check_dlogits(np64(r.dlogits), ref, "aux-only dlogits")
    bad = meta["slot"].copy()
    bad[3, 1] = T * k + 10
    moe.moe_router_bwd(torch.zeros(T, d, dtype=torch.bfloat16).cuda(), Ye.cuda(), _dev(bad),
                       _dev(idx), _dev(lg), _dev(meta["counts"]))
    assert moe.moe_get_status(clear=True) & moe.MOE_DEVERR_BAD_INDEX
    assert moe.moe_get_status() == 0


@pytest.mark.parametrize("T,E,k", [(1, 4, 2), (1000, 64, 8), (4097, 384, 8), (33, 512, 32)])
def test_aux_loss_matches_oracle(T, E, k):
    moe = _moe()
    lg, idx, meta = _routing(T, E, k, seed=E + T)
    got = float(moe.moe_aux_loss(_dev(lg), _dev(meta["counts"])).item())
    ref = O.aux_loss(lg, idx)
    # per token: softmax in fp32 (a few ulp); sums over up to T tokens and E
    # experts in fp32
    assert abs(got - ref) <= 4 * (T + E + 16) * U32 * ref, (got, ref)


def _linear_case(T, d, E, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    dl = torch.randn(T, E, generator=g) * 1e-2
    x = torch.randn(T, d, generator=g).to(dtype)
    Wr = (torch.randn(E, d, generator=g) * 0.02).to(dtype)
    dx0 = torch.randn(T, d, generator=g).to(dtype)
    return dl, x, Wr, dx0


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T,d,E", [(333, 260, 20), (64, 128, 64), (7, 4, 1), (1500, 2048, 64),
                                   (1000, 512, 20), (4100, 256, 100), (600, 768, 200)])
def test_router_linear_bwd_matches_oracle(dtype, T, d, E):
    """bf16 with d % 256 == 0 runs on the tensor cores with dlogits rounded to
    bf16 once (relative error at most 2^-9 per element, so 2^-9 of the sum of
    |products| more); the rest on the CUDA cores from the fp32 dlogits. The
    fp32 summation term is doubled for the tensor core's own order."""
    moe = _moe()
    dl, x, Wr, dx0 = _linear_case(T, d, E, dtype, seed=T + d + E)
    dx = dx0.cuda().clone()
    _, dWr = moe.moe_router_linear_bwd(dl.cuda(), x.cuda(), Wr.cuda(), dx=dx)
    gx, gW = O.router_linear_grad(dl.double().numpy(), x, Wr)
    bf16 = dtype == torch.bfloat16
    unit = 2.0 ** -8 if bf16 else U32
    dl_round = 2.0 ** -9 if bf16 else 0.0
    # dx: one rounding of (dx0 + fp32 sum of E products)
    want = np64(dx0) + gx
    sp = np.abs(dl.double().numpy()) @ np.abs(np64(Wr))
    sx = np.abs(np64(dx0)) + sp
    assert np.all(np.abs(np64(dx) - want) <=
                  unit * np.abs(want) + 2 * (E + 2) * U32 * sx + dl_round * sp + 1e-30)
    # dWr: one rounding of a two-level fp32 sum over the T tokens
    sW = np.abs(dl.double().numpy()).T @ np.abs(np64(x))
    assert np.all(np.abs(np64(dWr) - gW) <=
                  unit * np.abs(gW) + 2 * (T + 2) * U32 * sW + dl_round * sW + 1e-30)


def test_router_backward_chain_through_the_layer():
    """route -> dispatch -> grouped SwiGLU -> the router backward and router
    GEMM backward on the GPU, against the oracle layer's own (unrounded)
    expert outputs: the layer-level tolerance."""
    moe = _moe()
    T, d, E, k, F = 512, 256, 16, 4, 256
    g = torch.Generator().manual_seed(21)
    x = torch.randn(T, d, generator=g).to(torch.bfloat16)
    Wr = (torch.randn(E, d, generator=g) * 0.05).to(torch.bfloat16)
    W1 = (torch.randn(E, F, d, generator=g) * d ** -0.5).to(torch.bfloat16)
    W3 = (torch.randn(E, F, d, generator=g) * d ** -0.5).to(torch.bfloat16)
    W2 = (torch.randn(E, d, F, generator=g) * F ** -0.5).to(torch.bfloat16)
    dOut = torch.randn(T, d, generator=g).to(torch.bfloat16)
    xd, Wrd = x.cuda(), Wr.cuda()
    rt = moe.moe_route(k, x=xd, Wr=Wrd, keep_logits=True)
    Xe = moe.moe_dispatch(xd, rt.slot)
    _, Ye = moe.moe_grouped_swiglu(Xe, W1.cuda(), W3.cuda(), W2.cuda(), rt.offsets)
    r = moe.moe_router_bwd(dOut.cuda(), Ye, rt.slot, rt.idx, rt.logits, rt.counts,
                           aux_coef=0.01)
    dx = torch.zeros(T, d, dtype=torch.bfloat16, device="cuda")
    _, dWr = moe.moe_router_linear_bwd(r.dlogits, xd, Wrd, dx=dx)
    assert moe.moe_get_status() == 0
    lg = router_logits_checked(rt.logits.cpu().numpy(), x, Wr)
    ref = O.moe_layer(x, k, W1, W3, W2, logits=lg)
    idx = ref["idx"]
    assert np.array_equal(rt.idx.cpu().numpy(), idx)
    Y = ref["Ye"][ref["slot"]]
    dlog = O.router_grad(ref["logits"], idx, O.gate_grad(np64(dOut), Y), aux_coef=0.01)
    gx, gW = O.router_linear_grad(dlog, x, Wr)
    assert_close_layer(np64(r.dlogits), dlog, "dlogits", max_abs=2e-2 * np.abs(dlog).max())
    assert_close_layer(np64(dx), gx, "dx (router)", max_abs=2e-2 * np.abs(gx).max())
    assert_close_layer(np64(dWr), gW, "dWr", max_abs=2e-2 * np.abs(gW).max())


def test_router_backward_deterministic():
    moe = _moe()
    T, d, E, k = 700, 512, 32, 4
    lg, idx, meta = _routing(T, E, k, seed=9)
    Ye = torch.randn(T * k, d).to(torch.bfloat16).cuda()
    dOut = torch.randn(T, d).to(torch.bfloat16).cuda()
    x = torch.randn(T, d).to(torch.bfloat16).cuda()
    args = (dOut, Ye, _dev(meta["slot"]), _dev(idx), _dev(lg), _dev(meta["counts"]))
    a = moe.moe_router_bwd(*args, aux_coef=0.01)
    b = moe.moe_router_bwd(*args, aux_coef=0.01)
    assert torch.equal(a.dlogits, b.dlogits) and torch.equal(a.dgate, b.dgate)
    Wr = torch.randn(E, d).to(torch.bfloat16).cuda()
    _, w1 = moe.moe_router_linear_bwd(a.dlogits, x, Wr)
    _, w2 = moe.moe_router_linear_bwd(a.dlogits, x, Wr)
    assert torch.equal(w1, w2)
    l1 = moe.moe_aux_loss(_dev(lg), _dev(meta["counts"]))
    l2 = moe.moe_aux_loss(_dev(lg), _dev(meta["counts"]))
    assert torch.equal(l1, l2)


@pytest.mark.slow
def test_router_backward_full_size_olmoe():
    """The OLMoE-shaped layer (T=16384, d=2048, E=64, k=8) in the launch
    configuration the layer uses: dlogits on 64 sampled tokens and dWr in
    full against the oracle fed the GPU's own Ye rows, the aux loss in full."""
    moe = _moe()
    w = WORKLOADS["olmoe_1b7b"]
    inp = make_inputs(w, "cuda")
    x, Wr = inp["x"], inp["Wr"]
    T, d, E, k = w.T, w.d, w.E, w.k
    rt = moe.moe_route(k, x=x, Wr=Wr, keep_logits=True)
    Xe = moe.moe_dispatch(x, rt.slot)
    _, Ye = moe.moe_grouped_swiglu(Xe, inp["W1"], inp["W3"], inp["W2"], rt.offsets)
    dOut = torch.randn(T, d, generator=torch.Generator(device="cuda").manual_seed(1),
                       device="cuda").to(torch.bfloat16)
    r = moe.moe_router_bwd(dOut, Ye, rt.slot, rt.idx, rt.logits, rt.counts, aux_coef=0.01)
    _, dWr = moe.moe_router_linear_bwd(r.dlogits, x, Wr)
    aux = float(moe.moe_aux_loss(rt.logits, rt.counts).item())
    assert moe.moe_get_status() == 0
    lg = rt.logits.cpu().numpy()
    idx = rt.idx.cpu().numpy()
    slot = rt.slot.cpu().numpy()
    assert abs(aux - O.aux_loss(lg, idx)) <= 4 * (T + E + 16) * U32 * O.aux_loss(lg, idx)
    toks = np.sort(np.random.default_rng(0).choice(T, size=64, replace=False))
    Y = np64(Ye[torch.as_tensor(slot[toks].ravel(), device="cuda")]).reshape(64, k, d)
    dg = O.gate_grad(np64(dOut[torch.as_tensor(toks, device="cuda")]), Y)
    # the aux term needs the whole batch's counts: add it to the sampled rows
    p = O.softmax_fp64(lg[toks])
    f = np.bincount(idx.ravel(), minlength=E) / T
    ref = O.router_grad(lg[toks], idx[toks], dg)
    dp_aux = 0.01 * E * f / T
    ref += p * (dp_aux - (p * dp_aux).sum(axis=1, keepdims=True))
    _check_dlogits(np64(r.dlogits[torch.as_tensor(toks, device="cuda")]), ref, "dlogits sample")
    gW = np64(r.dlogits).T @ np64(x)
    sW = np.abs(np64(r.dlogits)).T @ np.abs(np64(x))
    # tensor-core path: dlogits rounded to bf16 (2^-9), fp32 sums in two levels
    assert np.all(np.abs(np64(dWr) - gW) <=
                  2.0 ** -8 * np.abs(gW) + (2 * (T + 2) * U32 + 2.0 ** -9) * sW)
