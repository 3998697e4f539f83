"""Route step on the GPU against the oracle: indices, counts, offsets, slots
and tile offsets bit-exact; gates within the fp32 softmax bound."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from dropless_top_mixture_b200.workloads import WORKLOADS, adversarial_logits, make_inputs
from tests._util import gate_tolerance, router_logits_checked

pytestmark = pytest.mark.gpu


def _moe():
    from dropless_top_mixture_b200 import moe
    return moe


def _check_route(r, lg_np, k, E, renorm=False):
    idx, gate, _ = O.route(lg_np, k, renorm)
    meta = O.routing_metadata(idx, E)
    g_idx = r.idx.cpu().numpy()
    assert np.array_equal(g_idx, idx), "top-k indices differ"
    assert np.array_equal(r.counts.cpu().numpy(), meta["counts"])
    assert np.array_equal(r.offsets.cpu().numpy(), meta["offsets"])
    assert np.array_equal(r.slot.cpu().numpy(), meta["slot"])
    assert np.array_equal(r.tile_offsets.cpu().numpy(), meta["tile_offsets"])
    g = r.gate.cpu().numpy().astype(np.float64)
    tol = gate_tolerance(lg_np, idx, renorm)
    err = np.abs(g - gate) / np.maximum(np.abs(gate), 1e-300)
    assert np.all((err <= tol) | (gate == 0)), f"gate rel err {err.max():.3e}"


@pytest.mark.parametrize("kind", ["normal", "dups", "constant", "signed_zero"])
@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (7, 8, 8), (37, 33, 5), (300, 64, 8), (1000, 128, 4),
                                   (257, 384, 8), (64, 512, 32), (50, 1, 1),
                                   # small batches: the lanes per token double up to
                                   # 16 while each keeps >= 8 logits
                                   (40, 16, 3), (129, 20, 6), (65, 32, 32), (70, 52, 7),
                                   (100, 80, 8), (70, 160, 8), (90, 256, 16), (33, 500, 9),
                                   (20, 12, 4), (30, 129, 8)])
def test_route_from_logits_bitexact(kind, T, E, k):
    moe = _moe()
    lg = adversarial_logits(T, E, kind, seed=T + E)
    r = moe.moe_route(k, logits=lg.cuda())
    _check_route(r, lg.numpy(), k, E)


@pytest.mark.parametrize("T,E,k", [(160_000, 12, 2), (160_000, 20, 6), (160_000, 30, 8),
                                   (80_000, 40, 8), (80_000, 60, 8), (40_000, 80, 8),
                                   (40_000, 120, 4), (20_000, 160, 8), (20_000, 240, 8)])
def test_route_large_batches(T, E, k):
    """Batches large enough that the top-k keeps the fewest lanes per token
    (up to 32 logits per lane; 148 SMs x 1024 threads reached)."""
    moe = _moe()
    lg = adversarial_logits(T, E, "dups", seed=T % 1000 + E)
    r = moe.moe_route(k, logits=lg.cuda())
    _check_route(r, lg.numpy(), k, E)


def test_route_logits_not_16_byte_aligned():
    """Logits whose rows are not 16-byte aligned take the scalar loads."""
    moe = _moe()
    T, E, k = 95, 64, 8
    lg = adversarial_logits(T, E, "dups", seed=3)
    flat = torch.empty(T * E + 1, device="cuda")
    view = flat[1:].view(T, E)
    view.copy_(lg.cuda())
    assert view.data_ptr() % 16 != 0
    r = moe.moe_route(k, logits=view)
    _check_route(r, lg.numpy(), k, E)


def test_route_renorm():
    moe = _moe()
    lg = adversarial_logits(333, 64, "normal", seed=5)
    r = moe.moe_route(8, logits=lg.cuda(), renorm=True)
    _check_route(r, lg.numpy(), 8, 64, renorm=True)


def test_route_skewed_with_empty_experts():
    moe = _moe()
    T, E, k = 2000, 40, 3
    lg = adversarial_logits(T, E, "normal", seed=11)
    lg[:, 10:30] -= 50.0  # experts 10..29 never chosen
    lg[:, 0] += 5.0       # expert 0 always chosen (> 128 rows: several tiles)
    r = moe.moe_route(k, logits=lg.cuda())
    _check_route(r, lg.numpy(), k, E)
    assert (r.counts.cpu().numpy()[10:30] == 0).all()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("T,d,E,k", [(5, 128, 8, 2), (130, 256, 64, 8), (77, 128, 33, 3),
                                     (64, 384, 17, 4), (300, 256, 100, 6), (257, 128, 300, 8),
                                     (129, 512, 128, 4), (3, 128, 1, 1), (1, 256, 512, 32)])
def test_router_logits_match_oracle(dtype, T, d, E, k):
    """fp32: the oracle's fixed-order chains bit for bit; bf16 (tensor cores):
    within the fp32 summation bound; routing on the GPU's logits bit-exact."""
    moe = _moe()
    g = torch.Generator().manual_seed(T * d + E)
    x = torch.randn(T, d, generator=g).to(dtype)
    Wr = (torch.randn(E, d, generator=g) * 0.02).to(dtype)
    r = moe.moe_route(k, x=x.cuda(), Wr=Wr.cuda(), keep_logits=True)
    lg = router_logits_checked(r.logits.cpu().numpy(), x, Wr)
    _check_route(r, lg, k, E)


def test_route_empty_batch():
    moe = _moe()
    lg = torch.zeros((0, 16), device="cuda")
    r = moe.moe_route(4, logits=lg)
    assert (r.counts.cpu() == 0).all() and (r.offsets.cpu() == 0).all()


@pytest.mark.slow
@pytest.mark.parametrize("name", ["tiny_fp32", "olmoe_1b7b", "sweep_e8", "sweep_e128_zipf",
                                  "fine_grained_e384"])
def test_route_full_size_workloads(name):
    moe = _moe()
    w = WORKLOADS[name]
    inp = make_inputs(w, "cpu", weights=False)
    if w.logits == "router":
        r = moe.moe_route(w.k, x=inp["x"].cuda(), Wr=inp["Wr"].cuda(), keep_logits=True)
        lg = router_logits_checked(r.logits.cpu().numpy(), inp["x"], inp["Wr"])
    else:
        r = moe.moe_route(w.k, logits=inp["logits"].cuda())
        lg = inp["logits"].numpy()
    _check_route(r, lg, w.k, w.E)
    assert moe.moe_get_status() == 0


@pytest.mark.slow
def test_bf16_router_routing_against_oracle_logits_full_size():
    """OLMoE-shaped layer (T=16384, d=2048, E=64, top-8), router from x·Wr on
    the tensor cores, against the oracle routing on its own fixed-order fp32
    logits: the indices must agree on every token except where two adjacent
    logits among the oracle's top k + 1 lie within twice the largest
    difference between the token's two logit vectors (a near-tie the two
    roundings may break differently); there the GPU's choices must still
    reach no lower than that band."""
    moe = _moe()
    w = WORKLOADS["olmoe_1b7b"]
    inp = make_inputs(w, "cpu", weights=False)
    x, Wr = inp["x"], inp["Wr"]
    r = moe.moe_route(w.k, x=x.cuda(), Wr=Wr.cuda(), keep_logits=True)
    got_lg = router_logits_checked(r.logits.cpu().numpy(), x, Wr).astype(np.float64)
    ref_lg = O.router_logits(x, Wr).astype(np.float64)
    idx_ref, _, _ = O.route(ref_lg.astype(np.float32), w.k)
    idx_gpu = r.idx.cpu().numpy()
    # the two logit vectors of a token differ by at most delta (checked above
    # against the derived bound), so their orders can only differ between
    # logits closer than 2 delta
    srt = np.sort(ref_lg, axis=1)[:, ::-1]
    kth = srt[:, w.k - 1]
    band = 2.0 * np.abs(got_lg - ref_lg).max(axis=1)
    # a near-tie anywhere among the top k + 1 can reorder or swap indices
    near_tie = (np.diff(-srt[:, :w.k + 1], axis=1) <= band[:, None]).any(axis=1)
    same = (idx_gpu == idx_ref).all(axis=1)
    assert np.all(same | near_tie), f"{int((~same & ~near_tie).sum())} tokens differ without a near-tie"
    for t in np.nonzero(~same)[0]:
        lo = kth[t] - band[t]
        # every expert the GPU chose is at least as large as the band's bottom
        assert np.all(ref_lg[t, idx_gpu[t]] >= lo), t
    print(f"\nnear-ties (adjacent top-{w.k + 1} logits within 2 delta): {int(near_tie.sum())} of {w.T} tokens; "
          f"tokens whose index list differs: {int((~same).sum())}")
