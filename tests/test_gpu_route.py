"""Route step on the GPU against the oracle: indices, counts, offsets, slots
and tile offsets bit-exact; gates within the fp32 softmax bound."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from dropless_top_mixture_b200.workloads import WORKLOADS, adversarial_logits, make_inputs
from tests._util import gate_tolerance, route_equals_oracle_own_logits, router_logits_checked

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
    # a probability below fp32's normal range (logits more than ~87 below the
    # token's maximum) underflows in the fp32 exponential: absolute there
    tiny = np.abs(g - gate) <= 2.0 ** -120
    assert np.all((err <= tol) | tiny), f"gate rel err {err[~tiny].max():.3e}"


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
    route_equals_oracle_own_logits(r, x, Wr, k, E)


@pytest.mark.parametrize("case", ["tied_experts", "near_tied_experts", "zero_tokens",
                                  "duplicate_tokens", "large_magnitudes"])
@pytest.mark.parametrize("T,d,E,k", [(300, 256, 64, 8), (129, 512, 128, 4), (70, 128, 300, 8)])
def test_bf16_router_ties_route_as_oracle(case, T, d, E, k):
    """bf16 router inputs built to put logits at or near exact ties: the GPU
    must still route exactly as the oracle does on its own fixed-order
    logits (ties to the lower expert index)."""
    moe = _moe()
    g = torch.Generator().manual_seed(T + d + E)
    x = torch.randn(T, d, generator=g)
    Wr = torch.randn(E, d, generator=g) * 0.02
    if case == "tied_experts":
        Wr[5] = Wr[2]
        Wr[E - 1] = Wr[0]
        Wr[7] = Wr[3]
        Wr[9] = Wr[3]
    elif case == "near_tied_experts":
        for a, b in ((5, 2), (E - 1, 0), (7, 3)):
            Wr[a] = Wr[b]
            Wr[a, (a * 7) % d] += 2.0 ** -12   # logits differ by x_j 2^-12 (one product)
    elif case == "zero_tokens":
        x[::3] = 0.0                           # every logit of those tokens is zero
    elif case == "duplicate_tokens":
        x[1::2] = x[0::2][: T // 2]
    elif case == "large_magnitudes":
        x *= 64.0
        x[:, :8] *= 1024.0
    x, Wr = x.to(torch.bfloat16), Wr.to(torch.bfloat16)
    r = moe.moe_route(k, x=x.cuda(), Wr=Wr.cuda(), keep_logits=True)
    torch.cuda.synchronize()
    assert moe.moe_get_status() == 0
    lg = router_logits_checked(r.logits.cpu().numpy(), x, Wr, tight=1e9)
    _check_route(r, lg, k, E)
    route_equals_oracle_own_logits(r, x, Wr, k, E)


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
    the tensor cores with the fixed-order recomputation of the undecided
    experts, against the oracle routing on its own fixed-order fp32 logits:
    idx, counts, offsets, slot and tile offsets identical for all tokens."""
    moe = _moe()
    w = WORKLOADS["olmoe_1b7b"]
    inp = make_inputs(w, "cpu", weights=False)
    x, Wr = inp["x"], inp["Wr"]
    r = moe.moe_route(w.k, x=x.cuda(), Wr=Wr.cuda(), keep_logits=True)
    torch.cuda.synchronize()
    assert moe.moe_get_status() == 0
    router_logits_checked(r.logits.cpu().numpy(), x, Wr)
    n_exact = route_equals_oracle_own_logits(r, x, Wr, w.k, w.E)
    print(f"\nlogits in the oracle's bits: {n_exact} of {w.T * w.E} "
          f"({n_exact / w.T:.2f} per token)")
