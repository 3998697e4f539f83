"""Pins for the CPU oracle: each check ties the oracle to something other than
itself — brute force, a closed form, an invariant, or a library routine
(torch) computing the same mathematical object a different way."""
import itertools
import math

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from dropless_top_mixture_b200.workloads import (WORKLOADS, adversarial_logits, make_inputs)


# ---------------------------------------------------------------- router logits

def _bf16(shape, seed, std=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * std).to(torch.bfloat16)


def test_router_logits_bf16_matches_unfused_fp32_sum():
    # bf16 x bf16 products are exact in fp32, so each quarter's fmaf chain
    # equals the sequential fp32 sum of its exact products (numpy here); the
    # four quarter sums are then added in order.
    x = _bf16((37, 96), 1)
    W = _bf16((11, 96), 2, 0.02)
    got = O.router_logits(x, W)
    xf = x.float().numpy()
    wf = W.float().numpy()
    total = None
    for q in range(4):
        acc = np.zeros((37, 11), dtype=np.float32)
        for j in range(24 * q, 24 * q + 24):
            acc = (acc + np.outer(xf[:, j], wf[:, j]).astype(np.float32)).astype(np.float32)
        total = acc if total is None else (total + acc).astype(np.float32)
    assert np.array_equal(got.view(np.uint32), total.view(np.uint32))


def test_router_logits_quarter_order_closed_form():
    # products [2^24, 0, 1, 1 | -2^24, 0, 0, 0] (d = 8, quarters of 2): a
    # single sequential chain loses both 1s against 2^24 and gives 0; the
    # quarter chains give (2^24 + 2) - 2^24 = 2 exactly
    x = torch.tensor([[4096.0, 0, 1, 1, 4096.0, 0, 0, 0]], dtype=torch.bfloat16)
    W = torch.tensor([[4096.0, 0, 1, 1, -4096.0, 0, 0, 0]], dtype=torch.bfloat16)
    assert O.router_logits(x, W)[0, 0] == 2.0
    assert O.router_logits(x.float(), W.float())[0, 0] == 2.0


def test_router_logits_error_bound_vs_fp64():
    # Four chains of d/4 terms and three adds: the error is at most
    # gamma_{d/4+3} * sum|x_j w_j|.
    x = torch.randn(64, 128, generator=torch.Generator().manual_seed(3))
    W = torch.randn(8, 128, generator=torch.Generator().manual_seed(4)) * 0.02
    got = O.router_logits(x, W).astype(np.float64)
    ref = x.double().numpy() @ W.double().numpy().T
    absdot = np.abs(x.double().numpy()) @ np.abs(W.double().numpy()).T
    u = 2.0 ** -24
    n = 128 // 4 + 3
    gamma = n * u / (1 - n * u)
    assert np.all(np.abs(got - ref) <= gamma * absdot + 1e-30)


def test_router_logits_one_hot_picks_weight_column():
    W = _bf16((5, 64), 7)
    x = torch.zeros(64, 64, dtype=torch.bfloat16)
    x[torch.arange(64), torch.arange(64)] = 1.0
    got = O.router_logits(x, W)
    assert np.array_equal(got, W.float().numpy().T)


def test_router_logits_fp32_small_integers_exact():
    g = torch.Generator().manual_seed(9)
    x = torch.randint(-8, 8, (10, 52), generator=g).float()
    W = torch.randint(-8, 8, (6, 52), generator=g).float()
    got = O.router_logits(x, W)
    assert np.array_equal(got, (x.double() @ W.double().T).float().numpy())


# ---------------------------------------------------------------- softmax + top-k

def _brute_topk(row, k):
    keyed = sorted(range(len(row)), key=lambda e: (-float(row[e]), e))
    return keyed[:k]


@pytest.mark.parametrize("kind", ["constant", "dups", "signed_zero", "normal"])
@pytest.mark.parametrize("E,k", [(1, 1), (8, 2), (8, 8), (33, 5), (64, 8)])
def test_topk_matches_brute_force(kind, E, k):
    lg = adversarial_logits(40, E, kind, seed=E * 10 + k).numpy()
    idx = O.topk_select(lg, k)
    for t in range(lg.shape[0]):
        assert list(idx[t]) == _brute_topk(lg[t], k)


def test_topk_matches_torch_topk_without_ties():
    lg = torch.randn(200, 64, generator=torch.Generator().manual_seed(5))
    assert len(set(lg.flatten().tolist())) == lg.numel()
    v, i = torch.topk(lg, 8, dim=1, largest=True, sorted=True)
    assert np.array_equal(O.topk_select(lg.numpy(), 8), i.numpy())


def test_constant_logits_closed_form():
    E, k = 16, 4
    idx, gate, probs = O.route(np.full((3, E), 1.5, np.float32), k)
    assert (idx == np.arange(k)).all()
    assert np.allclose(gate, 1.0 / E, rtol=0, atol=1e-15)


def test_nan_logit_ranks_last():
    lg = np.array([[np.nan, -100.0, 3.0, -np.inf]], np.float32)
    assert list(O.topk_select(lg, 4)[0]) == [2, 1, 0, 3]


def test_softmax_matches_torch():
    lg = torch.randn(50, 40, generator=torch.Generator().manual_seed(6)) * 3
    p = O.softmax_fp64(lg.numpy())
    assert np.allclose(p, torch.softmax(lg.double(), dim=1).numpy(), rtol=1e-14, atol=0)


def test_gates_are_probs_of_selected_and_renorm():
    lg = torch.randn(30, 12, generator=torch.Generator().manual_seed(8)).numpy()
    idx, gate, probs = O.route(lg, 3)
    for t in range(30):
        for j in range(3):
            assert gate[t, j] == probs[t, idx[t, j]]
    assert np.all(np.diff(gate, axis=1) <= 0)  # descending
    _, g2, _ = O.route(lg, 3, renorm=True)
    assert np.allclose(g2.sum(1), 1.0, atol=1e-15)
    _, gall, _ = O.route(lg, 12)
    assert np.allclose(gall.sum(1), 1.0, atol=1e-14)


# ---------------------------------------------------------------- routing metadata

def _brute_slots(idx, E):
    T, k = idx.shape
    counts = [0] * E
    for t in range(T):
        for j in range(k):
            counts[idx[t, j]] += 1
    offs = [0]
    for e in range(E):
        offs.append(offs[-1] + counts[e])
    seen = [0] * E
    slot = np.zeros_like(idx)
    for t in range(T):           # token-major walk = stable order
        for j in range(k):
            e = idx[t, j]
            slot[t, j] = offs[e] + seen[e]
            seen[e] += 1
    return counts, offs, slot


@pytest.mark.parametrize("E,k,T", [(8, 2, 64), (33, 5, 50), (128, 4, 300), (3, 3, 7), (1, 1, 5)])
def test_metadata_brute_force_and_invariants(E, k, T):
    lg = adversarial_logits(T, E, "normal", seed=E + T).numpy()
    # skew: make some experts empty
    lg[:, E // 2:] -= 5.0 if E > k + 1 else 0.0
    idx = O.topk_select(lg, k)
    m = O.routing_metadata(idx, E)
    counts, offs, slot = _brute_slots(idx, E)
    assert list(m["counts"]) == counts
    assert list(m["offsets"]) == offs
    assert np.array_equal(m["slot"], slot)
    assert m["counts"].sum() == T * k and m["offsets"][-1] == T * k
    assert np.all(np.diff(m["offsets"]) >= 0)
    assert sorted(m["slot"].reshape(-1).tolist()) == list(range(T * k))
    for e in range(E):  # within an expert, slots increase with t
        rows = [(t, m["slot"][t, j]) for t in range(T) for j in range(k) if idx[t, j] == e]
        assert [s for _, s in rows] == sorted(s for _, s in rows)
    tiles = [(c + 127) // 128 for c in counts]
    assert list(m["tile_offsets"]) == [0] + list(itertools.accumulate(tiles))
    assert all(m["row_token"][m["slot"][t, j]] == t for t in range(T) for j in range(k))


def test_dispatch_is_bitwise_copy_and_combine_identity_experts():
    T, E, k, d = 50, 8, 3, 24
    x = _bf16((T, d), 11)
    lg = adversarial_logits(T, E, "dups", seed=3).numpy()
    idx, gate, _ = O.route(lg, k)
    m = O.routing_metadata(idx, E)
    xb = x.view(torch.int16).numpy()
    Xe = O.dispatch(xb, m["slot"])
    for t in range(T):
        for j in range(k):
            assert np.array_equal(Xe[m["slot"][t, j]], xb[t])
    # identity experts: Ye := Xe gives (sum_j gate) * x
    x64 = x.double().numpy()
    out = O.combine(O.dispatch(x64, m["slot"]), m["slot"], gate)
    assert np.allclose(out, gate.sum(1, keepdims=True) * x64, rtol=1e-14, atol=1e-14)


# ---------------------------------------------------------------- expert FFN / layer

def _torch_swiglu(x, w1, w3, w2):
    return (torch.nn.functional.silu(x @ w1.T) * (x @ w3.T)) @ w2.T


def test_single_expert_top1_is_dense_swiglu():
    T, d, F = 20, 16, 24
    g = torch.Generator().manual_seed(12)
    x = torch.randn(T, d, generator=g, dtype=torch.float64)
    W1 = torch.randn(1, F, d, generator=g, dtype=torch.float64) * 0.3
    W3 = torch.randn(1, F, d, generator=g, dtype=torch.float64) * 0.3
    W2 = torch.randn(1, d, F, generator=g, dtype=torch.float64) * 0.3
    r = O.moe_layer(x, 1, W1, W3, W2, logits=np.zeros((T, 1), np.float32))
    ref = _torch_swiglu(x, W1[0], W3[0], W2[0]).numpy()
    assert np.allclose(r["gate"], 1.0)
    assert np.allclose(r["out"], ref, rtol=1e-12, atol=1e-12)


def test_k_equals_E_is_dense_softmax_mixture():
    T, d, F, E = 9, 8, 12, 5
    g = torch.Generator().manual_seed(13)
    x = torch.randn(T, d, generator=g, dtype=torch.float64)
    W1 = torch.randn(E, F, d, generator=g, dtype=torch.float64) * 0.3
    W3 = torch.randn(E, F, d, generator=g, dtype=torch.float64) * 0.3
    W2 = torch.randn(E, d, F, generator=g, dtype=torch.float64) * 0.3
    lg = torch.randn(T, E, generator=g).numpy()
    r = O.moe_layer(x, E, W1, W3, W2, logits=lg)
    p = torch.softmax(torch.from_numpy(lg).double(), dim=1)
    ref = sum(p[:, e:e + 1] * _torch_swiglu(x, W1[e], W3[e], W2[e]) for e in range(E))
    assert np.allclose(r["out"], ref.numpy(), rtol=1e-12, atol=1e-12)


def test_per_expert_layer_matches_per_token_formula_and_torch_index_add():
    T, d, F, E, k = 33, 16, 24, 6, 2
    g = torch.Generator().manual_seed(14)
    x = torch.randn(T, d, generator=g, dtype=torch.float64)
    W1 = torch.randn(E, F, d, generator=g, dtype=torch.float64) * 0.3
    W3 = torch.randn(E, F, d, generator=g, dtype=torch.float64) * 0.3
    W2 = torch.randn(E, d, F, generator=g, dtype=torch.float64) * 0.3
    lg = torch.randn(T, E, generator=g).numpy()
    lg[:, 4] -= 20  # expert 4 receives nothing
    r = O.moe_layer(x, k, W1, W3, W2, logits=lg)
    assert r["counts"][4] == 0
    per_tok = O.moe_layer_tokens(x, np.arange(T), r["idx"], r["gate"], W1, W3, W2)
    assert np.allclose(r["out"], per_tok, rtol=1e-12, atol=1e-12)
    # the same layer via torch's index_add_ over a hit mask (library routine)
    idx = torch.from_numpy(r["idx"]).long()
    gate = torch.from_numpy(r["gate"])
    ref = torch.zeros(T, d, dtype=torch.float64)
    for e in range(E):
        tok, j = torch.nonzero(idx == e, as_tuple=True)
        if tok.numel():
            y = _torch_swiglu(x[tok], W1[e], W3[e], W2[e]) * gate[tok, j, None]
            ref.index_add_(0, tok, y)
    assert np.allclose(r["out"], ref.numpy(), rtol=1e-12, atol=1e-12)


def test_workload_generator_is_deterministic_and_shaped():
    w = WORKLOADS["tiny_fp32"]
    a = make_inputs(w)
    b = make_inputs(w)
    for key in a:
        assert torch.equal(a[key], b[key])
    assert a["x"].shape == (256, 128) and a["Wr"].shape == (8, 128)
    assert a["W1"].shape == (8, 256, 128) and a["W2"].shape == (8, 128, 256)
    assert a["x"].dtype == torch.float32
    assert abs(a["W1"].std().item() - 0.02) < 0.002


# ---------------------------------------------------------------- E4M3 / MXFP8

ALL = np.arange(256, dtype=np.uint8)


def test_e4m3_decode_matches_torch_float8():
    ref = torch.from_numpy(ALL.copy()).view(torch.float8_e4m3fn).float().numpy()
    got = O.e4m3_decode(ALL)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan].astype(np.float64))
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x08] == 2.0 ** -6


def test_e4m3_roundtrip_every_code():
    vals = O.e4m3_decode(ALL).astype(np.float32)
    ok = ~np.isnan(vals)
    assert np.array_equal(O.e4m3_encode(vals[ok]), ALL[ok])


def test_e4m3_encode_matches_torch_cast_in_range():
    g = torch.Generator().manual_seed(21)
    v = torch.cat([torch.randn(1 << 18, generator=g) * s for s in (1e-3, 0.05, 1.0, 30.0, 150.0)])
    v = v[v.abs() < 464]
    ref = v.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.e4m3_encode(v.numpy()), ref)


def test_e4m3_rounding_and_saturation_closed_forms():
    f = lambda x: int(O.e4m3_encode(np.array([x], np.float32))[0])
    assert f(1.0625) == 0x38          # midpoint of 1.0 / 1.125 -> even
    assert f(1.1875) == 0x3A          # midpoint of 1.125 / 1.25 -> even
    assert f(2.0 ** -10) == 0x00      # half the smallest subnormal -> 0
    assert f(3 * 2.0 ** -10) == 0x02  # midpoint of 1 and 2 units -> even
    for big in (448.0, 460.0, 464.0, 1e6, np.inf):
        assert f(big) == 0x7E and f(-big) == 0xFE
    assert f(-0.0) == 0x80 and f(np.nan) & 0x7F == 0x7F


@pytest.mark.parametrize("mode", ["f32", "e8m0"])
def test_mxfp8_roundtrip_bound_and_zero_block(mode):
    g = torch.Generator().manual_seed(22)
    v = torch.randn(64, 256, generator=g) * torch.logspace(-3, 3, 64).unsqueeze(1)
    v[3, 32:64] = 0.0
    v = v.to(torch.bfloat16).float().numpy()
    q, s = O.mxfp8_quantize(v, mode)
    back = O.mxfp8_dequantize_f32(q, s, mode).astype(np.float64)
    sc = np.repeat(O.mxfp8_scales_to_f32(s, mode).astype(np.float64), 32, axis=1)
    err = np.abs(back - v)
    bound = np.maximum(2.0 ** -4 * np.abs(v), 2.0 ** -10 * sc) * (1 + 2.0 ** -20)
    assert np.all(err <= bound)
    assert np.all(q[3, 32:64] == 0)
    zero_scale = s[3, 1]
    assert (zero_scale == 1.0) if mode == "f32" else (zero_scale == 127)
    amax = np.abs(v.reshape(64, 8, 32)).max(2)
    if mode == "e8m0":
        s32 = O.mxfp8_scales_to_f32(s, mode)
        nz = amax > 0
        # the smallest power of two at or above amax/448
        assert np.all(s32[nz] >= (amax[nz] / np.float32(448)).astype(np.float32))
        assert np.all(s32[nz] / 2 < (amax[nz] / np.float32(448)).astype(np.float32))
        assert np.all(np.abs(O.e4m3_decode(q)).max() <= 448)
    else:
        assert np.all(np.abs(O.e4m3_decode(q.reshape(64, 8, 32))).max(2)[amax > 0] >= 416)


def test_mxfp8_dequantize_bf16_rounds_fp32_product():
    v = torch.randn(4, 64, generator=torch.Generator().manual_seed(23)).numpy()
    q, s = O.mxfp8_quantize(v, "f32")
    b = O.mxfp8_dequantize(q, s, "f32")
    f = torch.from_numpy(O.mxfp8_dequantize_f32(q, s, "f32"))
    assert torch.equal(b, f.to(torch.bfloat16))


# ---------------------------------------------------------------- backward

def _tiny_problem(seed, T=12, d=6, F=8, E=4, k=2):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, d, generator=g, dtype=torch.float64)
    W1 = torch.randn(E, F, d, generator=g, dtype=torch.float64) * 0.5
    W3 = torch.randn(E, F, d, generator=g, dtype=torch.float64) * 0.5
    W2 = torch.randn(E, d, F, generator=g, dtype=torch.float64) * 0.5
    lg = torch.randn(T, E, generator=g).numpy()
    lg[:, E - 1] -= 30.0  # one expert with zero rows
    dOut = torch.randn(T, d, generator=g, dtype=torch.float64)
    return x, W1, W3, W2, lg, dOut


def test_backward_matches_torch_autograd():
    x, W1, W3, W2, lg, dOut = _tiny_problem(31)
    k = 2
    r = O.moe_layer_bwd(x, dOut, k, W1, W3, W2, lg)
    xs = x.clone().requires_grad_(True)
    ws = [w.clone().requires_grad_(True) for w in (W1, W3, W2)]
    idx = torch.from_numpy(r["idx"]).long()
    gate = torch.from_numpy(r["gate"])
    out = torch.zeros_like(x)
    for t in range(x.shape[0]):
        for j in range(k):
            e = int(idx[t, j])
            out[t] = out[t] + gate[t, j] * _torch_swiglu(xs[t:t + 1], ws[0][e], ws[1][e], ws[2][e])[0]
    out.backward(dOut)
    assert np.allclose(r["dx"], xs.grad.numpy(), rtol=1e-11, atol=1e-12)
    for name, w in zip(("dW1", "dW3", "dW2"), ws):
        assert np.allclose(r[name], w.grad.numpy(), rtol=1e-11, atol=1e-12)
    assert np.all(r["dW1"][3] == 0) and np.all(r["dW2"][3] == 0)


def test_backward_finite_differences():
    x, W1, W3, W2, lg, dOut = _tiny_problem(32, T=6, d=4, F=5, E=3, k=2)
    k = 2
    r = O.moe_layer_bwd(x, dOut, k, W1, W3, W2, lg)

    def loss(xv, w1, w3, w2):
        o = O.moe_layer(xv, k, w1, w3, w2, logits=lg)["out"]
        return float((o * dOut.numpy()).sum())

    h = 1e-6
    for (t, j) in [(0, 0), (3, 2), (5, 3)]:
        xp, xm = x.clone(), x.clone()
        xp[t, j] += h
        xm[t, j] -= h
        fd = (loss(xp, W1, W3, W2) - loss(xm, W1, W3, W2)) / (2 * h)
        assert math.isclose(fd, r["dx"][t, j], rel_tol=1e-6, abs_tol=1e-8)
    for (e, a, b) in [(0, 1, 2), (1, 4, 0)]:
        Wp, Wm = W2.clone(), W2.clone()
        Wp[e, b, a] += h
        Wm[e, b, a] -= h
        fd = (loss(x, W1, W3, Wp) - loss(x, W1, W3, Wm)) / (2 * h)
        assert math.isclose(fd, r["dW2"][e, b, a], rel_tol=1e-6, abs_tol=1e-8)
        Wp, Wm = W1.clone(), W1.clone()
        Wp[e, a, b] += h
        Wm[e, a, b] -= h
        fd = (loss(x, Wp, W3, W2) - loss(x, Wm, W3, W2)) / (2 * h)
        assert math.isclose(fd, r["dW1"][e, a, b], rel_tol=1e-6, abs_tol=1e-8)


def test_sampled_backward_matches_full_backward():
    x, W1, W3, W2, lg, dOut = _tiny_problem(33, T=20, d=6, F=8, E=5, k=2)
    full = O.moe_layer_bwd(x, dOut, 2, W1, W3, W2, lg)
    toks = np.array([0, 7, 19])
    smp = O.moe_layer_bwd_sampled(x, dOut, 2, W1, W3, W2, lg, toks, [0, 2, 4])
    assert np.allclose(smp["dx"], full["dx"][toks], rtol=1e-12, atol=1e-13)
    for e in (0, 2, 4):
        for n, g in zip(("dW1", "dW3", "dW2"), smp["dW"][e]):
            assert np.allclose(g, full[n][e], rtol=1e-12, atol=1e-13)
    assert np.all(smp["dW"][4][0] == 0)  # expert 4 has no rows


# ------------------------------------------- f2: router backward, aux loss

def _grid_logits(T, E, seed):
    """Logits on a 2^-10 grid in [-4, 4): exact in fp32, and so are their
    perturbations by 2^-12, so finite differences see the fp32 softmax
    input move by exactly eps."""
    rng = np.random.default_rng(seed)
    return (rng.integers(-4096, 4096, size=(T, E)) / 1024.0).astype(np.float32)


def _expert_rows(x, idx, W1, W3, W2):
    """Y[t, j] = FFN_{idx[t,j]}(x_t), the un-gated expert outputs."""
    T, k = idx.shape
    x64 = O.to64(x)
    Y = np.zeros((T, k, x64.shape[1]))
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            a = O.to64(W1[e]) @ x64[t]
            b = O.to64(W3[e]) @ x64[t]
            Y[t, j] = O.to64(W2[e]) @ (O.silu(a) * b)
    return Y


def test_aux_loss_closed_forms():
    T, E, k = 64, 8, 2
    rng = np.random.default_rng(0)
    # a uniform router gives aux = k whatever the counts (sum_e f_e = k)
    flat = np.zeros((T, E), np.float32)
    assert O.aux_loss(flat, O.topk_select(flat, k)) == pytest.approx(k, rel=1e-12)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    assert O.aux_loss(flat, idx) == pytest.approx(k, rel=1e-12)
    # exactly balanced counts give aux = k whatever the probabilities
    bal = np.array([[(2 * t) % E, (2 * t + 1) % E] for t in range(T)], np.int32)
    assert np.all(np.bincount(bal.ravel(), minlength=E) == T * k // E)
    assert O.aux_loss(rng.normal(size=(T, E)).astype(np.float32), bal) == pytest.approx(k, rel=1e-12)
    # a collapsed router (every token picks the same k experts, probability
    # 1/k on each) gives aux = E
    col = np.zeros((T, E), np.float32)
    col[:, :k] = 60.0
    assert O.aux_loss(col, O.topk_select(col, k)) == pytest.approx(E, rel=1e-12)


def test_gate_grad_finite_differences():
    rng = np.random.default_rng(1)
    T, k, d = 5, 3, 7
    Y = rng.normal(size=(T, k, d))
    dOut = rng.normal(size=(T, d))
    g = rng.random((T, k))
    L = lambda gg: float((dOut * np.einsum("tj,tjd->td", gg, Y)).sum())
    got = O.gate_grad(dOut, Y)
    for t, j in itertools.product(range(T), range(k)):
        e = np.zeros((T, k)); e[t, j] = 1.0
        assert got[t, j] == pytest.approx(L(g + e) - L(g), rel=1e-9, abs=1e-12)


@pytest.mark.parametrize("renorm", [False, True])
@pytest.mark.parametrize("aux_coef", [0.0, 0.37])
def test_router_grad_finite_differences_through_the_layer(renorm, aux_coef):
    """dlogits of <dOut, out(logits)> + aux_coef * aux(logits) by central
    differences of the oracle layer itself (top-k choice and counts fixed:
    the logits are far from ties, and eps is small)."""
    T, d, E, k, F = 6, 8, 5, 2, 6
    g = torch.Generator().manual_seed(5)
    x = torch.randn(T, d, generator=g, dtype=torch.float64)
    W1 = torch.randn(E, F, d, generator=g, dtype=torch.float64) * 0.3
    W3 = torch.randn(E, F, d, generator=g, dtype=torch.float64) * 0.3
    W2 = torch.randn(E, d, F, generator=g, dtype=torch.float64) * 0.3
    dOut = np.random.default_rng(6).normal(size=(T, d))
    lg = _grid_logits(T, E, 7)
    idx0 = O.topk_select(lg, k)

    def loss(l):
        assert np.array_equal(O.topk_select(l, k), idx0)
        out = O.moe_layer(x, k, W1, W3, W2, logits=l, renorm=renorm)["out"]
        return float((dOut * out).sum()) + aux_coef * O.aux_loss(l, idx0)

    Y = _expert_rows(x, idx0, W1, W3, W2)
    got = O.router_grad(lg, idx0, O.gate_grad(dOut, Y), renorm=renorm, aux_coef=aux_coef)
    eps = 2.0 ** -12
    fd = np.zeros((T, E))
    for t, e in itertools.product(range(T), range(E)):
        lp, lm = lg.copy(), lg.copy()
        lp[t, e] += eps
        lm[t, e] -= eps
        fd[t, e] = (loss(lp) - loss(lm)) / (2 * eps)
    assert np.abs(got - fd).max() <= 1e-6 * max(1.0, np.abs(fd).max())
    assert np.abs(got).max() > 1e-3   # not vacuous


@pytest.mark.parametrize("renorm", [False, True])
def test_router_grad_matches_torch_autograd(renorm):
    T, E, k = 40, 9, 3
    lg = np.random.default_rng(8).normal(size=(T, E)).astype(np.float32)
    dg = np.random.default_rng(9).normal(size=(T, k))
    idx = O.topk_select(lg, k)
    c = 0.21
    L = torch.tensor(lg.astype(np.float64), requires_grad=True)
    p = torch.softmax(L, dim=1)
    sel = torch.gather(p, 1, torch.as_tensor(idx, dtype=torch.long))
    if renorm:
        sel = sel / sel.sum(dim=1, keepdim=True)
    f = torch.bincount(torch.as_tensor(idx.ravel(), dtype=torch.long), minlength=E).double() / T
    total = (sel * torch.as_tensor(dg)).sum() + c * E * (f * p.mean(dim=0)).sum()
    total.backward()
    got = O.router_grad(lg, idx, dg, renorm=renorm, aux_coef=c)
    assert np.allclose(got, L.grad.numpy(), rtol=1e-10, atol=1e-13)


def test_router_grad_closed_forms():
    T, E = 30, 6
    rng = np.random.default_rng(10)
    lg = rng.normal(size=(T, E)).astype(np.float32)
    # k = E, the same upstream gradient on every gate: the gates are the whole
    # softmax, whose outputs sum to 1, so the logits get no gradient
    idx = O.topk_select(lg, E)
    assert np.abs(O.router_grad(lg, idx, np.full((T, E), 0.7))).max() < 1e-15
    # renormalised gates are invariant to a common shift of the chosen
    # logits' probabilities' scale: k = E renorm equals plain softmax
    dg = rng.normal(size=(T, E))
    assert np.allclose(O.router_grad(lg, idx, dg, renorm=True), O.router_grad(lg, idx, dg),
                       rtol=1e-12, atol=1e-15)
    # the aux term alone vanishes for a uniform router with balanced counts
    flat = np.zeros((T, E), np.float32)
    bal = np.array([[t % E, (t + 1) % E] for t in range(T)], np.int32)
    assert np.abs(O.router_grad(flat, bal, np.zeros((T, 2)), aux_coef=1.0)).max() < 1e-15


def test_router_linear_grad_finite_differences():
    """logits = x Wr^T is linear in each operand, so a unit step gives the
    exact derivative (no truncation error)."""
    T, d, E = 5, 7, 3
    rng = np.random.default_rng(11)
    x = rng.normal(size=(T, d))
    Wr = rng.normal(size=(E, d))
    G = rng.normal(size=(T, E))
    L = lambda xx, ww: float((G * (xx @ ww.T)).sum())
    dx, dWr = O.router_linear_grad(G, x, Wr)
    assert dx.shape == (T, d) and dWr.shape == (E, d)
    for t, c in itertools.product(range(T), range(d)):
        e = np.zeros((T, d)); e[t, c] = 1.0
        assert dx[t, c] == pytest.approx(L(x + e, Wr) - L(x, Wr), rel=1e-9, abs=1e-12)
    for r, c in itertools.product(range(E), range(d)):
        e = np.zeros((E, d)); e[r, c] = 1.0
        assert dWr[r, c] == pytest.approx(L(x, Wr + e) - L(x, Wr), rel=1e-9, abs=1e-12)


# ---------------------------------------------------------------- MXFP8 backward

def _torch_qdq_rows(m):
    """Quantise-dequantise along the last axis written independently of the
    oracle's codec: torch's float8_e4m3fn cast of the fp32 quotient, the
    scale 2^e with e = ceil(log2(fp32(amax / 448))) found by frexp (1 for an
    all-zero block)."""
    v = torch.as_tensor(np.ascontiguousarray(np.asarray(m, np.float32)))
    rows, K = v.shape
    b = v.reshape(rows, K // 32, 32)
    amax = b.abs().amax(dim=2)
    s32 = amax / 448.0
    mant, ex = torch.frexp(s32)
    e = torch.where(mant == 0.5, ex - 1, ex).clamp(-127, 127)
    e = torch.where(amax == 0, torch.zeros_like(e), e)
    scale = torch.ldexp(torch.ones_like(s32), e)
    q = (b / scale[..., None]).to(torch.float8_e4m3fn).to(torch.float32)
    return (q * scale[..., None]).reshape(rows, K).double().numpy()


def _bf16_of(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).double().numpy()


def _mx_problem(seed, T=40, d=64, F=64, E=4, k=2, skew=False):
    g = torch.Generator().manual_seed(seed)

    def mod(shape):
        # skew=True: magnitudes spread over 2^-3..2^3 along both of the last
        # two axes, so 32-blocks along one axis and along the other get
        # different scales (iid data would give the same scale either way)
        if not skew:
            return 1.0
        r = torch.exp2(torch.randint(-3, 4, (shape[-2], 1), generator=g).float())
        c = torch.exp2(torch.randint(-3, 4, (1, shape[-1]), generator=g).float())
        return r * c

    x = (torch.randn(T, d, generator=g) * mod((T, d))).to(torch.bfloat16)
    W1 = (torch.randn(E, F, d, generator=g) * 0.15 * mod((F, d))).to(torch.bfloat16)
    W3 = (torch.randn(E, F, d, generator=g) * 0.15 * mod((F, d))).to(torch.bfloat16)
    W2 = (torch.randn(E, d, F, generator=g) * 0.15 * mod((d, F))).to(torch.bfloat16)
    dOut = (torch.randn(T, d, generator=g) * mod((T, d))).to(torch.bfloat16)
    lg = torch.randn(T, E, generator=g).numpy().astype(np.float32)
    lg[:, E - 1] -= 30.0  # one expert with zero rows
    return x, W1, W3, W2, lg, dOut


def test_mxfp8_backward_exact_mode_is_the_backward():
    # every quantisation and bf16 rounding replaced by the identity: the
    # wiring (operands, transposes, gates, combine) must give the plain
    # backward, itself pinned against torch autograd above
    x, W1, W3, W2, lg, dOut = _mx_problem(61)
    r = O.mxfp8_layer_bwd(x, dOut, 2, W1, W3, W2, lg, exact=True)
    b = O.moe_layer_bwd(x, dOut, 2, W1, W3, W2, lg)
    for name in ("dx", "dW1", "dW3", "dW2"):
        assert np.allclose(r[name], b[name], rtol=1e-12, atol=1e-12), name
    assert np.all(r["dW1"][3] == 0) and np.all(r["dW2"][3] == 0)


def test_mxfp8_backward_operands_quantised_along_contraction():
    # each quantised operand equals an independent torch restatement of the
    # codec applied along the stated axis to the stated source
    x, W1, W3, W2, lg, dOut = _mx_problem(62, skew=True)
    k = 2
    with np.errstate(over="ignore"):  # exp(-a) of large negative pre-activations: silu -> -0
        r = O.mxfp8_layer_bwd(x, dOut, k, W1, W3, W2, lg, return_ops=True)
    idx, gate = r["idx"], r["gate"]
    assert set(r["ops"]) == {0, 1, 2}
    x64, d64 = x.double().numpy(), dOut.double().numpy()
    for e, op in r["ops"].items():
        toks, js = np.nonzero(idx == e)     # token-major: the expert's row order
        # forward operand: the token rows of x quantised along d
        assert np.array_equal(op["X"], _torch_qdq_rows(x64[toks]))
        w1, w3, w2 = (t[e].double().numpy() for t in (W1, W3, W2))
        A = _bf16_of(op["X"] @ _torch_qdq_rows(w1).T)
        assert np.array_equal(op["A"], A)
        # dYe rows: bf16 of the fp32 product gate * dOut
        dy = _bf16_of((gate[toks, js][:, None] * d64[toks]).astype(np.float32))
        assert np.array_equal(op["dy"], dy)
        assert np.array_equal(op["dyd"], _torch_qdq_rows(dy))          # along d
        assert np.array_equal(op["w2td"], _torch_qdq_rows(w2.T))       # W2_e along d
        both = np.concatenate([w1.T, w3.T], axis=1)                    # [d, 2F]
        assert np.array_equal(op["w13td"], _torch_qdq_rows(both))      # along F
        dab = np.concatenate([op["da"], op["db"]], axis=1)
        assert np.array_equal(op["dabd"], _torch_qdq_rows(dab))        # along F


def test_mxfp8_backward_error_against_exact_backward():
    # the format's error: a few percent of relative L2, never a gross mistake
    x, W1, W3, W2, lg, dOut = _mx_problem(63, T=96, d=128, F=128)
    r = O.mxfp8_layer_bwd(x, dOut, 2, W1, W3, W2, lg)
    b = O.moe_layer_bwd(x, dOut, 2, W1, W3, W2, lg)
    for name in ("dx", "dW1", "dW3", "dW2"):
        rel = np.linalg.norm(r[name] - b[name]) / np.linalg.norm(b[name])
        assert 1e-3 < rel < 0.15, (name, rel)


# ---------------------------------------------------------------- MXFP8 forward

def test_mxfp8_forward_exact_mode_is_the_layer():
    # every quantise-dequantise (and the fp32 rounding of H) replaced by the
    # identity: the wiring (which operand, gates, the per-token sum) must give
    # the plain layer, itself pinned against torch above
    x, W1, W3, W2, lg, _ = _mx_problem(71)
    k = 2
    r = O.mxfp8_layer(x, k, W1, W3, W2, lg, exact=True)
    b = O.moe_layer(x, k, W1, W3, W2, logits=lg)
    assert np.allclose(r["out"], b["out"], rtol=1e-12, atol=1e-12)
    toks = np.array([0, 5, 17, 39])
    rs = O.mxfp8_layer(x, k, W1, W3, W2, lg, tokens=toks, exact=True)
    assert np.allclose(rs["out"], b["out"][toks], rtol=1e-12, atol=1e-12)
    assert np.array_equal(r["idx"], b["idx"]) and np.array_equal(r["slot"], b["slot"])


def test_mxfp8_forward_operands_quantised_along_contraction():
    # each quantised operand equals an independent torch restatement of the
    # codec applied along the stated axis to the stated source; the skewed
    # magnitudes make the other axis give other scales, which is checked too
    x, W1, W3, W2, lg, _ = _mx_problem(72, skew=True)
    k = 2
    toks = np.arange(4, 36)  # 32 tokens, so blocks along the token axis exist too
    with np.errstate(over="ignore"):
        r = O.mxfp8_layer(x, k, W1, W3, W2, lg, tokens=toks, return_ops=True)
    ops = r["ops"]
    x64 = x.double().numpy()
    assert np.array_equal(ops["xd"], _torch_qdq_rows(x64[toks]))            # x along d
    assert not np.array_equal(ops["xd"], _torch_qdq_rows(x64[toks].T).T)
    for e, (w1d, w3d, w2d) in ops["w"].items():
        w1, w3, w2 = (t[e].double().numpy() for t in (W1, W3, W2))
        assert np.array_equal(w1d, _torch_qdq_rows(w1))                    # [F, d] along d
        assert np.array_equal(w3d, _torch_qdq_rows(w3))
        assert np.array_equal(w2d, _torch_qdq_rows(w2))                    # [d, F] along F
        # the other axis gives another result on these inputs
        assert not np.array_equal(w1d, _torch_qdq_rows(w1.T).T)
        assert not np.array_equal(w2d, _torch_qdq_rows(w2.T).T)
    idx, gate = r["idx"], r["gate"]
    out = np.zeros((len(toks), x.shape[1]))
    for (i, j), (h, hd) in ops["h"].items():
        e = int(idx[toks[i], j])
        w1d, w3d, w2d = ops["w"][e]
        xi = ops["xd"][i]
        a, b = w1d @ xi, w3d @ xi
        h_ref = (a / (1.0 + np.exp(-a)) * b).astype(np.float32).astype(np.float64)
        assert np.array_equal(h, h_ref)                                    # H from its fp32 value
        assert np.array_equal(hd, _torch_qdq_rows(h[None, :])[0])          # H along F
        out[i] += gate[toks[i], j] * (w2d @ hd)
    assert np.allclose(out, r["out"], rtol=1e-13, atol=1e-13)


def test_mxfp8_forward_error_against_exact_layer():
    # the format's error: a few percent of relative L2, never a gross mistake
    x, W1, W3, W2, lg, _ = _mx_problem(73, T=96, d=128, F=128)
    r = O.mxfp8_layer(x, 2, W1, W3, W2, lg)
    b = O.moe_layer(x, 2, W1, W3, W2, logits=lg)
    rel = np.linalg.norm(r["out"] - b["out"]) / np.linalg.norm(b["out"])
    assert 1e-3 < rel < 0.15, rel


def test_mxfp8_sampled_backward_matches_full_backward():
    # the per-row restatement used at full size equals the whole-batch MXFP8
    # backward on the sampled tokens and experts (empty expert included)
    x, W1, W3, W2, lg, dOut = _mx_problem(64, T=60, d=64, F=64, E=4, k=2, skew=True)
    with np.errstate(over="ignore"):
        full = O.mxfp8_layer_bwd(x, dOut, 2, W1, W3, W2, lg)
        toks = np.array([0, 7, 31, 59])
        smp = O.mxfp8_layer_bwd_sampled(x, dOut, 2, W1, W3, W2, lg, toks, [0, 2, 3])
    assert np.allclose(smp["dx"], full["dx"][toks], rtol=1e-12, atol=1e-12)
    for e in (0, 2, 3):
        for got, ref in zip(smp["dW"][e], (full["dW1"][e], full["dW3"][e], full["dW2"][e])):
            assert np.allclose(got, ref, rtol=1e-12, atol=1e-12), e
    assert all(np.all(m == 0) for m in smp["dW"][3])  # expert 3 gets no rows
