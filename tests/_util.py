"""Helpers shared by the GPU parity tests (comparison only, no layer math)."""
import math

import numpy as np
import torch

# Floating-point bars for outputs stored in bf16 (and the fp32 layer run on
# tf32 tensor cores): max-abs 2e-2 and relative L2 1e-2 against the
# fp32-or-better oracle.
MAX_ABS = 2e-2
REL_L2 = 1e-2


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().to(torch.float64).numpy()


def rel_l2(got, ref) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    den = math.sqrt(float((ref * ref).sum()))
    return math.sqrt(float(((got - ref) ** 2).sum())) / (den if den > 0 else 1.0)


def assert_close_layer(got, ref, what="", max_abs=MAX_ABS, rel=REL_L2):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    ma = float(np.abs(got - ref).max()) if got.size else 0.0
    rl = rel_l2(got, ref)
    assert ma <= max_abs and rl <= rel, f"{what}: max-abs {ma:.3e} rel-L2 {rl:.3e}"
    return ma, rl


def gate_tolerance(logits: np.ndarray, idx: np.ndarray, renorm: bool) -> np.ndarray:
    """Relative error bound of the fp32 softmax gate computed on the GPU.

    exp(l - max) in fp32: the subtraction rounds (|l-max| * 2^-24 absolute in
    the exponent's argument), expf adds at most 2 ulp; the denominator is a
    sum of E positive terms done as a pairwise tree over each lane's (at most
    32) terms and a butterfly over the lanes of the token's group, so a term
    passes through at most ceil(log2 E) + 1 roundings (adding an exact zero
    for an absent expert is exact); one division. Each rounding contributes
    at most 2^-24 relative; the bound below doubles it for margin.
    """
    T, E = logits.shape
    lg = logits.astype(np.float64)
    mx = lg.max(axis=1, keepdims=True)
    sel = np.take_along_axis(lg, idx.astype(np.int64), axis=1)
    terms = np.abs(sel - mx) + math.ceil(math.log2(E)) + 1 + 2 + 2
    if renorm:
        terms = terms + idx.shape[1] + 2
    return terms * 2.0 ** -23


def assert_close_scaled(got, ref, what="", max_abs=MAX_ABS, rel=REL_L2):
    """For intermediates of O(1) or larger magnitude (H, Ye of the unit
    tests): the max-abs bar applies relative to max(1, max|ref|), since bf16
    storage alone rounds each value by up to 2^-8 of its magnitude."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    scale = max(1.0, float(np.abs(ref).max()) if ref.size else 1.0)
    ma = float(np.abs(got - ref).max()) / scale if got.size else 0.0
    rl = rel_l2(got, ref)
    assert ma <= max_abs and rl <= rel, f"{what}: scaled max-abs {ma:.3e} rel-L2 {rl:.3e}"
    return ma, rl


def router_logits_checked(got, x: torch.Tensor, Wr: torch.Tensor, tight: float = 64.0) -> np.ndarray:
    """Router logits from the GPU against the oracle's fixed-order fp32 logits,
    returning the logits the GPU routed on.

    fp32 inputs: the GPU runs the oracle's four in-order fmaf chains, so the
    bits must agree. bf16 inputs: every logit is either the oracle's value
    bit for bit (the experts the route step recomputes in the fixed order)
    or the tensor cores' fp32 sum of the same exact products in another
    order. Two bounds apply to the difference, with P = sum_j |x_j w_j|:
      * the worst case of the two summation orders, 1.25 d 2^-23 P (the
        four in-order chains (d/4 + 3) 2^-24 P, the tensor core at most
        18 units of 2^-23 P per 16-product instruction);
      * an empirical bar, ``tight`` 2^-24 P, about eight times the largest
        difference measured on the OLMoE-shaped workload (7.5 2^-24 P):
        a reduced-precision accumulation or a dropped product, which the
        worst-case bound would let through, fails it.
    """
    from oracle import moe_oracle as O
    got = np.asarray(got, dtype=np.float32)
    ref = O.router_logits(x, Wr)
    if x.dtype == torch.float32:
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32)), "fp32 router logits"
        return got
    xa = np.abs(x.detach().cpu().double().numpy())
    wa = np.abs(Wr.detach().cpu().double().numpy())
    d = x.shape[1]
    P = xa @ wa.T
    err = np.abs(got.astype(np.float64) - ref.astype(np.float64))
    worst = 1.25 * d * 2.0 ** -23 * P
    assert np.all(err <= worst), f"bf16 router logits: worst err/bound {np.max(err / worst):.3e}"
    bar = tight * 2.0 ** -24 * P
    ratio = np.max(np.where(P > 0, err / np.where(P > 0, P, 1.0), 0.0)) / 2.0 ** -24
    assert np.all(err <= bar), f"bf16 router logits: max err = {ratio:.2f} 2^-24 P (bar {tight})"
    return got


def route_equals_oracle_own_logits(r, x: torch.Tensor, Wr: torch.Tensor, k: int, E: int,
                                   renorm: bool = False):
    """Routing computed on the GPU from x and Wr against the oracle routing on
    its own fixed-order logits: idx (order of j included), counts, offsets,
    slot and tile offsets identical for every token. Returns the number of
    logits the GPU holds in the oracle's bits (the recomputed ones)."""
    from oracle import moe_oracle as O
    ref_lg = O.router_logits(x, Wr)
    idx, _, _ = O.route(ref_lg, k, renorm)
    meta = O.routing_metadata(idx, E)
    g_idx = r.idx.cpu().numpy()
    bad = np.nonzero((g_idx != idx).any(axis=1))[0]
    assert bad.size == 0, f"{bad.size} tokens route differently from the oracle's logits, first {bad[:5]}"
    assert np.array_equal(r.counts.cpu().numpy(), meta["counts"])
    assert np.array_equal(r.offsets.cpu().numpy(), meta["offsets"])
    assert np.array_equal(r.slot.cpu().numpy(), meta["slot"])
    to = getattr(r, "tile_offsets", None)
    if to is not None:
        assert np.array_equal(to.cpu().numpy(), meta["tile_offsets"])
    if getattr(r, "logits", None) is not None:
        got = r.logits.cpu().numpy().astype(np.float32)
        return int((got.view(np.uint32) == ref_lg.view(np.uint32)).sum())
    return -1
