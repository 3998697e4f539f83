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


def router_logits_checked(got, x: torch.Tensor, Wr: torch.Tensor) -> np.ndarray:
    """Router logits from the GPU against the oracle's fixed-order fp32 logits,
    returning the logits both sides route on (the GPU's).

    fp32 inputs: the GPU runs the oracle's four in-order fmaf chains, so the
    bits must agree. bf16 inputs: every product is exact in fp32 and both
    sides are fp32 sums of the same d products, the tensor core in its own
    order; a recursive fp32 sum of d terms errs by at most (d-1) 2^-24
    sum|terms|, so the two differ by at most 2 (d-1) 2^-24 sum_j |x_j w_j|;
    the bound doubles that for the tensor core's internal accumulation.
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
    bound = 4.0 * (d - 1) * 2.0 ** -24 * (xa @ wa.T)
    err = np.abs(got.astype(np.float64) - ref.astype(np.float64))
    assert np.all(err <= bound), f"bf16 router logits: worst err/bound {np.max(err / bound):.3e}"
    return got
