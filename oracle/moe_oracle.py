"""CPU oracle for the dropless top-k MoE expert layer.

TEST INFRASTRUCTURE ONLY. Only the test-suite, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this module. The CUDA path
never imports it and shares no code with it; the only shared module is the
seeded input generator, which holds none of the layer's arithmetic.

Plain, slow, obviously-correct restatement of what the layer computes, in
numpy float64 unless the pages fix the precision (they fix the router's
softmax to fp32; the fp32 router logits come from ``router_logits.c``).

Sources (page title, section):
  [HF]   "Transformers 中的 OLMoE：稀疏 MoE 语言模型架构解析与推理实践"
         (blog.gitcode.com): §2 router (fp32 softmax over experts, torch.topk,
         optional norm_topk_prob, bias-free (E, hidden) weight); §3 experts
         (3-D gate_up / down tensors, per-expert gather -> gate/up -> SiLU
         product -> down -> scale by the top-k weight -> index_add back);
         OlmoeConfig table (norm_topk_prob defaults to False).
  [OF]   "olmoforge" README (git.onestrm.cn/huzjie/olmoforge): capability
         table (row-wise EP writes tokens straight into the expert input
         buffer; grouped GEMM; GPU-resident routing table; MXFP8 with a
         shared scale per block) and the MXFP8 block-quantisation sketch.
  [NEWS] "专家池 8→128 只慢 5%：Ai2 开源万亿参数 MoE 训练框架 Olmo-core 3"
         (xxqk.cn), section "三招拆分、三项优化、一个精度开关".
  [REL]  "OLMo-core 3 发布：主攻混合专家训练与导出校验" (wedoingai.com),
         section "主要功能": pairwise SwiGLU backward, bf16 weight gradients.

Readings of points the pages leave open (each is also listed in the design
notes):
  * top-k ties go to the lower expert index; selection is made on the fp32
    logits (softmax is strictly increasing, so this is the exact-arithmetic
    top-k of the probabilities without exp-rounding ties); NaN logits count
    as -inf; +0.0 and -0.0 compare equal.
  * gates are the softmax probabilities of the chosen experts, in descending
    logit order, not renormalised unless ``renorm``.
  * routing metadata is the stable counting sort of the token-major list of
    (token, j) pairs by expert: slot = offsets[e] + (number of earlier
    tokens routed to e). Offsets are unpadded.
  * router logits x·Wrᵀ: four sequential fp32 fmaf chains over the
    contiguous quarters of the hidden dimension, added in order (the
    summation order decides the top-k bits, so it is fixed on both sides).
  * the expert FFN and the combine are evaluated without intermediate
    rounding (float64); the CUDA path stores H and Ye in the layer dtype.
  * MXFP8: blocks of 32 consecutive elements along the contraction axis;
    scale = amax/448 in fp32 (1.0 for an all-zero block), or that value
    rounded up to a power of two (UE8M0, what block-scaled MMA consumes);
    payload = E4M3 with round-to-nearest-even and saturation to ±448 of the
    fp32 quotient v/scale. The sketch in [OF] rounds v/scale to an integer,
    which is not an E4M3 payload; the E4M3 reading is taken.
  * MXFP8 backward (the pages leave its precision open): the input-gradient
    GEMMs quantise each operand along its own contraction dimension (dYe
    and W2 along d, [dA | dB] and [W1; W3] along F); the weight gradients
    are exact GEMMs of the unquantised gradients with the forward's
    dequantised operands. Values that decide a code are taken in the
    precision the layer stores them in (bf16 dYe, dH, A, B).

Where a function has no independent pin it says "parity unpinned"; every
function below is pinned by tests/test_oracle.py.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from typing import Dict, Optional

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "_router_logits.so")
_lib = None

E4M3_MAX = 448.0
MX_BLOCK = 32
TILE_M = 128  # rows per M-tile in the tile table (an output of the route step)


# --------------------------------------------------------------------------
# build / load of the C part
# --------------------------------------------------------------------------

def build(force: bool = False) -> str:
    """Compile router_logits.c into a shared object next to it."""
    src = os.path.join(_HERE, "router_logits.c")
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(src)):
        return _LIB_PATH
    cmd = ["gcc", "-O2", "-fPIC", "-shared", "-ffp-contract=off", "-fopenmp",
           src, "-o", _LIB_PATH, "-lm"]
    subprocess.run(cmd, check=True)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        for name, pt in (("oracle_router_logits_f32", ctypes.c_void_p),
                         ("oracle_router_logits_bf16", ctypes.c_void_p)):
            f = getattr(lib, name)
            f.argtypes = [pt, pt, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                          ctypes.c_void_p]
            f.restype = None
        _lib = lib
    return _lib


# --------------------------------------------------------------------------
# a0: router logits  [HF §2]
# --------------------------------------------------------------------------

def router_logits(x: torch.Tensor, Wr: torch.Tensor) -> np.ndarray:
    """fp32 logits[t, e]: four sequential fmaf chains over the contiguous
    quarters of j (each from +0.0), the quarter sums added in order
    ((c0 + c1) + c2) + c3. d must be a multiple of 4."""
    lib = _load()
    x = x.detach().cpu().contiguous()
    Wr = Wr.detach().cpu().contiguous()
    T, d = x.shape
    if d % 4:
        raise ValueError("the router's hidden size must be a multiple of 4")
    E = Wr.shape[0]
    out = np.empty((T, E), dtype=np.float32)
    if x.dtype == torch.float32:
        xa, wa = x.numpy(), Wr.numpy()
        lib.oracle_router_logits_f32(xa.ctypes.data, wa.ctypes.data, T, d, E,
                                     out.ctypes.data)
    elif x.dtype == torch.bfloat16:
        xa = x.view(torch.int16).numpy()
        wa = Wr.view(torch.int16).numpy()
        lib.oracle_router_logits_bf16(xa.ctypes.data, wa.ctypes.data, T, d, E,
                                      out.ctypes.data)
    else:
        raise TypeError(x.dtype)
    return out


# --------------------------------------------------------------------------
# a1: softmax + top-k  [HF §2]
# --------------------------------------------------------------------------

def topk_select(logits: np.ndarray, k: int) -> np.ndarray:
    """idx[t, j]: the k experts with the largest logit, descending, ties to
    the lower index (stable sort of -logit; NaN counts as -inf)."""
    lg = np.asarray(logits, dtype=np.float32).astype(np.float64)
    lg = np.where(np.isnan(lg), -np.inf, lg)
    # np.argsort(kind="stable") keeps equal keys in index order; -0.0 == +0.0.
    order = np.argsort(-lg, axis=1, kind="stable")
    return order[:, :k].astype(np.int32)


def softmax_fp64(logits: np.ndarray) -> np.ndarray:
    """Row softmax of the fp32 logits, evaluated in float64."""
    lg = np.asarray(logits, dtype=np.float32).astype(np.float64)
    m = lg.max(axis=1, keepdims=True)
    p = np.exp(lg - m)
    return p / p.sum(axis=1, keepdims=True)


def route(logits: np.ndarray, k: int, renorm: bool = False):
    """(idx int32 [T,k], gate float64 [T,k], probs float64 [T,E])."""
    idx = topk_select(logits, k)
    probs = softmax_fp64(logits)
    gate = np.take_along_axis(probs, idx.astype(np.int64), axis=1)
    if renorm:
        gate = gate / gate.sum(axis=1, keepdims=True)
    return idx, gate, probs


# --------------------------------------------------------------------------
# a2: GPU-resident routing metadata  [OF capability table; NEWS]
# --------------------------------------------------------------------------

def routing_metadata(idx: np.ndarray, E: int, tile_m: int = TILE_M) -> Dict[str, np.ndarray]:
    """Stable counting sort of the token-major (t, j) list by expert.

    counts[e]   number of (t, j) with idx[t, j] == e
    offsets     exclusive prefix sum of counts, length E+1, offsets[E] = T*k
    slot[t, j]  row of (t, j) in the expert-sorted buffers
    tile_offsets exclusive prefix sum of ceil(counts / tile_m), length E+1
    row_token   inverse map: row -> token
    """
    idx = np.asarray(idx)
    T, k = idx.shape
    flat = idx.reshape(-1).astype(np.int64)
    counts = np.bincount(flat, minlength=E).astype(np.int64)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    order = np.argsort(flat, kind="stable")  # token-major order kept inside an expert
    slot_flat = np.empty(T * k, dtype=np.int64)
    slot_flat[order] = np.arange(T * k, dtype=np.int64)
    tiles = (counts + tile_m - 1) // tile_m
    tile_offsets = np.zeros(E + 1, dtype=np.int64)
    tile_offsets[1:] = np.cumsum(tiles)
    row_token = np.empty(T * k, dtype=np.int64)
    row_token[slot_flat] = np.repeat(np.arange(T, dtype=np.int64), k)
    return {
        "counts": counts.astype(np.int32),
        "offsets": offsets.astype(np.int32),
        "slot": slot_flat.reshape(T, k).astype(np.int32),
        "tile_offsets": tile_offsets.astype(np.int32),
        "row_token": row_token.astype(np.int32),
    }


# --------------------------------------------------------------------------
# a3: row-wise dispatch  [OF capability table]
# --------------------------------------------------------------------------

def dispatch(x: np.ndarray, slot: np.ndarray, gate: Optional[np.ndarray] = None) -> np.ndarray:
    """Xe[slot[t, j]] = x[t] (or gate[t, j] * x[t] when gate is given).

    Works on any numpy dtype; with gate=None it is a pure copy.
    """
    T, k = slot.shape
    Xe = np.empty((T * k,) + x.shape[1:], dtype=np.float64 if gate is not None else x.dtype)
    for j in range(k):
        if gate is None:
            Xe[slot[:, j]] = x
        else:
            Xe[slot[:, j]] = gate[:, j:j + 1] * x.astype(np.float64)
    return Xe


# --------------------------------------------------------------------------
# a4: SwiGLU expert FFN over each expert's rows  [HF §3]
# --------------------------------------------------------------------------

def silu(a: np.ndarray) -> np.ndarray:
    return a / (1.0 + np.exp(-a))


def expert_ffn(Xe: np.ndarray, offsets: np.ndarray, W1: np.ndarray, W3: np.ndarray,
               W2: np.ndarray, keep: bool = False):
    """Ye[r] = W2_e (silu(W1_e Xe[r]) * W3_e Xe[r]) for r in expert e's rows.

    W1, W3: [E, F, d]; W2: [E, d, F]; everything float64. Returns Ye (and
    A, B, H when keep=True).
    """
    E = W1.shape[0]
    R = Xe.shape[0]
    F = W1.shape[1]
    d = W2.shape[1]
    Ye = np.zeros((R, d), dtype=np.float64)
    if keep:
        A = np.zeros((R, F)); B = np.zeros((R, F)); H = np.zeros((R, F))
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 == r0:
            continue
        X = Xe[r0:r1]
        a = X @ W1[e].T
        b = X @ W3[e].T
        h = silu(a) * b
        Ye[r0:r1] = h @ W2[e].T
        if keep:
            A[r0:r1], B[r0:r1], H[r0:r1] = a, b, h
    if keep:
        return Ye, A, B, H
    return Ye


# --------------------------------------------------------------------------
# a5: gate-weighted combine  [HF §3, index_add back to token order]
# --------------------------------------------------------------------------

def combine(Ye: np.ndarray, slot: np.ndarray, gate: Optional[np.ndarray]) -> np.ndarray:
    """out[t] = sum_j gate[t, j] * Ye[slot[t, j]] (gate None = unit gates)."""
    T, k = slot.shape
    out = np.zeros((T,) + Ye.shape[1:], dtype=np.float64)
    for j in range(k):
        g = 1.0 if gate is None else gate[:, j:j + 1]
        out += g * Ye[slot[:, j]].astype(np.float64)
    return out


# --------------------------------------------------------------------------
# the whole layer, as the pages describe it  [HF §3]
# --------------------------------------------------------------------------

def to64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().cpu().to(torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def moe_layer(x: torch.Tensor, k: int, W1, W3, W2, *, logits: Optional[np.ndarray] = None,
              Wr: Optional[torch.Tensor] = None, renorm: bool = False,
              keep: bool = False) -> Dict[str, np.ndarray]:
    """Route, then for every expert gather its tokens, run the SwiGLU FFN,
    scale by the top-k weight and add back in token order.

    The per-expert loop is the pages' formulation; the expert-sorted buffer
    and slots are the routing metadata written out.
    """
    if logits is None:
        logits = router_logits(x, Wr)
    E = W1.shape[0]
    idx, gate, probs = route(logits, k, renorm)
    meta = routing_metadata(idx, E)
    x64 = to64(x)
    Xe = dispatch(x64, meta["slot"])
    W1_, W3_, W2_ = to64(W1), to64(W3), to64(W2)
    res = expert_ffn(Xe, meta["offsets"], W1_, W3_, W2_, keep=keep)
    Ye = res[0] if keep else res
    out = combine(Ye, meta["slot"], gate)
    r = dict(logits=np.asarray(logits, np.float32), idx=idx, gate=gate, probs=probs,
             Xe=Xe, Ye=Ye, out=out, **meta)
    if keep:
        r["A"], r["B"], r["H"] = res[1], res[2], res[3]
    return r


def moe_layer_tokens(x: torch.Tensor, tokens: np.ndarray, idx: np.ndarray, gate: np.ndarray,
                     W1, W3, W2) -> np.ndarray:
    """out[t] for a sample of tokens (for full-size workloads where the whole
    layer would take too long on the CPU): the per-token formula
    out[t] = sum_j gate[t,j] W2_e(silu(W1_e x_t) * W3_e x_t), visiting each
    needed expert once."""
    tokens = np.asarray(tokens)
    xs = to64(x[torch.as_tensor(tokens, dtype=torch.long)])
    out = np.zeros((len(tokens), xs.shape[1]))
    sel = idx[tokens]
    for e in np.unique(sel):
        e = int(e)
        rows, js = np.nonzero(sel == e)
        w1, w3, w2 = to64(W1[e]), to64(W3[e]), to64(W2[e])
        X = xs[rows]
        h = silu(X @ w1.T) * (X @ w3.T)
        y = h @ w2.T
        out[rows] += gate[tokens[rows], js][:, None] * y
    return out


# --------------------------------------------------------------------------
# a6: E4M3 codec and MXFP8 block quantisation  [OF "MXFP8 分块量化"; NEWS]
# --------------------------------------------------------------------------

def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """OCP FP8 E4M3: 1 sign, 4 exponent bits (bias 7), 3 mantissa bits; no
    infinities; S.1111.111 is NaN; exponent field 0 holds subnormals
    m * 2^-9."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    ex = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(ex == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(ex - 7.0))
    val = np.where((ex == 15) & (m == 7), np.nan, val)
    return s * val


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """fp32 -> E4M3, round to nearest even, saturating to ±448; NaN -> 0x7F
    with the sign kept."""
    with np.errstate(invalid="ignore", divide="ignore", over="ignore"):
        return _e4m3_encode(v)


def _e4m3_encode(v: np.ndarray) -> np.ndarray:
    v = np.asarray(v, dtype=np.float32).astype(np.float64)  # exact
    sign = np.where(np.signbit(v), 0x80, 0x00).astype(np.int64)
    a = np.abs(v)
    nan = np.isnan(a)
    a = np.where(nan, 0.0, a)
    a = np.where(np.isinf(a), 2.0 * E4M3_MAX, a)
    code = np.zeros(a.shape, dtype=np.int64)
    # subnormal range: a < 2^-6, unit 2^-9
    sub = a < 2.0 ** -6
    qs = np.rint(a * 2.0 ** 9)  # rint is round-half-even; exact scaling
    code = np.where(sub, qs.astype(np.int64), code)  # qs == 8 is min normal 0x08
    # normal range
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    # guard log2 rounding at exact powers of two
    e = np.where(np.exp2(e) > a, e - 1, e)
    e = np.where(np.exp2(e + 1) <= a, e + 1, e)
    mant = np.rint((a / np.exp2(e) - 1.0) * 8.0)
    e = np.where(mant == 8, e + 1, e)
    mant = np.where(mant == 8, 0, mant)
    ncode = ((e + 7).astype(np.int64) << 3) | mant.astype(np.int64)
    code = np.where(sub, code, ncode)
    # saturate: anything at or above 448 (after rounding) is 448 = 0x7E
    code = np.where(~sub & ((e > 8) | ((e == 8) & (mant > 6))), 0x7E, code)
    code = np.where(a >= E4M3_MAX, 0x7E, code)
    code = np.where(nan, 0x7F, code)
    return (code | sign).astype(np.uint8)


def _pow2_ceil_exponent(s: np.ndarray) -> np.ndarray:
    """Smallest integer e with 2^e >= s (s > 0, float32 values), clamped to
    the UE8M0 range [-127, 127]."""
    s = np.asarray(s, dtype=np.float32).astype(np.float64)
    m, ex = np.frexp(s)  # s = m * 2^ex, m in [0.5, 1)
    e = np.where(m == 0.5, ex - 1, ex)
    return np.clip(e, -127, 127).astype(np.int64)


def mxfp8_quantize(v, mode: str = "e8m0"):
    """Block-quantise a [rows, K] array along K in blocks of 32.

    mode "f32":  scale = fp32(amax / 448), 1.0 when amax == 0; scales are
                 returned as float32 [rows, K/32].
    mode "e8m0": scale = smallest power of two >= fp32(amax / 448) (1.0 when
                 amax == 0); returned as the biased exponent byte
                 (uint8 = e + 127) [rows, K/32].
    codes = E4M3(fp32(v / scale)) as uint8 [rows, K].
    """
    if isinstance(v, torch.Tensor):
        v = v.detach().cpu().to(torch.float32).numpy()
    v = np.asarray(v, dtype=np.float32)
    rows, K = v.shape
    assert K % MX_BLOCK == 0
    blk = v.reshape(rows, K // MX_BLOCK, MX_BLOCK)
    amax = np.abs(blk).max(axis=2).astype(np.float32)
    s32 = (amax / np.float32(E4M3_MAX)).astype(np.float32)  # IEEE fp32 division
    zero = amax == 0
    if mode == "f32":
        scale = np.where(zero, np.float32(1.0), s32).astype(np.float32)
        stored = scale
    elif mode == "e8m0":
        e = np.where(zero, 0, _pow2_ceil_exponent(np.where(zero, 1.0, s32)))
        scale = np.exp2(e.astype(np.float64)).astype(np.float32)
        stored = (e + 127).astype(np.uint8)
    else:
        raise ValueError(mode)
    q32 = (blk / scale[:, :, None]).astype(np.float32)  # fp32 division, rounded once
    codes = e4m3_encode(q32).reshape(rows, K)
    return codes, stored


def mxfp8_scales_to_f32(stored: np.ndarray, mode: str) -> np.ndarray:
    if mode == "f32":
        return np.asarray(stored, dtype=np.float32)
    return np.exp2(np.asarray(stored, dtype=np.int64) - 127.0).astype(np.float32)


def mxfp8_dequantize_f32(codes: np.ndarray, stored: np.ndarray, mode: str) -> np.ndarray:
    """fp32 values decode(q) * scale (the product rounded to fp32)."""
    rows, K = codes.shape
    dec = e4m3_decode(codes).reshape(rows, K // MX_BLOCK, MX_BLOCK)
    sc = mxfp8_scales_to_f32(stored, mode).astype(np.float64)
    return (dec * sc[:, :, None]).astype(np.float32).reshape(rows, K)


def mxfp8_dequantize(codes: np.ndarray, stored: np.ndarray, mode: str) -> torch.Tensor:
    """bf16 output: fp32 product decode(q) * scale, then round-to-nearest-even
    to bf16."""
    return torch.from_numpy(mxfp8_dequantize_f32(codes, stored, mode)).to(torch.bfloat16)


def mxfp8_layer(x: torch.Tensor, k: int, W1, W3, W2, logits: np.ndarray,
                mode: str = "e8m0", tokens: Optional[np.ndarray] = None,
                exact: bool = False, return_ops: bool = False) -> Dict[str, np.ndarray]:
    """MXFP8 variant of the layer ([OF] capability table and "MXFP8 分块量化":
    32-element blocks sharing one scale, E4M3 payload; [NEWS] "三招拆分、三项
    优化、一个精度开关": the FFN runs on MXFP8 operands). Every GEMM operand
    is quantised along its contraction dimension: the token rows of x and
    the rows of W1_e, W3_e ([F, d]) along d; the rows of W2_e ([d, F]) and
    H along F, H from its fp32 value silu(a) * b. The GEMMs then run on the
    dequantised values in float64, per (token, choice) as in the per-token
    formula out[t] = sum_j gate[t,j] W2_e(silu(W1_e x_t) * W3_e x_t).
    ``tokens`` restricts the output to a sample.

    exact=True replaces every quantise-dequantise (and the fp32 rounding of
    H) by the identity, which must give the plain layer (a wiring check).
    return_ops=True adds the operands as quantised: "xd" (the sampled token
    rows), "w" {e: (w1d, w3d, w2d)}, "h" {(i, j): (H fp32 row, Hd row)}."""
    if exact:
        qdq = lambda m: np.asarray(m, np.float64)  # noqa: E731
        h32 = lambda m: np.asarray(m, np.float64)  # noqa: E731
    else:
        qdq = lambda m: _qdq_rows(m, mode)  # noqa: E731
        h32 = lambda m: np.asarray(m, np.float32).astype(np.float64)  # noqa: E731
    E = W1.shape[0]
    idx, gate, _ = route(logits, k)
    meta = routing_metadata(idx, E)
    T = x.shape[0]
    toks = np.arange(T) if tokens is None else np.asarray(tokens)
    xd = qdq(to64(x[torch.as_tensor(toks, dtype=torch.long)]))      # along d
    out = np.zeros((len(toks), x.shape[1]))
    wq = {}
    hs = {}
    for i, t in enumerate(toks):
        for j in range(k):
            e = int(idx[t, j])
            if e not in wq:
                wq[e] = (qdq(to64(W1[e])),   # [F, d] along d
                         qdq(to64(W3[e])),   # [F, d] along d
                         qdq(to64(W2[e])))   # [d, F] along F
            w1d, w3d, w2d = wq[e]
            h = h32(silu(w1d @ xd[i]) * (w3d @ xd[i]))
            hd = qdq(h[None, :])[0]                                  # along F
            out[i] += gate[t, j] * (w2d @ hd)
            if return_ops:
                hs[(i, j)] = (h, hd)
    res = dict(out=out, idx=idx, gate=gate, tokens=toks, **meta)
    if return_ops:
        res["ops"] = dict(xd=xd, w=wq, h=hs)
    return res


# --------------------------------------------------------------------------
# a8: backward of the expert layer (router and gate gradients excluded)
#     [REL "主要功能": pairwise SwiGLU backward, bf16 weight gradients]
# --------------------------------------------------------------------------

def dsilu(a: np.ndarray) -> np.ndarray:
    s = 1.0 / (1.0 + np.exp(-a))
    return s * (1.0 + a * (1.0 - s))


def expert_ffn_bwd(Xe: np.ndarray, offsets: np.ndarray, W1, W3, W2, dYe: np.ndarray):
    """Gradients of Ye = W2_e(silu(W1_e x) * W3_e x) per expert.

    Returns dXe [R,d], dW1 [E,F,d], dW3 [E,F,d], dW2 [E,d,F] (float64). An
    expert with no rows gets zero weight gradients.
    """
    E, F, d = W1.shape
    R = Xe.shape[0]
    dXe = np.zeros((R, d))
    dW1 = np.zeros((E, F, d)); dW3 = np.zeros((E, F, d)); dW2 = np.zeros((E, d, F))
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 == r0:
            continue
        X = Xe[r0:r1]
        a = X @ W1[e].T
        b = X @ W3[e].T
        h = silu(a) * b
        dy = dYe[r0:r1]
        dh = dy @ W2[e]
        da = dh * b * dsilu(a)
        db = dh * silu(a)
        dXe[r0:r1] = da @ W1[e] + db @ W3[e]
        dW1[e] = da.T @ X
        dW3[e] = db.T @ X
        dW2[e] = dy.T @ h
    return dXe, dW1, dW3, dW2


def moe_layer_bwd(x: torch.Tensor, dOut: torch.Tensor, k: int, W1, W3, W2,
                  logits: np.ndarray) -> Dict[str, np.ndarray]:
    """dx and dW for out = sum_j gate[t,j] FFN_e(x_t), gates held constant."""
    E = W1.shape[0]
    idx, gate, _ = route(logits, k)
    meta = routing_metadata(idx, E)
    Xe = dispatch(to64(x), meta["slot"])
    dYe = dispatch(to64(dOut), meta["slot"], gate=gate)
    dXe, dW1, dW3, dW2 = expert_ffn_bwd(Xe, meta["offsets"], to64(W1), to64(W3), to64(W2), dYe)
    dx = combine(dXe, meta["slot"], None)
    return dict(dx=dx, dW1=dW1, dW3=dW3, dW2=dW2, dYe=dYe, dXe=dXe, idx=idx, gate=gate, **meta)


def moe_layer_bwd_sampled(x: torch.Tensor, dOut: torch.Tensor, k: int, W1, W3, W2,
                          logits: np.ndarray, tokens, experts) -> Dict[str, np.ndarray]:
    """The same gradients as moe_layer_bwd, restricted to a sample: dx for the
    given tokens (each (t, j) row's dXe from the per-row formula) and dW1,
    dW3, dW2 for the given experts (from all of that expert's rows). For
    full-size workloads whose whole backward would take too long on the CPU."""
    E = W1.shape[0]
    idx, gate, _ = route(logits, k)
    meta = routing_metadata(idx, E)
    tokens = np.asarray(tokens)
    dx = np.zeros((len(tokens), x.shape[1]))
    for i, t in enumerate(tokens):
        xt = to64(x[int(t)])
        dot = to64(dOut[int(t)])
        for j in range(k):
            e = int(idx[t, j])
            w1, w3, w2 = to64(W1[e]), to64(W3[e]), to64(W2[e])
            a, b = w1 @ xt, w3 @ xt
            dh = w2.T @ (gate[t, j] * dot)
            dx[i] += w1.T @ (dh * b * dsilu(a)) + w3.T @ (dh * silu(a))
    dW = {}
    for e in experts:
        e = int(e)
        toks, js = np.nonzero(idx == e)   # token-major order, as in the expert buffer
        X = to64(x[torch.as_tensor(toks, dtype=torch.long)]) if len(toks) else np.zeros((0, x.shape[1]))
        dY = (gate[toks, js][:, None] * to64(dOut[torch.as_tensor(toks, dtype=torch.long)])
              if len(toks) else np.zeros((0, x.shape[1])))
        off = np.array([0, len(toks)])
        _, g1, g3, g2 = expert_ffn_bwd(X, off, to64(W1[e:e + 1]), to64(W3[e:e + 1]),
                                       to64(W2[e:e + 1]), dY)
        dW[e] = (g1[0], g3[0], g2[0])
    return dict(dx=dx, dW=dW, idx=idx, gate=gate, tokens=tokens, **meta)


# --------------------------------------------------------------------------
# f3: backward of the MXFP8 layer
#     [NEWS "三招拆分、三项优化、一个精度开关": the MXFP8 switch speeds up
#      training through the FFN and the expert data movement; OF capability
#      table and "MXFP8 分块量化": 32-element blocks sharing one scale;
#      REL "主要功能": bf16 weight gradients]
# --------------------------------------------------------------------------

def _qdq_rows(m: np.ndarray, mode: str) -> np.ndarray:
    """Quantise-dequantise along the last axis (blocks of 32), float64 out."""
    q, st = mxfp8_quantize(np.asarray(m, np.float32), mode)
    return mxfp8_dequantize_f32(q, st, mode).astype(np.float64)


def _bf16(m: np.ndarray) -> np.ndarray:
    """fp32 value rounded to bf16 (round-to-nearest-even), as float64."""
    t = torch.from_numpy(np.ascontiguousarray(np.asarray(m, np.float32)))
    return t.to(torch.bfloat16).to(torch.float64).numpy()


def mxfp8_layer_bwd(x: torch.Tensor, dOut: torch.Tensor, k: int, W1, W3, W2,
                    logits: np.ndarray, mode: str = "e8m0", exact: bool = False,
                    return_ops: bool = False) -> Dict[str, np.ndarray]:
    """Backward of the MXFP8 layer (gates held constant). Reading (the pages
    leave the backward's precision open): the forward is mxfp8_layer's; the
    two input-gradient GEMMs quantise each operand along its contraction
    dimension,
        dH  = Q_d(dYe) Q_d(W2_e)                 (W2_e [d,F] quantised along d)
        dXe = Q_F([dA | dB]) Q_F([W1_e; W3_e])   ([W1_e; W3_e] along F)
    with dYe = gate * dOut[t] and dA = dH B silu'(A), dB = dH silu(A); the
    weight gradients use the forward's dequantised operands without a
    further quantisation: dW1 = dA^T Xd, dW3 = dB^T Xd, dW2 = dYe^T Hd.

    Values that decide a quantised code are taken in the precision the
    layer stores them in: dYe, dH and the pre-activations A, B are bf16
    tensors (rounded once from their fp32 value); dA, dB are formed from
    those and quantised from their fp32 value. Everything else is float64.

    exact=True replaces every quantise-dequantise and bf16 rounding by the
    identity, which must give moe_layer_bwd's gradients (a wiring check).
    return_ops=True adds, per expert, the operands as quantised."""
    qdq = (lambda m: np.asarray(m, np.float64)) if exact else (lambda m: _qdq_rows(m, mode))
    rnd = (lambda m: np.asarray(m, np.float64)) if exact else _bf16
    E, F, d = W1.shape
    idx, gate, _ = route(logits, k)
    meta = routing_metadata(idx, E)
    slot, offsets = meta["slot"], meta["offsets"]
    xd = qdq(to64(x))                              # token rows along d
    Xd = dispatch(xd, slot)
    dYe = rnd(dispatch(to64(dOut), slot, gate=gate))
    R = Xd.shape[0]
    dXe = np.zeros((R, d))
    dW1 = np.zeros((E, F, d)); dW3 = np.zeros((E, F, d)); dW2 = np.zeros((E, d, F))
    ops = {}
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 == r0:
            continue
        w1, w3, w2 = to64(W1[e]), to64(W3[e]), to64(W2[e])
        X = Xd[r0:r1]
        # forward (mxfp8_layer): weights along d, H along F from its fp32 value
        a_ex = X @ qdq(w1).T
        b_ex = X @ qdq(w3).T
        Hd = qdq(silu(a_ex) * b_ex)
        A, B = rnd(a_ex), rnd(b_ex)
        # backward
        dy = dYe[r0:r1]
        dyd = qdq(dy)                               # along d
        w2t = w2.T                                  # [F, d]: row f = column f of W2_e
        w2td = qdq(w2t)                             # along d
        dH = rnd(dyd @ w2td.T)
        da = dH * B * dsilu(A)
        db = dH * silu(A)
        dab = np.concatenate([da, db], axis=1)      # [rows, 2F]
        dabd = qdq(dab)                             # along F
        w13t = np.concatenate([w1.T, w3.T], axis=1)  # [d, 2F]: row i = W1_e[:, i] | W3_e[:, i]
        w13td = qdq(w13t)                           # along F
        dXe[r0:r1] = dabd @ w13td.T
        dW1[e] = da.T @ X
        dW3[e] = db.T @ X
        dW2[e] = dy.T @ Hd
        if return_ops:
            ops[e] = dict(dy=dy, dyd=dyd, w2t=w2t, w2td=w2td, dH=dH, A=A, B=B, da=da, db=db,
                          dab=dab, dabd=dabd, w13t=w13t, w13td=w13td, Hd=Hd, X=X)
    dx = combine(dXe, slot, None)
    res = dict(dx=dx, dW1=dW1, dW3=dW3, dW2=dW2, dXe=dXe, dYe=dYe, idx=idx, gate=gate, **meta)
    if return_ops:
        res["ops"] = ops
    return res


def mxfp8_layer_bwd_sampled(x: torch.Tensor, dOut: torch.Tensor, k: int, W1, W3, W2,
                            logits: np.ndarray, tokens, experts,
                            mode: str = "e8m0") -> Dict[str, np.ndarray]:
    """mxfp8_layer_bwd's gradients restricted to a sample, for full-size
    workloads: dx for the given tokens and dW1, dW3, dW2 for the given
    experts (from all of that expert's rows). Every quantisation in that
    reading is per row of an activation (the token rows of x, dYe, [dA | dB],
    H) or per weight, so a (token, choice) row's chain needs only its own
    row and its expert's weights, quantised once per expert here."""
    E, F, d = W1.shape
    idx, gate, _ = route(logits, k)
    meta = routing_metadata(idx, E)
    qdq = lambda m: _qdq_rows(m, mode)  # noqa: E731
    cache = {}

    def wq(e):
        if e not in cache:
            w1, w3, w2 = to64(W1[e]), to64(W3[e]), to64(W2[e])
            cache[e] = dict(w1d=qdq(w1), w3d=qdq(w3), w2td=qdq(w2.T),
                            w13td=qdq(np.concatenate([w1.T, w3.T], axis=1)))
        return cache[e]

    def rows(e, toks, js):
        w = wq(e)
        tt = torch.as_tensor(np.asarray(toks), dtype=torch.long)
        X = qdq(to64(x[tt]))                                   # token rows along d
        a, b = X @ w["w1d"].T, X @ w["w3d"].T
        Hd = qdq(silu(a) * b)                                  # H along F
        A, B = _bf16(a), _bf16(b)
        dy = _bf16(gate[toks, js][:, None] * to64(dOut[tt]))   # bf16 of gate * dOut
        dH = _bf16(qdq(dy) @ w["w2td"].T)                      # dYe along d
        da = dH * B * dsilu(A)
        db = dH * silu(A)
        dXe = qdq(np.concatenate([da, db], axis=1)) @ w["w13td"].T  # [dA | dB] along F
        return X, Hd, dy, da, db, dXe

    tokens = np.asarray(tokens)
    dx = np.zeros((len(tokens), d))
    for i, t in enumerate(tokens):
        for j in range(k):
            dx[i] += rows(int(idx[t, j]), np.array([t]), np.array([j]))[5][0]
    dW = {}
    for e in experts:
        e = int(e)
        toks, js = np.nonzero(idx == e)  # token-major: the expert buffer's order
        if len(toks) == 0:
            dW[e] = (np.zeros((F, d)), np.zeros((F, d)), np.zeros((d, F)))
            continue
        X, Hd, dy, da, db, _ = rows(e, toks, js)
        dW[e] = (da.T @ X, db.T @ X, dy.T @ Hd)
    return dict(dx=dx, dW=dW, idx=idx, gate=gate, tokens=tokens, **meta)


# --------------------------------------------------------------------------
# f2: router backward and the load-balancing auxiliary loss
#     [HF §2 router (fp32 softmax, top-k, optional norm_topk_prob);
#      HF §4 "负载均衡辅助损失": Switch-Transformer-style loss from the
#      per-expert assignment frequency and the routing probability
#      distribution, multiplied and summed; router_aux_loss_coef (0.01 by
#      default) scales it into the total loss]
# --------------------------------------------------------------------------

def aux_loss(logits: np.ndarray, idx: np.ndarray) -> float:
    """aux = E * sum_e f_e * P_e with f_e = (number of (t, j) routed to e) / T
    and P_e = mean over tokens of softmax(logits_t)_e. Reading: every one of a
    token's k choices counts toward f (so a uniform router gives aux = k),
    and the factor E is Switch Transformer's expert-count scaling."""
    T, E = np.asarray(logits).shape
    p = softmax_fp64(logits)
    f = np.bincount(np.asarray(idx).reshape(-1), minlength=E).astype(np.float64) / T
    P = p.mean(axis=0)
    return float(E * (f * P).sum())


def gate_grad(dOut: np.ndarray, Y: np.ndarray) -> np.ndarray:
    """dgate[t, j] = <dOut[t], Y[t, j]>, Y[t, j] = the j-th chosen expert's
    output for token t (before gating): the gradient of out[t] = sum_j
    gate[t, j] Y[t, j] with respect to the gate."""
    return np.einsum("td,tjd->tj", np.asarray(dOut, np.float64), np.asarray(Y, np.float64))


def router_grad(logits: np.ndarray, idx: np.ndarray, dgate: np.ndarray, renorm: bool = False,
                aux_coef: float = 0.0) -> np.ndarray:
    """dlogits [T,E] for a loss L(gates) + aux_coef * aux_loss, with the top-k
    choice and the counts held fixed (both are piecewise constant).

    gate[t,j] = p[t, idx[t,j]] (renorm: divided by S_t = sum_j p[t, idx[t,j]]),
    p = softmax(logits[t]). Chain rule: the gradient reaching p,
      dp[t,e] = sum_j [idx[t,j] = e] dsel[t,j] + aux_coef * E * f_e / T,
      dsel = dgate (renorm: (dgate - sum_i gate_i dgate_i) / S_t),
    then the softmax Jacobian: dlogits = p * (dp - sum_e p dp)."""
    p = softmax_fp64(logits)
    T, E = p.shape
    idx = np.asarray(idx).astype(np.int64)
    dg = np.asarray(dgate, np.float64)
    if renorm:
        sel = np.take_along_axis(p, idx, axis=1)
        S = sel.sum(axis=1, keepdims=True)
        g = sel / S
        dsel = (dg - (g * dg).sum(axis=1, keepdims=True)) / S
    else:
        dsel = dg
    dp = np.zeros((T, E))
    for j in range(idx.shape[1]):
        dp[np.arange(T), idx[:, j]] += dsel[:, j]
    if aux_coef:
        f = np.bincount(idx.reshape(-1), minlength=E).astype(np.float64) / T
        dp += aux_coef * E * f / T
    return p * (dp - (p * dp).sum(axis=1, keepdims=True))


def router_linear_grad(dlogits: np.ndarray, x, Wr):
    """logits = x Wr^T: dx = dlogits Wr [T,d], dWr = dlogits^T x [E,d]."""
    dl = np.asarray(dlogits, np.float64)
    return dl @ to64(Wr), dl.T @ to64(x)


# --------------------------------------------------------------------------
# error measures used by the parity tests
# --------------------------------------------------------------------------

def rel_l2(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = math.sqrt(float((ref * ref).sum()))
    num = math.sqrt(float(((got - ref) ** 2).sum()))
    return num / den if den > 0 else num


def max_abs(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(got - ref).max()) if got.size else 0.0
