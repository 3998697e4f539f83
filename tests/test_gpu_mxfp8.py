"""MXFP8 path on the GPU against the oracle: the quantising dispatch
(codes and scales bit-exact), the block-scaled grouped GEMMs on operands the
oracle quantised, and the whole MXFP8 layer against the MXFP8 oracle, with
its distance to the bf16 oracle measured."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from dropless_top_mixture_b200.workloads import WORKLOADS, adversarial_logits, make_inputs
from tests._util import assert_close_layer, assert_close_scaled, np64, rel_l2

pytestmark = pytest.mark.gpu


def _moe():
    from dropless_top_mixture_b200 import moe
    return moe


def _deq(q, s):
    return O.mxfp8_dequantize_f32(q, s, "e8m0").astype(np.float64)


def _quant_w(W):
    """Oracle quantisation of [E, N, K] weights along K -> codes, scales."""
    E, N, K = W.shape
    q, s = O.mxfp8_quantize(W.reshape(E * N, K).float().numpy(), "e8m0")
    return q.reshape(E, N, K), s.reshape(E, N, K // 32)


def _problem(T, d, F, E, k, seed):
    g = torch.Generator().manual_seed(seed)
    bf = torch.bfloat16
    x = torch.randn(T, d, generator=g).to(bf)
    W1 = (torch.randn(E, F, d, generator=g) * d ** -0.5).to(bf)
    W3 = (torch.randn(E, F, d, generator=g) * d ** -0.5).to(bf)
    W2 = (torch.randn(E, d, F, generator=g) * F ** -0.5).to(bf)
    lg = adversarial_logits(T, E, "normal", seed=seed).numpy()
    if E >= 4:
        lg[:, 1] -= 40.0
        lg[:, 0] += 3.0
    return x, W1, W3, W2, lg


def test_dispatch_mxfp8_bitexact():
    moe = _moe()
    T, d, E, k = 300, 512, 8, 3
    x, *_ , lg = _problem(T, d, 128, E, k, seed=3)
    idx, gate, _ = O.route(lg, k)
    meta = O.routing_metadata(idx, E)
    Xq, Xs = moe.moe_dispatch_mxfp8(x.cuda(), torch.from_numpy(meta["slot"]).cuda())
    q, s = O.mxfp8_quantize(x.float().numpy(), "e8m0")
    assert np.array_equal(Xq.cpu().numpy(), O.dispatch(q, meta["slot"]))
    assert np.array_equal(Xs.cpu().numpy(), O.dispatch(s, meta["slot"]))


@pytest.mark.parametrize("T,d,F,E,k", [(300, 256, 256, 5, 2), (700, 512, 384, 16, 4),
                                       (37, 128, 128, 4, 2), (200, 384, 256, 6, 3)])
def test_grouped_mxfp8_gemms(T, d, F, E, k):
    moe = _moe()
    x, W1, W3, W2, lg = _problem(T, d, F, E, k, seed=T + d + F)
    idx, gate, _ = O.route(lg, k)
    meta = O.routing_metadata(idx, E)
    offs = meta["offsets"]
    xq, xs = O.mxfp8_quantize(x.float().numpy(), "e8m0")
    Xq, Xs = O.dispatch(xq, meta["slot"]), O.dispatch(xs, meta["slot"])
    (w1q, w1s), (w3q, w3s), (w2q, w2s) = _quant_w(W1), _quant_w(W3), _quant_w(W2)
    dev = "cuda"
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    w = moe.MxWeights(t(w1q), t(w1s), t(w3q), t(w3s), t(w2q), t(w2s))
    Hq, Hs = moe.moe_grouped_gate_up_mxfp8(t(Xq), t(Xs), w, t(offs))
    # oracle: exact products of the dequantised operands, then SwiGLU
    Xd = _deq(Xq, Xs)
    H = np.zeros((T * k, F))
    for e in range(E):
        r0, r1 = offs[e], offs[e + 1]
        if r1 > r0:
            a = Xd[r0:r1] @ _deq(w1q[e], w1s[e]).T
            b = Xd[r0:r1] @ _deq(w3q[e], w3s[e]).T
            H[r0:r1] = O.silu(a) * b
    Hq_g, Hs_g = Hq.cpu().numpy(), Hs.cpu().numpy()
    Hd_g = _deq(Hq_g, Hs_g)
    hq_ref, hs_ref = O.mxfp8_quantize(H.astype(np.float32), "e8m0")
    # fp32 accumulation on the GPU moves a few values across a rounding
    # boundary of the E4M3 grid; almost every code and scale is identical
    assert np.mean(Hq_g == hq_ref) > 0.99 and np.mean(Hs_g == hs_ref) > 0.99
    assert rel_l2(Hd_g, _deq(hq_ref, hs_ref)) < 1e-2
    # down GEMM on the oracle's own quantised H
    Ye = moe.moe_grouped_down_mxfp8(t(hq_ref), t(hs_ref), w, t(offs))
    Hd = _deq(hq_ref, hs_ref)
    Ye_ref = np.zeros((T * k, d))
    for e in range(E):
        r0, r1 = offs[e], offs[e + 1]
        if r1 > r0:
            Ye_ref[r0:r1] = Hd[r0:r1] @ _deq(w2q[e], w2s[e]).T
    assert moe.moe_get_status() == 0
    assert_close_scaled(np64(Ye), Ye_ref, "Ye")


def test_layer_mxfp8_small():
    moe = _moe()
    T, d, F, E, k = 500, 256, 256, 8, 2
    x, W1, W3, W2, lg = _problem(T, d, F, E, k, seed=11)
    dev = "cuda"
    w = moe.mxfp8_quantize_weights(W1.to(dev), W3.to(dev), W2.to(dev))
    r = moe.moe_layer_fwd_mxfp8(x.to(dev), k, w, logits=torch.from_numpy(lg).to(dev))
    torch.cuda.synchronize()
    assert moe.moe_get_status() == 0
    ref = O.mxfp8_layer(x, k, W1, W3, W2, lg)
    assert np.array_equal(r.idx.cpu().numpy(), ref["idx"])
    assert_close_layer(np64(r.out), ref["out"], "out vs MXFP8 oracle")


@pytest.mark.slow
def test_layer_mxfp8_full_size_sampled():
    """The MXFP8 variant of the 128-expert sweep workload (T=8192, d=4096,
    F=2048, top-4): the output on sampled tokens against the MXFP8 oracle
    (bar: rel-L2 1e-2) and, measured, against the bf16 oracle."""
    moe = _moe()
    wl = WORKLOADS["mxfp8_e128"]
    inp = make_inputs(wl, "cuda")
    w = moe.mxfp8_quantize_weights(inp["W1"], inp["W3"], inp["W2"])
    r = moe.moe_layer_fwd_mxfp8(inp["x"], wl.k, w, logits=inp["logits"])
    torch.cuda.synchronize()
    assert moe.moe_get_status() == 0
    rng = np.random.default_rng(2)
    toks = np.sort(rng.choice(wl.T, size=16, replace=False))
    lg = inp["logits"].cpu().numpy()
    x_cpu = inp["x"].cpu()
    ref = O.mxfp8_layer(x_cpu, wl.k, inp["W1"], inp["W3"], inp["W2"], lg, tokens=toks)
    got = np64(r.out[torch.as_tensor(toks, device="cuda")])
    assert_close_layer(got, ref["out"], "MXFP8 layer vs MXFP8 oracle")
    idx, gate, _ = O.route(lg, wl.k)
    bf = O.moe_layer_tokens(x_cpu, toks, idx, gate, inp["W1"], inp["W3"], inp["W2"])
    gap = rel_l2(got, bf)
    print(f"\nMXFP8 layer vs bf16 oracle: rel-L2 {gap:.4f}; "
          f"MXFP8 oracle vs bf16 oracle: rel-L2 {rel_l2(ref['out'], bf):.4f}")
    assert gap < 0.1


@pytest.mark.parametrize("E,d,F", [(3, 256, 128), (2, 128, 384), (2, 384, 256)])
def test_pack_weight_scales_layout(E, d, F):
    """The packed weight scales are a permutation of the row-layout scale
    bytes, as the header defines it: for block (e, nb, s, half) of 512 bytes,
    the row m of that half's 128 tile rows has its four K-block bytes at
    16*(m % 32) + 4*(m / 32); rows past the matrix are zero."""
    moe = _moe()
    g = torch.Generator().manual_seed(E + d + F)
    s1 = torch.randint(0, 256, (E, F, d // 32), generator=g, dtype=torch.uint8)
    s3 = torch.randint(0, 256, (E, F, d // 32), generator=g, dtype=torch.uint8)
    s2 = torch.randint(0, 256, (E, d, F // 32), generator=g, dtype=torch.uint8)
    z = lambda *sh: torch.zeros(*sh, dtype=torch.uint8, device="cuda")
    w = moe.MxWeights(z(E, F, d), s1.cuda(), z(E, F, d), s3.cuda(), z(E, d, F), s2.cuda())
    moe.mxfp8_pack_weight_scales(w)
    got13 = w.Ps13.cpu().numpy()
    got2 = w.Ps2.cpu().numpy()

    def block(rows_bytes):            # rows_bytes: [<= 128 rows, 4 bytes]
        b = np.zeros(512, dtype=np.uint8)
        for m in range(rows_bytes.shape[0]):
            o = 16 * (m % 32) + 4 * (m // 32)
            b[o:o + 4] = rows_bytes[m]
        return b

    want13 = []
    for e in range(E):
        for nb in range(F // 128):
            halves = [s1[e, 128 * nb:128 * nb + 128].numpy(),
                      s3[e, 128 * nb:128 * nb + 128].numpy()]
            for s in range(d // 128):
                for rows in halves:
                    want13.append(block(rows[:, 4 * s:4 * s + 4]))
    want2 = []
    for e in range(E):
        for nb in range((d + 255) // 256):
            halves = [s2[e, 256 * nb:256 * nb + 128].numpy(),
                      s2[e, 256 * nb + 128:256 * nb + 256].numpy()]
            for s in range(F // 128):
                for rows in halves:
                    want2.append(block(rows[:, 4 * s:4 * s + 4]))
    assert np.array_equal(got13, np.concatenate(want13))
    assert np.array_equal(got2, np.concatenate(want2))


@pytest.mark.parametrize("counts,K", [([0, 130, 1, 256, 5], 256), ([300], 128), ([7, 0, 0, 129], 512),
                                      ([200, 57], 4352), ([128, 256], 4096)])
def test_act_scales_pack_layout_and_roundtrip(counts, K):
    """Tile-packed activation scales as the header defines them: row tiles
    of 128 per expert (ceil(count/128) each, numbered in expert order), one
    512-byte block per (tile, K slab), word of tile row m at
    16*(m % 32) + 4*(m / 32), tile rows past the expert's rows zero; unpack
    restores the rows."""
    moe = _moe()
    E = len(counts)
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R = int(offs[-1])
    g = torch.Generator().manual_seed(R + K)
    S = torch.randint(0, 256, (R, K // 32), generator=g, dtype=torch.uint8)
    Sp = moe.mxfp8_pack_act_scales(S.cuda(), torch.from_numpy(offs).cuda(), E)
    got = Sp.cpu().numpy()
    ks = K // 128
    want = []
    for e in range(E):
        rows = S[offs[e]:offs[e + 1]].numpy()
        for mt in range((counts[e] + 127) // 128):
            tile = rows[128 * mt:128 * mt + 128]
            for s in range(ks):
                b = np.zeros(512, dtype=np.uint8)
                for m in range(tile.shape[0]):
                    o = 16 * (m % 32) + 4 * (m // 32)
                    b[o:o + 4] = tile[m, 4 * s:4 * s + 4]
                want.append(b)
    want = np.concatenate(want) if want else np.zeros(0, np.uint8)
    assert np.array_equal(got[:want.size], want)
    back = moe.mxfp8_unpack_act_scales(Sp, torch.from_numpy(offs).cuda(), E, R, K)
    assert np.array_equal(back.cpu().numpy(), S.numpy())
    assert moe.moe_get_status() == 0


def test_act_scales_bad_offsets_flagged():
    moe = _moe()
    offs = torch.tensor([0, 40, 30, 64], dtype=torch.int32, device="cuda")  # not monotone
    S = torch.zeros((64, 4), dtype=torch.uint8, device="cuda")
    Sp = torch.full((moe.lib.mxfp8_act_scales_packed_size(3, 64, 128),), 7, dtype=torch.uint8,
                    device="cuda")
    moe.mxfp8_pack_act_scales(S, offs, 3, Sp)
    torch.cuda.synchronize()
    assert moe.moe_get_status(clear=True) & moe.MOE_DEVERR_BAD_OFFSETS
    assert (Sp.cpu() == 7).all()  # nothing written
    assert moe.moe_get_status() == 0
