"""MXFP8 backward on the GPU against the oracle: the backward weights
(transposed re-quantisation, codes and scales bit-exact), the SwiGLU
backward step with its quantisation, and the whole MXFP8 layer backward
against the oracle's MXFP8 backward (the same reading: FP8 input-gradient
GEMMs with operands quantised along their contraction dimension, bf16 weight
gradients on the forward's dequantised operands)."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from dropless_top_mixture_b200.workloads import adversarial_logits
from tests._util import assert_close_scaled, np64, rel_l2

pytestmark = pytest.mark.gpu


def _moe():
    from dropless_top_mixture_b200 import moe
    return moe


def _weights(E, d, F, seed):
    g = torch.Generator().manual_seed(seed)
    bf = torch.bfloat16
    W1 = (torch.randn(E, F, d, generator=g) * d ** -0.5).to(bf)
    W3 = (torch.randn(E, F, d, generator=g) * d ** -0.5).to(bf)
    W2 = (torch.randn(E, d, F, generator=g) * F ** -0.5).to(bf)
    return W1, W3, W2


@pytest.mark.parametrize("E,d,F,fused", [(2, 256, 128, False), (3, 128, 256, False),
                                         (2, 256, 256, True)])
def test_quantize_weights_bwd_bit_exact(E, d, F, fused):
    """W13tq row i = (column i of W1_e | column i of W3_e) quantised along F,
    W2tq row f = column f of W2_e quantised along d: codes and UE8M0 scale
    bytes equal the oracle's codec on the transposed weights."""
    moe = _moe()
    W1, W3, W2 = _weights(E, d, F, seed=E * 7 + d + F)
    g = torch.Generator().manual_seed(5)
    W1[0, :, :32] *= 64.0  # blocks of very different scale
    W2[-1, :32, :] *= 2.0 ** -12
    if fused:
        W13 = torch.cat([W1, W3], dim=1).cuda()  # [E, 2F, d]; views with expert stride 2F*d
        w1d, w3d = W13[:, :F], W13[:, F:]
    else:
        w1d, w3d = W1.cuda(), W3.cuda()
    wb = moe.mxfp8_quantize_weights_bwd(w1d, w3d, W2.cuda())
    torch.cuda.synchronize()
    assert moe.moe_get_status() == 0
    for e in range(E):
        both = np.concatenate([W1[e].float().numpy().T, W3[e].float().numpy().T], axis=1)
        q, s = O.mxfp8_quantize(both, "e8m0")
        assert np.array_equal(wb.W13tq[e].cpu().numpy(), q)
        assert np.array_equal(wb.W13ts[e].cpu().numpy(), s)
        q, s = O.mxfp8_quantize(W2[e].float().numpy().T, "e8m0")
        assert np.array_equal(wb.W2tq[e].cpu().numpy(), q)
        assert np.array_equal(wb.W2ts[e].cpu().numpy(), s)


def test_swiglu_bwd_mxfp8_step():
    """dA = dH B silu'(A), dB = dH silu(A) from bf16 inputs, stored in bf16
    (one rounding of an fp32 value), and the MXFP8 codes of [dA | dB]
    quantised from the fp32 values: against the oracle's codec on the exact
    values, codes may differ only where the fp32 and float64 values fall on
    either side of a rounding boundary."""
    moe = _moe()
    R, F = 300, 256
    g = torch.Generator().manual_seed(41)
    dH = torch.randn(R, F, generator=g).to(torch.bfloat16)
    A = (torch.randn(R, F, generator=g) * 3).to(torch.bfloat16)
    B = torch.randn(R, F, generator=g).to(torch.bfloat16)
    dA, dB, q, s = moe.moe_swiglu_bwd_mxfp8(dH.cuda(), A.cuda(), B.cuda())
    torch.cuda.synchronize()
    assert moe.moe_get_status() == 0
    h, a, b = (t.double().numpy() for t in (dH, A, B))
    da = h * b * O.dsilu(a)
    db = h * O.silu(a)
    for got, ref, mag in ((dA, da, np.abs(h * b)), (dB, db, np.abs(h * a))):
        err = np.abs(np64(got) - ref)
        assert np.all(err <= 2.0 ** -8 * np.abs(ref) + 1e-6 * mag)
    qr, sr = O.mxfp8_quantize(np.concatenate([da, db], axis=1), "e8m0")
    qg, sg = q.cpu().numpy(), s.cpu().numpy()
    assert np.mean(qg == qr) > 0.999 and np.mean(sg == sr) > 0.999
    deq_g = O.mxfp8_dequantize_f32(qg, sg, "e8m0").astype(np.float64)
    deq_r = O.mxfp8_dequantize_f32(qr, sr, "e8m0").astype(np.float64)
    assert rel_l2(deq_g, deq_r) < 1e-3


def _layer_problem(T, d, F, E, k, seed):
    W1, W3, W2 = _weights(E, d, F, seed)
    g = torch.Generator().manual_seed(seed + 1)
    x = torch.randn(T, d, generator=g).to(torch.bfloat16)
    dOut = torch.randn(T, d, generator=g).to(torch.bfloat16)
    lg = adversarial_logits(T, E, "normal", seed=seed).numpy()
    if E >= 4:
        lg[:, 1] -= 40.0  # expert 1 gets no rows: zero weight gradients
    return x, dOut, W1, W3, W2, lg


def _run_layer(moe, x, dOut, W1, W3, W2, lg, k):
    dev = "cuda"
    w = moe.mxfp8_quantize_weights(W1.to(dev), W3.to(dev), W2.to(dev))
    wb = moe.mxfp8_quantize_weights_bwd(W1.to(dev), W3.to(dev), W2.to(dev))
    fw = moe.moe_layer_fwd_mxfp8(x.to(dev), k, w, logits=torch.from_numpy(lg).to(dev), save=True)
    gr = moe.moe_layer_bwd_mxfp8(fw, dOut.to(dev), k, wb)
    torch.cuda.synchronize()
    assert moe.moe_get_status() == 0
    return w, wb, fw, gr


@pytest.mark.parametrize("T,d,F,E,k", [(300, 256, 256, 8, 2), (77, 512, 256, 4, 3),
                                       (1, 256, 256, 2, 1)])
def test_layer_bwd_mxfp8_against_oracle(T, d, F, E, k):
    moe = _moe()
    x, dOut, W1, W3, W2, lg = _layer_problem(T, d, F, E, k, seed=T + d + E)
    _, _, fw, gr = _run_layer(moe, x, dOut, W1, W3, W2, lg, k)
    ref = O.mxfp8_layer_bwd(x, dOut, k, W1, W3, W2, lg, return_ops=True)
    assert np.array_equal(fw.idx.cpu().numpy(), ref["idx"])
    # the saved pre-activations: bf16 of the fp32 accumulation
    off = ref["offsets"]
    for e, op in ref["ops"].items():
        r0, r1 = int(off[e]), int(off[e + 1])
        for name in ("A", "B"):
            got = np64(getattr(fw, name)[r0:r1])
            assert rel_l2(got, op[name]) < 1e-3, (e, name)
    for name in ("dx", "dW1", "dW3", "dW2"):
        assert_close_scaled(np64(getattr(gr, name)), ref[name], f"{name} vs MXFP8 oracle")
    if E >= 4:
        for name in ("dW1", "dW3", "dW2"):
            assert torch.count_nonzero(getattr(gr, name)[1]) == 0
    exact = O.moe_layer_bwd(x, dOut, k, W1, W3, W2, lg)
    print(f"\nMXFP8 backward vs exact backward: "
          + ", ".join(f"{n} {rel_l2(np64(getattr(gr, n)), exact[n]):.4f}"
                      for n in ("dx", "dW1", "dW3", "dW2")))


def test_layer_bwd_mxfp8_medium_against_oracle():
    """A larger case: many ragged experts, several 128-row tiles each."""
    moe = _moe()
    T, d, F, E, k = 2048, 1024, 512, 16, 4
    x, dOut, W1, W3, W2, lg = _layer_problem(T, d, F, E, k, seed=5)
    _, _, fw, gr = _run_layer(moe, x, dOut, W1, W3, W2, lg, k)
    ref = O.mxfp8_layer_bwd(x, dOut, k, W1, W3, W2, lg)
    for name in ("dx", "dW1", "dW3", "dW2"):
        assert_close_scaled(np64(getattr(gr, name)), ref[name], f"{name} vs MXFP8 oracle")


def test_layer_bwd_mxfp8_matches_its_steps_and_is_deterministic():
    """moe_layer_bwd_mxfp8 equals, bit for bit, the chain of its public
    steps (the calls the benchmark times one by one), and two runs agree."""
    moe = _moe()
    T, d, F, E, k = 300, 256, 512, 8, 2
    x, dOut, W1, W3, W2, lg = _layer_problem(T, d, F, E, k, seed=9)
    w, wb, fw, gr = _run_layer(moe, x, dOut, W1, W3, W2, lg, k)
    dO = dOut.cuda()
    R = T * k
    off = fw.offsets
    dYe = moe.moe_dispatch(dO, fw.slot, gate=fw.gate)
    dYq, dYs = moe.mxfp8_quantize(dYe)
    dYsp = moe.mxfp8_pack_act_scales(dYs, off, E)
    dH = moe.moe_grouped_mxfp8_gemm(dYq, dYsp, wb.W2tq, wb.Ps2t, off)
    dA, dB, dq, ds = moe.moe_swiglu_bwd_mxfp8(dH, fw.A, fw.B)
    dsp = moe.mxfp8_pack_act_scales(ds, off, E)
    dXe = moe.moe_grouped_mxfp8_gemm(dq, dsp, wb.W13tq, wb.Ps13t, off)
    dx = moe.moe_combine(dXe, fw.slot, None)
    Xd = moe.mxfp8_dequantize(fw.Xq, fw.Xs)
    Hs = moe.mxfp8_unpack_act_scales(fw.Hsp, off, E, R, F)
    Hd = moe.mxfp8_dequantize(fw.Hq, Hs)
    dW1, dW3, dW2 = moe.moe_grouped_swiglu_wgrad(Xd, dA, dB, dYe, Hd, off)
    torch.cuda.synchronize()
    assert moe.moe_get_status() == 0
    for got, step in ((gr.dx, dx), (gr.dW1, dW1), (gr.dW3, dW3), (gr.dW2, dW2)):
        assert torch.equal(got, step)
    gr2 = moe.moe_layer_bwd_mxfp8(fw, dO, k, wb)
    torch.cuda.synchronize()
    for name in ("dx", "dW1", "dW3", "dW2"):
        assert torch.equal(getattr(gr, name), getattr(gr2, name))


def test_layer_bwd_mxfp8_rejects_bad_arguments():
    moe = _moe()
    T, d, F, E, k = 64, 256, 256, 4, 2
    x, dOut, W1, W3, W2, lg = _layer_problem(T, d, F, E, k, seed=3)
    w = moe.mxfp8_quantize_weights(W1.cuda(), W3.cuda(), W2.cuda())
    wb = moe.mxfp8_quantize_weights_bwd(W1.cuda(), W3.cuda(), W2.cuda())
    fw = moe.moe_layer_fwd_mxfp8(x.cuda(), k, w, logits=torch.from_numpy(lg).cuda())
    with pytest.raises(ValueError):
        moe.moe_layer_bwd_mxfp8(fw, dOut.cuda(), k, wb)  # forward without save
    fw = moe.moe_layer_fwd_mxfp8(x.cuda(), k, w, logits=torch.from_numpy(lg).cuda(), save=True)
    gr = moe.moe_layer_bwd_mxfp8(fw, dOut.cuda(), k, wb)
    ws = gr.workspace
    gr.workspace = ws[: ws.numel() // 2]
    with pytest.raises(RuntimeError):
        moe.moe_layer_bwd_mxfp8(fw, dOut.cuda(), k, wb, out=gr)
    torch.cuda.synchronize()
    assert moe.moe_get_status() == 0


@pytest.mark.slow
def test_layer_bwd_mxfp8_full_size_sampled():
    """The MXFP8 backward of the 128-expert workload (T=8192, d=4096,
    F=2048, top-4) at full size, in the launch configuration the benchmark
    times, against the oracle's MXFP8 backward restricted to a sample: dx of
    one token and the weight gradients of one of its experts (the oracle
    re-quantises each expert's weights in numpy, about 18 s per expert)."""
    from dropless_top_mixture_b200.workloads import WORKLOADS, make_inputs
    moe = _moe()
    wl = WORKLOADS["mxfp8_e128"].scaled(backward=True)
    inp = make_inputs(wl, "cuda")
    w = moe.mxfp8_quantize_weights(inp["W1"], inp["W3"], inp["W2"])
    wb = moe.mxfp8_quantize_weights_bwd(inp["W1"], inp["W3"], inp["W2"])
    fw = moe.moe_layer_fwd_mxfp8(inp["x"], wl.k, w, logits=inp["logits"], save=True)
    gr = moe.moe_layer_bwd_mxfp8(fw, inp["dOut"], wl.k, wb)
    torch.cuda.synchronize()
    assert moe.moe_get_status() == 0
    lg = inp["logits"].cpu().numpy()
    tok = wl.T // 2 + 17
    e = int(fw.idx[tok, 0].item())
    W1, W3, W2 = (inp[n].cpu() for n in ("W1", "W3", "W2"))
    ref = O.mxfp8_layer_bwd_sampled(inp["x"].cpu(), inp["dOut"].cpu(), wl.k, W1, W3, W2, lg,
                                    [tok], [e])
    assert np.array_equal(fw.idx.cpu().numpy(), ref["idx"])
    assert_close_scaled(np64(gr.dx[tok:tok + 1]), ref["dx"], "dx (sampled token)")
    for name, r in zip(("dW1", "dW3", "dW2"), ref["dW"][e]):
        assert_close_scaled(np64(getattr(gr, name)[e]), r, f"{name} of expert {e}")
