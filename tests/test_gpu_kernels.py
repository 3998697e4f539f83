"""Dispatch, combine and the MXFP8 codec on the GPU against the oracle."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from dropless_top_mixture_b200.workloads import adversarial_logits
from tests._util import np64

pytestmark = pytest.mark.gpu


def _moe():
    from dropless_top_mixture_b200 import moe
    return moe


def _routing(T, E, k, seed):
    lg = adversarial_logits(T, E, "normal", seed=seed).numpy()
    idx, gate, _ = O.route(lg, k)
    meta = O.routing_metadata(idx, E)
    return gate, meta


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T,d,E,k", [(1, 8, 4, 2), (33, 136, 8, 3), (517, 2048, 64, 8),
                                     (64, 7168, 384, 8), (100, 4096, 128, 4)])
def test_dispatch_bitwise(dtype, T, d, E, k):
    moe = _moe()
    gate, meta = _routing(T, E, k, seed=T + d)
    x = torch.randn(T, d, generator=torch.Generator().manual_seed(d)).to(dtype)
    slot = torch.from_numpy(meta["slot"])
    Xe = moe.moe_dispatch(x.cuda(), slot.cuda()).cpu()
    view = torch.int16 if dtype == torch.bfloat16 else torch.int32
    ref = O.dispatch(x.view(view).numpy(), meta["slot"])
    assert np.array_equal(Xe.view(view).numpy(), ref)


def test_dispatch_scaled_by_gate():
    moe = _moe()
    T, d, E, k = 200, 256, 16, 4
    gate, meta = _routing(T, E, k, seed=3)
    x = torch.randn(T, d, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    g32 = torch.from_numpy(gate).float()
    Xe = moe.moe_dispatch(x.cuda(), torch.from_numpy(meta["slot"]).cuda(), gate=g32.cuda())
    ref = O.dispatch(x.double().numpy(), meta["slot"], gate=g32.double().numpy())
    # one fp32 product rounded to bf16: bf16 unit roundoff is 2^-8 (8 significant bits)
    got = np64(Xe)
    assert np.all(np.abs(got - ref) <= (2.0 ** -8 + 2.0 ** -23) * np.abs(ref) + 1e-30)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T,d,E,k", [(1, 8, 4, 2), (33, 136, 8, 3), (517, 2048, 64, 8)])
def test_dispatch_gate_records_row_gates(dtype, T, d, E, k):
    """The gate-recording dispatch writes the same rows as moe_dispatch, bit
    for bit, and row_gate[slot[t,j]] = gate[t,j] exactly."""
    moe = _moe()
    gate, meta = _routing(T, E, k, seed=T + 7)
    x = torch.randn(T, d, generator=torch.Generator().manual_seed(d + 1)).to(dtype).cuda()
    slot = torch.from_numpy(meta["slot"]).cuda()
    g32 = torch.from_numpy(gate).float().cuda()
    Xe, row_gate = moe.moe_dispatch_gate(x, slot, g32)
    assert moe.moe_get_status() == 0
    assert torch.equal(Xe, moe.moe_dispatch(x, slot))
    want = np.empty(T * k, dtype=np.float32)
    want[meta["slot"].reshape(-1)] = gate.astype(np.float32).reshape(-1)
    assert np.array_equal(row_gate.cpu().numpy(), want)


def test_dispatch_gate_flags_bad_slot():
    moe = _moe()
    x = torch.ones(2, 64, dtype=torch.bfloat16, device="cuda")
    slot = torch.tensor([[0, 1], [2, 9]], dtype=torch.int32, device="cuda")  # 9 >= R = 4
    gate = torch.full((2, 2), 0.5, device="cuda")
    row_gate = torch.full((4,), -1.0, device="cuda")
    moe.moe_dispatch_gate(x, slot, gate, row_gate=row_gate)
    assert moe.moe_get_status() == moe.MOE_DEVERR_BAD_INDEX
    assert row_gate.tolist() == [0.5, 0.5, 0.5, -1.0]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T,d,E,k", [(1, 8, 4, 2), (33, 136, 8, 3), (517, 2048, 64, 8),
                                     (64, 7168, 384, 8)])
def test_combine(dtype, T, d, E, k):
    moe = _moe()
    gate, meta = _routing(T, E, k, seed=T * 7 + d)
    R = T * k
    Ye = torch.randn(R, d, generator=torch.Generator().manual_seed(R)).to(dtype)
    g32 = torch.from_numpy(gate).float()
    out = moe.moe_combine(Ye.cuda(), torch.from_numpy(meta["slot"]).cuda(), g32.cuda())
    ref = O.combine(Ye.double().numpy(), meta["slot"], g32.double().numpy())
    got = np64(out)
    absum = O.combine(np.abs(Ye.double().numpy()), meta["slot"], np.abs(g32.double().numpy()))
    # fp32 fma chain of k terms (k * 2^-24 of sum|terms|) + final rounding
    unit = 2.0 ** -8 if dtype == torch.bfloat16 else 2.0 ** -24
    assert np.all(np.abs(got - ref) <= unit * np.abs(ref) + (k + 1) * 2.0 ** -24 * absum * 2)


def test_combine_identity_experts_and_unit_gates():
    moe = _moe()
    T, d, E, k = 300, 512, 32, 4
    gate, meta = _routing(T, E, k, seed=9)
    x = torch.randn(T, d, generator=torch.Generator().manual_seed(2)).to(torch.float32)
    slot = torch.from_numpy(meta["slot"]).cuda()
    Xe = moe.moe_dispatch(x.cuda(), slot)
    g32 = torch.from_numpy(gate).float()
    out = moe.moe_combine(Xe, slot, g32.cuda()).cpu().double().numpy()
    expect = g32.double().sum(1, keepdim=True).numpy() * x.double().numpy()
    assert np.allclose(out, expect, rtol=1e-6, atol=1e-6)
    out1 = moe.moe_combine(Xe, slot, None).cpu().double().numpy()
    assert np.allclose(out1, k * x.double().numpy(), rtol=1e-6, atol=1e-6)


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_mxfp8_quantize_bitexact(mode, dtype):
    moe = _moe()
    g = torch.Generator().manual_seed(17 + mode)
    v = torch.randn(96, 512, generator=g) * torch.logspace(-6, 4, 96).unsqueeze(1)
    v[5, 64:96] = 0
    v[6, :32] = 1e-40  # fp32 subnormal block
    v[7, 0] = 3e38
    v = v.to(dtype)
    q, s = moe.mxfp8_quantize(v.cuda(), mode)
    mname = "f32" if mode == 0 else "e8m0"
    rq, rs = O.mxfp8_quantize(v.float().numpy(), mname)
    assert np.array_equal(q.cpu().numpy(), rq)
    if mode == 0:
        assert np.array_equal(s.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    else:
        assert np.array_equal(s.cpu().numpy(), rs)
    back = moe.mxfp8_dequantize(q, s, mode).cpu()
    rb = O.mxfp8_dequantize(rq, rs, mname)
    assert torch.equal(back.view(torch.int16), rb.view(torch.int16))


def test_mxfp8_every_code_roundtrips():
    moe = _moe()
    codes = np.arange(256, dtype=np.uint8)
    vals = O.e4m3_decode(codes)
    ok = ~np.isnan(vals)
    # one block per code: [code value, 448 to pin the scale to exactly 1.0 ...]
    blocks = np.zeros((int(ok.sum()), 32), np.float32)
    blocks[:, 0] = vals[ok]
    blocks[:, 1] = 448.0
    q, s = moe.mxfp8_quantize(torch.from_numpy(blocks).cuda(), 1)
    assert (s.cpu().numpy() == 127).all()
    assert np.array_equal(q.cpu().numpy()[:, 0], codes[ok])
