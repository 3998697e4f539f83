"""The C-ABI library loads, exports every symbol include/*.h declares, and
rejects bad arguments on the host before any CUDA call (no GPU needed)."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names += re.findall(r"MOE_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from dropless_top_mixture_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("moe_route", "moe_dispatch", "moe_grouped_swiglu", "moe_combine", "mxfp8_quantize",
              "mxfp8_dequantize", "moe_layer_fwd"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_covers_every_symbol():
    from dropless_top_mixture_b200 import moe
    assert set(_declared()) <= set(moe.exported_symbols())


def test_host_validation_rejects_without_launch(lib):
    from dropless_top_mixture_b200 import moe as m
    L = m.lib
    buf = ctypes.create_string_buffer(1 << 16)
    p = ctypes.addressof(buf)
    p16 = (p + 255) & ~255
    # k > E
    assert L.moe_route(p16, None, None, 0, 10, 0, 4, 5, 0, None, p16, p16, p16, p16, p16, None,
                       p16, 4096, None) == m.MOE_ERR_INVALID
    # E beyond the build limit
    assert L.moe_route(p16, None, None, 0, 10, 0, 1000, 2, 0, None, p16, p16, p16, p16, p16, None,
                       p16, 4096, None) == m.MOE_ERR_INVALID
    # logits from x need d % 128 == 0 (four quarters of whole 32-column chunks)
    assert L.moe_route(None, p16, p16, m.MOE_BF16, 10, 96, 4, 2, 0, None, p16, p16, p16, p16,
                       p16, None, p16, 1 << 15, None) == m.MOE_ERR_INVALID
    # workspace too small
    assert L.moe_route(p16, None, None, 0, 1000, 0, 64, 2, 0, None, p16, p16, p16, p16, p16, None,
                       p16, 16, None) == m.MOE_ERR_INVALID
    # d not a multiple of 128 for the grouped GEMM
    assert L.moe_grouped_gate_up(p16, p16, p16, 96 * 128, p16, 4, 100, 96, 128, m.MOE_BF16, p16,
                                 None) == m.MOE_ERR_UNSUPPORTED
    # unsupported dtype
    assert L.moe_dispatch(p16, p16, None, 4, 64, 2, 7, p16, None) == m.MOE_ERR_UNSUPPORTED
    # misaligned pointer
    assert L.moe_combine(p16 + 2, p16, None, 4, 64, 2, m.MOE_BF16, p16, None) == m.MOE_ERR_INVALID
    # MXFP8 columns must be whole blocks
    assert L.mxfp8_quantize(p16, m.MOE_BF16, 4, 48, m.MOE_SCALE_E8M0, p16, p16, None) == m.MOE_ERR_INVALID
    # gathered gate/up: no row_token, or rows to compute but no token to gather
    assert L.moe_grouped_gate_up_gather(p16, None, 10, p16, p16, 128 * 128, p16, 4, 20, 128, 128,
                                        m.MOE_BF16, p16, None) == m.MOE_ERR_INVALID
    assert L.moe_grouped_gate_up_gather(p16, p16, 0, p16, p16, 128 * 128, p16, 4, 20, 128, 128,
                                        m.MOE_BF16, p16, None) == m.MOE_ERR_INVALID
    assert L.moe_row_token(p16, 4, 0, p16, None) == m.MOE_ERR_INVALID
    # the gate-recording dispatch needs the gates and somewhere to put them;
    # the gated down GEMM needs the row gates
    assert L.moe_dispatch_gate(p16, p16, None, 4, 64, 2, m.MOE_BF16, p16, p16, None) == m.MOE_ERR_INVALID
    assert L.moe_dispatch_gate(p16, p16, p16, 4, 64, 2, m.MOE_BF16, p16, None, None) == m.MOE_ERR_INVALID
    assert L.moe_dispatch_gate(p16, p16, None, 0, 64, 2, m.MOE_BF16, p16, None, None) == m.MOE_OK
    assert L.moe_grouped_down_gated(p16, p16, 128 * 128, p16, None, 2, 8, 128, 128, m.MOE_BF16,
                                    p16, None) == m.MOE_ERR_INVALID
    assert L.moe_grouped_down_gated(p16, p16, 128 * 128, p16, None, 2, 0, 128, 128, m.MOE_BF16,
                                    p16, None) == m.MOE_OK
    # tile-form hook: 0, 1, 2 only
    assert L.moe_debug_set_gemm_form(3) == m.MOE_ERR_INVALID
    assert L.moe_debug_set_gemm_form(0) == m.MOE_OK
    # T == 0 is a no-op
    assert L.moe_dispatch(p16, p16, None, 0, 64, 2, m.MOE_BF16, p16, None) == m.MOE_OK
    assert L.moe_row_token(p16, 0, 2, p16, None) == m.MOE_OK
    assert L.moe_layer_fwd(None, None) == m.MOE_ERR_INVALID
    # MXFP8 backward: weights need d, F % 128; the SwiGLU step needs F % 32;
    # the layer needs its arguments and d, F % 256
    assert L.mxfp8_quantize_weights_bwd(p16, p16, p16, 96 * 128, 96 * 128, 2, 96, 128, p16, p16,
                                        p16, p16, None) == m.MOE_ERR_UNSUPPORTED
    assert L.mxfp8_quantize_weights_bwd(p16, None, p16, 128 * 128, 128 * 128, 2, 128, 128, p16,
                                        p16, p16, p16, None) == m.MOE_ERR_INVALID
    assert L.moe_swiglu_bwd_mxfp8(p16, p16, p16, 4, 48, p16, p16, p16, p16, None) == m.MOE_ERR_INVALID
    assert L.moe_swiglu_bwd_mxfp8(p16, p16, p16, 0, 64, p16, p16, p16, p16, None) == m.MOE_OK
    assert L.moe_layer_bwd_mxfp8(None, None) == m.MOE_ERR_INVALID
    a = m.LayerBwdMxArgs(T=4, d=128, E=2, F=256, k=1, workspace=p16, workspace_bytes=1 << 15)
    assert L.moe_layer_bwd_mxfp8(ctypes.byref(a), None) == m.MOE_ERR_UNSUPPORTED
    a.d = 256
    assert L.moe_layer_bwd_mxfp8(ctypes.byref(a), None) == m.MOE_ERR_INVALID  # no tensors
    for f in ("slot", "gate", "offsets", "Xq", "Xs", "Hq", "Hsp", "A", "B", "W13tq", "Ps13t",
              "W2tq", "Ps2t", "dOut", "dx", "dW1", "dW3", "dW2"):
        setattr(a, f, p16)
    a.dx = p16 + 2  # a misaligned output is caught before the first launch
    assert L.moe_layer_bwd_mxfp8(ctypes.byref(a), None) == m.MOE_ERR_INVALID
    assert L.moe_grouped_swiglu_wgrad(p16, p16, p16, p16, p16, p16, 2, 8, 256, 256, m.MOE_F32,
                                      p16, p16, p16, None) == m.MOE_ERR_UNSUPPORTED
    # the MXFP8 forward's save buffers: all or none; not in the sliced host entry
    f = m.LayerMxArgs(T=4, d=256, E=2, F=256, k=1, workspace=p16, workspace_bytes=1 << 15,
                      save_A=p16)
    assert L.moe_layer_fwd_mxfp8_host(ctypes.byref(f), p16, None, p16, 2, p16, p16 + 1,
                                      p16 + 2) == m.MOE_ERR_INVALID


def test_workspace_sizes_are_consistent(lib):
    from dropless_top_mixture_b200 import moe as m
    a = m.lib.moe_route_workspace_size(16384, 64, 1)
    b = m.lib.moe_route_workspace_size(16384, 64, 0)
    assert a - b >= 16384 * 64 * 4
    T, d, E, F, k = 16384, 2048, 64, 1024, 8
    ws = m.lib.moe_layer_workspace_size(T, d, E, F, k, m.MOE_BF16, 0)
    R = T * k
    assert ws >= 2 * (R * d * 2 + R * F * 2 // 2) + b


def _aligned(nbytes, fill=0):
    """A zero-offset-aligned (256-byte) numpy byte buffer and its address."""
    import numpy as np
    raw = np.full(nbytes + 512, fill, dtype=np.uint8)
    off = (-raw.ctypes.data) % 256
    return raw, raw.ctypes.data + off


def test_layer_entries_check_every_step_before_launch(lib):
    """A misaligned weight of a late step (W2 of the down GEMM, dW2 of the
    weight gradients, W2 codes of the MXFP8 down GEMM) is reported as
    MOE_ERR_INVALID before the first step is enqueued: the host buffers
    passed as every output stay as they were (no GPU is touched: every
    check runs on the host)."""
    import numpy as np
    from dropless_top_mixture_b200 import moe as m
    L = m.lib
    T, d, E, F, k = 64, 256, 8, 256, 2
    R = T * k
    keep = []

    def buf(nbytes, fill=0):
        raw, p = _aligned(nbytes, fill)
        keep.append(raw)
        return raw, p

    _, x = buf(T * d * 2)
    _, lg = buf(T * E * 4)
    _, W1 = buf(E * F * d * 2)
    _, W3 = buf(E * F * d * 2)
    _, W2 = buf(E * d * F * 2 + 16)
    outs = {n: buf(sz, 0xA5) for n, sz in (("out", T * d * 2), ("idx", R * 4), ("gate", R * 4),
                                            ("counts", E * 4), ("offsets", (E + 1) * 4),
                                            ("slot", R * 4))}
    ws_bytes = L.moe_layer_workspace_size(T, d, E, F, k, m.MOE_BF16, 1)
    _, ws = buf(ws_bytes)
    a = m.LayerArgs(T=T, d=d, E=E, F=F, k=k, dtype=m.MOE_BF16, x=x, logits=lg, W1=W1, W3=W3,
                    W2=W2 + 2, w13_expert_stride=F * d, w2_expert_stride=F * d,
                    out=outs["out"][1], idx=outs["idx"][1], gate=outs["gate"][1],
                    counts=outs["counts"][1], offsets=outs["offsets"][1], slot=outs["slot"][1],
                    workspace=ws, workspace_bytes=ws_bytes)
    assert L.moe_layer_fwd(ctypes.byref(a), None) == m.MOE_ERR_INVALID
    for n, (raw, _) in outs.items():
        assert (raw == 0xA5).all(), n
    # the sliced host pipeline checks every slice's call before its first copy
    xh_raw, xh = buf(T * d * 2, 0x11)
    oh_raw, oh = buf(T * d * 2, 0x5A)
    lh_raw, lh = buf(T * E * 4)
    assert L.moe_layer_fwd_host(ctypes.byref(a), xh, lh, oh, 3, 1, 2, 3) == m.MOE_ERR_INVALID
    assert (oh_raw == 0x5A).all()
    for n, (raw, _) in outs.items():
        assert (raw == 0xA5).all(), n
    a.W2 = W2
    a.w2_expert_stride = F * d + 3  # not a multiple of 8 elements: the down GEMM rejects it
    assert L.moe_layer_fwd(ctypes.byref(a), None) == m.MOE_ERR_INVALID
    for n, (raw, _) in outs.items():
        assert (raw == 0xA5).all(), n

    # backward: dW2 misaligned (the last GEMM of the chain)
    grads = {n: buf(sz, 0xC3) for n, sz in (("dx", T * d * 2), ("dW1", E * F * d * 2),
                                             ("dW3", E * F * d * 2), ("dW2", E * d * F * 2 + 16))}
    bws = L.moe_layer_bwd_workspace_size(T, d, F, k, m.MOE_BF16)
    _, bw = buf(bws)
    _, tok = buf(R * d * 2)
    _, rowsF = buf(R * F * 2)
    b = m.LayerBwdArgs(T=T, d=d, E=E, F=F, k=k, dtype=m.MOE_BF16, slot=outs["slot"][1],
                       gate=outs["gate"][1], offsets=outs["offsets"][1], Xe=tok, A=rowsF,
                       B=rowsF, H=rowsF, W1=W1, W3=W3, W2=W2, w13_expert_stride=F * d,
                       w2_expert_stride=F * d, dOut=x, dx=grads["dx"][1], dW1=grads["dW1"][1],
                       dW3=grads["dW3"][1], dW2=grads["dW2"][1] + 2, workspace=bw,
                       workspace_bytes=bws)
    assert L.moe_layer_bwd(ctypes.byref(b), None) == m.MOE_ERR_INVALID
    for n, (raw, _) in grads.items():
        assert (raw == 0xC3).all(), n

    # MXFP8 forward: the W2 codes misaligned
    mws = L.moe_layer_mxfp8_workspace_size(T, d, E, F, k, 1)
    _, mw = buf(mws)
    _, q13 = buf(E * F * d)
    _, q2 = buf(E * d * F + 16)
    _, ps = buf(1 << 20)
    f = m.LayerMxArgs(T=T, d=d, E=E, F=F, k=k, x=x, logits=lg, W1q=q13, W3q=q13, Ps13=ps,
                      W2q=q2 + 1, Ps2=ps, w13_expert_stride=F * d, w2_expert_stride=F * d,
                      out=outs["out"][1], idx=outs["idx"][1], gate=outs["gate"][1],
                      counts=outs["counts"][1], offsets=outs["offsets"][1],
                      slot=outs["slot"][1], workspace=mw, workspace_bytes=mws)
    assert L.moe_layer_fwd_mxfp8(ctypes.byref(f), None) == m.MOE_ERR_INVALID
    for n, (raw, _) in outs.items():
        assert (raw == 0xA5).all(), n


@pytest.mark.gpu
def test_layer_entry_rejects_before_launch_on_device():
    """The same on the GPU with device buffers: a misaligned W2 returns
    MOE_ERR_INVALID and idx, the workspace's Xe rows and out keep their
    sentinel bytes after the stream drains."""
    import torch
    from dropless_top_mixture_b200 import moe as m
    T, d, E, F, k = 256, 256, 8, 256, 2
    dev = "cuda"
    x = torch.randn(T, d, device=dev).to(torch.bfloat16)
    lg = torch.randn(T, E, device=dev)
    W1 = torch.randn(E, F, d, device=dev).to(torch.bfloat16)
    W3 = torch.randn(E, F, d, device=dev).to(torch.bfloat16)
    W2 = torch.randn(E * d * F + 8, device=dev).to(torch.bfloat16)
    i32 = dict(dtype=torch.int32, device=dev)
    out = torch.full((T, d), 7.0, dtype=torch.bfloat16, device=dev)
    idx = torch.full((T, k), -5, **i32)
    gate = torch.full((T, k), 3.0, device=dev)
    counts = torch.full((E,), -5, **i32)
    offsets = torch.full((E + 1,), -5, **i32)
    slot = torch.full((T, k), -5, **i32)
    ws_bytes = m.lib.moe_layer_workspace_size(T, d, E, F, k, m.MOE_BF16, 1)
    ws = torch.full((ws_bytes,), 0x3C, dtype=torch.uint8, device=dev)
    a = m.LayerArgs(T=T, d=d, E=E, F=F, k=k, dtype=m.MOE_BF16, x=x.data_ptr(),
                    logits=lg.data_ptr(), W1=W1.data_ptr(), W3=W3.data_ptr(),
                    W2=W2.data_ptr() + 2, w13_expert_stride=F * d, w2_expert_stride=F * d,
                    out=out.data_ptr(), idx=idx.data_ptr(), gate=gate.data_ptr(),
                    counts=counts.data_ptr(), offsets=offsets.data_ptr(), slot=slot.data_ptr(),
                    workspace=ws.data_ptr(), workspace_bytes=ws_bytes)
    stream = torch.cuda.current_stream().cuda_stream
    assert m.lib.moe_layer_fwd(ctypes.byref(a), stream) == m.MOE_ERR_INVALID
    torch.cuda.synchronize()
    assert (out == 7.0).all() and (idx == -5).all() and (gate == 3.0).all()
    assert (counts == -5).all() and (offsets == -5).all() and (slot == -5).all()
    assert (ws == 0x3C).all()  # Xe, H, Ye and the route workspace untouched
    assert m.moe_get_status() == 0
