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
