"""Python binding of the C ABI in include/moe.h.

Argument marshalling only: tensors become ``data_ptr()`` values, the stream
is torch's current stream on the tensors' device, and a non-zero return code
raises :class:`MoeError`. Every step of the layer runs in the sm_100a
library ``lib/libdtm_b200.so``; if it is missing, importing this module
fails — there is no other implementation behind these names.

Output tensors may be passed in; when omitted they are allocated with
``torch.empty`` on the input's device (allocation only, no compute).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libdtm_b200.so")

MOE_OK, MOE_ERR_INVALID, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA = 0, -1, -2, -3
MOE_F32, MOE_BF16, MOE_E4M3 = 0, 1, 2
MOE_SCALE_F32, MOE_SCALE_E8M0 = 0, 1
MOE_DEVERR_TIMEOUT, MOE_DEVERR_BAD_OFFSETS, MOE_DEVERR_BAD_INDEX = 1, 2, 4
TILE_M = 128

_ERRNAMES = {MOE_ERR_INVALID: "MOE_ERR_INVALID", MOE_ERR_UNSUPPORTED: "MOE_ERR_UNSUPPORTED",
             MOE_ERR_CUDA: "MOE_ERR_CUDA"}


class MoeError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {_ERRNAMES.get(code, code)}")
        self.code = code


if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"{_LIB_PATH} is missing: build it with `python -m dropless_top_mixture_b200.build`")

lib = ctypes.CDLL(_LIB_PATH)

_p = ctypes.c_void_p
_i64 = ctypes.c_int64
_i32 = ctypes.c_int
_sz = ctypes.c_size_t


class LayerArgs(ctypes.Structure):
    _fields_ = [
        ("T", _i64), ("d", _i64), ("E", _i64), ("F", _i64),
        ("k", ctypes.c_int32), ("dtype", ctypes.c_int32), ("renorm", ctypes.c_int32),
        ("reserved0", ctypes.c_int32),
        ("x", _p), ("logits", _p), ("Wr", _p), ("W1", _p), ("W3", _p), ("W2", _p),
        ("w13_expert_stride", _i64), ("w2_expert_stride", _i64),
        ("out", _p), ("idx", _p), ("gate", _p), ("counts", _p), ("offsets", _p), ("slot", _p),
        ("workspace", _p), ("workspace_bytes", _sz),
        ("save_Xe", _p), ("save_H", _p), ("save_A", _p), ("save_B", _p),
        ("save_Ye", _p), ("save_logits", _p),
    ]


class LayerBwdArgs(ctypes.Structure):
    _fields_ = [
        ("T", _i64), ("d", _i64), ("E", _i64), ("F", _i64),
        ("k", ctypes.c_int32), ("dtype", ctypes.c_int32), ("reserved0", ctypes.c_int32),
        ("reserved1", ctypes.c_int32),
        ("slot", _p), ("gate", _p), ("offsets", _p),
        ("Xe", _p), ("A", _p), ("B", _p), ("H", _p), ("W1", _p), ("W3", _p), ("W2", _p),
        ("w13_expert_stride", _i64), ("w2_expert_stride", _i64),
        ("dOut", _p), ("dx", _p), ("dW1", _p), ("dW3", _p), ("dW2", _p),
        ("workspace", _p), ("workspace_bytes", _sz),
        ("logits", _p), ("idx", _p), ("counts", _p), ("Ye", _p), ("x", _p), ("Wr", _p),
        ("aux_coef", ctypes.c_float), ("renorm", ctypes.c_int32),
        ("dgate", _p), ("dlogits", _p), ("dWr", _p),
        ("router_workspace", _p), ("router_workspace_bytes", _sz),
    ]


class LayerMxArgs(ctypes.Structure):
    _fields_ = [
        ("T", _i64), ("d", _i64), ("E", _i64), ("F", _i64),
        ("k", ctypes.c_int32), ("renorm", ctypes.c_int32), ("reserved0", ctypes.c_int32),
        ("reserved1", ctypes.c_int32),
        ("x", _p), ("logits", _p), ("Wr", _p),
        ("W1q", _p), ("W3q", _p), ("W2q", _p), ("Ps13", _p), ("Ps2", _p),
        ("w13_expert_stride", _i64), ("w2_expert_stride", _i64),
        ("out", _p), ("idx", _p), ("gate", _p), ("counts", _p), ("offsets", _p), ("slot", _p),
        ("workspace", _p), ("workspace_bytes", _sz),
        ("save_Xq", _p), ("save_Xs", _p), ("save_Hq", _p), ("save_Hsp", _p), ("save_A", _p),
        ("save_B", _p),
    ]


class LayerBwdMxArgs(ctypes.Structure):
    _fields_ = [
        ("T", _i64), ("d", _i64), ("E", _i64), ("F", _i64),
        ("k", ctypes.c_int32), ("reserved0", ctypes.c_int32), ("reserved1", ctypes.c_int32),
        ("reserved2", ctypes.c_int32),
        ("slot", _p), ("gate", _p), ("offsets", _p),
        ("Xq", _p), ("Xs", _p), ("Hq", _p), ("Hsp", _p), ("A", _p), ("B", _p),
        ("W13tq", _p), ("Ps13t", _p), ("W2tq", _p), ("Ps2t", _p),
        ("dOut", _p), ("dx", _p), ("dW1", _p), ("dW3", _p), ("dW2", _p),
        ("workspace", _p), ("workspace_bytes", _sz),
    ]


_SIGS = {
    "moe_route_workspace_size": (_sz, [_i64, _i64, _i32]),
    "moe_route": (_i32, [_p, _p, _p, _i32, _i64, _i64, _i64, _i32, _i32, _p, _p, _p, _p, _p, _p,
                         _p, _p, _sz, _p]),
    "moe_route_noalloc": (_i32, [_p, _p, _p, _i32, _i64, _i64, _i64, _i32, _i32, _p, _p, _p, _p,
                                 _p, _p, _p, _p]),
    "moe_dispatch": (_i32, [_p, _p, _p, _i64, _i64, _i32, _i32, _p, _p]),
    "moe_dispatch_gate": (_i32, [_p, _p, _p, _i64, _i64, _i32, _i32, _p, _p, _p]),
    "moe_grouped_down_gated": (_i32, [_p, _p, _i64, _p, _p, _i64, _i64, _i64, _i64, _i32, _p, _p]),
    "moe_grouped_gate_up": (_i32, [_p, _p, _p, _i64, _p, _i64, _i64, _i64, _i64, _i32, _p, _p]),
    "moe_grouped_down": (_i32, [_p, _p, _i64, _p, _i64, _i64, _i64, _i64, _i32, _p, _p]),
    "moe_row_token": (_i32, [_p, _i64, _i32, _p, _p]),
    "moe_grouped_gate_up_gather": (_i32, [_p, _p, _i64, _p, _p, _i64, _p, _i64, _i64, _i64, _i64,
                                          _i32, _p, _p]),
    "moe_grouped_swiglu": (_i32, [_p, _p, _p, _p, _i64, _i64, _p, _i64, _i64, _i64, _i64, _i32,
                                  _p, _p, _p]),
    "moe_grouped_gate_up_save": (_i32, [_p, _p, _p, _i64, _p, _i64, _i64, _i64, _i64, _i32, _p,
                                        _p, _p, _p]),
    "moe_grouped_swiglu_bwd": (_i32, [_p, _p, _p, _p, _p, _p, _p, _p, _i64, _i64, _p, _i64, _i64,
                                      _i64, _i64, _i32, _p, _p, _p, _p, _p, _p, _p]),
    "moe_combine": (_i32, [_p, _p, _p, _i64, _i64, _i32, _i32, _p, _p]),
    "mxfp8_quantize": (_i32, [_p, _i32, _i64, _i64, _i32, _p, _p, _p]),
    "mxfp8_dequantize": (_i32, [_p, _p, _i32, _i64, _i64, _p, _p]),
    "moe_dispatch_mxfp8": (_i32, [_p, _p, _i64, _i64, _i32, _p, _p, _p]),
    "mxfp8_pack_weight_scales": (_i32, [_p, _p, _p, _i64, _i64, _i64, _p, _p, _p]),
    "mxfp8_act_scales_packed_size": (_sz, [_i64, _i64, _i64]),
    "mxfp8_pack_act_scales": (_i32, [_p, _p, _i64, _i64, _i64, _p, _p]),
    "mxfp8_unpack_act_scales": (_i32, [_p, _p, _i64, _i64, _i64, _p, _p]),
    "moe_grouped_gate_up_mxfp8": (_i32, [_p, _p, _p, _p, _p, _i64, _p, _i64, _i64, _i64, _i64,
                                         _p, _p, _p]),
    "moe_grouped_down_mxfp8": (_i32, [_p, _p, _p, _p, _i64, _p, _i64, _i64, _i64, _i64, _p, _p]),
    "moe_layer_mxfp8_workspace_size": (_sz, [_i64, _i64, _i64, _i64, _i32, _i32]),
    "moe_grouped_gate_up_mxfp8_save": (_i32, [_p, _p, _p, _p, _p, _i64, _p, _i64, _i64, _i64,
                                              _i64, _p, _p, _p, _p, _p]),
    "mxfp8_quantize_weights_bwd": (_i32, [_p, _p, _p, _i64, _i64, _i64, _i64, _i64, _p, _p, _p,
                                          _p, _p]),
    "moe_swiglu_bwd_mxfp8": (_i32, [_p, _p, _p, _i64, _i64, _p, _p, _p, _p, _p]),
    "moe_layer_bwd_mxfp8_workspace_size": (_sz, [_i64, _i64, _i64, _i64, _i32]),
    "moe_layer_bwd_mxfp8": (_i32, [ctypes.POINTER(LayerBwdMxArgs), _p]),
    "moe_grouped_swiglu_wgrad": (_i32, [_p, _p, _p, _p, _p, _p, _i64, _i64, _i64, _i64, _i32, _p,
                                        _p, _p, _p]),
    "moe_layer_fwd_mxfp8": (_i32, [ctypes.POINTER(LayerMxArgs), _p]),
    "moe_layer_fwd_mxfp8_host": (_i32, [ctypes.POINTER(LayerMxArgs), _p, _p, _p, _i32, _p, _p,
                                        _p]),
    "moe_layer_workspace_size": (_sz, [_i64, _i64, _i64, _i64, _i32, _i32, _i32]),
    "moe_layer_fwd": (_i32, [ctypes.POINTER(LayerArgs), _p]),
    "moe_layer_fwd_host": (_i32, [ctypes.POINTER(LayerArgs), _p, _p, _p, _i32, _p, _p, _p]),
    "moe_layer_bwd_workspace_size": (_sz, [_i64, _i64, _i64, _i32, _i32]),
    "moe_layer_bwd": (_i32, [ctypes.POINTER(LayerBwdArgs), _p]),
    "moe_aux_loss_workspace_size": (_sz, [_i64, _i64]),
    "moe_aux_loss": (_i32, [_p, _p, _i64, _i64, _p, _p, _sz, _p]),
    "moe_router_bwd": (_i32, [_p, _p, _p, _p, _p, _p, _i64, _i64, _i64, _i32, _i32, _i32,
                              ctypes.c_float, _p, _p, _p]),
    "moe_router_linear_bwd_workspace_size": (_sz, [_i64, _i64, _i64]),
    "moe_router_linear_bwd": (_i32, [_p, _p, _p, _i64, _i64, _i64, _i32, _p, _p, _p, _sz, _p]),
    "moe_get_status": (_i32, [ctypes.POINTER(ctypes.c_int32), _i32, _p]),
    "moe_ep_workspace_size": (_sz, [_i64]),
    "moe_ep_plan": (_i32, [_p, _i32, _i32, _p, _p, _p, _i64, _i64, _i32, _p, _p, _p, _p, _sz, _p]),
    "moe_dispatch_ep": (_i32, [_p, _p, _p, _i64, _i64, _i32, _i32, _p, _i32, _i64, _p]),
    "moe_combine_ep": (_i32, [_p, _p, _p, _p, _i64, _i64, _i32, _i32, _i32, _i64, _p, _p]),
    "moe_debug_set_wait_limit_ns": (_i32, [ctypes.c_uint64]),
    "moe_debug_set_gemm_form": (_i32, [_i32]),
    "moe_version": (ctypes.c_char_p, []),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args


def exported_symbols():
    return list(_SIGS)


# ----------------------------------------------------------------- helpers

def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream(t: torch.Tensor):
    return torch.cuda.current_stream(t.device).cuda_stream


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return MOE_BF16
    if dt == torch.float32:
        return MOE_F32
    raise TypeError(f"unsupported dtype {dt}")


def _check(fn: str, rc: int):
    if rc != MOE_OK:
        raise MoeError(fn, rc)


def _need(t: torch.Tensor, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _alloc_ws(nbytes: int, device) -> torch.Tensor:
    # 256-byte aligned: torch's caching allocator hands out 512-byte aligned blocks
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


# ----------------------------------------------------------------- API

@dataclass
class Route:
    idx: torch.Tensor
    gate: torch.Tensor
    counts: torch.Tensor
    offsets: torch.Tensor
    slot: torch.Tensor
    tile_offsets: torch.Tensor
    logits: Optional[torch.Tensor] = None


def moe_route(k: int, *, logits: Optional[torch.Tensor] = None, x: Optional[torch.Tensor] = None,
              Wr: Optional[torch.Tensor] = None, renorm: bool = False, E: Optional[int] = None,
              keep_logits: bool = False, out: Optional[Route] = None,
              workspace: Optional[torch.Tensor] = None) -> Route:
    if logits is not None:
        _need(logits, "logits")
        T, E = logits.shape
        dev = logits.device
        dtype, d = MOE_F32, 0
    else:
        _need(x, "x"); _need(Wr, "Wr")
        T, d = x.shape
        E = Wr.shape[0]
        dev = x.device
        dtype = _dtype_code(x.dtype)
    i32 = dict(dtype=torch.int32, device=dev)
    if out is None:
        out = Route(idx=torch.empty((T, k), **i32), gate=torch.empty((T, k), dtype=torch.float32, device=dev),
                    counts=torch.empty(E, **i32), offsets=torch.empty(E + 1, **i32),
                    slot=torch.empty((T, k), **i32), tile_offsets=torch.empty(E + 1, **i32))
        if logits is None and keep_logits:
            out.logits = torch.empty((T, E), dtype=torch.float32, device=dev)
    ws_bytes = lib.moe_route_workspace_size(T, E, int(logits is None))
    if workspace is None:
        workspace = _alloc_ws(ws_bytes, dev)
    rc = lib.moe_route(_ptr(logits), _ptr(x), _ptr(Wr), dtype, T, d, E, k, int(renorm),
                       _ptr(out.logits), _ptr(out.idx), _ptr(out.gate), _ptr(out.counts),
                       _ptr(out.offsets), _ptr(out.slot), _ptr(out.tile_offsets),
                       _ptr(workspace), workspace.numel(), _stream(workspace))
    _check("moe_route", rc)
    return out


def moe_route_noalloc(k: int, *, logits: Optional[torch.Tensor] = None,
                      x: Optional[torch.Tensor] = None, Wr: Optional[torch.Tensor] = None,
                      renorm: bool = False, out: Route) -> Route:
    """moe_route with the library's own scratch: the caller passes every
    output (``out``) and no workspace; nothing is allocated here either."""
    if logits is not None:
        _need(logits, "logits")
        T, E = logits.shape
        dtype, d, dev_t = MOE_F32, 0, logits
    else:
        _need(x, "x"); _need(Wr, "Wr")
        T, d = x.shape
        E = Wr.shape[0]
        dtype, dev_t = _dtype_code(x.dtype), x
    rc = lib.moe_route_noalloc(_ptr(logits), _ptr(x), _ptr(Wr), dtype, T, d, E, k, int(renorm),
                               _ptr(out.logits), _ptr(out.idx), _ptr(out.gate), _ptr(out.counts),
                               _ptr(out.offsets), _ptr(out.slot), _ptr(out.tile_offsets),
                               _stream(dev_t))
    _check("moe_route_noalloc", rc)
    return out


def moe_dispatch(x: torch.Tensor, slot: torch.Tensor, gate: Optional[torch.Tensor] = None,
                 out: Optional[torch.Tensor] = None) -> torch.Tensor:
    _need(x, "x"); _need(slot, "slot")
    T, d = x.shape
    k = slot.shape[1]
    if out is None:
        out = torch.empty((T * k, d), dtype=x.dtype, device=x.device)
    rc = lib.moe_dispatch(_ptr(x), _ptr(slot), _ptr(gate), T, d, k, _dtype_code(x.dtype),
                          _ptr(out), _stream(x))
    _check("moe_dispatch", rc)
    return out


def moe_dispatch_gate(x: torch.Tensor, slot: torch.Tensor, gate: torch.Tensor,
                      out: Optional[torch.Tensor] = None,
                      row_gate: Optional[torch.Tensor] = None):
    """Unscaled dispatch that also records row_gate[slot[t,j]] = gate[t,j];
    returns (Xe, row_gate)."""
    _need(x, "x"); _need(slot, "slot"); _need(gate, "gate")
    T, d = x.shape
    k = slot.shape[1]
    if out is None:
        out = torch.empty((T * k, d), dtype=x.dtype, device=x.device)
    if row_gate is None:
        row_gate = torch.empty(T * k, dtype=torch.float32, device=x.device)
    rc = lib.moe_dispatch_gate(_ptr(x), _ptr(slot), _ptr(gate), T, d, k, _dtype_code(x.dtype),
                               _ptr(out), _ptr(row_gate), _stream(x))
    _check("moe_dispatch_gate", rc)
    return out, row_gate


def _w13(W1: torch.Tensor, W3: torch.Tensor):
    # [E,F,d] tensors, or views into a fused [E,2F,d] gate/up tensor
    E, F, d = W1.shape
    stride = W1.stride(0)
    if W3.stride(0) != stride or W1.stride(1) != d or W1.stride(2) != 1:
        raise ValueError("W1/W3 must be [E,F,d] with rows contiguous and a common expert stride")
    return E, F, d, stride


def moe_grouped_gate_up(Xe, W1, W3, offsets, H: Optional[torch.Tensor] = None) -> torch.Tensor:
    _need(Xe, "Xe"); _need(offsets, "offsets")
    E, F, d, s13 = _w13(W1, W3)
    R = Xe.shape[0]
    if H is None:
        H = torch.empty((R, F), dtype=Xe.dtype, device=Xe.device)
    rc = lib.moe_grouped_gate_up(_ptr(Xe), _ptr(W1), _ptr(W3), s13, _ptr(offsets), E, R, d, F,
                                 _dtype_code(Xe.dtype), _ptr(H), _stream(Xe))
    _check("moe_grouped_gate_up", rc)
    return H


def moe_row_token(slot, row_token: Optional[torch.Tensor] = None) -> torch.Tensor:
    _need(slot, "slot")
    T, k = slot.shape
    if row_token is None:
        row_token = torch.empty(T * k, dtype=torch.int32, device=slot.device)
    rc = lib.moe_row_token(_ptr(slot), T, k, _ptr(row_token), _stream(slot))
    _check("moe_row_token", rc)
    return row_token


def moe_grouped_gate_up_gather(x, row_token, W1, W3, offsets,
                               H: Optional[torch.Tensor] = None) -> torch.Tensor:
    _need(x, "x"); _need(row_token, "row_token"); _need(offsets, "offsets")
    E, F, d, s13 = _w13(W1, W3)
    R = row_token.numel()
    if H is None:
        H = torch.empty((R, F), dtype=x.dtype, device=x.device)
    rc = lib.moe_grouped_gate_up_gather(_ptr(x), _ptr(row_token), x.shape[0], _ptr(W1), _ptr(W3),
                                        s13, _ptr(offsets), E, R, d, F, _dtype_code(x.dtype),
                                        _ptr(H), _stream(x))
    _check("moe_grouped_gate_up_gather", rc)
    return H


def moe_grouped_gate_up_save(Xe, W1, W3, offsets, H=None, A=None, B=None):
    _need(Xe, "Xe"); _need(offsets, "offsets")
    E, F, d, s13 = _w13(W1, W3)
    R = Xe.shape[0]
    mk = lambda t: torch.empty((R, F), dtype=Xe.dtype, device=Xe.device) if t is None else t
    H, A, B = mk(H), mk(A), mk(B)
    rc = lib.moe_grouped_gate_up_save(_ptr(Xe), _ptr(W1), _ptr(W3), s13, _ptr(offsets), E, R, d,
                                      F, _dtype_code(Xe.dtype), _ptr(H), _ptr(A), _ptr(B),
                                      _stream(Xe))
    _check("moe_grouped_gate_up_save", rc)
    return H, A, B


@dataclass
class ExpertGrads:
    dXe: torch.Tensor
    dW1: torch.Tensor
    dW3: torch.Tensor
    dW2: torch.Tensor
    dA: torch.Tensor
    dB: torch.Tensor


def moe_grouped_swiglu_bwd(Xe, A, B, H, dYe, W1, W3, W2, offsets,
                           out: Optional[ExpertGrads] = None) -> ExpertGrads:
    for t, n in ((Xe, "Xe"), (A, "A"), (B, "B"), (H, "H"), (dYe, "dYe"), (offsets, "offsets")):
        _need(t, n)
    E, F, d, s13 = _w13(W1, W3)
    R = Xe.shape[0]
    dev, dt = Xe.device, Xe.dtype
    if out is None:
        out = ExpertGrads(dXe=torch.empty((R, d), dtype=dt, device=dev),
                          dW1=torch.empty((E, F, d), dtype=dt, device=dev),
                          dW3=torch.empty((E, F, d), dtype=dt, device=dev),
                          dW2=torch.empty((E, d, F), dtype=dt, device=dev),
                          dA=torch.empty((R, F), dtype=dt, device=dev),
                          dB=torch.empty((R, F), dtype=dt, device=dev))
    rc = lib.moe_grouped_swiglu_bwd(_ptr(Xe), _ptr(A), _ptr(B), _ptr(H), _ptr(dYe), _ptr(W1),
                                    _ptr(W3), _ptr(W2), s13, _w2(W2)[3], _ptr(offsets), E, R, d,
                                    F, _dtype_code(dt), _ptr(out.dA), _ptr(out.dB), _ptr(out.dXe),
                                    _ptr(out.dW1), _ptr(out.dW3), _ptr(out.dW2), _stream(Xe))
    _check("moe_grouped_swiglu_bwd", rc)
    return out


def _w2(W2: torch.Tensor):
    # [E,d,F] with rows contiguous; experts any (multiple of 8) stride apart
    if not W2.is_cuda:
        raise ValueError("W2 must be a CUDA tensor")
    E, d, F = W2.shape
    if W2.stride(2) != 1 or W2.stride(1) != F:
        raise ValueError("W2 must be [E,d,F] with rows contiguous")
    return E, d, F, W2.stride(0)


def moe_grouped_down(H, W2, offsets, Ye: Optional[torch.Tensor] = None) -> torch.Tensor:
    _need(H, "H"); _need(offsets, "offsets")
    E, d, F, s2 = _w2(W2)
    R = H.shape[0]
    if Ye is None:
        Ye = torch.empty((R, d), dtype=H.dtype, device=H.device)
    rc = lib.moe_grouped_down(_ptr(H), _ptr(W2), s2, _ptr(offsets), E, R, d, F,
                              _dtype_code(H.dtype), _ptr(Ye), _stream(H))
    _check("moe_grouped_down", rc)
    return Ye


def moe_grouped_down_gated(H, W2, offsets, row_gate, Ye: Optional[torch.Tensor] = None):
    """moe_grouped_down with each row's sums scaled by row_gate[r] before
    rounding (the gates from moe_dispatch_gate)."""
    _need(H, "H"); _need(offsets, "offsets"); _need(row_gate, "row_gate")
    E, d, F, s2 = _w2(W2)
    R = H.shape[0]
    if Ye is None:
        Ye = torch.empty((R, d), dtype=H.dtype, device=H.device)
    rc = lib.moe_grouped_down_gated(_ptr(H), _ptr(W2), s2, _ptr(offsets), _ptr(row_gate), E, R,
                                    d, F, _dtype_code(H.dtype), _ptr(Ye), _stream(H))
    _check("moe_grouped_down_gated", rc)
    return Ye


def moe_grouped_swiglu(Xe, W1, W3, W2, offsets, H: Optional[torch.Tensor] = None,
                       Ye: Optional[torch.Tensor] = None):
    _need(Xe, "Xe"); _need(offsets, "offsets")
    E, F, d, s13 = _w13(W1, W3)
    R = Xe.shape[0]
    if H is None:
        H = torch.empty((R, F), dtype=Xe.dtype, device=Xe.device)
    if Ye is None:
        Ye = torch.empty((R, d), dtype=Xe.dtype, device=Xe.device)
    rc = lib.moe_grouped_swiglu(_ptr(Xe), _ptr(W1), _ptr(W3), _ptr(W2), s13, _w2(W2)[3],
                                _ptr(offsets), E, R, d, F, _dtype_code(Xe.dtype), _ptr(H),
                                _ptr(Ye), _stream(Xe))
    _check("moe_grouped_swiglu", rc)
    return H, Ye


def moe_combine(Ye, slot, gate: Optional[torch.Tensor], out: Optional[torch.Tensor] = None):
    _need(Ye, "Ye"); _need(slot, "slot")
    T, k = slot.shape
    d = Ye.shape[1]
    if out is None:
        out = torch.empty((T, d), dtype=Ye.dtype, device=Ye.device)
    rc = lib.moe_combine(_ptr(Ye), _ptr(slot), _ptr(gate), T, d, k, _dtype_code(Ye.dtype),
                         _ptr(out), _stream(Ye))
    _check("moe_combine", rc)
    return out


def mxfp8_quantize(v: torch.Tensor, scale_mode: int = MOE_SCALE_E8M0, q=None, scales=None):
    _need(v, "v")
    rows, cols = v.shape
    if q is None:
        q = torch.empty((rows, cols), dtype=torch.uint8, device=v.device)
    if scales is None:
        sdt = torch.float32 if scale_mode == MOE_SCALE_F32 else torch.uint8
        scales = torch.empty((rows, cols // 32), dtype=sdt, device=v.device)
    rc = lib.mxfp8_quantize(_ptr(v), _dtype_code(v.dtype), rows, cols, scale_mode, _ptr(q),
                            _ptr(scales), _stream(v))
    _check("mxfp8_quantize", rc)
    return q, scales


def mxfp8_dequantize(q: torch.Tensor, scales: torch.Tensor, scale_mode: int = MOE_SCALE_E8M0,
                     out=None) -> torch.Tensor:
    _need(q, "q"); _need(scales, "scales")
    rows, cols = q.shape
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.bfloat16, device=q.device)
    rc = lib.mxfp8_dequantize(_ptr(q), _ptr(scales), scale_mode, rows, cols, _ptr(out), _stream(q))
    _check("mxfp8_dequantize", rc)
    return out


def moe_layer_workspace_size(T, d, E, F, k, dtype: torch.dtype, logits_given: bool) -> int:
    return lib.moe_layer_workspace_size(T, d, E, F, k, _dtype_code(dtype), int(logits_given))


@dataclass
class LayerOut:
    out: torch.Tensor
    idx: torch.Tensor
    gate: torch.Tensor
    counts: torch.Tensor
    offsets: torch.Tensor
    slot: torch.Tensor
    workspace: torch.Tensor
    Xe: Optional[torch.Tensor] = None   # rows kept for the backward (save=True)
    H: Optional[torch.Tensor] = None
    A: Optional[torch.Tensor] = None
    B: Optional[torch.Tensor] = None
    Ye: Optional[torch.Tensor] = None   # expert outputs, for the router backward
    logits: Optional[torch.Tensor] = None  # fp32 logits (computed or given)
    renorm: bool = False
    Xq: Optional[torch.Tensor] = None   # MXFP8 forward, save=True: codes and scales
    Xs: Optional[torch.Tensor] = None   # the backward reads (row-layout Xs,
    Hq: Optional[torch.Tensor] = None   # tile-packed Hsp)
    Hsp: Optional[torch.Tensor] = None


def moe_layer_fwd(x, k: int, W1, W3, W2, *, logits=None, Wr=None, renorm: bool = False,
                  out: Optional[LayerOut] = None, save: bool = False) -> LayerOut:
    _need(x, "x")
    T, d = x.shape
    E, F, _, s13 = _w13(W1, W3)
    dev = x.device
    if out is None:
        i32 = dict(dtype=torch.int32, device=dev)
        ws = _alloc_ws(moe_layer_workspace_size(T, d, E, F, k, x.dtype, logits is not None), dev)
        out = LayerOut(out=torch.empty((T, d), dtype=x.dtype, device=dev),
                       idx=torch.empty((T, k), **i32),
                       gate=torch.empty((T, k), dtype=torch.float32, device=dev),
                       counts=torch.empty(E, **i32), offsets=torch.empty(E + 1, **i32),
                       slot=torch.empty((T, k), **i32), workspace=ws)
        if save:
            R = T * k
            out.Xe = torch.empty((R, d), dtype=x.dtype, device=dev)
            out.H, out.A, out.B = (torch.empty((R, F), dtype=x.dtype, device=dev) for _ in range(3))
            out.Ye = torch.empty((R, d), dtype=x.dtype, device=dev)
            if logits is None:
                out.logits = torch.empty((T, E), dtype=torch.float32, device=dev)
    if logits is not None:
        out.logits = logits
    out.renorm = bool(renorm)
    save_logits = out.logits if (save and logits is None) else None
    a = LayerArgs(T=T, d=d, E=E, F=F, k=k, dtype=_dtype_code(x.dtype), renorm=int(renorm),
                  reserved0=0, x=_ptr(x), logits=_ptr(logits), Wr=_ptr(Wr), W1=_ptr(W1),
                  W3=_ptr(W3), W2=_ptr(W2), w13_expert_stride=s13, w2_expert_stride=_w2(W2)[3],
                  out=_ptr(out.out), idx=_ptr(out.idx), gate=_ptr(out.gate),
                  counts=_ptr(out.counts), offsets=_ptr(out.offsets), slot=_ptr(out.slot),
                  workspace=_ptr(out.workspace), workspace_bytes=out.workspace.numel(),
                  save_Xe=_ptr(out.Xe), save_H=_ptr(out.H), save_A=_ptr(out.A), save_B=_ptr(out.B),
                  save_Ye=_ptr(out.Ye), save_logits=_ptr(save_logits))
    rc = lib.moe_layer_fwd(ctypes.byref(a), _stream(x))
    _check("moe_layer_fwd", rc)
    return out


# Nominal bandwidths for choosing the host pipeline's slice count: pinned
# host <-> device copies over PCIe Gen5 x16, and HBM for re-streaming the
# expert weights once per slice.
PCIE_GBS = 55.0
HBM_GBS = 6500.0


def choose_chunks(T: int, d: int, act_esize: int, weight_bytes: int, max_chunks: int = 8) -> int:
    """Slice count for the host pipeline. With c slices the time is about
    compute + c * Wt + Ct * h(c): every slice streams the weights once (Wt),
    and of the copies (Ct per direction) what nothing overlaps is 2 Ct for
    one slice, Ct for two, and Ct / (c - 1) from three on (half-size first
    and last slices). Returns the c that minimises c * Wt + Ct * h(c)."""
    ct = T * d * act_esize / (PCIE_GBS * 1e9)
    wt = weight_bytes / (HBM_GBS * 1e9)
    h = lambda c: 2.0 if c == 1 else (1.0 if c == 2 else 1.0 / (c - 1))
    return min(range(1, max_chunks + 1), key=lambda c: c * wt + ct * h(c))


class HostLayer:
    """moe_layer_fwd_host: the layer from pinned host x (and logits) to
    pinned host out, cut into `chunks` token slices whose copy-in, compute
    and copy-out overlap. Holds the device staging buffers, the routing
    outputs (idx, gate, slot for every token) and the two copy streams, so
    repeated calls of one shape allocate nothing."""

    def __init__(self, T: int, d: int, E: int, F: int, k: int, dtype: torch.dtype, device,
                 *, logits_given: bool, chunks: int = 3):
        if not 1 <= chunks <= 64:
            raise ValueError("chunks must be in [1, 64]")
        dev = torch.device(device)
        i32 = dict(dtype=torch.int32, device=dev)
        self.T, self.d, self.E, self.F, self.k, self.dtype = T, d, E, F, k, dtype
        self.chunks = chunks
        self.x = torch.empty((T, d), dtype=dtype, device=dev)
        self.logits = torch.empty((T, E), dtype=torch.float32, device=dev) if logits_given else None
        self.res = LayerOut(out=torch.empty((T, d), dtype=dtype, device=dev),
                            idx=torch.empty((T, k), **i32),
                            gate=torch.empty((T, k), dtype=torch.float32, device=dev),
                            counts=torch.empty(E, **i32), offsets=torch.empty(E + 1, **i32),
                            slot=torch.empty((T, k), **i32),
                            workspace=_alloc_ws(moe_layer_workspace_size(
                                T, d, E, F, k, dtype, logits_given), dev))
        self.s_h2d = torch.cuda.Stream(dev)
        self.s_d2h = torch.cuda.Stream(dev)

    def __call__(self, x_host: torch.Tensor, W1, W3, W2, *, logits_host=None, Wr=None,
                 renorm: bool = False, out_host: Optional[torch.Tensor] = None) -> torch.Tensor:
        if x_host.is_cuda or tuple(x_host.shape) != (self.T, self.d) or x_host.dtype != self.dtype:
            raise ValueError("x_host must be a [T, d] host tensor of the layer's dtype")
        if (logits_host is None) != (self.logits is None):
            raise ValueError("logits_host must be given exactly when the layer was built for it")
        if logits_host is not None and (logits_host.is_cuda or logits_host.dtype != torch.float32
                                        or tuple(logits_host.shape) != (self.T, self.E)):
            raise ValueError("logits_host must be a [T, E] fp32 host tensor")
        if out_host is None:
            out_host = torch.empty((self.T, self.d), dtype=self.dtype, pin_memory=True)
        E, F, _, s13 = _w13(W1, W3)
        r = self.res
        a = LayerArgs(T=self.T, d=self.d, E=E, F=F, k=self.k, dtype=_dtype_code(self.dtype),
                      renorm=int(renorm), reserved0=0, x=_ptr(self.x), logits=_ptr(self.logits),
                      Wr=_ptr(Wr), W1=_ptr(W1), W3=_ptr(W3), W2=_ptr(W2),
                      w13_expert_stride=s13, w2_expert_stride=_w2(W2)[3], out=_ptr(r.out),
                      idx=_ptr(r.idx), gate=_ptr(r.gate), counts=_ptr(r.counts),
                      offsets=_ptr(r.offsets), slot=_ptr(r.slot), workspace=_ptr(r.workspace),
                      workspace_bytes=r.workspace.numel(), save_Xe=None, save_H=None,
                      save_A=None, save_B=None)
        rc = lib.moe_layer_fwd_host(ctypes.byref(a), x_host.data_ptr(), _ptr(logits_host),
                                    out_host.data_ptr(), self.chunks, _stream(self.x),
                                    self.s_h2d.cuda_stream, self.s_d2h.cuda_stream)
        _check("moe_layer_fwd_host", rc)
        return out_host


@dataclass
class LayerGrads:
    dx: torch.Tensor
    dW1: torch.Tensor
    dW3: torch.Tensor
    dW2: torch.Tensor
    workspace: torch.Tensor
    dlogits: Optional[torch.Tensor] = None    # router backward (router=True)
    dgate: Optional[torch.Tensor] = None
    dWr: Optional[torch.Tensor] = None
    router_workspace: Optional[torch.Tensor] = None


def moe_layer_bwd(fwd: LayerOut, dOut, k: int, W1, W3, W2,
                  out: Optional[LayerGrads] = None, *, router: bool = False, x=None, Wr=None,
                  aux_coef: float = 0.0) -> LayerGrads:
    """Backward of moe_layer_fwd(save=True). With router=False the gates are
    held constant; with router=True the gates are differentiated through the
    softmax too (plus aux_coef times the load-balancing loss), giving dlogits,
    dgate and, when Wr is given, the router GEMM backward (dx += dlogits Wr,
    dWr = dlogits^T x, which needs x)."""
    _need(dOut, "dOut")
    if fwd.Xe is None:
        raise ValueError("moe_layer_bwd needs the forward run with save=True")
    if router and (fwd.Ye is None or fwd.logits is None):
        raise ValueError("the router backward needs the forward's Ye and logits (save=True)")
    if router and Wr is not None and x is None:
        raise ValueError("dWr needs the forward input x")
    T, d = dOut.shape
    E, F, _, s13 = _w13(W1, W3)
    dev, dt = dOut.device, dOut.dtype
    if out is None:
        ws = _alloc_ws(lib.moe_layer_bwd_workspace_size(T, d, F, k, _dtype_code(dt)), dev)
        out = LayerGrads(dx=torch.empty((T, d), dtype=dt, device=dev),
                         dW1=torch.empty((E, F, d), dtype=dt, device=dev),
                         dW3=torch.empty((E, F, d), dtype=dt, device=dev),
                         dW2=torch.empty((E, d, F), dtype=dt, device=dev), workspace=ws)
        if router:
            out.dlogits = torch.empty((T, E), dtype=torch.float32, device=dev)
            out.dgate = torch.empty((T, k), dtype=torch.float32, device=dev)
            if Wr is not None:
                out.dWr = torch.empty((E, d), dtype=dt, device=dev)
                out.router_workspace = _alloc_ws(
                    lib.moe_router_linear_bwd_workspace_size(T, d, E), dev)
    rws = out.router_workspace
    a = LayerBwdArgs(T=T, d=d, E=E, F=F, k=k, dtype=_dtype_code(dt), reserved0=0, reserved1=0,
                     slot=_ptr(fwd.slot), gate=_ptr(fwd.gate), offsets=_ptr(fwd.offsets),
                     Xe=_ptr(fwd.Xe), A=_ptr(fwd.A), B=_ptr(fwd.B), H=_ptr(fwd.H), W1=_ptr(W1),
                     W3=_ptr(W3), W2=_ptr(W2), w13_expert_stride=s13,
                     w2_expert_stride=_w2(W2)[3], dOut=_ptr(dOut), dx=_ptr(out.dx),
                     dW1=_ptr(out.dW1), dW3=_ptr(out.dW3), dW2=_ptr(out.dW2),
                     workspace=_ptr(out.workspace), workspace_bytes=out.workspace.numel())
    if router:
        a.logits, a.idx, a.counts, a.Ye = (_ptr(fwd.logits), _ptr(fwd.idx), _ptr(fwd.counts),
                                           _ptr(fwd.Ye))
        a.x, a.Wr = _ptr(x), _ptr(Wr)
        a.aux_coef, a.renorm = float(aux_coef), int(fwd.renorm)
        a.dgate, a.dlogits, a.dWr = _ptr(out.dgate), _ptr(out.dlogits), _ptr(out.dWr)
        a.router_workspace = _ptr(rws)
        a.router_workspace_bytes = 0 if rws is None else rws.numel()
    rc = lib.moe_layer_bwd(ctypes.byref(a), _stream(dOut))
    _check("moe_layer_bwd", rc)
    return out


def moe_aux_loss(logits, counts, out: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Load-balancing loss E * sum_e (counts_e/T) * mean_t softmax(logits_t)_e,
    as a one-element fp32 device tensor."""
    _need(logits, "logits"); _need(counts, "counts")
    T, E = logits.shape
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=logits.device)
    if workspace is None:
        workspace = _alloc_ws(lib.moe_aux_loss_workspace_size(T, E), logits.device)
    rc = lib.moe_aux_loss(_ptr(logits), _ptr(counts), T, E, _ptr(out), _ptr(workspace),
                          workspace.numel(), _stream(logits))
    _check("moe_aux_loss", rc)
    return out


@dataclass
class RouterGrads:
    dgate: Optional[torch.Tensor]
    dlogits: torch.Tensor


def moe_router_bwd(dOut, Ye, slot, idx, logits, counts=None, *, renorm: bool = False,
                   aux_coef: float = 0.0, dgate=None, dlogits=None,
                   want_dgate: bool = True) -> RouterGrads:
    """Gate and router-logit gradients (top-k choice and counts held fixed)."""
    for t, n in ((dOut, "dOut"), (Ye, "Ye"), (slot, "slot"), (idx, "idx"), (logits, "logits")):
        _need(t, n)
    T, d = dOut.shape
    k = slot.shape[1]
    E = logits.shape[1]
    if dgate is None and want_dgate:
        dgate = torch.empty((T, k), dtype=torch.float32, device=dOut.device)
    if dlogits is None:
        dlogits = torch.empty((T, E), dtype=torch.float32, device=dOut.device)
    rc = lib.moe_router_bwd(_ptr(dOut), _ptr(Ye), _ptr(slot), _ptr(idx), _ptr(logits),
                            _ptr(counts), T, d, E, k, _dtype_code(dOut.dtype), int(renorm),
                            float(aux_coef), _ptr(dgate), _ptr(dlogits), _stream(dOut))
    _check("moe_router_bwd", rc)
    return RouterGrads(dgate=dgate, dlogits=dlogits)


def moe_router_linear_bwd(dlogits, x, Wr, dx=None, want_dWr: bool = True, dWr=None,
                          workspace: Optional[torch.Tensor] = None):
    """logits = x Wr^T backward: dx += dlogits Wr (in place, when dx is given)
    and dWr = dlogits^T x. Returns (dx, dWr)."""
    _need(dlogits, "dlogits"); _need(x, "x"); _need(Wr, "Wr")
    T, d = x.shape
    E = Wr.shape[0]
    if dWr is None and want_dWr:
        dWr = torch.empty((E, d), dtype=x.dtype, device=x.device)
    if dWr is not None and workspace is None:
        workspace = _alloc_ws(lib.moe_router_linear_bwd_workspace_size(T, d, E), x.device)
    rc = lib.moe_router_linear_bwd(_ptr(dlogits), _ptr(x), _ptr(Wr), T, d, E,
                                   _dtype_code(x.dtype), _ptr(dx), _ptr(dWr), _ptr(workspace),
                                   0 if workspace is None else workspace.numel(), _stream(x))
    _check("moe_router_linear_bwd", rc)
    return dx, dWr


# ----------------------------------------------------------------- expert parallelism

@dataclass
class EPPlan:
    """Where this rank's (token, choice) rows live on their experts' ranks."""
    dst_rank: torch.Tensor      # [T,k] int32
    dst_row: torch.Tensor       # [T,k] int32
    recv_offsets: torch.Tensor  # [E/G + 1] int32: this rank's receive buffer by local expert


def moe_ep_plan(counts_all: torch.Tensor, me: int, route: "Route",
                out: Optional[EPPlan] = None,
                workspace: Optional[torch.Tensor] = None) -> EPPlan:
    """counts_all [G,E] int32 (row s = rank s's per-expert counts); `route`
    is this rank's moe_route result."""
    _need(counts_all, "counts_all")
    G, E = counts_all.shape
    T, k = route.idx.shape
    dev = counts_all.device
    if out is None:
        i32 = dict(dtype=torch.int32, device=dev)
        out = EPPlan(dst_rank=torch.empty((T, k), **i32), dst_row=torch.empty((T, k), **i32),
                     recv_offsets=torch.empty(E // G + 1 if G and E % G == 0 else 1, **i32))
    if workspace is None:
        workspace = _alloc_ws(lib.moe_ep_workspace_size(E), dev)
    rc = lib.moe_ep_plan(_ptr(counts_all), G, me, _ptr(route.idx), _ptr(route.slot),
                         _ptr(route.offsets), T, E, k, _ptr(out.dst_rank), _ptr(out.dst_row),
                         _ptr(out.recv_offsets), _ptr(workspace), workspace.numel(),
                         _stream(counts_all))
    _check("moe_ep_plan", rc)
    return out


def _ptr_table(bufs, dev) -> torch.Tensor:
    return torch.tensor([b.data_ptr() for b in bufs], dtype=torch.int64, device=dev)


def moe_dispatch_ep(x: torch.Tensor, plan: EPPlan, recv_table: torch.Tensor,
                    rows_max: int) -> None:
    """Write every (token, choice) row of x into its owner's receive buffer;
    recv_table is a device int64 tensor of the G buffers' addresses."""
    _need(x, "x")
    T, d = x.shape
    k = plan.dst_rank.shape[1]
    rc = lib.moe_dispatch_ep(_ptr(x), _ptr(plan.dst_rank), _ptr(plan.dst_row), T, d, k,
                             _dtype_code(x.dtype), _ptr(recv_table), recv_table.numel(),
                             rows_max, _stream(x))
    _check("moe_dispatch_ep", rc)


def moe_combine_ep(ye_table: torch.Tensor, plan: EPPlan, gate: torch.Tensor, d: int,
                   dtype: torch.dtype, rows_max: int,
                   out: Optional[torch.Tensor] = None) -> torch.Tensor:
    T, k = plan.dst_rank.shape
    if out is None:
        out = torch.empty((T, d), dtype=dtype, device=gate.device)
    rc = lib.moe_combine_ep(_ptr(ye_table), _ptr(plan.dst_rank), _ptr(plan.dst_row), _ptr(gate),
                            T, d, k, _dtype_code(dtype), ye_table.numel(), rows_max, _ptr(out),
                            _stream(gate))
    _check("moe_combine_ep", rc)
    return out


def moe_get_status(clear: bool = True, device=None) -> int:
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    v = ctypes.c_int32(0)
    with torch.cuda.device(dev):
        rc = lib.moe_get_status(ctypes.byref(v), int(clear), torch.cuda.current_stream(dev).cuda_stream)
    _check("moe_get_status", rc)
    return int(v.value)


def moe_version() -> str:
    return lib.moe_version().decode()


def moe_debug_set_wait_limit_ns(ns: int, device=None) -> None:
    """Test-only: time limit of the kernels' pipeline waits on the device
    (0 = the default 2 s)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        rc = lib.moe_debug_set_wait_limit_ns(int(ns))
    _check("moe_debug_set_wait_limit_ns", rc)


GEMM_FORM_AUTO, GEMM_FORM_ROWS, GEMM_FORM_TOKENS = 0, 1, 2


def moe_debug_set_gemm_form(form: int) -> None:
    """Test-only: tile form of the grouped GEMMs (GEMM_FORM_AUTO by shape,
    GEMM_FORM_ROWS, GEMM_FORM_TOKENS where the weight layout allows)."""
    _check("moe_debug_set_gemm_form", lib.moe_debug_set_gemm_form(int(form)))


# ----------------------------------------------------------------- MXFP8 path

@dataclass
class MxWeights:
    """E4M3 codes and UE8M0 scales of W1, W3 [E,F,d] and W2 [E,d,F], and the
    scales packed for the GEMMs (mxfp8_pack_weight_scales; filled by
    mxfp8_quantize_weights, or on first use)."""
    W1q: torch.Tensor
    W1s: torch.Tensor
    W3q: torch.Tensor
    W3s: torch.Tensor
    W2q: torch.Tensor
    W2s: torch.Tensor
    Ps13: Optional[torch.Tensor] = None
    Ps2: Optional[torch.Tensor] = None


def mxfp8_pack_weight_scales(w: MxWeights) -> MxWeights:
    E, F, d = w.W1q.shape
    dev = w.W1q.device
    w.Ps13 = torch.empty(E * (F // 128) * (d // 128) * 1024, dtype=torch.uint8, device=dev)
    w.Ps2 = torch.empty(E * ((d + 255) // 256) * (F // 128) * 1024, dtype=torch.uint8, device=dev)
    for t in (w.W1s, w.W3s, w.W2s):
        _need(t, "weight scales")
    rc = lib.mxfp8_pack_weight_scales(_ptr(w.W1s), _ptr(w.W3s), _ptr(w.W2s), E, d, F,
                                      _ptr(w.Ps13), _ptr(w.Ps2), _stream(w.W1q))
    _check("mxfp8_pack_weight_scales", rc)
    return w


def _packed(w: MxWeights) -> MxWeights:
    return w if w.Ps13 is not None else mxfp8_pack_weight_scales(w)


def mxfp8_quantize_weights(W1, W3, W2) -> MxWeights:
    """Offline quantisation of the expert weights along their contraction
    dimension (d for W1/W3, F for W2) with UE8M0 block scales, plus the
    scales packed for the GEMMs."""
    E, F, d = W1.shape
    q1, s1 = mxfp8_quantize(W1.reshape(E * F, d), MOE_SCALE_E8M0)
    q3, s3 = mxfp8_quantize(W3.reshape(E * F, d), MOE_SCALE_E8M0)
    q2, s2 = mxfp8_quantize(W2.reshape(E * d, F), MOE_SCALE_E8M0)
    w = MxWeights(q1.view(E, F, d), s1.view(E, F, d // 32), q3.view(E, F, d),
                  s3.view(E, F, d // 32), q2.view(E, d, F), s2.view(E, d, F // 32))
    return mxfp8_pack_weight_scales(w)


def moe_dispatch_mxfp8(x, slot, Xq=None, Xs=None):
    _need(x, "x"); _need(slot, "slot")
    T, d = x.shape
    k = slot.shape[1]
    if Xq is None:
        Xq = torch.empty((T * k, d), dtype=torch.uint8, device=x.device)
    if Xs is None:
        Xs = torch.empty((T * k, d // 32), dtype=torch.uint8, device=x.device)
    rc = lib.moe_dispatch_mxfp8(_ptr(x), _ptr(slot), T, d, k, _ptr(Xq), _ptr(Xs), _stream(x))
    _check("moe_dispatch_mxfp8", rc)
    return Xq, Xs


def mxfp8_pack_act_scales(S, offsets, E: int, Sp=None):
    """Row-layout activation scales [R, K/32] -> the tile-packed layout the
    MXFP8 GEMMs read (blocks of 512 bytes per 128-row tile and K slab)."""
    _need(S, "S"); _need(offsets, "offsets")
    R, kb = S.shape
    if Sp is None:
        Sp = torch.empty(lib.mxfp8_act_scales_packed_size(E, R, kb * 32), dtype=torch.uint8,
                         device=S.device)
    rc = lib.mxfp8_pack_act_scales(_ptr(S), _ptr(offsets), E, R, kb * 32, _ptr(Sp), _stream(S))
    _check("mxfp8_pack_act_scales", rc)
    return Sp


def mxfp8_unpack_act_scales(Sp, offsets, E: int, R: int, K: int, S=None):
    """Tile-packed activation scales -> row layout [R, K/32]."""
    _need(Sp, "Sp"); _need(offsets, "offsets")
    if S is None:
        S = torch.empty((R, K // 32), dtype=torch.uint8, device=Sp.device)
    rc = lib.mxfp8_unpack_act_scales(_ptr(Sp), _ptr(offsets), E, R, K, _ptr(S), _stream(Sp))
    _check("mxfp8_unpack_act_scales", rc)
    return S


def moe_grouped_gate_up_mxfp8(Xq, Xs, w: MxWeights, offsets, Hq=None, Hs=None, *,
                              packed: bool = False, A=None, B=None):
    """H = quantised SwiGLU of the block-scaled FP8 gate/up GEMMs. With
    packed=False, Xs and the returned Hs are in row layout (packed and
    unpacked here); with packed=True both are in the tile-packed layout.
    A, B ([R,F] bf16, both or neither) receive the pre-activations."""
    _need(Xq, "Xq"); _need(Xs, "Xs"); _need(offsets, "offsets")
    E, F, d = w.W1q.shape
    R = Xq.shape[0]
    dev = Xq.device
    if Hq is None:
        Hq = torch.empty((R, F), dtype=torch.uint8, device=dev)
    Xsp = Xs if packed else mxfp8_pack_act_scales(Xs, offsets, E)
    Hsp = Hs if (packed and Hs is not None) else torch.empty(
        lib.mxfp8_act_scales_packed_size(E, R, F), dtype=torch.uint8, device=dev)
    w = _packed(w)
    rc = lib.moe_grouped_gate_up_mxfp8_save(_ptr(Xq), _ptr(Xsp), _ptr(w.W1q), _ptr(w.W3q),
                                            _ptr(w.Ps13), w.W1q.stride(0), _ptr(offsets), E, R, d,
                                            F, _ptr(Hq), _ptr(Hsp), _ptr(A), _ptr(B), _stream(Xq))
    _check("moe_grouped_gate_up_mxfp8", rc)
    if packed:
        return Hq, Hsp
    return Hq, mxfp8_unpack_act_scales(Hsp, offsets, E, R, F, Hs)


def moe_grouped_down_mxfp8(Hq, Hs, w: MxWeights, offsets, Ye=None, *, packed: bool = False):
    """Ye = the block-scaled FP8 down GEMM; Hs in row layout unless packed."""
    _need(Hq, "Hq"); _need(Hs, "Hs"); _need(offsets, "offsets")
    E, d, F = w.W2q.shape
    R = Hq.shape[0]
    if Ye is None:
        Ye = torch.empty((R, d), dtype=torch.bfloat16, device=Hq.device)
    Hsp = Hs if packed else mxfp8_pack_act_scales(Hs, offsets, E)
    w = _packed(w)
    rc = lib.moe_grouped_down_mxfp8(_ptr(Hq), _ptr(Hsp), _ptr(w.W2q), _ptr(w.Ps2), w.W2q.stride(0),
                                    _ptr(offsets), E, R, d, F, _ptr(Ye), _stream(Hq))
    _check("moe_grouped_down_mxfp8", rc)
    return Ye


def moe_grouped_mxfp8_gemm(Aq, Asp, Bq, Pb, offsets, out=None):
    """out[r] = A[r] · B_eᵀ for each expert e's rows on block-scaled FP8
    (the down GEMM's kernel): Aq [R,K] E4M3 codes with tile-packed scales
    Asp (K = the contraction), Bq [E,N,K] codes with scales packed as a W2
    operand (mxfp8_pack_weight_scales); out [R,N] bf16."""
    for t, n in ((Aq, "Aq"), (Asp, "Asp"), (Bq, "Bq"), (Pb, "Pb"), (offsets, "offsets")):
        _need(t, n)
    E, N, K = Bq.shape
    R = Aq.shape[0]
    if out is None:
        out = torch.empty((R, N), dtype=torch.bfloat16, device=Aq.device)
    rc = lib.moe_grouped_down_mxfp8(_ptr(Aq), _ptr(Asp), _ptr(Bq), _ptr(Pb), Bq.stride(0),
                                    _ptr(offsets), E, R, N, K, _ptr(out), _stream(Aq))
    _check("moe_grouped_down_mxfp8", rc)
    return out


def moe_grouped_swiglu_wgrad(Xe, dA, dB, dYe, H, offsets, out=None):
    """dW1 = dAᵀ Xe, dW3 = dBᵀ Xe, dW2 = dYeᵀ H per expert (bf16); returns
    (dW1, dW3, dW2), or fills `out` = (dW1, dW3, dW2)."""
    for t, n in ((Xe, "Xe"), (dA, "dA"), (dB, "dB"), (dYe, "dYe"), (H, "H"),
                 (offsets, "offsets")):
        _need(t, n)
    R, d = Xe.shape
    F = dA.shape[1]
    E = offsets.numel() - 1
    if out is None:
        kw = dict(dtype=Xe.dtype, device=Xe.device)
        out = (torch.empty((E, F, d), **kw), torch.empty((E, F, d), **kw),
               torch.empty((E, d, F), **kw))
    dW1, dW3, dW2 = out
    rc = lib.moe_grouped_swiglu_wgrad(_ptr(Xe), _ptr(dA), _ptr(dB), _ptr(dYe), _ptr(H),
                                      _ptr(offsets), E, R, d, F, _dtype_code(Xe.dtype), _ptr(dW1),
                                      _ptr(dW3), _ptr(dW2), _stream(Xe))
    _check("moe_grouped_swiglu_wgrad", rc)
    return out


def moe_layer_fwd_mxfp8(x, k: int, w: MxWeights, *, logits=None, Wr=None, renorm: bool = False,
                        out: Optional[LayerOut] = None, save: bool = False) -> LayerOut:
    """The MXFP8 layer. save=True keeps what moe_layer_bwd_mxfp8 reads:
    Xq/Xs (dispatched codes, row-layout scales), Hq/Hsp (H codes, tile-packed
    scales) and the bf16 pre-activations A, B."""
    _need(x, "x")
    w = _packed(w)
    T, d = x.shape
    E, F, _ = w.W1q.shape
    dev = x.device
    if out is None:
        i32 = dict(dtype=torch.int32, device=dev)
        ws = _alloc_ws(lib.moe_layer_mxfp8_workspace_size(T, d, E, F, k, int(logits is not None)), dev)
        out = LayerOut(out=torch.empty((T, d), dtype=torch.bfloat16, device=dev),
                       idx=torch.empty((T, k), **i32),
                       gate=torch.empty((T, k), dtype=torch.float32, device=dev),
                       counts=torch.empty(E, **i32), offsets=torch.empty(E + 1, **i32),
                       slot=torch.empty((T, k), **i32), workspace=ws)
        if save:
            R = T * k
            u8 = dict(dtype=torch.uint8, device=dev)
            out.Xq = torch.empty((R, d), **u8)
            out.Xs = torch.empty((R, d // 32), **u8)
            out.Hq = torch.empty((R, F), **u8)
            out.Hsp = torch.empty(max(1, lib.mxfp8_act_scales_packed_size(E, R, F)), **u8)
            out.A = torch.empty((R, F), dtype=torch.bfloat16, device=dev)
            out.B = torch.empty((R, F), dtype=torch.bfloat16, device=dev)
    if save and out.Xq is None:
        raise ValueError("save=True needs an `out` made with save=True")
    a = LayerMxArgs(T=T, d=d, E=E, F=F, k=k, renorm=int(renorm), reserved0=0, reserved1=0,
                    x=_ptr(x), logits=_ptr(logits), Wr=_ptr(Wr), W1q=_ptr(w.W1q), W3q=_ptr(w.W3q),
                    W2q=_ptr(w.W2q), Ps13=_ptr(w.Ps13), Ps2=_ptr(w.Ps2),
                    w13_expert_stride=w.W1q.stride(0), w2_expert_stride=w.W2q.stride(0),
                    out=_ptr(out.out), idx=_ptr(out.idx), gate=_ptr(out.gate),
                    counts=_ptr(out.counts), offsets=_ptr(out.offsets), slot=_ptr(out.slot),
                    workspace=_ptr(out.workspace), workspace_bytes=out.workspace.numel())
    if save:
        a.save_Xq, a.save_Xs, a.save_Hq = _ptr(out.Xq), _ptr(out.Xs), _ptr(out.Hq)
        a.save_Hsp, a.save_A, a.save_B = _ptr(out.Hsp), _ptr(out.A), _ptr(out.B)
    rc = lib.moe_layer_fwd_mxfp8(ctypes.byref(a), _stream(x))
    _check("moe_layer_fwd_mxfp8", rc)
    return out


@dataclass
class MxWeightsBwd:
    """Backward weights of the MXFP8 layer: W13tq [E,d,2F] (row i = column i
    of W1_e then of W3_e, blocks of 32 along F) and W2tq [E,F,d] (row f =
    column f of W2_e, blocks along d), their UE8M0 scales and the scales
    packed for the FP8 GEMMs."""
    W13tq: torch.Tensor
    W13ts: torch.Tensor
    W2tq: torch.Tensor
    W2ts: torch.Tensor
    Ps13t: torch.Tensor
    Ps2t: torch.Tensor


def mxfp8_quantize_weights_bwd(W1, W3, W2) -> MxWeightsBwd:
    """Re-quantise the bf16 expert weights along the contraction dimensions
    of the backward's input-gradient GEMMs (F for W1/W3, d for W2) and pack
    their scales; once per weight update."""
    for t, n in ((W1, "W1"), (W3, "W3"), (W2, "W2")):
        if not t.is_cuda:
            raise ValueError(f"{n} must be a CUDA tensor")
    E, F, d, s13 = _w13(W1, W3)  # views into a fused [E,2F,d] tensor are accepted
    if tuple(W2.shape) != (E, d, F) or W2.stride(1) != F or W2.stride(2) != 1:
        raise ValueError("W2 must be [E,d,F] with rows contiguous")
    dev = W1.device
    u8 = dict(dtype=torch.uint8, device=dev)
    wb = MxWeightsBwd(W13tq=torch.empty((E, d, 2 * F), **u8),
                      W13ts=torch.empty((E, d, 2 * F // 32), **u8),
                      W2tq=torch.empty((E, F, d), **u8), W2ts=torch.empty((E, F, d // 32), **u8),
                      Ps13t=torch.empty(E * ((d + 255) // 256) * (2 * F // 128) * 1024, **u8),
                      Ps2t=torch.empty(E * ((F + 255) // 256) * (d // 128) * 1024, **u8))
    st = _stream(W1)
    rc = lib.mxfp8_quantize_weights_bwd(_ptr(W1), _ptr(W3), _ptr(W2), s13, _w2(W2)[3], E, d, F,
                                        _ptr(wb.W13tq), _ptr(wb.W13ts), _ptr(wb.W2tq),
                                        _ptr(wb.W2ts), st)
    _check("mxfp8_quantize_weights_bwd", rc)
    # both packed as the down GEMM's W2 operand: [E, rows, K]
    rc = lib.mxfp8_pack_weight_scales(None, None, _ptr(wb.W2ts), E, F, d, None, _ptr(wb.Ps2t), st)
    _check("mxfp8_pack_weight_scales", rc)
    rc = lib.mxfp8_pack_weight_scales(None, None, _ptr(wb.W13ts), E, d, 2 * F, None,
                                      _ptr(wb.Ps13t), st)
    _check("mxfp8_pack_weight_scales", rc)
    return wb


def moe_swiglu_bwd_mxfp8(dH, A, B, dA=None, dB=None, dABq=None, dABs=None):
    """dA = dH*B*silu'(A), dB = dH*silu(A) (bf16) and the MXFP8 codes and
    row-layout scales of [dA | dB] quantised from the fp32 values."""
    for t, n in ((dH, "dH"), (A, "A"), (B, "B")):
        _need(t, n)
    R, F = dH.shape
    dev = dH.device
    dA = torch.empty_like(dH) if dA is None else dA
    dB = torch.empty_like(dH) if dB is None else dB
    dABq = torch.empty((R, 2 * F), dtype=torch.uint8, device=dev) if dABq is None else dABq
    dABs = torch.empty((R, 2 * F // 32), dtype=torch.uint8, device=dev) if dABs is None else dABs
    rc = lib.moe_swiglu_bwd_mxfp8(_ptr(dH), _ptr(A), _ptr(B), R, F, _ptr(dA), _ptr(dB),
                                  _ptr(dABq), _ptr(dABs), _stream(dH))
    _check("moe_swiglu_bwd_mxfp8", rc)
    return dA, dB, dABq, dABs


def moe_layer_bwd_mxfp8(fwd: LayerOut, dOut, k: int, wb: MxWeightsBwd,
                        out: Optional[LayerGrads] = None) -> LayerGrads:
    """Backward of moe_layer_fwd_mxfp8(save=True) with the gates held
    constant: FP8 input-gradient GEMMs with wb's weights, bf16 weight
    gradients on the forward's dequantised operands."""
    _need(dOut, "dOut")
    if fwd.Xq is None or fwd.A is None:
        raise ValueError("moe_layer_bwd_mxfp8 needs the MXFP8 forward run with save=True")
    T, d = dOut.shape
    E, F = wb.W2tq.shape[0], wb.W2tq.shape[1]
    dev = dOut.device
    if out is None:
        ws = _alloc_ws(lib.moe_layer_bwd_mxfp8_workspace_size(T, d, E, F, k), dev)
        bf = dict(dtype=torch.bfloat16, device=dev)
        out = LayerGrads(dx=torch.empty((T, d), **bf), dW1=torch.empty((E, F, d), **bf),
                         dW3=torch.empty((E, F, d), **bf), dW2=torch.empty((E, d, F), **bf),
                         workspace=ws)
    a = LayerBwdMxArgs(T=T, d=d, E=E, F=F, k=k, reserved0=0, reserved1=0, reserved2=0,
                       slot=_ptr(fwd.slot), gate=_ptr(fwd.gate), offsets=_ptr(fwd.offsets),
                       Xq=_ptr(fwd.Xq), Xs=_ptr(fwd.Xs), Hq=_ptr(fwd.Hq), Hsp=_ptr(fwd.Hsp),
                       A=_ptr(fwd.A), B=_ptr(fwd.B), W13tq=_ptr(wb.W13tq), Ps13t=_ptr(wb.Ps13t),
                       W2tq=_ptr(wb.W2tq), Ps2t=_ptr(wb.Ps2t), dOut=_ptr(dOut), dx=_ptr(out.dx),
                       dW1=_ptr(out.dW1), dW3=_ptr(out.dW3), dW2=_ptr(out.dW2),
                       workspace=_ptr(out.workspace), workspace_bytes=out.workspace.numel())
    rc = lib.moe_layer_bwd_mxfp8(ctypes.byref(a), _stream(dOut))
    _check("moe_layer_bwd_mxfp8", rc)
    return out


class HostLayerMxfp8:
    """moe_layer_fwd_mxfp8_host: the MXFP8 layer from pinned host x (bf16,
    and logits) to pinned host out (bf16), in `chunks` token slices whose
    copies overlap the compute. Holds the staging buffers, routing outputs,
    workspace and copy streams, so repeated calls of one shape allocate
    nothing."""

    def __init__(self, T: int, d: int, E: int, F: int, k: int, device, *, logits_given: bool,
                 chunks: int = 3):
        if not 1 <= chunks <= 64:
            raise ValueError("chunks must be in [1, 64]")
        dev = torch.device(device)
        i32 = dict(dtype=torch.int32, device=dev)
        self.T, self.d, self.E, self.F, self.k = T, d, E, F, k
        self.chunks = chunks
        self.x = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
        self.logits = torch.empty((T, E), dtype=torch.float32, device=dev) if logits_given else None
        self.res = LayerOut(out=torch.empty((T, d), dtype=torch.bfloat16, device=dev),
                            idx=torch.empty((T, k), **i32),
                            gate=torch.empty((T, k), dtype=torch.float32, device=dev),
                            counts=torch.empty(E, **i32), offsets=torch.empty(E + 1, **i32),
                            slot=torch.empty((T, k), **i32),
                            workspace=_alloc_ws(lib.moe_layer_mxfp8_workspace_size(
                                T, d, E, F, k, int(logits_given)), dev))
        self.s_h2d = torch.cuda.Stream(dev)
        self.s_d2h = torch.cuda.Stream(dev)

    def __call__(self, x_host: torch.Tensor, w: MxWeights, *, logits_host=None, Wr=None,
                 renorm: bool = False, out_host: Optional[torch.Tensor] = None) -> torch.Tensor:
        if x_host.is_cuda or tuple(x_host.shape) != (self.T, self.d) or x_host.dtype != torch.bfloat16:
            raise ValueError("x_host must be a [T, d] bf16 host tensor")
        if (logits_host is None) != (self.logits is None):
            raise ValueError("logits_host must be given exactly when the layer was built for it")
        if logits_host is not None and (logits_host.is_cuda or logits_host.dtype != torch.float32
                                        or tuple(logits_host.shape) != (self.T, self.E)):
            raise ValueError("logits_host must be a [T, E] fp32 host tensor")
        if out_host is None:
            out_host = torch.empty((self.T, self.d), dtype=torch.bfloat16, pin_memory=True)
        w = _packed(w)
        r = self.res
        a = LayerMxArgs(T=self.T, d=self.d, E=self.E, F=self.F, k=self.k, renorm=int(renorm),
                        reserved0=0, reserved1=0, x=_ptr(self.x), logits=_ptr(self.logits),
                        Wr=_ptr(Wr), W1q=_ptr(w.W1q), W3q=_ptr(w.W3q), W2q=_ptr(w.W2q),
                        Ps13=_ptr(w.Ps13), Ps2=_ptr(w.Ps2), w13_expert_stride=w.W1q.stride(0),
                        w2_expert_stride=w.W2q.stride(0), out=_ptr(r.out), idx=_ptr(r.idx),
                        gate=_ptr(r.gate), counts=_ptr(r.counts), offsets=_ptr(r.offsets),
                        slot=_ptr(r.slot), workspace=_ptr(r.workspace),
                        workspace_bytes=r.workspace.numel())
        rc = lib.moe_layer_fwd_mxfp8_host(ctypes.byref(a), x_host.data_ptr(), _ptr(logits_host),
                                          out_host.data_ptr(), self.chunks, _stream(self.x),
                                          self.s_h2d.cuda_stream, self.s_d2h.cuda_stream)
        _check("moe_layer_fwd_mxfp8_host", rc)
        return out_host
