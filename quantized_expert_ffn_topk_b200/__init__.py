"""Python binding of libmoeq.so, the B200 (sm_100a) quantized MoE FFN step.

Argument marshalling only: every step runs in the library's CUDA kernels.
Functions carry the C names of ``include/moeq.h`` and accept torch CUDA
tensors (or raw device addresses as ints); the stream defaults to torch's
current stream. A non-OK status raises ``MoeError``. PyTorch is used for
device memory and streams only.

The library must be built (``build.build()``); importing this module on a
machine without it raises instead of falling back to anything else.
"""
from __future__ import annotations

import ctypes
import os

from . import build as _build

LIB_PATH = _build.LIB

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_ALIGN, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA = 0, 1, 2, 3, 4
MOE_ERR_INDEX, MOE_ERR_TIMEOUT, MOE_ERR_WORKSPACE, MOE_ERR_RANGE = 5, 6, 7, 8
MOEQ_MAX_K = 8
MOEQ_MAX_B = 128
MOEQ_STATIC_SCRATCH_BYTES = 2 << 20


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s: %s (status %d)" % (where, status_str(status), status))


class moe_layer_q(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int), ("I", ctypes.c_int), ("E", ctypes.c_int), ("K", ctypes.c_int),
                ("group", ctypes.c_int), ("bits_routed", ctypes.c_int), ("bits_shared", ctypes.c_int),
                ("experts", ctypes.c_void_p), ("shared", ctypes.c_void_p), ("router_w", ctypes.c_void_p),
                ("shared_gate_w", ctypes.c_void_p)]


_lib = None
_VP, _SZ, _INT, _FLT = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_float
_LP = ctypes.POINTER(moe_layer_q)

_SIGS = {
    "moe_abi_version": (_INT, []),
    "moe_status_str": (ctypes.c_char_p, [_INT]),
    "moe_expert_bytes": (_SZ, [_INT, _INT, _INT, _INT]),
    "moe_expert_layout": (_INT, [_INT, _INT, _INT, _INT, ctypes.POINTER(_SZ)]),
    "moe_workspace_bytes": (_SZ, [_INT, _INT, _INT, _INT, _INT]),
    "moe_workspace_init": (_INT, [_VP, _SZ, _VP]),
    "moe_workspace_debug": (_INT, [_VP, _SZ, ctypes.c_uint, _INT, _VP]),
    "moe_rmsnorm": (_INT, [_VP, _VP, _INT, _INT, _FLT, _VP, _VP]),
    "moe_pack_q": (_INT, [_VP, _VP, _VP, _INT, _INT, _INT, _INT, _VP, _VP, _VP, _VP]),
    "moe_pack_expert": (_INT, [_VP] * 9 + [_INT, _INT, _INT, _INT, _VP, _VP, _VP]),
    "moe_quantize": (_INT, [_VP, _INT, _INT, _INT, _INT, _INT, _VP, _VP, _VP, _VP, _VP]),
    "moe_router_topk": (_INT, [_VP, _VP, _INT, _INT, _INT, _INT, _INT, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "moe_expert_ffn_q": (_INT, [_LP, _VP, _INT, _VP, _VP, _VP, _SZ, _VP]),
    "moe_combine_residual": (_INT, [_LP, _VP, _VP, _VP, _VP, _INT, _VP, _VP, _FLT, _VP]),
    "moe_decode_layers": (_INT, [_LP, _INT, _VP, _VP, _INT, _VP, _VP, _VP, _VP, _VP, _FLT, _VP, _SZ, _VP]),
    "moe_get_device_error": (_INT, [_VP, _VP]),
    "moe_expert_ffn_q_static": (_INT, [_LP, _VP, _INT, _VP, _VP, _VP, _VP]),
}


def lib() -> ctypes.CDLL:
    """Load libmoeq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libmoeq.so not found at %s: build it with __graft_entry__.build()" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def exported_symbols():
    return sorted(_SIGS)


def status_str(status: int) -> str:
    return lib().moe_status_str(int(status)).decode()


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str) -> None:
    if status != MOE_OK:
        raise MoeError(status, where)


# ---- sizes ------------------------------------------------------------------

def moe_expert_bytes(H: int, I: int, bits: int, group: int) -> int:
    return int(lib().moe_expert_bytes(H, I, bits, group))


def moe_expert_layout(H: int, I: int, bits: int, group: int):
    """[unit bytes U, down offset, down block bytes D, rows per block, gate/up code row bytes, down code row bytes]"""
    lay = (ctypes.c_size_t * 6)()
    _check(lib().moe_expert_layout(H, I, bits, group, lay), "moe_expert_layout")
    return [int(v) for v in lay]


def moe_workspace_bytes(B: int, K: int, H: int, I: int, E: int) -> int:
    return int(lib().moe_workspace_bytes(B, K, H, I, E))


def moe_workspace_init(ws, ws_bytes: int = None, stream=None) -> None:
    n = ws_bytes if ws_bytes is not None else ws.numel() * ws.element_size()
    _check(lib().moe_workspace_init(_ptr(ws), n, _stream(stream)), "moe_workspace_init")


def moe_workspace_debug(ws, ws_bytes: int, wait_budget_us: int, withhold_cta: int, stream=None) -> None:
    """Testing hook of the bounded waits (see include/moeq.h)."""
    _check(lib().moe_workspace_debug(_ptr(ws), ws_bytes, int(wait_budget_us), int(withhold_cta), _stream(stream)),
           "moe_workspace_debug")


# ---- the four calls ---------------------------------------------------------

def moe_pack_q(codes, scale_bf16, bias_bf16, rows: int, cols: int, bits: int, group: int, packed_out, sb_out,
               ws=None, stream=None) -> None:
    _check(lib().moe_pack_q(_ptr(codes), _ptr(scale_bf16), _ptr(bias_bf16), rows, cols, bits, group,
                            _ptr(packed_out), _ptr(sb_out), _ptr(ws), _stream(stream)), "moe_pack_q")


def moe_quantize(w, in_bf16: bool, rows: int, cols: int, bits: int, group: int, codes_out, scale_out, bias_out,
                 ws=None, stream=None) -> None:
    _check(lib().moe_quantize(_ptr(w), int(bool(in_bf16)), rows, cols, bits, group, _ptr(codes_out), _ptr(scale_out),
                              _ptr(bias_out), _ptr(ws), _stream(stream)), "moe_quantize")


def moe_pack_expert(gate, up, down, H: int, I: int, bits: int, group: int, record_out, ws=None, stream=None) -> None:
    """gate/up/down = (codes u8, scale bf16, bias bf16) device buffers."""
    args = [_ptr(t) for m in (gate, up, down) for t in m]
    _check(lib().moe_pack_expert(*args, H, I, bits, group, _ptr(record_out), _ptr(ws), _stream(stream)),
           "moe_pack_expert")


def moe_router_topk(x_bf16, router_w_bf16, B: int, H: int, E: int, K: int, renorm: bool, forced_idx, idx_out, w_out,
                    logits_out, ws, ws_bytes: int, stream=None) -> None:
    _check(lib().moe_router_topk(_ptr(x_bf16), _ptr(router_w_bf16), B, H, E, K, int(bool(renorm)), _ptr(forced_idx),
                                 _ptr(idx_out), _ptr(w_out), _ptr(logits_out), _ptr(ws), ws_bytes, _stream(stream)),
           "moe_router_topk")


def moe_expert_ffn_q(layer: moe_layer_q, x_bf16, B: int, idx, y_out, ws, ws_bytes: int, stream=None) -> None:
    _check(lib().moe_expert_ffn_q(ctypes.byref(layer), _ptr(x_bf16), B, _ptr(idx), _ptr(y_out), _ptr(ws), ws_bytes,
                                  _stream(stream)), "moe_expert_ffn_q")


def moe_combine_residual(layer: moe_layer_q, y, w, x_bf16, resid_in, B: int, resid_out, xnorm_bf16_out, eps: float,
                         stream=None) -> None:
    _check(lib().moe_combine_residual(ctypes.byref(layer), _ptr(y), _ptr(w), _ptr(x_bf16), _ptr(resid_in), B,
                                      _ptr(resid_out), _ptr(xnorm_bf16_out), float(eps), _stream(stream)),
           "moe_combine_residual")


def moe_rmsnorm(r, weight_bf16, B: int, H: int, eps: float, xnorm_bf16_out, stream=None) -> None:
    _check(lib().moe_rmsnorm(_ptr(r), _ptr(weight_bf16), B, H, float(eps), _ptr(xnorm_bf16_out), _stream(stream)),
           "moe_rmsnorm")


def layer_table(layers):
    """A C array of moe_layer_q for moe_decode_layers, built once and reused
    across calls (saves rebuilding it on every token)."""
    return (moe_layer_q * len(layers))(*layers)


def moe_decode_layers(layers, x_bf16, resid_in, renorm: bool, forced_idx, idx_out, w_out, resid_out, xnorm_bf16_out,
                      eps: float, ws, ws_bytes: int, stream=None) -> None:
    """layers: a sequence of moe_layer_q (one token through all of them), or
    a table from layer_table()."""
    arr = layers if isinstance(layers, ctypes.Array) else (moe_layer_q * len(layers))(*layers)
    _check(lib().moe_decode_layers(arr, len(layers), _ptr(x_bf16), _ptr(resid_in), int(bool(renorm)),
                                   _ptr(forced_idx), _ptr(idx_out), _ptr(w_out), _ptr(resid_out),
                                   _ptr(xnorm_bf16_out), float(eps), _ptr(ws), ws_bytes, _stream(stream)),
           "moe_decode_layers")


def moe_expert_ffn_q_static(layer: moe_layer_q, x_bf16, B: int, idx, y_out, error_out=None, stream=None) -> None:
    """moe_expert_ffn_q on the library's own static scratch (no workspace argument)."""
    _check(lib().moe_expert_ffn_q_static(ctypes.byref(layer), _ptr(x_bf16), B, _ptr(idx), _ptr(y_out),
                                         _ptr(error_out), _stream(stream)), "moe_expert_ffn_q_static")


def moe_get_device_error(ws, stream=None) -> int:
    """Synchronises the stream; returns the device error status (and clears it)."""
    st = lib().moe_get_device_error(_ptr(ws), _stream(stream))
    if st == MOE_ERR_CUDA:
        raise MoeError(st, "moe_get_device_error")
    return int(st)


from .layer import QuantLayer, Workspace  # noqa: E402  (device-memory owners built on the calls above)
