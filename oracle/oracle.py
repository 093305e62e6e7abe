"""Python access to the oracle (plain single-threaded fp64 C, ``moe_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg use it; the library's code path never does.
It shares no code with the CUDA path. ``build()`` compiles ``liboracle.so``
next to this file with gcc; every wrapper takes and returns numpy arrays.
Sources and the readings taken where the pages are silent are listed in
``moe_oracle.h``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_HDR = os.path.join(_HERE, "moe_oracle.h")
_LIB = os.path.join(_HERE, "liboracle.so")

_lib = None

_u8p = ctypes.POINTER(ctypes.c_uint8)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_i32p = ctypes.POINTER(ctypes.c_int32)
_f64p = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compile liboracle.so (gcc, C99, -O2, no fp contraction)."""
    stale = (not os.path.exists(_LIB)) or max(os.path.getmtime(_SRC), os.path.getmtime(_HDR)) > os.path.getmtime(_LIB)
    if force or stale:
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        L.moe_ref_bf16_to_f64.restype = ctypes.c_double
        L.moe_ref_bf16_to_f64.argtypes = [ctypes.c_uint16]
        L.moe_ref_f64_to_bf16.restype = ctypes.c_uint16
        L.moe_ref_f64_to_bf16.argtypes = [ctypes.c_double]
        L.moe_ref_expert_bytes.restype = ctypes.c_size_t
        L.moe_ref_expert_bytes.argtypes = [ctypes.c_int] * 4
        for name in ("moe_ref_pack", "moe_ref_unpack"):
            getattr(L, name).restype = ctypes.c_int
        L.moe_ref_pack.argtypes = [_u8p, _u16p, _u16p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                   ctypes.c_int, _u8p, _u16p]
        L.moe_ref_unpack.argtypes = [_u8p, _u16p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                     _u8p, _u16p, _u16p]
        L.moe_ref_quantize.restype = ctypes.c_int
        L.moe_ref_quantize.argtypes = [ctypes.POINTER(ctypes.c_float), ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, _u8p, _u16p, _u16p]
        for name in ("moe_ref_dequant_gemv", "moe_ref_dequant_gemv_fma", "moe_ref_dequant_gemv_grouped"):
            f = getattr(L, name)
            f.restype = None
            f.argtypes = [_u8p, _u16p, _u16p, ctypes.c_int, ctypes.c_int, ctypes.c_int, _f64p, _f64p]
        L.moe_ref_router_logits.restype = None
        L.moe_ref_router_logits.argtypes = [_u16p, _u16p, ctypes.c_int, ctypes.c_int, _f64p]
        L.moe_ref_softmax.restype = None
        L.moe_ref_softmax.argtypes = [_f64p, ctypes.c_int, _f64p]
        L.moe_ref_topk.restype = ctypes.c_int
        L.moe_ref_topk.argtypes = [_f64p, ctypes.c_int, ctypes.c_int, ctypes.c_int, _i32p, _i32p, _f64p]
        L.moe_ref_silu.restype = ctypes.c_double
        L.moe_ref_silu.argtypes = [ctypes.c_double]
        L.moe_ref_swiglu.restype = None
        L.moe_ref_swiglu.argtypes = [_f64p, _f64p, ctypes.c_int, _f64p]
        L.moe_ref_expert_ffn.restype = None
        L.moe_ref_expert_ffn.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         _u8p, _u16p, _u16p, _u8p, _u16p, _u16p, _u8p, _u16p, _u16p,
                                         _f64p, _f64p]
        L.moe_ref_shared_gate.restype = ctypes.c_double
        L.moe_ref_shared_gate.argtypes = [_u16p, _u16p, ctypes.c_int]
        L.moe_ref_combine.restype = None
        L.moe_ref_combine.argtypes = [ctypes.c_int, ctypes.c_int, _f64p, _f64p, ctypes.c_double, _f64p, _f64p]
        L.moe_ref_rmsnorm.restype = None
        L.moe_ref_rmsnorm.argtypes = [_f64p, ctypes.c_int, ctypes.c_double, _f64p]
        L.moe_ref_rmsnorm_bf16.restype = None
        L.moe_ref_rmsnorm_bf16.argtypes = [_f64p, ctypes.c_int, ctypes.c_double, _u16p]
        L.moe_ref_rmsnorm_weighted_bf16.restype = None
        L.moe_ref_rmsnorm_weighted_bf16.argtypes = [_f64p, _u16p, ctypes.c_int, ctypes.c_double, _u16p]
        _lib = L
    return _lib


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a: np.ndarray, ptype):
    return a.ctypes.data_as(ptype)


# ---- scalar helpers ---------------------------------------------------------

def bf16_to_f64(bits) -> np.ndarray:
    b = _c(np.atleast_1d(bits), np.uint16)
    L = lib()
    return np.array([L.moe_ref_bf16_to_f64(int(v)) for v in b.ravel()], dtype=np.float64).reshape(b.shape)


def f64_to_bf16(values) -> np.ndarray:
    v = _c(np.atleast_1d(values), np.float64)
    L = lib()
    return np.array([L.moe_ref_f64_to_bf16(float(t)) for t in v.ravel()], dtype=np.uint16).reshape(v.shape)


def expert_bytes(H: int, I: int, bits: int, group: int) -> int:
    return int(lib().moe_ref_expert_bytes(H, I, bits, group))


# ---- packing ----------------------------------------------------------------

def pack(codes, scale, bias, bits: int, group: int):
    """codes u8 [rows, cols], scale/bias bf16 bits [rows, cols/group] ->
    (packed u8 [rows, cols*bits/8], sb bf16 bits [rows, cols/group, 2])."""
    codes = _c(codes, np.uint8)
    rows, cols = codes.shape
    scale = _c(scale, np.uint16)
    bias = _c(bias, np.uint16)
    packed = np.zeros((rows, cols * bits // 8), dtype=np.uint8)
    sb = np.zeros((rows, cols // group, 2), dtype=np.uint16)
    rc = lib().moe_ref_pack(_p(codes, _u8p), _p(scale, _u16p), _p(bias, _u16p), rows, cols, bits, group,
                            _p(packed, _u8p), _p(sb, _u16p))
    if rc != 0:
        raise ValueError("moe_ref_pack rejected its arguments")
    return packed, sb


def unpack(packed, sb, rows: int, cols: int, bits: int, group: int):
    packed = _c(packed, np.uint8)
    sb = _c(sb, np.uint16)
    codes = np.zeros((rows, cols), dtype=np.uint8)
    scale = np.zeros((rows, cols // group), dtype=np.uint16)
    bias = np.zeros((rows, cols // group), dtype=np.uint16)
    rc = lib().moe_ref_unpack(_p(packed, _u8p), _p(sb, _u16p), rows, cols, bits, group,
                              _p(codes, _u8p), _p(scale, _u16p), _p(bias, _u16p))
    if rc != 0:
        raise ValueError("moe_ref_unpack rejected its arguments")
    return codes, scale, bias


def quantize(w, bits: int, group: int):
    """fp32 weights [rows, cols] -> (codes u8 [rows, cols], scale bf16 bits
    [rows, cols/group], bias bf16 bits [rows, cols/group]), min-max per group."""
    w = _c(w, np.float32)
    rows, cols = w.shape
    codes = np.zeros((rows, cols), dtype=np.uint8)
    scale = np.zeros((rows, cols // group), dtype=np.uint16)
    bias = np.zeros((rows, cols // group), dtype=np.uint16)
    rc = lib().moe_ref_quantize(w.ctypes.data_as(ctypes.POINTER(ctypes.c_float)), rows, cols, bits, group,
                                _p(codes, _u8p), _p(scale, _u16p), _p(bias, _u16p))
    if rc != 0:
        raise ValueError("moe_ref_quantize rejected its arguments")
    return codes, scale, bias


# ---- dequant GEMV -----------------------------------------------------------

def _gemv(fn, codes, scale, bias, group, x):
    codes = _c(codes, np.uint8)
    rows, cols = codes.shape
    scale = _c(scale, np.uint16)
    bias = _c(bias, np.uint16)
    x = _c(x, np.float64)
    assert x.shape == (cols,)
    y = np.zeros(rows, dtype=np.float64)
    fn(_p(codes, _u8p), _p(scale, _u16p), _p(bias, _u16p), rows, cols, group, _p(x, _f64p), _p(y, _f64p))
    return y


def dequant_gemv(codes, scale, bias, group, x):
    return _gemv(lib().moe_ref_dequant_gemv, codes, scale, bias, group, x)


def dequant_gemv_fma(codes, scale, bias, group, x):
    return _gemv(lib().moe_ref_dequant_gemv_fma, codes, scale, bias, group, x)


def dequant_gemv_grouped(codes, scale, bias, group, x):
    return _gemv(lib().moe_ref_dequant_gemv_grouped, codes, scale, bias, group, x)


# ---- router -----------------------------------------------------------------

def router_logits(x_bf16, wr_bf16):
    """x bf16 bits [H], W_r bf16 bits [E, H] -> logits fp64 [E]."""
    x = _c(x_bf16, np.uint16)
    wr = _c(wr_bf16, np.uint16)
    E, H = wr.shape
    out = np.zeros(E, dtype=np.float64)
    lib().moe_ref_router_logits(_p(x, _u16p), _p(wr, _u16p), H, E, _p(out, _f64p))
    return out


def softmax(logits):
    lg = _c(logits, np.float64)
    p = np.zeros_like(lg)
    lib().moe_ref_softmax(_p(lg, _f64p), lg.shape[0], _p(p, _f64p))
    return p


def topk(logits, K: int, renorm: bool = False, forced=None):
    lg = _c(logits, np.float64)
    E = lg.shape[0]
    idx = np.zeros(K, dtype=np.int32)
    w = np.zeros(K, dtype=np.float64)
    fp = None
    if forced is not None:
        f = _c(forced, np.int32)
        fp = _p(f, _i32p)
    rc = lib().moe_ref_topk(_p(lg, _f64p), E, K, int(bool(renorm)), fp, _p(idx, _i32p), _p(w, _f64p))
    if rc != 0:
        raise ValueError("moe_ref_topk rejected its arguments")
    return idx, w


# ---- SwiGLU, expert FFN -----------------------------------------------------

def silu(z: float) -> float:
    return float(lib().moe_ref_silu(float(z)))


def swiglu(g, u):
    g = _c(g, np.float64)
    u = _c(u, np.float64)
    h = np.zeros_like(g)
    lib().moe_ref_swiglu(_p(g, _f64p), _p(u, _f64p), g.shape[0], _p(h, _f64p))
    return h


def expert_ffn(H: int, I: int, group: int, gate, up, down, x):
    """gate/up/down = (codes, scale, bias) with codes [I,H], [I,H], [H,I];
    x fp64 [H] -> y fp64 [H]."""
    arrs = []
    for (codes, scale, bias) in (gate, up, down):
        arrs += [_c(codes, np.uint8), _c(scale, np.uint16), _c(bias, np.uint16)]
    x = _c(x, np.float64)
    y = np.zeros(H, dtype=np.float64)
    ptrs = []
    for i, a in enumerate(arrs):
        ptrs.append(_p(a, _u8p if i % 3 == 0 else _u16p))
    lib().moe_ref_expert_ffn(H, I, group, *ptrs, _p(x, _f64p), _p(y, _f64p))
    return y


# ---- combine, gate, norm ----------------------------------------------------

def shared_gate(wsg_bf16, x_bf16) -> float:
    w = _c(wsg_bf16, np.uint16)
    x = _c(x_bf16, np.uint16)
    return float(lib().moe_ref_shared_gate(_p(w, _u16p), _p(x, _u16p), w.shape[0]))


def combine(y, w, gamma: float, r):
    """y fp64 [K+1, H] (row K = shared expert), w [K], r [H] -> out [H]."""
    y = _c(y, np.float64)
    K = y.shape[0] - 1
    H = y.shape[1]
    w = _c(w, np.float64)
    r = _c(r, np.float64)
    out = np.zeros(H, dtype=np.float64)
    lib().moe_ref_combine(H, K, _p(y, _f64p), _p(w, _f64p), float(gamma), _p(r, _f64p), _p(out, _f64p))
    return out


def rmsnorm(v, eps: float):
    v = _c(v, np.float64)
    out = np.zeros_like(v)
    lib().moe_ref_rmsnorm(_p(v, _f64p), v.shape[0], float(eps), _p(out, _f64p))
    return out


def rmsnorm_bf16(v, eps: float):
    v = _c(v, np.float64)
    out = np.zeros(v.shape[0], dtype=np.uint16)
    lib().moe_ref_rmsnorm_bf16(_p(v, _f64p), v.shape[0], float(eps), _p(out, _u16p))
    return out


def rmsnorm_weighted_bf16(v, w_bf16, eps: float):
    """bf16 bits of v / rms(v) * w (w: bf16 bits [H], or None for unit weight)."""
    v = _c(v, np.float64)
    out = np.zeros(v.shape[0], dtype=np.uint16)
    wp = None
    if w_bf16 is not None:
        w = _c(w_bf16, np.uint16)
        assert w.shape == v.shape
        wp = _p(w, _u16p)
    lib().moe_ref_rmsnorm_weighted_bf16(_p(v, _f64p), wp, v.shape[0], float(eps), _p(out, _u16p))
    return out
