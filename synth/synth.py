"""Seeded synthetic inputs for the quantized MoE FFN step.

Input-generation infrastructure shared by the tests, the oracle's callers and
the benchmark. It holds none of the method's arithmetic: it only produces
codes, scales, biases, activations, router weights and forced routings with
stated distributions.

* Dense tensors come from the counter-based generator in ``synth_gen.h``:
  ``synth_host.c`` (CPU, numpy out) and ``synth_dev.cu`` (GPU, in place)
  produce identical bytes for the same (seed, tuple, element).
* Forced routings (the 24-layer stack with 27 % overlap between consecutive
  tokens, and Zipf(1.1)-popularity batches) come from numpy's PCG64.

Workload recipes (all seed 0):

``tiny``      H=256, E=8, I=128, top-2 + 1 shared, 4-bit, group 32
``layer4``    H=4096, E=512, I=1024, top-4 + 1 shared, 4-bit, group 64
``layer2``    as ``layer4`` with 2-bit routed experts (shared stays 4-bit)
``layer3``    as ``layer4`` with 3-bit routed experts (shared stays 4-bit)
``stack24``   24 ``layer4`` layers, 256 sequential tokens, forced routing
              with 27 % per-layer overlap between consecutive tokens
``batch32``   ``layer4`` with 32 tokens per step, forced Zipf(1.1) routing

Distributions: scale ~ U(0.005, 0.02) (24-bit grid), bias ~ 0.01 * Z,
router weights ~ 0.02 * Z, x ~ Z, with Z the Irwin-Hall(12) stand-in for a
standard normal; codes uniform over [0, 2^bits). With router weights of
standard deviation 0.02 and H=4096 the router logits have standard deviation
about 1.28, so routing is close to uniform over the experts.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, replace

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_HOST_SRC = os.path.join(_HERE, "synth_host.c")
_DEV_SRC = os.path.join(_HERE, "synth_dev.cu")
_GEN_H = os.path.join(_HERE, "synth_gen.h")
_HOST_LIB = os.path.join(_HERE, "libsynth_host.so")
_DEV_LIB = os.path.join(_HERE, "libsynth_dev.so")

TAG_CODES, TAG_SCALE, TAG_BIAS, TAG_ROUTER, TAG_X, TAG_SHARED_GATE, TAG_RESID = 1, 2, 3, 4, 5, 6, 7
GATE, UP, DOWN = 0, 1, 2


def _stale(lib: str, *srcs: str) -> bool:
    return (not os.path.exists(lib)) or max(os.path.getmtime(s) for s in srcs) > os.path.getmtime(lib)


def build(force: bool = False, device: bool = True) -> None:
    """Compile the host generator (gcc) and, unless device=False, the GPU one (nvcc)."""
    if force or _stale(_HOST_LIB, _HOST_SRC, _GEN_H):
        tmp = _HOST_LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fPIC", "-shared",
                               "-o", tmp, _HOST_SRC])
        os.replace(tmp, _HOST_LIB)
    if device and (force or _stale(_DEV_LIB, _DEV_SRC, _GEN_H)):
        tmp = _DEV_LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
                               "-Xcompiler", "-fPIC", "-shared", "-o", tmp, _DEV_SRC])
        os.replace(tmp, _DEV_LIB)


_host = None
_dev = None
_U64, _U32, _I64, _F32 = ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int64, ctypes.c_float


def host_lib():
    global _host
    if _host is None:
        build(device=False)
        L = ctypes.CDLL(_HOST_LIB)
        key = [_U64, _U32, _U32, _U32, _U32]
        L.syn_fill_codes.argtypes = key + [ctypes.c_int, _I64, _I64, ctypes.c_void_p]
        L.syn_fill_uniform_bf16.argtypes = key + [_F32, _F32, _I64, _I64, ctypes.c_void_p]
        L.syn_fill_normal_bf16.argtypes = key + [_F32, _I64, _I64, ctypes.c_void_p]
        L.syn_fill_normal_f32.argtypes = key + [_F32, _I64, _I64, ctypes.c_void_p]
        for f in (L.syn_fill_codes, L.syn_fill_uniform_bf16, L.syn_fill_normal_bf16, L.syn_fill_normal_f32):
            f.restype = ctypes.c_int
        _host = L
    return _host


def dev_lib():
    global _dev
    if _dev is None:
        if not os.path.exists(_DEV_LIB):
            raise RuntimeError("libsynth_dev.so is not built; run __graft_entry__.build()")
        L = ctypes.CDLL(_DEV_LIB)
        key = [_U64, _U32, _U32, _U32, _U32]
        L.syn_fill_codes_dev.argtypes = key + [ctypes.c_int, _I64, _I64, ctypes.c_void_p, ctypes.c_void_p]
        L.syn_fill_uniform_bf16_dev.argtypes = key + [_F32, _F32, _I64, _I64, ctypes.c_void_p, ctypes.c_void_p]
        L.syn_fill_normal_bf16_dev.argtypes = key + [_F32, _I64, _I64, ctypes.c_void_p, ctypes.c_void_p]
        L.syn_fill_normal_f32_dev.argtypes = key + [_F32, _I64, _I64, ctypes.c_void_p, ctypes.c_void_p]
        for f in (L.syn_fill_codes_dev, L.syn_fill_uniform_bf16_dev, L.syn_fill_normal_bf16_dev,
                  L.syn_fill_normal_f32_dev):
            f.restype = ctypes.c_int
        _dev = L
    return _dev


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise RuntimeError("%s failed with code %d" % (what, rc))


# ---- workload recipes -------------------------------------------------------

@dataclass(frozen=True)
class Workload:
    name: str
    H: int
    E: int
    I: int
    K: int
    group: int
    bits_routed: int = 4
    bits_shared: int = 4
    B: int = 1                 # tokens per step
    layers: int = 1
    tokens: int = 1            # sequential tokens (stack)
    routing: str = "router"    # "router" | "overlap" | "zipf"
    overlap: float = 0.27
    zipf_s: float = 1.1
    scale_lo: float = 0.005
    scale_span: float = 0.015
    bias_sigma: float = 0.01
    router_sigma: float = 0.02
    x_sigma: float = 1.0
    gate_sigma: float = 0.02   # shared-gate vector, when one is used
    seed: int = 0

    def bits_of(self, expert: int) -> int:
        return self.bits_shared if expert == self.E else self.bits_routed

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", H=256, E=8, I=128, K=2, group=32),
    "layer4": Workload("layer4", H=4096, E=512, I=1024, K=4, group=64),
    "layer2": Workload("layer2", H=4096, E=512, I=1024, K=4, group=64, bits_routed=2),
    "layer3": Workload("layer3", H=4096, E=512, I=1024, K=4, group=64, bits_routed=3),
    "stack24": Workload("stack24", H=4096, E=512, I=1024, K=4, group=64, layers=24, tokens=256,
                        routing="overlap"),
    "batch32": Workload("batch32", H=4096, E=512, I=1024, K=4, group=64, B=32, routing="zipf"),
}


def matrix_shape(w: Workload, matrix: int):
    return (w.I, w.H) if matrix in (GATE, UP) else (w.H, w.I)


# ---- host (numpy) tensors ---------------------------------------------------

def codes_host(w: Workload, layer: int, expert: int, matrix: int) -> np.ndarray:
    rows, cols = matrix_shape(w, matrix)
    out = np.empty((rows, cols), dtype=np.uint8)
    _check(host_lib().syn_fill_codes(w.seed, layer, expert, TAG_CODES, matrix, w.bits_of(expert), 0,
                                     rows * cols, out.ctypes.data), "syn_fill_codes")
    return out


def scale_host(w: Workload, layer: int, expert: int, matrix: int) -> np.ndarray:
    rows, cols = matrix_shape(w, matrix)
    out = np.empty((rows, cols // w.group), dtype=np.uint16)
    _check(host_lib().syn_fill_uniform_bf16(w.seed, layer, expert, TAG_SCALE, matrix, w.scale_lo, w.scale_span,
                                            0, out.size, out.ctypes.data), "syn_fill_uniform_bf16")
    return out


def bias_host(w: Workload, layer: int, expert: int, matrix: int) -> np.ndarray:
    rows, cols = matrix_shape(w, matrix)
    out = np.empty((rows, cols // w.group), dtype=np.uint16)
    _check(host_lib().syn_fill_normal_bf16(w.seed, layer, expert, TAG_BIAS, matrix, w.bias_sigma, 0, out.size,
                                           out.ctypes.data), "syn_fill_normal_bf16")
    return out


def expert_host(w: Workload, layer: int, expert: int):
    """(gate, up, down), each (codes, scale, bias), for expert id `expert`
    (id E is the shared expert)."""
    return tuple((codes_host(w, layer, expert, m), scale_host(w, layer, expert, m), bias_host(w, layer, expert, m))
                 for m in (GATE, UP, DOWN))


def router_host(w: Workload, layer: int) -> np.ndarray:
    out = np.empty((w.E, w.H), dtype=np.uint16)
    _check(host_lib().syn_fill_normal_bf16(w.seed, layer, 0, TAG_ROUTER, 0, w.router_sigma, 0, out.size,
                                           out.ctypes.data), "syn_fill_normal_bf16")
    return out


def shared_gate_host(w: Workload, layer: int) -> np.ndarray:
    out = np.empty(w.H, dtype=np.uint16)
    _check(host_lib().syn_fill_normal_bf16(w.seed, layer, 0, TAG_SHARED_GATE, 0, w.gate_sigma, 0, out.size,
                                           out.ctypes.data), "syn_fill_normal_bf16")
    return out


def x_host(w: Workload, token: int, n: int = 1) -> np.ndarray:
    """bf16 bits [n, H] for tokens token .. token+n-1."""
    out = np.empty((n, w.H), dtype=np.uint16)
    for t in range(n):
        _check(host_lib().syn_fill_normal_bf16(w.seed, token + t, 0, TAG_X, 0, w.x_sigma, 0, w.H,
                                               out[t].ctypes.data), "syn_fill_normal_bf16")
    return out


def resid_host(w: Workload, token: int, n: int = 1) -> np.ndarray:
    out = np.empty((n, w.H), dtype=np.float32)
    for t in range(n):
        _check(host_lib().syn_fill_normal_f32(w.seed, token + t, 0, TAG_RESID, 0, 1.0, 0, w.H,
                                              out[t].ctypes.data), "syn_fill_normal_f32")
    return out


# ---- device fills (raw device pointers; used to build large arenas) --------

def codes_dev(w: Workload, layer: int, expert: int, matrix: int, ptr: int, stream: int = 0) -> None:
    rows, cols = matrix_shape(w, matrix)
    _check(dev_lib().syn_fill_codes_dev(w.seed, layer, expert, TAG_CODES, matrix, w.bits_of(expert), 0,
                                        rows * cols, ptr, stream), "syn_fill_codes_dev")


def scale_dev(w: Workload, layer: int, expert: int, matrix: int, ptr: int, stream: int = 0) -> None:
    rows, cols = matrix_shape(w, matrix)
    _check(dev_lib().syn_fill_uniform_bf16_dev(w.seed, layer, expert, TAG_SCALE, matrix, w.scale_lo,
                                               w.scale_span, 0, rows * cols // w.group, ptr, stream),
           "syn_fill_uniform_bf16_dev")


def bias_dev(w: Workload, layer: int, expert: int, matrix: int, ptr: int, stream: int = 0) -> None:
    rows, cols = matrix_shape(w, matrix)
    _check(dev_lib().syn_fill_normal_bf16_dev(w.seed, layer, expert, TAG_BIAS, matrix, w.bias_sigma, 0,
                                              rows * cols // w.group, ptr, stream), "syn_fill_normal_bf16_dev")


def router_dev(w: Workload, layer: int, ptr: int, stream: int = 0) -> None:
    _check(dev_lib().syn_fill_normal_bf16_dev(w.seed, layer, 0, TAG_ROUTER, 0, w.router_sigma, 0, w.E * w.H,
                                              ptr, stream), "syn_fill_normal_bf16_dev")


def shared_gate_dev(w: Workload, layer: int, ptr: int, stream: int = 0) -> None:
    _check(dev_lib().syn_fill_normal_bf16_dev(w.seed, layer, 0, TAG_SHARED_GATE, 0, w.gate_sigma, 0, w.H,
                                              ptr, stream), "syn_fill_normal_bf16_dev")


def x_dev(w: Workload, token: int, n: int, ptr: int, stream: int = 0) -> None:
    for t in range(n):
        _check(dev_lib().syn_fill_normal_bf16_dev(w.seed, token + t, 0, TAG_X, 0, w.x_sigma, 0, w.H,
                                                  ptr + 2 * w.H * t, stream), "syn_fill_normal_bf16_dev")


# ---- forced routings (inputs to both sides) --------------------------------

def overlap_routing(E: int, K: int, tokens: int, layers: int, p: float, seed: int = 0) -> np.ndarray:
    """int32 [tokens, layers, K]. Token 0 draws K distinct experts uniformly.
    For token t > 0 at layer l, each slot independently reuses, with
    probability p, one not-yet-reused expert of token t-1's set at layer l;
    otherwise it draws uniformly among experts outside token t-1's set and not
    already picked. The expected overlap |S_t & S_{t-1}| / K is exactly p."""
    rng = np.random.Generator(np.random.PCG64(seed))
    out = np.empty((tokens, layers, K), dtype=np.int32)
    for l in range(layers):
        prev = rng.choice(E, size=K, replace=False)
        out[0, l] = prev
        for t in range(1, tokens):
            prev_list = list(prev)
            rng.shuffle(prev_list)
            chosen = []
            for _ in range(K):
                if rng.random() < p and prev_list:
                    chosen.append(prev_list.pop())
                else:
                    banned = set(prev.tolist()) | set(chosen)
                    while True:
                        e = int(rng.integers(E))
                        if e not in banned:
                            break
                    chosen.append(e)
            prev = np.array(chosen, dtype=np.int64)
            out[t, l] = prev
    return out


def measured_overlap(routing: np.ndarray) -> float:
    """Mean |S_t & S_{t-1}| / K over consecutive tokens and layers."""
    T, Lyr, K = routing.shape
    tot = 0
    for t in range(1, T):
        for l in range(Lyr):
            tot += len(set(routing[t, l].tolist()) & set(routing[t - 1, l].tolist()))
    return tot / float((T - 1) * Lyr * K)


def zipf_routing(E: int, K: int, B: int, steps: int, s: float = 1.1, seed: int = 0) -> np.ndarray:
    """int32 [steps, B, K]. Expert popularity p(rank r) ~ r^-s (r = 1..E), rank
    mapped to expert id by a seeded permutation; each token draws K distinct
    experts by successive weighted draws without replacement."""
    rng = np.random.Generator(np.random.PCG64(seed))
    perm = rng.permutation(E)
    pop = np.arange(1, E + 1, dtype=np.float64) ** (-s)
    out = np.empty((steps, B, K), dtype=np.int32)
    for st in range(steps):
        for b in range(B):
            wgt = pop.copy()
            for k in range(K):
                r = int(rng.choice(E, p=wgt / wgt.sum()))
                out[st, b, k] = perm[r]
                wgt[r] = 0.0
    return out


def fill_matrix_dev(w: Workload, layer: int, expert: int, matrix: int, codes_ptr: int, scale_ptr: int,
                    bias_ptr: int, stream: int = 0) -> None:
    """Write one matrix's codes and bf16 scale/bias into device buffers."""
    codes_dev(w, layer, expert, matrix, codes_ptr, stream)
    scale_dev(w, layer, expert, matrix, scale_ptr, stream)
    bias_dev(w, layer, expert, matrix, bias_ptr, stream)
