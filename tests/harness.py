"""Helpers shared by the GPU tests: build a layer arena from the seeded
generator on the device, and get the same weights on the host for the oracle."""
from __future__ import annotations

import functools

import numpy as np

from synth import synth


def torch_cuda():
    import torch
    return torch


def build_layer(w: synth.Workload, layer: int = 0, shared_gate: bool = False):
    torch = torch_cuda()
    import quantized_expert_ffn_topk_b200 as moeq
    synth.build()
    L = moeq.QuantLayer(w.H, w.I, w.E, w.K, w.group, w.bits_routed, w.bits_shared, shared_gate=shared_gate)
    stream = torch.cuda.current_stream().cuda_stream
    L.fill(lambda e, m, c, s, b: synth.fill_matrix_dev(w, layer, e, m, c, s, b, stream))
    synth.router_dev(w, layer, L.router_w.data_ptr(), stream)
    if shared_gate:
        synth.shared_gate_dev(w, layer, L.shared_gate_w.data_ptr(), stream)
    return L


def x_device(w: synth.Workload, token: int, n: int):
    torch = torch_cuda()
    x = torch.empty((n, w.H), dtype=torch.bfloat16, device="cuda")
    synth.x_dev(w, token, n, x.data_ptr(), torch.cuda.current_stream().cuda_stream)
    return x


def bf16_bits(t) -> np.ndarray:
    """torch bf16 tensor -> numpy uint16 bit patterns."""
    torch = torch_cuda()
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_to_f64(bits) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def oracle_experts(w: synth.Workload, layer: int):
    @functools.lru_cache(maxsize=64)
    def get(e: int):
        return synth.expert_host(w, layer, e)
    return get


def max_rel_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    scale = np.abs(ref).max()
    return float(np.abs(got - ref).max() / (scale if scale > 0 else 1.0))


def check_topk(gpu_idx, gpu_logits, ref_logits, K: int, logit_tol: float):
    """Router indices: bit-exact against the oracle where the oracle's ranking
    is decided by more than twice the observed logit error; otherwise (a near
    tie) the GPU's picks must be the exact top-K of its own logits. Returns
    True when the exact comparison applied."""
    gpu_idx = [int(v) for v in gpu_idx]
    gl = np.asarray(gpu_logits, dtype=np.float64)
    rl = np.asarray(ref_logits, dtype=np.float64)
    err = float(np.abs(gl - rl).max())
    assert err <= logit_tol, (err, logit_tol)
    own = sorted(range(len(gl)), key=lambda e: (-np.float32(gl[e]), e))[:K]
    assert gpu_idx == own, (gpu_idx, own)
    order = sorted(range(len(rl)), key=lambda e: (-rl[e], e))
    gaps = [rl[order[i]] - rl[order[i + 1]] for i in range(min(K, len(rl) - 1))]
    if min(gaps) > 2 * err:
        assert gpu_idx == order[:K], (gpu_idx, order[:K])
        return True
    return False
