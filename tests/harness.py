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


# ---- router exactness: a-priori error bound of the GPU's fp32 logits ---------

U32 = 2.0 ** -24  # unit roundoff of fp32


def logit_bound(x_bits, wr_bits) -> np.ndarray:
    """Per-expert bound on |GPU logit - exact logit| for a bf16 input x and
    bf16 router rows. Each bf16 x bf16 product is exact in fp32; the router
    kernels sum a row in a tree whose every term passes through at most
    D = H/32 + 8 fp32 additions (per lane a run of H/256 eight-term dot
    products, then the warp and quarter reductions), so
    |err_e| <= gamma_D * sum_h |w_eh x_h| with gamma_D = D u / (1 - D u)."""
    xd = bf16_to_f64(x_bits)
    wd = bf16_to_f64(wr_bits)
    H = xd.shape[0]
    D = H // 32 + 8
    gamma = D * U32 / (1.0 - D * U32)
    return gamma * np.abs(wd * xd[None, :]).sum(axis=1)


def ranking_decided(ref_logits, K: int, bound: float) -> bool:
    """True when the exact ranking of the top K (their order and the cut
    between rank K and K+1) is decided by more than twice the error bound, so
    any fp32 evaluation within the bound must give the same picks."""
    rl = np.asarray(ref_logits, dtype=np.float64)
    order = sorted(range(len(rl)), key=lambda e: (-rl[e], e))
    n = min(K, len(rl) - 1)
    gaps = [rl[order[i]] - rl[order[i + 1]] for i in range(n)]
    return n == 0 or min(gaps) > 2.0 * bound


def picks_valid_within(gpu_idx, ref_logits, bound: float) -> bool:
    """The GPU's picks at a near tie: distinct, in an order the exact logits
    allow within twice the bound, and no unpicked expert above the last pick
    by more than that."""
    rl = np.asarray(ref_logits, dtype=np.float64)
    p = [int(v) for v in gpu_idx]
    if len(set(p)) != len(p) or min(p) < 0 or max(p) >= len(rl):
        return False
    slack = 2.0 * bound
    if any(rl[p[i]] < rl[p[i + 1]] - slack for i in range(len(p) - 1)):
        return False
    rest = [e for e in range(len(rl)) if e not in set(p)]
    return all(rl[e] <= rl[p[-1]] + slack for e in rest)


def decided_tokens(w: synth.Workload, layer: int, n: int, first: int, oracle_logits, limit: int = 400):
    """The first n token ids from `first` on whose oracle top-K is decided
    (ranking_decided with logit_bound); tokens with a near tie are skipped
    and returned separately so that a test can report them."""
    wr = synth.router_host(w, layer)
    chosen, skipped = [], []
    for t in range(first, first + limit):
        xb = synth.x_host(w, t)[0]
        rl = oracle_logits(xb, wr)
        if ranking_decided(rl, w.K, float(logit_bound(xb, wr).max())):
            chosen.append(t)
            if len(chosen) == n:
                return chosen, skipped
        else:
            skipped.append(t)
    raise AssertionError("fewer than %d decided tokens in %d candidates" % (n, limit))


def x_tokens_device(w: synth.Workload, tokens):
    """bf16 [len(tokens), H] on the GPU holding the generator's x of each token id."""
    torch = torch_cuda()
    bits = np.stack([synth.x_host(w, t)[0] for t in tokens]).astype(np.uint16)
    return torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
