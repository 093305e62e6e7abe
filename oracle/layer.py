"""One MoE layer for one token, composed from the oracle's C steps.

TEST INFRASTRUCTURE ONLY (see ``oracle.py``). The order of the steps is the
method's: router logits -> softmax/top-K -> per selected expert and the
shared expert: gate/up dequant mat-vecs, SwiGLU, down dequant mat-vec ->
weighted combine with the shared expert and the residual -> optional RMSNorm
to bf16 for the next layer ("Flash-MoE" page, sections "Metal Compute
Shaders" and "Deferred GPU Expert Compute").
"""
from __future__ import annotations

import numpy as np

from . import oracle as ref


def bf16_bits_to_f64(bits) -> np.ndarray:
    """Exact widening of bf16 bit patterns (the upper half of a binary32)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def layer_token(H, I, E, K, group, x_bf16, router_w, expert_weights, shared_weights,
                renorm=False, forced=None, resid=None, shared_gate_w=None, eps=None):
    """Returns a dict with logits [E], idx [K], w [K], y [K+1, H] (row K is the
    shared expert), gamma, out [H] and, when eps is given, xn (bf16 bits [H]).

    expert_weights(e) -> (gate, up, down), each (codes, scale, bias).
    resid: fp64 [H] or None (then r = x widened)."""
    x_bf16 = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    logits = ref.router_logits(x_bf16, router_w)
    idx, w = ref.topk(logits, K, renorm=renorm, forced=forced)
    x = bf16_bits_to_f64(x_bf16)
    y = np.zeros((K + 1, H), dtype=np.float64)
    for k in range(K):
        g, u, d = expert_weights(int(idx[k]))
        y[k] = ref.expert_ffn(H, I, group, g, u, d, x)
    g, u, d = shared_weights
    y[K] = ref.expert_ffn(H, I, group, g, u, d, x)
    gamma = 1.0 if shared_gate_w is None else ref.shared_gate(shared_gate_w, x_bf16)
    r = x if resid is None else np.asarray(resid, dtype=np.float64)
    out = ref.combine(y, w, gamma, r)
    res = dict(logits=logits, idx=idx, w=w, y=y, gamma=gamma, out=out)
    if eps is not None:
        res["xn"] = ref.rmsnorm_bf16(out, eps)
    return res
