"""GPU parity of the fused persistent decode (moe_decode_layers) against the
oracle: one layer (router-driven), the 24-layer resident stack (router-driven
and with the workload's forced overlap routing, every layer checked on its
own GPU input), the residual input and renormalisation, the device error
path, the bounded-wait timeout path and repeat calls on one workspace."""
import os

import numpy as np
import pytest

from synth import synth
from tests import harness as hz

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import quantized_expert_ffn_topk_b200 as moeq  # noqa: E402
from oracle import layer as ref_layer  # noqa: E402
from oracle import oracle as ref  # noqa: E402

FFN_TOL = 2e-3
W_TOL = 1e-5
EPS = 1e-6

_cache = {}


def layers_for(name, n, **over):
    w = synth.WORKLOADS[name].with_(**over) if over else synth.WORKLOADS[name]
    key = (w, n)
    if key not in _cache:
        _cache.clear()
        torch.cuda.empty_cache()
        _cache[key] = (w, [hz.build_layer(w, l) for l in range(n)])
    return _cache[key]


def run(w, Ls, x, resid=None, forced=None, renorm=False):
    n = len(Ls)
    ws = moeq.Workspace(1, w.K, w.H, w.I, w.E)
    idx = torch.empty((n, w.K), dtype=torch.int32, device="cuda")
    wt = torch.empty((n, w.K), dtype=torch.float32, device="cuda")
    out = torch.empty(w.H, dtype=torch.float32, device="cuda")
    xn = torch.empty(w.H, dtype=torch.bfloat16, device="cuda")
    fi = None if forced is None else torch.as_tensor(np.ascontiguousarray(forced, np.int32), device="cuda")
    moeq.moe_decode_layers([L.struct for L in Ls], x, resid, renorm, fi, idx, wt, out, xn, EPS, ws.buf, ws.nbytes)
    torch.cuda.synchronize()
    return ws, idx.cpu().numpy(), wt.cpu().numpy(), out.cpu().numpy().astype(np.float64), hz.bf16_bits(xn)


def oracle_chain(w, n, x_bits, forced=None):
    """Chain the oracle over n layers from x (r_0 = x widened)."""
    x = x_bits
    r = None
    res = []
    for l in range(n):
        experts = hz.oracle_experts(w, l)
        f = None if forced is None else forced[l]
        ro = ref_layer.layer_token(w.H, w.I, w.E, w.K, w.group, x, synth.router_host(w, l), experts, experts(w.E),
                                   forced=f, resid=r, eps=EPS)
        res.append(ro)
        x, r = ro["xn"], ro["out"]
    return res


@pytest.mark.parametrize("name", ["tiny", "layer4", "layer2", "layer3"])
def test_one_layer_matches_oracle(name):
    w, Ls = layers_for(name, 1)
    toks, skipped = hz.decided_tokens(w, 0, 1, 321, ref.router_logits)
    x = hz.x_tokens_device(w, toks)[0]
    ws, idx, wt, out, xn = run(w, Ls, x)
    assert moeq.moe_get_device_error(ws.buf) == moeq.MOE_OK
    ro = oracle_chain(w, 1, synth.x_host(w, toks[0])[0])[0]
    assert list(idx[0]) == list(ro["idx"])
    assert np.abs(wt[0] - ro["w"]).max() <= W_TOL
    assert hz.max_rel_err(out, ro["out"]) <= FFN_TOL
    # RMSNorm'd bf16 output: one bf16 rounding plus the propagated FFN error
    xg = hz.bf16_to_f64(xn)
    rn = ro["out"] / np.sqrt(np.mean(ro["out"] ** 2) + EPS)
    assert (np.abs(xg - rn) <= np.abs(rn) * 2.0 ** -8 + FFN_TOL * np.abs(rn).max()).all()


@pytest.mark.parametrize("over", [dict(E=1024, K=8, group=128), dict(bits_routed=2, bits_shared=2),
                                  dict(bits_routed=3, bits_shared=3, group=128)],
                         ids=["E1024-K8-g128", "2bit-both", "3bit-both-g128"])
def test_one_layer_other_shapes(over):
    """The fused kernel at the most experts and picks it takes (its largest
    item plan), at group 128 (four k-steps per group) and with the shared
    expert at the routed width, one layer against the oracle."""
    w, Ls = layers_for("layer4", 1, **over)
    toks, skipped = hz.decided_tokens(w, 0, 1, 321, ref.router_logits)
    x = hz.x_tokens_device(w, toks)[0]
    ws, idx, wt, out, xn = run(w, Ls, x)
    assert moeq.moe_get_device_error(ws.buf) == moeq.MOE_OK
    ro = oracle_chain(w, 1, synth.x_host(w, toks[0])[0])[0]
    assert list(idx[0]) == list(ro["idx"])
    assert np.abs(wt[0] - ro["w"]).max() <= W_TOL
    assert hz.max_rel_err(out, ro["out"]) <= FFN_TOL


# ---- the 24-layer stack (87 GB resident) ------------------------------------------

N_STACK = 24


def prefix_states(w, Ls, x, forced=None, resid=None, renorm=False):
    """Run the first n layers for n = 1..len(Ls) (the kernel is deterministic,
    so layer n-1 of every run is the same computation): returns the inputs
    (x_l bf16 bits, r_l fp64 or None) of every layer, the picks and weights of
    the full run, and r_n after each prefix."""
    n = len(Ls)
    xs = [hz.bf16_bits(x)]
    rs = [None]
    outs = []
    full = None
    for m in range(1, n + 1):
        ws, idx, wt, out, xn = run(w, Ls[:m], x, resid=resid, forced=None if forced is None else forced[:m],
                                   renorm=renorm)
        assert moeq.moe_get_device_error(ws.buf) == moeq.MOE_OK
        xs.append(xn)
        rs.append(out)
        outs.append(out)
        if full is not None:
            assert (idx[:m - 1] == full[0][:m - 1]).all() and (wt[:m - 1] == full[1][:m - 1]).all()
        full = (idx, wt)
    return xs, rs, full[0], full[1]


def check_layers_on_gpu_inputs(w, xs, rs, idx, wt, forced=None, exact=True, renorm=False):
    """Every layer l against the oracle evaluated on the GPU's own input of
    that layer (x_l, r_l): picks exact (their ranking decided beyond twice the
    fp32 bound), weights within 1e-5, r_{l+1} within the FFN bar. The layers
    are independent, so the oracle runs them on a thread pool."""
    from concurrent.futures import ThreadPoolExecutor

    def one(l):
        experts = hz.oracle_experts(w, l)
        wr = synth.router_host(w, l)
        ro = ref_layer.layer_token(w.H, w.I, w.E, w.K, w.group, xs[l], wr, experts, experts(w.E),
                                   forced=None if forced is None else forced[l], resid=rs[l], eps=EPS,
                                   renorm=renorm)
        decided = forced is not None or hz.ranking_decided(ro["logits"], w.K, float(hz.logit_bound(xs[l], wr).max()))
        return l, ro, decided

    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as pool:
        res = list(pool.map(one, range(len(xs) - 1)))
    for l, ro, decided in res:
        if exact:
            assert decided, l
        assert list(idx[l]) == list(ro["idx"]), (l, idx[l], ro["idx"])
        assert np.abs(wt[l] - ro["w"]).max() <= W_TOL, l
        assert hz.max_rel_err(rs[l + 1], ro["out"]) <= FFN_TOL, l
    return res


def test_stack24_router_driven_every_layer():
    """A token through all 24 resident layer4 layers with the router picking:
    each layer's picks are bit-exact against the oracle on that layer's GPU
    input. The token is the first candidate whose ranking is decided at every
    layer (the others are reported); the final residual also matches the
    oracle chained from the start."""
    w, Ls = layers_for("layer4", N_STACK)
    chosen = None
    tried = []
    for t in range(11, 31):
        x = hz.x_tokens_device(w, [t])[0]
        xs, rs, idx, wt = prefix_states(w, Ls, x)
        ok = all(hz.ranking_decided(ref.router_logits(xs[l], synth.router_host(w, l)), w.K,
                                    float(hz.logit_bound(xs[l], synth.router_host(w, l)).max()))
                 for l in range(N_STACK))
        if ok:
            chosen = (t, xs, rs, idx, wt)
            break
        tried.append(t)
    assert chosen is not None, "no candidate token decided at all 24 layers: %s" % tried
    t, xs, rs, idx, wt = chosen
    print("token %d; candidates with a near tie at some layer: %s" % (t, tried))
    check_layers_on_gpu_inputs(w, xs, rs, idx, wt)
    res = oracle_chain(w, N_STACK, synth.x_host(w, t)[0], forced=idx)
    assert hz.max_rel_err(rs[-1], res[-1]["out"]) <= FFN_TOL


def test_stack24_forced_overlap_routing():
    """The 24-layer workload itself: three tokens with the stack's forced
    routing (27 % overlap between consecutive tokens), every layer against
    the oracle on the GPU's input of that layer, and the final residual
    against the oracle chained over all 24 layers."""
    w, Ls = layers_for("layer4", N_STACK)
    routing = synth.overlap_routing(w.E, w.K, 3, N_STACK, 0.27, seed=0)
    for t in range(3):
        x = hz.x_device(w, 1000 + t, 1)[0]
        xs, rs, idx, wt = prefix_states(w, Ls, x, forced=routing[t])
        assert (idx == routing[t]).all()
        check_layers_on_gpu_inputs(w, xs, rs, idx, wt, forced=routing[t])
        res = oracle_chain(w, N_STACK, synth.x_host(w, 1000 + t)[0], forced=routing[t])
        for l in range(N_STACK):
            assert np.abs(wt[l] - res[l]["w"]).max() <= (W_TOL if l == 0 else FFN_TOL)
        assert hz.max_rel_err(rs[-1], res[-1]["out"]) <= FFN_TOL


def test_residual_input_and_renorm():
    """A given residual stream and renormalised weights, two layers, each
    layer checked on its own GPU input with exact picks."""
    w, Ls = layers_for("tiny", 2)
    x = hz.x_device(w, 5, 1)[0]
    resid = torch.from_numpy(synth.resid_host(w, 5)[0]).cuda()
    xs, rs, idx, wt = prefix_states(w, Ls, x, resid=resid, renorm=True)
    rs[0] = resid.cpu().numpy().astype(np.float64)
    check_layers_on_gpu_inputs(w, xs, rs, idx, wt, renorm=True)


def test_bad_forced_index_and_repeat_calls():
    w, Ls = layers_for("tiny", 1)
    x = hz.x_device(w, 9, 1)[0]
    ws, idx, wt, out, xn = run(w, Ls, x)
    ws2, idx2, wt2, out2, xn2 = run(w, Ls, x)
    assert (out == out2).all() and (idx == idx2).all()
    # the same workspace twice in a row: counters come back to zero
    n = 1
    idx_t = torch.empty((n, w.K), dtype=torch.int32, device="cuda")
    wt_t = torch.empty((n, w.K), dtype=torch.float32, device="cuda")
    o = torch.empty(w.H, dtype=torch.float32, device="cuda")
    for _ in range(3):
        moeq.moe_decode_layers([Ls[0].struct], x, None, False, None, idx_t, wt_t, o, None, EPS, ws.buf, ws.nbytes)
    torch.cuda.synchronize()
    assert moeq.moe_get_device_error(ws.buf) == moeq.MOE_OK
    assert (o.cpu().numpy() == out.astype(np.float32)).all()
    bad = torch.tensor([[1, 8]], dtype=torch.int32, device="cuda")
    moeq.moe_decode_layers([Ls[0].struct], x, None, False, bad, idx_t, wt_t, o, None, EPS, ws.buf, ws.nbytes)
    assert moeq.moe_get_device_error(ws.buf) == moeq.MOE_ERR_INDEX


def test_graph_capture_of_decode_layers():
    w, Ls = layers_for("tiny", 2)
    x = hz.x_device(w, 4, 1)[0]
    ws = moeq.Workspace(1, w.K, w.H, w.I, w.E)
    o = torch.empty(w.H, dtype=torch.float32, device="cuda")
    xn = torch.empty(w.H, dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        moeq.moe_decode_layers([L.struct for L in Ls], x, None, False, None, None, None, o, xn, EPS, ws.buf, ws.nbytes)
        s.synchronize()
        ref_o = o.clone()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            moeq.moe_decode_layers([L.struct for L in Ls], x, None, False, None, None, None, o, xn, EPS, ws.buf,
                                   ws.nbytes)
        o.zero_()
        g.replay()
        g.replay()
        s.synchronize()
    assert (o == ref_o).all()
    assert moeq.moe_get_device_error(ws.buf) == moeq.MOE_OK


def test_bounded_wait_times_out_then_workspace_recovers():
    """A wait that runs out: one CTA withholds its arrival on the first
    logits exchange (a hook in the workspace, set from the host), so every
    CTA's bounded wait gives up after the short budget. The kernel must end
    by itself, report MOE_ERR_TIMEOUT, and leave the GPU usable; after
    moe_workspace_init the same workspace gives the normal result again."""
    import time
    w, Ls = layers_for("tiny", 2)
    x = hz.x_device(w, 13, 1)[0]
    _, idx0, wt0, out0, _ = run(w, Ls, x)
    ws = moeq.Workspace(1, w.K, w.H, w.I, w.E)
    o = torch.empty(w.H, dtype=torch.float32, device="cuda")
    structs = [L.struct for L in Ls]
    for withhold in (1, 7):
        moeq.moe_workspace_debug(ws.buf, ws.nbytes, 2000, withhold)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        moeq.moe_decode_layers(structs, x, None, False, None, None, None, o, None, EPS, ws.buf, ws.nbytes)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
        assert moeq.moe_get_device_error(ws.buf) == moeq.MOE_ERR_TIMEOUT
        assert elapsed < 0.5, elapsed  # the 2 ms budget, not the default second
        moeq.moe_workspace_init(ws.buf, ws.nbytes)
        moeq.moe_decode_layers(structs, x, None, False, None, None, None, o, None, EPS, ws.buf, ws.nbytes)
        torch.cuda.synchronize()
        assert moeq.moe_get_device_error(ws.buf) == moeq.MOE_OK
        assert (o.cpu().numpy() == out0.astype(np.float32)).all()
