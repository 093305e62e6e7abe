#!/usr/bin/env python3
"""Benchmark of the decode-time quantized MoE FFN step on B200.

Default workload ("layer4"): batch-1 MoE layers (H=4096, E=512 routed
experts, I=1024, top-4 + 1 shared expert, 4-bit group-64 affine codes with
bf16 scale/bias, bf16 router), i.e. per layer router GEMV + softmax/top-K +
gate/up/down dequant mat-vecs + SwiGLU + combine with shared expert and
residual + RMSNorm. A step is one decode token through `--layers` distinct
resident layers (one launch of the fused kernel); the metric counts
layer-tokens (one token through one MoE layer). Steps chain like decode
(x_{t+1} = RMSNorm(r_{t+1}) of step t), and every launch walks the whole
resident stack, so no weight byte is reused from L2 (126 MB) between visits.

Prints one JSON line (rank 0). `--impl reference` times the fp64 C oracle on
the host cores instead, on a bounded sample of the same workload.
Synthetic weights and inputs (seeded generator), no datasets.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="layer4", choices=["layer4", "layer2"])
    ap.add_argument("--layers", type=int, default=24, help="resident layers walked by the steps")
    ap.add_argument("--cpu-sample", type=int, default=12, help="tokens in the oracle CPU-baseline sample")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the C0/C2/C3/C4 report lines")
    ap.add_argument("--stat-replays", type=int, default=200, help="individually timed launches for the distribution")
    ap.add_argument("--profile-case", choices=["decode", "per_call", "batch"], default=None,
                    help="run one path on --layers resident layers for --steps steps and print no JSON "
                         "(a small case for ncu captures)")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, copy)"
    return FALLBACK_HBM_GBS, "fallback 6.65 TB/s"


def algorithmic_bytes(w):
    """Bytes the step must read: router matrix + K routed + 1 shared expert records."""
    import quantized_expert_ffn_topk_b200 as moeq
    router = w.E * w.H * 2
    rec_r = moeq.moe_expert_bytes(w.H, w.I, w.bits_routed, w.group)
    rec_s = moeq.moe_expert_bytes(w.H, w.I, w.bits_shared, w.group)
    return router + w.K * rec_r + rec_s, rec_r, rec_s


class ClockSampler:
    """Polls NVML (SM clock, throttle reasons) from a thread while the GPU works."""

    def __init__(self, dev_index: int, period_s: float = 0.005):
        self.samples = []
        self.reasons = set()
        self.period = period_s
        self._stop = threading.Event()
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(dev_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # no NVML: report no clocks
            self.nv = None
        self._t = threading.Thread(target=self._run, daemon=True)

    _NAMES = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
              0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
              0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self._NAMES.items():
                    if r & bit and bit != 0x1:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.nv is not None:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---- oracle timing (CPU baseline / reference arm) ---------------------------

def oracle_tokens_per_s(w, n_tokens: int, layers: int = 2, seed_token: int = 1_000_000):
    """Time the fp64 C oracle on n_tokens layer-token steps; returns (tok/s,
    seconds of oracle work). Input generation is outside the timed part."""
    from oracle import layer as ref_layer
    from oracle import oracle as ref
    from synth import synth
    ref.build()
    routers = [synth.router_host(w, l) for l in range(layers)]
    total = 0.0
    for t in range(n_tokens):
        l = t % layers
        xb = synth.x_host(w, seed_token + t)[0]
        lg = ref.router_logits(xb, routers[l])
        idx, _ = ref.topk(lg, w.K)
        experts = {int(e): synth.expert_host(w, l, int(e)) for e in list(idx) + [w.E]}
        t0 = time.perf_counter()
        ref_layer.layer_token(w.H, w.I, w.E, w.K, w.group, xb, routers[l], experts.__getitem__, experts[w.E],
                              eps=1e-6)
        total += time.perf_counter() - t0
    return n_tokens / total, total


def workload_config(w, nlayers: int, world: int = 1) -> dict:
    """The `config` object of both arms' JSON lines."""
    import quantized_expert_ffn_topk_b200 as moeq
    rec_r = moeq.moe_expert_bytes(w.H, w.I, w.bits_routed, w.group)
    rec_s = moeq.moe_expert_bytes(w.H, w.I, w.bits_shared, w.group)
    resident = nlayers * (w.E * rec_r + rec_s + w.E * w.H * 2)
    return {"workload": "%s: batch-1 MoE layer H%d E%d I%d top-%d + shared, %d-bit routed / %d-bit shared, group %d"
                        % (w.name, w.H, w.E, w.I, w.K, w.bits_routed, w.bits_shared, w.group),
            "batch": 1, "layers_resident": nlayers, "resident_bytes": resident,
            "step": "one decode token through the %d resident layers (%d layer-tokens)" % (nlayers, nlayers),
            "l2": "inputs larger than L2: each step walks %d resident layers (%.1f GB)" % (nlayers, resident / 1e9),
            "parallelism": "replicas" if world > 1 else "single GPU"}


def run_reference(args, w, rank: int):
    """The reference arm: the fp64 C oracle on the host cores (rank 0 only),
    each step one layer-token of the same workload (a bounded sample of a
    decode token through the stack), reported in the same unit."""
    if rank != 0:
        return
    n = args.warmup + args.steps
    tps, secs = oracle_tokens_per_s(w, n)
    line = {"impl": "reference", "metric": "MoE-layer decode tokens/s", "value": tps, "unit": "layer-tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 / tps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, args.layers, args.gpus),
            "cpu_baseline": {"value": tps, "unit": "layer-tokens/s", "cores": 1, "host_cores": os.cpu_count(),
                             "kind": "oracle",
                             "sample": "%d layer-token steps (router, top-K, 5 expert FFNs, combine, RMSNorm) of %s "
                                       "through the single-threaded fp64 C oracle, %.1f s of oracle work"
                                       % (n, w.name, secs)},
            "e2e": {"value": tps, "unit": "layer-tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---- our arm ------------------------------------------------------------------

def build_layers(w, nlayers, dev, s):
    import quantized_expert_ffn_topk_b200 as moeq
    from synth import synth
    layers = []
    for l in range(nlayers):
        L = moeq.QuantLayer(w.H, w.I, w.E, w.K, w.group, w.bits_routed, w.bits_shared, device=dev)
        L.fill(lambda e, m, c, sc, b, l=l: synth.fill_matrix_dev(w, l, e, m, c, sc, b, s), stream=s)
        synth.router_dev(w, l, L.router_w.data_ptr(), s)
        layers.append(L)
    return layers


def dist_of(ms_list):
    """median / p10 / p90 of per-replay times (ms)."""
    import numpy as np
    a = np.asarray(ms_list, dtype=np.float64)
    return {"median_ms": float(np.median(a)), "p10_ms": float(np.percentile(a, 10)),
            "p90_ms": float(np.percentile(a, 90)), "replays": int(a.size)}


def replay_times(stream, graphs, n: int, nvtx: str = None):
    """Replay the graphs in turn n times, each replay bracketed by its own
    events on `stream`; returns the per-replay times (ms). `nvtx` names the
    range (for profiler filters)."""
    import torch
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    torch.cuda.synchronize()
    if nvtx:
        torch.cuda.nvtx.range_push(nvtx)
    for i in range(n):
        ev[i][0].record(stream)
        graphs[i % len(graphs)].replay()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    if nvtx:
        torch.cuda.nvtx.range_pop()
    return [a.elapsed_time(b) for (a, b) in ev]


def capture(stream, fn):
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


def per_call_path(w, layers, ws, dev, stream, replays):
    """The per-token calls (router+top-K, expert FFN, combine) chained like
    decode over all resident layers in one CUDA graph (PDL between the
    kernels); each replay is timed on its own and reported per layer. Also
    the expert-FFN call alone (events around it, eager launches)."""
    import torch

    import quantized_expert_ffn_topk_b200 as moeq
    s = stream.cuda_stream
    nl = len(layers)
    xbuf = [torch.empty((1, w.H), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    xbuf[0].normal_()
    resid = xbuf[0].float().clone()
    outs = [L.alloc_outputs(1, logits=False, xnorm=False) for L in layers]
    for o in outs:
        o["resid"] = resid

    def step(t):
        l = t % nl
        o = outs[l]
        o["xnorm"] = xbuf[(l + 1) % 2]
        layers[l].forward(xbuf[l % 2], ws, o, resid_in=resid, eps=1e-6, stream=s)

    for l in range(nl):
        step(l)
    torch.cuda.synchronize()
    # one graph over all resident layers (a token through the stack, 4 launches
    # per layer), so that the host's graph launches stay off the device's path
    g_all = capture(stream, lambda: [step(l) for l in range(nl)])
    for _ in range(2):
        g_all.replay()
    times = [t / nl for t in replay_times(stream, [g_all], max(replays // nl, 20), nvtx="per_call")]
    graphs = [g_all]
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nl)]
    ffn_ms = []
    for t in range(max(nl, min(replays, 400))):
        l = t % nl
        L, o = layers[l], outs[l]
        xin = xbuf[l % 2]
        moeq.moe_router_topk(xin, L.router_w, 1, w.H, w.E, w.K, False, None, o["idx"], o["w"], None, ws.buf,
                             ws.nbytes, s)
        e0, e1 = ev[l]
        e0.record(stream)
        moeq.moe_expert_ffn_q(L.struct, xin, 1, o["idx"], o["y"], ws.buf, ws.nbytes, s)
        e1.record(stream)
        o["xnorm"] = xbuf[(l + 1) % 2]
        moeq.moe_combine_residual(L.struct, o["y"], o["w"], xin, resid, 1, resid, o["xnorm"], 1e-6, s)
        if l == nl - 1:
            torch.cuda.synchronize()
            ffn_ms += [x.elapsed_time(y) for (x, y) in ev]
    torch.cuda.synchronize()
    del graphs
    return times, ffn_ms


def replica_rate(ms: float, steps: int, world: int, device=None):
    """Whole-job rate of `world` independent replicas, each having processed
    `steps` units in `ms` milliseconds of its own device time: the job takes
    the slowest replica's time (max over ranks), and processes world * steps
    units in it. Returns (max ms, units per second)."""
    if world > 1:
        import torch
        import torch.distributed as dist
        t = torch.tensor([ms], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    return ms, world * steps / (ms / 1e3)


def extra_configs(layers, dev, stream, peak):
    """The other workloads, each timed on the device with the data resident,
    as a distribution over individually timed CUDA-graph replays: C0 (tiny,
    fused), C2 (2-bit routed experts, fused, own 8-layer arena), C3 (256
    tokens through all resident layer4 layers with forced 27 %-overlap
    routing), C4 (32 tokens per step, forced Zipf routing, grouped per-call
    path). Returns a dict of report lines."""
    import numpy as np
    import torch

    import quantized_expert_ffn_topk_b200 as moeq
    from synth import synth
    s = stream.cuda_stream
    out = {}
    eps = 1e-6

    def decode_stats(w, Ls, launches_per_graph, replays):
        ws_w = moeq.Workspace(1, w.K, w.H, w.I, w.E, device=dev, stream=s)
        x = torch.empty(w.H, dtype=torch.bfloat16, device=dev)
        synth.x_dev(w, 7, 1, x.data_ptr(), s)
        r = x.float().clone()
        table = moeq.layer_table([L.struct for L in Ls])
        g = capture(stream, lambda: [moeq.moe_decode_layers(table, x, r, False, None, None, None, r, x, eps,
                                                            ws_w.buf, ws_w.nbytes, s)
                                     for _ in range(launches_per_graph)])
        for _ in range(3):
            g.replay()
        d = dist_of(replay_times(stream, [g], replays))
        units = launches_per_graph * len(Ls)
        return units / (d["median_ms"] / 1e3), d

    # C0: tiny, one layer, fused (parity workload; a latency figure)
    w0 = synth.WORKLOADS["tiny"]
    L0 = build_layers(w0, 1, dev, s)
    tps0, d0 = decode_stats(w0, L0, 64, 50)
    b0 = algorithmic_bytes(w0)[0]
    out["C0"] = {"workload": "tiny H256 E8 I128 top-2 + shared, 4-bit, group 32", "tokens_per_s": tps0,
                 "step_bytes": b0, "gbs": b0 * tps0 / 1e9, "timing": d0, "graph": "64 one-layer launches"}
    del L0

    # C2: 2-bit routed experts (4-bit shared), own 8-layer arena
    w2 = synth.WORKLOADS["layer2"]
    L2 = build_layers(w2, 8, dev, s)
    tps2, d2 = decode_stats(w2, L2, 4, 100)
    b2 = algorithmic_bytes(w2)[0]
    out["C2"] = {"workload": "layer2: as layer4 with 2-bit routed experts (shared 4-bit)", "tokens_per_s": tps2,
                 "step_bytes": b2, "gbs": b2 * tps2 / 1e9, "frac_of_peak": b2 * tps2 / 1e9 / peak,
                 "layers_resident": 8, "timing": d2, "graph": "4 launches over the 8 resident layers"}
    del L2
    torch.cuda.empty_cache()

    # C3: 256 tokens x all resident layer4 layers, forced routing with 27 % overlap
    w = synth.WORKLOADS["layer4"]
    nl = len(layers)
    T, per = 256, 32
    routing = synth.overlap_routing(w.E, w.K, T, nl, 0.27, seed=3)
    rd = torch.from_numpy(np.ascontiguousarray(routing)).to(dev)
    xs = torch.empty((T, w.H), dtype=torch.bfloat16, device=dev)
    synth.x_dev(w, 9000, T, xs.data_ptr(), s)
    r3 = torch.empty(w.H, dtype=torch.float32, device=dev)
    table = moeq.layer_table([L.struct for L in layers])
    ws3 = moeq.Workspace(1, w.K, w.H, w.I, w.E, device=dev, stream=s)
    graphs3 = [capture(stream, lambda g0=g0: [moeq.moe_decode_layers(table, xs[t], None, False, rd[t], None, None, r3,
                                                                      None, eps, ws3.buf, ws3.nbytes, s)
                                              for t in range(g0, g0 + per)])
               for g0 in range(0, T, per)]
    graphs3[0].replay()
    d3 = dist_of(replay_times(stream, graphs3, 3 * len(graphs3)))
    tps3 = per / (d3["median_ms"] / 1e3)
    b3 = algorithmic_bytes(w)[0] * nl
    out["C3"] = {"workload": "%d layer4 layers resident, %d tokens, forced routing (overlap %.3f measured)" %
                             (nl, T, synth.measured_overlap(routing)),
                 "tokens_per_s": tps3, "layer_tokens_per_s": tps3 * nl, "token_bytes": b3, "gbs": b3 * tps3 / 1e9,
                 "frac_of_peak": b3 * tps3 / 1e9 / peak, "timing": d3,
                 "graph": "%d graphs of %d tokens (one launch per token over %d layers), replayed in turn" %
                          (len(graphs3), per, nl)}
    del graphs3

    # C4: 32 tokens per step, forced Zipf(1.1) routing, grouped per-call path
    B, S = 32, nl
    zr = synth.zipf_routing(w.E, w.K, B, S, 1.1, seed=5)
    zd = torch.from_numpy(np.ascontiguousarray(zr)).to(dev)
    wsb = moeq.Workspace(B, w.K, w.H, w.I, w.E, device=dev, stream=s)
    xb = torch.empty((B, w.H), dtype=torch.bfloat16, device=dev)
    synth.x_dev(w, 12000, B, xb.data_ptr(), s)
    resid = xb.float().clone()
    outs = [L.alloc_outputs(B, logits=False, xnorm=True) for L in layers]

    def c4_step(st):
        L, o = layers[st], outs[st]
        moeq.moe_router_topk(xb, L.router_w, B, w.H, w.E, w.K, False, zd[st], o["idx"], o["w"], None, wsb.buf,
                             wsb.nbytes, s)
        moeq.moe_expert_ffn_q(L.struct, xb, B, o["idx"], o["y"], wsb.buf, wsb.nbytes, s)
        moeq.moe_combine_residual(L.struct, o["y"], o["w"], xb, resid, B, resid, o["xnorm"], eps, s)

    graphs4 = [capture(stream, lambda st=st: c4_step(st)) for st in range(S)]
    for g in graphs4:
        g.replay()
    d4 = dist_of(replay_times(stream, graphs4, max(200, 4 * S), nvtx="batch"))
    step_s = d4["median_ms"] / 1e3
    rec = algorithmic_bytes(w)[1]
    distinct = float(np.mean([len(np.unique(zr[st])) for st in range(S)]))
    b4 = w.E * w.H * 2 + (1 + distinct) * rec
    out["C4"] = {"workload": "layer4, 32 tokens per step, forced Zipf(1.1) routing, grouped per expert",
                 "tokens_per_s": B / step_s, "distinct_experts_per_step": distinct, "step_bytes": b4,
                 "gbs": b4 / step_s / 1e9, "frac_of_peak": b4 / step_s / 1e9 / peak, "timing": d4,
                 "graph": "one graph per layer (router + grouped expert FFN + combine), layers in turn"}
    del graphs4
    return out


def kernel_source_digest() -> str:
    """Digest of the sources the fused decode kernel is built from."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(os.path.dirname(os.path.abspath(__file__)), "quantized_expert_ffn_topk_b200", "csrc")
    for f in ("common.cuh", "tiledot.cuh", "router.cuh", "stack.cuh"):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(w, nlayers):
    """DRAM bytes per launch of the fused kernel from the committed ncu
    capture (profiles/k_decode_layers.traffic.json: one launch over one
    layer, scaled by the layers a launch walks), or None when the kernel's
    sources changed since the capture or no capture matches the workload."""
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "profiles", "k_decode_layers.traffic.json")
    try:
        with open(path) as fh:
            rec = json.load(fh)
    except (OSError, ValueError):
        return None
    if rec.get("source_digest") != kernel_source_digest() or rec.get("workload") != w.name:
        return None
    return rec["dram_bytes_per_layer"] * nlayers


def profile_case(args, w, dev, stream):
    """A small run of one path for ncu (no JSON): `decode` (the fused kernel),
    `per_call` (router, expert FFN, combine per token) or `batch` (32 tokens
    per step, grouped), each over --layers resident layers for --steps steps."""
    import numpy as np
    import torch

    import quantized_expert_ffn_topk_b200 as moeq
    from synth import synth
    s = stream.cuda_stream
    with torch.cuda.stream(stream):
        layers = build_layers(w, args.layers, dev, s)
        nl = len(layers)
        if args.profile_case == "decode":
            ws = moeq.Workspace(1, w.K, w.H, w.I, w.E, device=dev, stream=s)
            x = torch.empty(w.H, dtype=torch.bfloat16, device=dev)
            synth.x_dev(w, 1, 1, x.data_ptr(), s)
            r = x.float().clone()
            table = moeq.layer_table([L.struct for L in layers])
            for _ in range(args.warmup + args.steps):
                moeq.moe_decode_layers(table, x, r, False, None, None, None, r, x, 1e-6, ws.buf, ws.nbytes, s)
        elif args.profile_case == "per_call":
            ws = moeq.Workspace(1, w.K, w.H, w.I, w.E, device=dev, stream=s)
            x = torch.empty((1, w.H), dtype=torch.bfloat16, device=dev)
            synth.x_dev(w, 1, 1, x.data_ptr(), s)
            r = x.float().clone()
            outs = [L.alloc_outputs(1, logits=False, xnorm=True) for L in layers]
            for t in range(args.warmup + args.steps):
                l = t % nl
                layers[l].forward(x, ws, outs[l], resid_in=r, eps=1e-6, stream=s)
                x.copy_(outs[l]["xnorm"])
        else:
            B = 32
            zr = synth.zipf_routing(w.E, w.K, B, args.warmup + args.steps, 1.1, seed=5)
            zd = torch.from_numpy(np.ascontiguousarray(zr)).to(dev)
            ws = moeq.Workspace(B, w.K, w.H, w.I, w.E, device=dev, stream=s)
            xb = torch.empty((B, w.H), dtype=torch.bfloat16, device=dev)
            synth.x_dev(w, 12000, B, xb.data_ptr(), s)
            resid = xb.float().clone()
            outs = [L.alloc_outputs(B, logits=False, xnorm=True) for L in layers]
            for t in range(args.warmup + args.steps):
                l = t % nl
                layers[l].forward(xb, ws, outs[l], resid_in=resid, forced_idx=zd[t], eps=1e-6, stream=s)
        torch.cuda.synchronize()
        err = moeq.moe_get_device_error(ws.buf, s)
    print("profile case %s: %d layers, %d steps, device status %s" %
          (args.profile_case, nl, args.warmup + args.steps, moeq.status_str(err)), flush=True)
    if err != moeq.MOE_OK:
        raise SystemExit(1)


def run_ours(args, w, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist

    import quantized_expert_ffn_topk_b200 as moeq
    from synth import synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    if args.profile_case:
        profile_case(args, w, dev, stream)
        return None
    nlayers = args.layers
    eps = 1e-6
    peak, peak_src = peaks()
    K, W = args.steps, args.warmup
    with torch.cuda.stream(stream):
        s = stream.cuda_stream
        layers = build_layers(w, nlayers, dev, s)
        ws = moeq.Workspace(1, w.K, w.H, w.I, w.E, device=dev, stream=s)
        x = torch.empty(w.H, dtype=torch.bfloat16, device=dev)
        synth.x_dev(w, 1000 * rank, 1, x.data_ptr(), s)
        resid = x.float().clone()
        table = moeq.layer_table([L.struct for L in layers])
        torch.cuda.synchronize()

        # a step is one decode token through all resident layers: one launch
        # (x <- RMSNorm(r) of the last layer, so steps chain like decode)
        def launch():
            moeq.moe_decode_layers(table, x, resid, False, None, None, None, resid, x, eps, ws.buf, ws.nbytes, s)

        launch()
        torch.cuda.synchronize()
        if moeq.moe_get_device_error(ws.buf, s) != moeq.MOE_OK:
            raise RuntimeError("device error in the first launch")
        g = capture(stream, launch)
        synth.x_dev(w, 1000 * rank, 1, x.data_ptr(), s)
        resid.copy_(x.float())
        for _ in range(W):
            g.replay()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(local_rank) as clk:
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            torch.cuda.nvtx.range_push("decode")
            start.record(stream)
            for _ in range(K):
                g.replay()
            end.record(stream)
            torch.cuda.synchronize()
            torch.cuda.nvtx.range_pop()
            if world > 1:
                dist.barrier()
            ms = start.elapsed_time(end)
            # the distribution: launches timed one by one, at least --stat-replays of them
            dist_ms = replay_times(stream, [g], max(args.stat_replays, 1), nvtx="decode_dist")
        err = moeq.moe_get_device_error(ws.buf, s)
        if err != moeq.MOE_OK:
            raise RuntimeError("device error in timed region: %s" % moeq.status_str(err))
        ms, tps = replica_rate(ms, K * nlayers, world, dev)
        del g

        # the per-call path (router_topk, expert_ffn_q, combine_residual)
        pc_times, ffn_ms = per_call_path(w, layers, ws, dev, stream, args.stat_replays)

        # end to end through the public call with host buffers: per step one
        # token through all resident layers (one call, prebuilt layer table),
        # x copied in from pinned memory and r copied back out
        e2e = None
        if not args.no_e2e:
            n_e2e = max(K, 100)
            tmp = torch.empty((n_e2e, w.H), dtype=torch.bfloat16, device=dev)
            synth.x_dev(w, 50_000, n_e2e, tmp.data_ptr(), s)
            torch.cuda.synchronize()
            xh = tmp.cpu().pin_memory()
            outh = torch.empty((n_e2e, w.H), dtype=torch.float32, pin_memory=True)
            xd = torch.empty(w.H, dtype=torch.bfloat16, device=dev)
            rd = torch.empty(w.H, dtype=torch.float32, device=dev)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.nvtx.range_push("e2e")
            e0.record(stream)
            for t in range(n_e2e):
                xd.copy_(xh[t], non_blocking=True)
                moeq.moe_decode_layers(table, xd, None, False, None, None, None, rd, None, eps, ws.buf, ws.nbytes, s)
                outh[t].copy_(rd, non_blocking=True)
            e1.record(stream)
            torch.cuda.synchronize()
            torch.cuda.nvtx.range_pop()
            e2e_ms, e2e_rate = replica_rate(e0.elapsed_time(e1), n_e2e * nlayers, world, dev)
            e2e = {"value": e2e_rate, "unit": "layer-tokens/s", "tokens_per_s": e2e_rate / nlayers,
                   "h2d_bytes_per_step": w.H * 2, "d2h_bytes_per_step": w.H * 4, "steps": n_e2e,
                   "path": "moe_decode_layers over the %d resident layers per call (one token per call), "
                           "pinned host input and output copies on the stream" % nlayers}

        # the other workloads (report lines), on one GPU only
        extra = None
        if not args.no_extra and world == 1 and w.name == "layer4":
            extra = extra_configs(layers, dev, stream, peak)

    step_bytes, rec_r, rec_s = algorithmic_bytes(w)
    launches = K
    bytes_per_launch = step_bytes * nlayers
    avg_launch_us = ms * 1e3 / launches
    achieved = bytes_per_launch / (avg_launch_us / 1e6) / 1e9
    dd = dist_of(dist_ms)
    ffn_bytes = w.K * rec_r + rec_s
    pc = dist_of(pc_times)
    ffn_mean = statistics.mean(ffn_ms)
    cfg = workload_config(w, nlayers, world)
    line = {
        "metric": "MoE-layer decode tokens/s", "value": tps, "unit": "layer-tokens/s", "n_gpus": world,
        "steps": K, "warmup": W, "ms_per_step": ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "u8xs8-mma+f32", "data": "synthetic",
        "config": cfg,
        "launch": "moe_decode_layers: one persistent kernel per step (%d layers), CUDA graph replay" % nlayers,
        "tokens_per_s": tps / nlayers,
        "step_bytes": bytes_per_launch,
        "effective_gbs": achieved,
        "frac_of_8tbs": achieved * 1e9 / 8e12,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": measured_traffic(w, nlayers), "kernel": "k_decode_layers",
                     "layers_per_launch": nlayers, "bytes_per_layer": step_bytes,
                     "bytes_per_launch": bytes_per_launch, "avg_launch_us": avg_launch_us,
                     "launches_timed": launches, "peak_source": peak_src,
                     "launch_distribution_us": {k.replace("_ms", "_us"): v * 1e3 if k.endswith("_ms") else v
                                                for k, v in dd.items()}},
        "per_call": {"value": 1.0 / (pc["median_ms"] / 1e3), "unit": "layer-tokens/s",
                     "path": "moe_router_topk + moe_expert_ffn_q + moe_combine_residual per layer, one graph per "
                             "token over the resident layers",
                     "timing": pc, "ffn_call_us": ffn_mean * 1e3,
                     "ffn_call_gbs": ffn_bytes / (ffn_mean / 1e3) / 1e9},
        "gpu_launches": launches,
        "clocks": clk.summary(),
    }
    if e2e is not None:
        line["e2e"] = e2e
    if extra is not None:
        line["configs"] = extra
    return line


def main():
    args = parse()
    from synth import synth
    w = synth.WORKLOADS[args.workload]
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, w, rank)
        return
    import torch
    import torch.distributed as dist
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    line = run_ours(args, w, rank, world, local_rank)
    if rank == 0 and line is not None:
        tps, secs = oracle_tokens_per_s(w, args.cpu_sample)
        line["cpu_baseline"] = {"value": tps, "unit": "layer-tokens/s", "cores": 1, "host_cores": os.cpu_count(),
                                "kind": "oracle",
                                "sample": "%d layer-token steps of %s through the single-threaded fp64 C oracle "
                                          "(%.1f s of oracle work)" % (args.cpu_sample, w.name, secs)}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
