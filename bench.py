#!/usr/bin/env python3
"""Benchmark of the decode-time quantized MoE FFN step on B200.

Default workload ("layer4"): one batch-1 MoE layer per step (H=4096, E=512
routed experts, I=1024, top-4 + 1 shared expert, 4-bit group-64 affine codes
with bf16 scale/bias, bf16 router), i.e. router GEMV + softmax/top-K +
gate/up/down dequant mat-vecs + SwiGLU + combine with shared expert and
residual + RMSNorm. A step is one layer-token; steps chain like decode
(x_{t+1} = RMSNorm(r_{t+1}) of step t) and walk `--layers` distinct resident
layers so that no weight byte is reused from L2 (126 MB) between visits.

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
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="layer4", choices=["layer4", "layer2"])
    ap.add_argument("--layers", type=int, default=24, help="resident layers walked by the steps")
    ap.add_argument("--cpu-sample", type=int, default=12, help="tokens in the oracle CPU-baseline sample")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the C0/C2/C3/C4 report lines")
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


def run_reference(args, w, rank: int):
    if rank != 0:
        return
    tps, secs = oracle_tokens_per_s(w, args.warmup + args.steps)
    line = {"impl": "reference", "metric": "MoE-layer decode tokens/s", "value": tps, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 / tps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "H": w.H, "E": w.E, "I": w.I, "K": w.K, "group": w.group,
                       "bits_routed": w.bits_routed, "bits_shared": w.bits_shared, "batch": 1},
            "cpu_baseline": {"value": tps, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                             "sample": "%d layer-token steps through the single-threaded fp64 C oracle "
                                       "(router, top-K, 5 expert FFNs, combine, RMSNorm)" % (args.warmup + args.steps)},
            "e2e": {"value": tps, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
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


def per_call_path(w, layers, ws, dev, stream, steps):
    """The four per-token calls (router+top-K, expert FFN, combine) chained
    like decode, each step one CUDA graph of 4 kernels with PDL; also times
    the expert-FFN call alone with events around it."""
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
    graphs = []
    for l in range(nl):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step(l)
        graphs.append(g)
    for t in range(2 * nl):
        graphs[t % nl].replay()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("per_call")
    a.record(stream)
    for t in range(steps):
        graphs[t % nl].replay()
    b.record(stream)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    ms = a.elapsed_time(b)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nl)]
    ffn_ms = []
    for t in range(max(nl, min(steps, 1600))):
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
    return steps / (ms / 1e3), statistics.mean(ffn_ms)


def replica_rate(ms: float, steps: int, world: int, device=None):
    """Whole-job rate of `world` independent replicas, each having run `steps`
    layer-token steps in `ms` milliseconds of its own device time: the job
    takes the slowest replica's time (max over ranks), and processes
    world * steps units in it. Returns (max ms, units per second)."""
    if world > 1:
        import torch
        import torch.distributed as dist
        t = torch.tensor([ms], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    return ms, world * steps / (ms / 1e3)


def timed_graph(stream, fn, reps: int = 2):
    """Capture fn() (a sequence of launches on `stream`) in a CUDA graph, replay
    it once to warm up, then time `reps` replays with events. Returns ms per replay."""
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(reps):
        g.replay()
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    del g
    return ms


def extra_configs(layers, ws, dev, stream, peak):
    """The other workloads, each timed on the device with the data resident:
    C0 (tiny, fused), C2 (2-bit routed experts, fused, own arena), C3 (256
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

    def decode_rate(w, Ls, steps_layers):
        x = torch.empty(w.H, dtype=torch.bfloat16, device=dev)
        synth.x_dev(w, 7, 1, x.data_ptr(), s)
        r = x.float().clone()
        structs = [L.struct for L in Ls]
        reps = max(1, steps_layers // len(Ls))
        ms = timed_graph(stream, lambda: [moeq.moe_decode_layers(structs, x, r, False, None, None, None, r, x, eps,
                                                                 ws_w.buf, ws_w.nbytes, s) for _ in range(reps)])
        return reps * len(Ls) / (ms / 1e3)

    # C0: tiny, one layer, fused (parity workload; a latency figure)
    w0 = synth.WORKLOADS["tiny"]
    L0 = build_layers(w0, 1, dev, s)
    ws_w = moeq.Workspace(1, w0.K, w0.H, w0.I, w0.E, device=dev, stream=s)
    tps0 = decode_rate(w0, L0, 256)
    b0 = algorithmic_bytes(w0)[0]
    out["C0"] = {"workload": "tiny H256 E8 I128 top-2 + shared, 4-bit, group 32", "tokens_per_s": tps0,
                 "step_bytes": b0, "gbs": b0 * tps0 / 1e9}
    del L0

    # C2: 2-bit routed experts (4-bit shared), own 8-layer arena
    w2 = synth.WORKLOADS["layer2"]
    L2 = build_layers(w2, 8, dev, s)
    ws_w = moeq.Workspace(1, w2.K, w2.H, w2.I, w2.E, device=dev, stream=s)
    tps2 = decode_rate(w2, L2, 8 * 64)
    b2 = algorithmic_bytes(w2)[0]
    out["C2"] = {"workload": "layer2: as layer4 with 2-bit routed experts (shared 4-bit)", "tokens_per_s": tps2,
                 "step_bytes": b2, "gbs": b2 * tps2 / 1e9, "frac_of_measured_hbm": b2 * tps2 / 1e9 / peak,
                 "layers_resident": 8}
    del L2
    torch.cuda.empty_cache()

    # C3: 256 tokens x all resident layer4 layers, forced routing with 27 % overlap
    w = synth.WORKLOADS["layer4"]
    nl = len(layers)
    T = 256
    routing = synth.overlap_routing(w.E, w.K, T, nl, 0.27, seed=3)
    rd = torch.from_numpy(np.ascontiguousarray(routing)).to(dev)
    xs = torch.empty((T, w.H), dtype=torch.bfloat16, device=dev)
    synth.x_dev(w, 9000, T, xs.data_ptr(), s)
    r3 = torch.empty(w.H, dtype=torch.float32, device=dev)
    structs = [L.struct for L in layers]
    ws_w = ws
    ms3 = timed_graph(stream, lambda: [moeq.moe_decode_layers(structs, xs[t], None, False, rd[t], None, None, r3, None,
                                                              eps, ws.buf, ws.nbytes, s) for t in range(T)])
    tps3 = T / (ms3 / 1e3)
    b3 = algorithmic_bytes(w)[0] * nl
    out["C3"] = {"workload": "%d layer4 layers resident, %d tokens, forced routing (overlap %.3f measured)" %
                             (nl, T, synth.measured_overlap(routing)),
                 "tokens_per_s": tps3, "token_bytes": b3, "gbs": b3 * tps3 / 1e9,
                 "frac_of_measured_hbm": b3 * tps3 / 1e9 / peak}

    # C4: 32 tokens per step, forced Zipf(1.1) routing, grouped per-call path
    B, S = 32, 2 * nl
    zr = synth.zipf_routing(w.E, w.K, B, S, 1.1, seed=5)
    zd = torch.from_numpy(np.ascontiguousarray(zr)).to(dev)
    wsb = moeq.Workspace(B, w.K, w.H, w.I, w.E, device=dev, stream=s)
    xb = torch.empty((B, w.H), dtype=torch.bfloat16, device=dev)
    synth.x_dev(w, 12000, B, xb.data_ptr(), s)
    resid = xb.float().clone()
    outs = [L.alloc_outputs(B, logits=False, xnorm=True) for L in layers]

    def c4():
        for st in range(S):
            l = st % nl
            L, o = layers[l], outs[l]
            moeq.moe_router_topk(xb, L.router_w, B, w.H, w.E, w.K, False, zd[st], o["idx"], o["w"], None, wsb.buf,
                                 wsb.nbytes, s)
            moeq.moe_expert_ffn_q(L.struct, xb, B, o["idx"], o["y"], wsb.buf, wsb.nbytes, s)
            moeq.moe_combine_residual(L.struct, o["y"], o["w"], xb, resid, B, resid, o["xnorm"], eps, s)

    ms4 = timed_graph(stream, c4)
    tps4 = B * S / (ms4 / 1e3)
    rec = algorithmic_bytes(w)[1]
    distinct = float(np.mean([len(np.unique(zr[st])) for st in range(S)]))
    b4 = w.E * w.H * 2 + (1 + distinct) * rec
    out["C4"] = {"workload": "layer4, 32 tokens per step, forced Zipf(1.1) routing, grouped per expert",
                 "tokens_per_s": tps4, "distinct_experts_per_step": distinct, "step_bytes": b4,
                 "gbs": b4 * (S / (ms4 / 1e3)) / 1e9, "frac_of_measured_hbm": b4 * (S / (ms4 / 1e3)) / 1e9 / peak}
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


def run_ours(args, w, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist

    import quantized_expert_ffn_topk_b200 as moeq
    from synth import synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    nlayers = args.layers
    eps = 1e-6
    with torch.cuda.stream(stream):
        s = stream.cuda_stream
        layers = build_layers(w, nlayers, dev, s)
        ws = moeq.Workspace(1, w.K, w.H, w.I, w.E, device=dev, stream=s)
        x = torch.empty(w.H, dtype=torch.bfloat16, device=dev)
        synth.x_dev(w, 1000 * rank, 1, x.data_ptr(), s)
        resid = x.float().clone()
        structs = [L.struct for L in layers]
        torch.cuda.synchronize()

        # a step is one layer-token; one launch walks all resident layers
        # (x <- RMSNorm(r) of the last layer, so passes chain like decode)
        def launch(n):
            moeq.moe_decode_layers(structs[:n], x, resid, False, None, None, None, resid, x, eps, ws.buf, ws.nbytes, s)

        launch(nlayers)
        torch.cuda.synchronize()
        if moeq.moe_get_device_error(ws.buf, s) != moeq.MOE_OK:
            raise RuntimeError("device error in the first launch")
        full, rem = divmod(args.steps, nlayers)
        g_full = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_full, stream=stream):
            launch(nlayers)
        g_rem = None
        if rem:
            g_rem = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_rem, stream=stream):
                launch(rem)
        synth.x_dev(w, 1000 * rank, 1, x.data_ptr(), s)
        resid.copy_(x.float())
        for _ in range(max(1, args.warmup // nlayers)):
            g_full.replay()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        with ClockSampler(local_rank) as clk:
            torch.cuda.nvtx.range_push("decode")
            start.record(stream)
            for _ in range(full):
                g_full.replay()
            if g_rem is not None:
                g_rem.replay()
            end.record(stream)
            torch.cuda.synchronize()
            torch.cuda.nvtx.range_pop()
        if world > 1:
            dist.barrier()
        ms = start.elapsed_time(end)
        err = moeq.moe_get_device_error(ws.buf, s)
        if err != moeq.MOE_OK:
            raise RuntimeError("device error in timed region: %s" % moeq.status_str(err))
        ms, tps = replica_rate(ms, args.steps, world, dev)
        launches = full + (1 if rem else 0)
        del g_full, g_rem

        # the per-call path (router_topk, expert_ffn_q, combine_residual)
        pc_tps, ffn_avg_ms = per_call_path(w, layers, ws, dev, stream, min(args.steps, 4000))

        # end to end through the public call with host buffers: per step one
        # layer-token, x copied in from pinned memory and r copied back out
        e2e = None
        if not args.no_e2e:
            n_e2e = min(args.steps, 4000)
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
                moeq.moe_decode_layers(structs[t % nlayers: t % nlayers + 1], xd, None, False, None, None, None, rd,
                                       None, eps, ws.buf, ws.nbytes, s)
                outh[t].copy_(rd, non_blocking=True)
            e1.record(stream)
            torch.cuda.synchronize()
            torch.cuda.nvtx.range_pop()
            e2e_ms = e0.elapsed_time(e1)
            e2e = {"value": n_e2e / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": w.H * 2,
                   "d2h_bytes_per_step": w.H * 4, "steps": n_e2e,
                   "path": "moe_decode_layers (1 layer per call) with pinned host input/output copies"}

        # the other workloads (report lines), on one GPU only
        extra = None
        if not args.no_extra and world == 1 and w.name == "layer4":
            extra = extra_configs(layers, ws, dev, stream, peaks()[0])

    step_bytes, rec_r, rec_s = algorithmic_bytes(w)
    peak, peak_src = peaks()
    achieved = step_bytes * args.steps / (ms / 1e3) / 1e9
    ffn_bytes = w.K * rec_r + rec_s
    resident = sum(L.nbytes() for L in layers)
    line = {
        "metric": "MoE-layer decode tokens/s", "value": tps, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "u8xs8-mma+f32", "data": "synthetic",
        "config": {"workload": "%s: batch-1 MoE layer H%d E%d I%d top-%d + shared, %d-bit routed / %d-bit shared, "
                               "group %d" % (w.name, w.H, w.E, w.I, w.K, w.bits_routed, w.bits_shared, w.group),
                   "batch": 1, "layers_resident": nlayers, "resident_bytes": resident,
                   "l2": "inputs larger than L2: each launch walks %d resident layers (%.1f GB)" %
                         (nlayers, resident / 1e9),
                   "parallelism": "replicas" if world > 1 else "single GPU",
                   "launch": "moe_decode_layers: one persistent kernel per %d layer-token steps, CUDA graph" % nlayers},
        "step_bytes": step_bytes,
        "effective_gbs": achieved,
        "frac_of_8tbs": achieved * 1e9 / 8e12,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": measured_traffic(w, nlayers), "kernel": "k_decode_layers",
                     "bytes_per_launch": step_bytes * nlayers, "avg_launch_us": ms * 1e3 / launches,
                     "peak_source": peak_src},
        "per_call": {"value": pc_tps, "unit": "tokens/s",
                     "path": "moe_router_topk + moe_expert_ffn_q + moe_combine_residual, graph per step",
                     "ffn_call_us": ffn_avg_ms * 1e3, "ffn_call_gbs": ffn_bytes / (ffn_avg_ms / 1e3) / 1e9},
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
    if rank == 0:
        tps, secs = oracle_tokens_per_s(w, args.cpu_sample)
        line["cpu_baseline"] = {"value": tps, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                "sample": "%d layer-token steps of %s through the single-threaded fp64 C oracle "
                                          "(%.1f s of oracle work)" % (args.cpu_sample, w.name, secs)}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
