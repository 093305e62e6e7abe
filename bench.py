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
    ap.add_argument("--layers", type=int, default=16, help="resident layers walked by the steps (even)")
    ap.add_argument("--cpu-sample", type=int, default=12, help="tokens in the oracle CPU-baseline sample")
    ap.add_argument("--no-e2e", action="store_true")
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

def run_ours(args, w, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist

    import quantized_expert_ffn_topk_b200 as moeq
    from synth import synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    nlayers = args.layers + (args.layers % 2)
    with torch.cuda.stream(stream):
        s = stream.cuda_stream
        layers = []
        for l in range(nlayers):
            L = moeq.QuantLayer(w.H, w.I, w.E, w.K, w.group, w.bits_routed, w.bits_shared, device=dev)
            L.fill(lambda e, m, c, sc, b, l=l: synth.fill_matrix_dev(w, l, e, m, c, sc, b, s), stream=s)
            synth.router_dev(w, l, L.router_w.data_ptr(), s)
            layers.append(L)
        ws = moeq.Workspace(1, w.K, w.H, w.I, w.E, device=dev, stream=s)
        xbuf = [torch.empty((1, w.H), dtype=torch.bfloat16, device=dev) for _ in range(2)]
        synth.x_dev(w, 1000 * rank, 1, xbuf[0].data_ptr(), s)
        resid = xbuf[0].float().clone()
        outs = [L.alloc_outputs(1, logits=False, xnorm=False) for L in layers]
        for o in outs:
            o["resid"] = resid
        torch.cuda.synchronize()

        def step(t):
            l = t % nlayers
            L, o = layers[l], outs[l]
            o["xnorm"] = xbuf[(l + 1) % 2]
            L.forward(xbuf[l % 2], ws, o, resid_in=resid, eps=1e-6, stream=s)

        # one CUDA graph per layer: the 4 kernels of a step, chained with PDL
        graphs = []
        for l in range(nlayers):
            step(l)  # warm the launch path outside capture
        torch.cuda.synchronize()
        for l in range(nlayers):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                step(l)
            graphs.append(g)
        torch.cuda.synchronize()
        # restart the chain from a clean input
        synth.x_dev(w, 1000 * rank, 1, xbuf[0].data_ptr(), s)
        resid.copy_(xbuf[0].float())
        if moeq.moe_get_device_error(ws.buf, s) != moeq.MOE_OK:
            raise RuntimeError("device error during warm-up")

        for t in range(args.warmup):
            graphs[t % nlayers].replay()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        with ClockSampler(local_rank) as clk:
            start.record(stream)
            for t in range(args.steps):
                graphs[(args.warmup + t) % nlayers].replay()
            end.record(stream)
            torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        ms = start.elapsed_time(end)
        err = moeq.moe_get_device_error(ws.buf, s)
        if err != moeq.MOE_OK:
            raise RuntimeError("device error in timed region: %s" % moeq.status_str(err))
        if world > 1:
            tt = torch.tensor([ms], device=dev)
            dist.all_reduce(tt, op=dist.ReduceOp.MAX)
            ms = float(tt.item())

        # dominant call: the expert FFN (gate/up + down kernels), timed per call
        # with events on the launching stream over the same kind of steps
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nlayers)]
        ffn_ms = []
        reps = max(nlayers, min(args.steps, 2000))
        for t in range(reps):
            l = t % nlayers
            L, o = layers[l], outs[l]
            xin = xbuf[l % 2]
            moeq.moe_router_topk(xin, L.router_w, 1, w.H, w.E, w.K, False, None, o["idx"], o["w"], None, ws.buf,
                                 ws.nbytes, s)
            a, b = ev[l]
            a.record(stream)
            moeq.moe_expert_ffn_q(L.struct, xin, 1, o["idx"], o["y"], ws.buf, ws.nbytes, s)
            b.record(stream)
            o["xnorm"] = xbuf[(l + 1) % 2]
            moeq.moe_combine_residual(L.struct, o["y"], o["w"], xin, resid, 1, resid, o["xnorm"], 1e-6, s)
            if l == nlayers - 1:
                torch.cuda.synchronize()
                ffn_ms += [x.elapsed_time(y) for (x, y) in ev]
        torch.cuda.synchronize()

        # end to end through the public calls with host buffers
        e2e = None
        if not args.no_e2e:
            n_e2e = min(args.steps, 2000)
            xh = torch.empty((n_e2e, w.H), dtype=torch.bfloat16, pin_memory=True)
            tmp = torch.empty((n_e2e, w.H), dtype=torch.bfloat16, device=dev)
            synth.x_dev(w, 50_000, n_e2e, tmp.data_ptr(), s)
            torch.cuda.synchronize()
            xh.copy_(tmp.cpu())
            outh = torch.empty((n_e2e, w.H), dtype=torch.float32, pin_memory=True)
            xd = torch.empty((1, w.H), dtype=torch.bfloat16, device=dev)
            e2e_out = outs[0]
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for t in range(n_e2e):
                L = layers[t % nlayers]
                xd.copy_(xh[t:t + 1], non_blocking=True)
                e2e_out["xnorm"] = xbuf[1]
                L.forward(xd, ws, e2e_out, resid_in=None, eps=1e-6, stream=s)
                outh[t:t + 1].copy_(e2e_out["resid"], non_blocking=True)
            e1.record(stream)
            torch.cuda.synchronize()
            e2e_ms = e0.elapsed_time(e1)
            e2e = {"value": n_e2e / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": w.H * 2,
                   "d2h_bytes_per_step": w.H * 4, "steps": n_e2e}

    step_bytes, rec_r, rec_s = algorithmic_bytes(w)
    ffn_bytes = w.K * rec_r + rec_s
    ffn_avg_ms = statistics.mean(ffn_ms)
    peak, peak_src = peaks()
    achieved = ffn_bytes / (ffn_avg_ms / 1e3) / 1e9
    tps = world * args.steps / (ms / 1e3)
    line = {
        "metric": "MoE-layer decode tokens/s", "value": tps, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": "%s: batch-1 MoE layer H%d E%d I%d top-%d + shared, %d-bit routed / %d-bit shared, "
                               "group %d" % (w.name, w.H, w.E, w.I, w.K, w.bits_routed, w.bits_shared, w.group),
                   "batch": 1, "layers_resident": nlayers,
                   "resident_bytes": sum(L.nbytes() for L in layers),
                   "l2": "inputs larger than L2: steps walk %d resident layers (%.1f GB)" %
                         (nlayers, sum(L.nbytes() for L in layers) / 1e9),
                   "parallelism": "replicas" if world > 1 else "single GPU",
                   "launch": "one CUDA graph per layer-step, 4 kernels chained with PDL"},
        "step_bytes": step_bytes,
        "effective_gbs": step_bytes / (ms / args.steps / 1e3) / 1e9,
        "frac_of_8tbs": step_bytes / (ms / args.steps / 1e3) / 8e12,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": None, "kernel": "moe_expert_ffn_q (gate/up + down)",
                     "bytes_per_launch": ffn_bytes, "avg_launch_us": ffn_avg_ms * 1e3, "peak_source": peak_src},
        "gpu_launches": 4 * args.steps,
        "clocks": clk.summary(),
    }
    if e2e is not None:
        line["e2e"] = e2e
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
