#!/usr/bin/env python3
"""Benchmark: MoE-layer forward tokens/s and fraction of roofline on B200.

One step = one call of colibri_moe_forward over one batch (all stages: Gate, Scatter,
Expert Compute, Gather).  Default workload: the Mixtral-shaped prefill layer (T=4096,
d_model=4096, 8 experts, top-2, SwiGLU d_ff=14336, bf16).  Inputs are seeded synthetic
tensors (random-init weights); the 2.8 GB of expert weights streamed per step is far larger
than L2, so no explicit flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl colibri|reference]

With --gpus N > 1 (launched by torch.distributed.run) every rank runs an independent replica
of the workload on its own GPU (weak scaling; the layer has no exchange step when tokens
are data-parallel); timing is the max over ranks.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/sec (prefill & decode) and % of roofline on 1 B200"
DEFAULT_WORKLOAD = "mixtral_prefill_bf16"
# T up to which the Scatter stage is one fused launch (histogram, prefix sum and scatter)
FUSED_ROUTE_MAX_T = 64


def kernels_per_step(wl):
    """Kernels one forward launches, following the library's launch sequence."""
    fused_int8 = wl.wdt == 2 and os.environ.get("COLIBRI_DEC_FUSED", "1") != "0"
    if fused_int8 and wl.T <= FUSED_ROUTE_MAX_T and os.environ.get("COLIBRI_DEC_ROUTE", "1") != "0":
        return 1                                     # router, grouping, experts, combine: one launch
    n = 1                                            # Gate: router + top-k
    n += 1 if wl.T <= FUSED_ROUTE_MAX_T else 3       # Scatter: fused, or count + scan + scatter
    if fused_int8:
        return n + 1                                 # int8: one fused launch, the combine inside
    if wl.wdt == 0:
        n += 2 + (2 if wl.fs else 0)                 # fp32: gate/up + down (+ the shared expert's)
    elif wl.wdt == 1:
        n += 2                                       # bf16: gate/up + down (shared expert inside)
    else:
        n += 3                                       # int8: gate/up stream, finish H, down stream
    return n + 1                                     # Gather


# DRAM bytes (read + write) per launch of the dominant kernel, from one ncu capture of the
# same kernel on the same workload (profiles/); None where no capture of the current kernel
# exists.  Keyed by (workload, dominant-kernel tag).
NCU_TRAFFIC = {
    ("mixtral_prefill_bf16", "tc2_ffn"): 3.1173e9 + 0.2305e9,      # tc2_ffn_traffic_mixtral_prefill_bf16.md
    ("fine_grained_shared_bf16", "tc_ffn"): 1.00698e9 + 74.0e6,   # launches_fine_grained_shared_bf16.md
    ("decode_int8_T1", "dec_fused"): 352.855e6 + 4.891e6,         # dec_fused_decode_int8_T1.md
}

# fp32 FMA peak: 148 SMs x 128 lanes x 2 FLOP x 1.965 GHz (the unit counts and clock of the part)
FP32_SIMT_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="colibri", choices=["colibri", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-sample-tokens", type=int, default=None,
                    help="tokens of the CPU-baseline sample (default sized for ~10-30 s)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    a = ap.parse_args()
    a.warmup = max(a.warmup, 3)
    return a


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            pk = json.load(fh)
        return dict(hbm=pk["hbm_gbs"], bf16=pk["bf16_tflops"], bf16_sus=pk.get("bf16_tflops_sustained"),
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


def work(wl, counts):
    """Algorithmic work of one call: only the k chosen experts per token, plus the shared expert."""
    rows = wl.T * wl.k
    d, f, fs = wl.d, wl.f, wl.fs
    wsize = {0: 4, 1: 2, 2: 1}[wl.wdt]
    touched = sum(1 for c in counts if c > 0)
    flops_gateup = 2.0 * rows * d * 2 * f + 2.0 * wl.T * d * 2 * fs
    flops_down = 2.0 * rows * f * d + 2.0 * wl.T * fs * d
    flops_router = 2.0 * wl.T * d * wl.E
    w13_bytes = touched * 2 * f * d * wsize + (2 * fs * d * wsize if fs else 0)
    w2_bytes = touched * d * f * wsize + (fs * d * wsize if fs else 0)
    scale_bytes = touched * (2 * f + d) * 4 if wl.wdt == 2 else 0
    return dict(flops_gateup=flops_gateup, flops_down=flops_down, flops_router=flops_router,
                flops=flops_gateup + flops_down + flops_router, w13_bytes=w13_bytes, w2_bytes=w2_bytes,
                scale_bytes=scale_bytes, touched=touched)


class ClockSampler:
    """Samples the SM clock and clock-event reasons through NVML (read-only queries) every
    20 ms on a background thread during the timed region."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, pci_bus_id: str):
        self.pci = pci_bus_id
        self.samples = []
        self.max_mhz = None
        self.error = None

    def __enter__(self):
        import threading

        self.stop = threading.Event()
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(self.pci.encode() if isinstance(self.pci, str) else self.pci)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.sample()
        except Exception as exc:  # NVML missing or unreadable: report unsampled
            self.error = repr(exc)
            self.nv = None
            return self
        self.thread = threading.Thread(target=self.loop, daemon=True)
        self.thread.start()
        return self

    def sample(self):
        nv = self.nv
        mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
        reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        self.samples.append((mhz, reasons))

    def loop(self):
        while not self.stop.wait(0.02):
            try:
                self.sample()
            except Exception:
                break

    def __exit__(self, *exc):
        self.stop.set()
        if self.nv is not None:
            self.thread.join(timeout=2)
            try:
                self.sample()
            except Exception:
                pass
        return False

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"], "samples": 0,
                    "error": self.error}
        nv = self.nv
        mhz = [m for m, _ in self.samples]
        active = sorted({name for _, bits in self.samples for name, const in self.REASONS
                         if bits & getattr(nv, const, 0)})
        return {"sm_mhz": statistics.median(mhz), "sm_min_mhz": min(mhz), "sm_max_mhz": self.max_mhz,
                "reasons": active, "samples": len(mhz), "source": "NVML, 20 ms"}


def cpu_baseline(p, n_tokens, seed_tokens=None):
    """The oracle, as it stands, on a bounded sample: routing for every token, the expert FFN
    and combine for n_tokens tokens spread over the batch; tokens/s extrapolated per token."""
    import oracle
    from inputgen import sample_tokens

    wl = p.wl
    t0 = time.perf_counter()
    logits = oracle.router_logits(p.x, p.router_w, p.router_b)
    idx, w, _ = oracle.topk(logits, wl.k)
    oracle.group(idx, wl.E)
    t_route = time.perf_counter() - t0
    toks = seed_tokens or sample_tokens(wl.T, n_tokens)
    t0 = time.perf_counter()
    oracle.combine(p.x, idx, w, p.expert_w, p.expert_stride, wl.f, p.expert_scales, p.shared_w, wl.fs, toks)
    t_ffn = time.perf_counter() - t0
    per_token = t_route / wl.T + t_ffn / len(toks)
    return dict(value=1.0 / per_token, unit="tokens/s", cores=1, kind="oracle",
                sample=f"routing (logits, top-k, grouping) of all {wl.T} tokens in {t_route:.2f} s; expert FFN + "
                       f"combine of {len(toks)} tokens spread over the batch in {t_ffn:.2f} s; tokens/s = 1 / "
                       f"(routing time per token + FFN time per token), single-threaded C++ oracle",
                seconds=t_route + t_ffn)


def default_sample(wl):
    per_token_macs = wl.k * 3 * wl.d * wl.f + 3 * wl.d * wl.fs
    # ~0.4 s per 3.5e8 multiply-adds on one core -> aim at ~12 s
    return int(max(2, min(wl.T, round(12.0 / (per_token_macs / 3.5e8 * 0.4)))))


def run_reference(a, rank, world):
    """--impl reference: the oracle on the host cores, rank 0 only, bounded sample per step."""
    if rank != 0:
        return 0
    import inputgen
    import oracle

    wl = inputgen.WORKLOADS[a.workload]
    p = inputgen.make_problem(wl, seed=a.seed)
    sample_tokens = inputgen.sample_tokens
    n = max(1, min(wl.T, (a.cpu_sample_tokens or max(1, default_sample(wl) // 4))))
    toks = sample_tokens(wl.T, n)
    logits = oracle.router_logits(p.x, p.router_w, p.router_b)
    idx, w, _ = oracle.topk(logits, wl.k)

    def step():
        # routing for the sampled tokens, then their FFN and combine
        rows = p.x[toks].contiguous()
        lg = oracle.router_logits(rows, p.router_w, p.router_b)
        oracle.topk(lg, wl.k)
        oracle.combine(p.x, idx, w, p.expert_w, p.expert_stride, wl.f, p.expert_scales, p.shared_w, wl.fs, toks)

    for _ in range(a.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(a.steps):
        step()
    dt = time.perf_counter() - t0
    value = len(toks) * a.steps / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": dt / a.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(wl),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": f"each step: routing and expert FFN + combine of {len(toks)} of the {wl.T} "
                                   f"tokens (single-threaded C++ oracle, double accumulation)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def max_over_ranks(ms, world, device):
    """The largest of the ranks' times: each rank times its own replica on its own device."""
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, tokens_per_step, steps, ms):
    """Whole-job tokens/s: every rank processed `steps` batches of `tokens_per_step` in `ms`."""
    return world * tokens_per_step * steps / (ms / 1e3)


def config_of(wl):
    cfg = {"workload": wl.name, "T": wl.T, "d_model": wl.d, "num_experts": wl.E, "top_k": wl.k, "d_ff": wl.f,
           "act_dtype": {0: "f32", 1: "bf16"}[wl.act], "weight_dtype": {0: "f32", 1: "bf16", 2: "i8"}[wl.wdt]}
    if wl.fs:
        cfg["shared_d_ff"] = wl.fs
    if wl.bias:
        cfg["router_bias"] = {str(e): v for e, v in wl.bias}
    return cfg


def main():
    a = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if a.impl == "reference":
        return run_reference(a, rank, world)

    import torch
    import torch.distributed as dist

    import inputgen
    import sparse_expert_ffn_router_b200 as colibri

    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    wl = inputgen.WORKLOADS[a.workload]
    p = inputgen.make_problem(wl, seed=a.seed, pin=True)
    dev = torch.device("cuda", local)
    x = p.x.to(dev)
    rw = p.router_w.to(dev)
    rb = None if p.router_b is None else p.router_b.to(dev)
    ew = p.expert_w.to(dev)
    sc = None if p.expert_scales is None else p.expert_scales.to(dev)
    sw = None if p.shared_w is None else p.shared_w.to(dev)
    y = torch.empty(wl.T, wl.d, dtype=x.dtype, device=dev)
    layer = colibri.MoELayer(wl.d, wl.f, wl.E, wl.k, wl.fs, wl.act, wl.wdt, max_tokens=wl.T, device_id=local)
    assert layer.expert_stride == p.expert_stride
    # a dedicated stream: the library replays a captured CUDA graph of the forward on it
    stream = torch.cuda.Stream(device=dev)

    def step(xin, yout):
        colibri.colibri_moe_forward(layer.ctx, xin, wl.T, rw, rb, ew, sc, sw, yout, stream)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(a.warmup):
        step(x, y)
    layer.sync_status()
    counts = torch.empty(wl.E, dtype=torch.int32, device=dev)
    colibri.colibri_get_routing(layer.ctx, counts=counts, stream=stream)
    stream.synchronize()
    counts = counts.cpu().tolist()
    wk = work(wl, counts)

    # ---- device-resident timed region (inputs already in HBM; graph replay of each forward)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    props = torch.cuda.get_device_properties(dev)
    pci = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
    with ClockSampler(pci) as clk:
        ev0.record(stream)
        h0 = time.perf_counter()
        for _ in range(a.steps):
            step(x, y)
        host_ms = (time.perf_counter() - h0) * 1e3 / a.steps
        ev1.record(stream)
        barrier()
    layer.sync_status()
    ms_total = ev0.elapsed_time(ev1)

    # ---- per-kernel durations: an equal region with per-stage CUDA events recorded on the
    # forward's stream between the launches (graph replay is bypassed while they are recorded)
    colibri.colibri_profile_begin(layer.ctx, a.steps)
    barrier()
    for _ in range(a.steps):
        step(x, y)
    barrier()
    stage_ms, ncalls = colibri.colibri_profile_end(layer.ctx)
    layer.sync_status()
    ms_max = max_over_ranks(ms_total, world, dev)
    value = job_throughput(world, wl.T, a.steps, ms_max)

    # ---- end to end through the same call with host buffers (pinned x in, y out).  Every step
    # copies its x from pinned host memory and its y back inside the call.  Serial: one context
    # on one stream.  Pipelined (the reported e2e value): two contexts on two streams taking
    # alternate steps, so one step's copies overlap the other's kernels, as a serving loop
    # would run it.
    x_host = p.x.pin_memory() if not p.x.is_pinned() else p.x
    y_hosts = [torch.empty(wl.T, wl.d, dtype=x.dtype).pin_memory() for _ in range(2)]
    for _ in range(2):
        step(x_host, y_hosts[0])
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(a.steps):
        step(x_host, y_hosts[0])
    e1.record(stream)
    barrier()
    e2e_serial = job_throughput(world, wl.T, a.steps, max_over_ranks(e0.elapsed_time(e1), world, dev))

    layer2 = colibri.MoELayer(wl.d, wl.f, wl.E, wl.k, wl.fs, wl.act, wl.wdt, max_tokens=wl.T, device_id=local)
    stream2 = torch.cuda.Stream(device=dev)
    ctxs, streams = (layer.ctx, layer2.ctx), (stream, stream2)

    def e2e_step(i):
        colibri.colibri_moe_forward(ctxs[i & 1], x_host, wl.T, rw, rb, ew, sc, sw, y_hosts[i & 1], streams[i & 1])

    for i in range(4):
        e2e_step(i)
    barrier()
    f0, f1, fj = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
                  torch.cuda.Event())
    f0.record(stream)
    stream2.wait_event(f0)
    for i in range(a.steps):
        e2e_step(i)
    fj.record(stream2)
    stream.wait_event(fj)
    f1.record(stream)
    barrier()
    layer2.sync_status()
    layer2.close()
    e2e_value = job_throughput(world, wl.T, a.steps, max_over_ranks(f0.elapsed_time(f1), world, dev))
    row_bytes = wl.d * (4 if wl.act == 0 else 2)

    # ---- roofline of the dominant kernel (per-launch averages over the timed region)
    pk = peaks()
    per_call = {k: v / max(ncalls, 1) for k, v in stage_ms.items()}
    if wl.wdt == 2:
        # the expert stage and the combine: one fused launch (or, with COLIBRI_DEC_FUSED=0, the
        # gate/up stream, H planes, down stream and combine launches), all touched weights
        wbytes = wk["w13_bytes"] + wk["w2_bytes"] + wk["scale_bytes"]
        ms_exp = per_call["expert_gateup"] + per_call["expert_down"] + per_call["gather"]
        achieved = wbytes / (ms_exp / 1e3) / 1e9
        fused = os.environ.get("COLIBRI_DEC_FUSED", "1") != "0"
        roof = {"kernel": ("dec_fused_kernel (one cooperative launch: tcgen05 kind::i8 gate/up stream, H planes, "
                           "down stream, combine)") if fused else
                ("dec_stream_kernel<gate/up> + dec_finish_h_kernel + dec_stream_kernel<down> + "
                 "combine_split_kernel (tcgen05 kind::i8 weight streams)"),
                "bound": "hbm", "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s", "frac": achieved / pk["hbm"],
                "algorithmic_bytes_per_launch": wbytes}
    elif wl.wdt == 1:
        achieved = wk["flops_gateup"] / (per_call["expert_gateup"] / 1e3) / 1e12
        mode = os.environ.get("COLIBRI_GEMM_CTA", "")[:1]
        if mode not in ("1", "2", "s"):
            mode = "2" if wl.T * wl.k // wl.E >= 512 else "1"
        name = {"1": "tc_ffn_kernel<gate/up> (tcgen05, 128x256 tiles)",
                "2": "tc2_ffn_kernel<gate/up> (tcgen05, 2-CTA 256x256 pair tiles)",
                "s": "tcs_ffn_kernel<gate/up> (tcgen05, weights x 16..256 token rows)"}[mode]
        roof = {"kernel": name, "bound": "tensor", "achieved": achieved,
                "peak": pk["bf16"], "unit": "TFLOP/s", "frac": achieved / pk["bf16"],
                "algorithmic_flops_per_launch": wk["flops_gateup"]}
    else:
        achieved = wk["flops_gateup"] / (per_call["expert_gateup"] / 1e3) / 1e12
        roof = {"kernel": "simt_ffn_kernel<gate/up> (fp32 FMA)", "bound": "alu", "achieved": achieved,
                "peak": FP32_SIMT_TFLOPS, "unit": "TFLOP/s",
                "frac": achieved / FP32_SIMT_TFLOPS, "algorithmic_flops_per_launch": wk["flops_gateup"]}
    roof["peak_source"] = pk["source"] + (" burst" if roof["bound"] == "tensor" else "")
    tag = {"dec_fused_kernel": "dec_fused", "tc_ffn_kernel<": "tc_ffn", "tc2_ffn_kernel<": "tc2_ffn",
           "tcs_ffn_kernel<": "tcs_ffn"}
    ktag = next((v for k, v in tag.items() if roof["kernel"].startswith(k)), None)
    roof["traffic"] = NCU_TRAFFIC.get((wl.name, ktag))
    roof["timing"] = "kernel stage events averaged over the profiling region's calls"
    kernels = kernels_per_step(wl)

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": ms_max / a.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": {0: "f32", 1: "bf16", 2: "bf16"}[wl.act],
        "data": "synthetic (seeded SplitMix64 + Box-Muller inputs, random-init weights)",
        "config": dict(config_of(wl), l2="inputs larger than L2: %.2f GB of expert weights per step" %
                       ((wk["w13_bytes"] + wk["w2_bytes"]) / 1e9), parallelism=f"replicas x{world}"),
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": wl.T * row_bytes,
                "d2h_bytes_per_step": wl.T * row_bytes, "serial_value": e2e_serial,
                "how": "colibri_moe_forward with pinned host x and y (copies inside the call, every step); "
                       "value: two contexts on two streams taking alternate steps; serial_value: one stream"},
        "gpu_launches": kernels * a.steps,
        "clocks": clk.summary(),
        "stage_ms_per_call": per_call,
        "stage_timing": "per-stage CUDA events on the forward's stream, second region of the same length",
        "host_ms_per_step": host_ms,
        "tflops_per_gpu_layer": wk["flops"] * a.steps / (ms_max / 1e3) / 1e12,
        "routing_counts": counts,
    }
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        n = a.cpu_sample_tokens or default_sample(wl)
        line["cpu_baseline"] = cpu_baseline(p, n)
    if rank == 0:
        print(json.dumps(line), flush=True)
    layer.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
