#!/usr/bin/env python3
"""Benchmark: MoE-layer forward tokens/s and fraction of roofline on B200.

One step = one call of colibri_moe_forward over one batch (all stages: Gate, Scatter,
Expert Compute, Gather).  Headline workload: the Mixtral-shaped prefill layer (T=4096,
d_model=4096, 8 experts, top-2, SwiGLU d_ff=14336, bf16).  Inputs are seeded synthetic
tensors (random-init weights); the 2.8 GB of expert weights streamed per step is far larger
than L2, so no explicit flush is needed between its steps.

The same line carries a `workloads` object with one entry per workload of the metric (the tiny
fp32 layer, the Mixtral prefill, the 128-expert layer with a shared expert, the skewed layer,
and int8 and group-wise int4 decode at T = 1, 8 and 32): the median time per call over at least
--calls calls with L2 flushed before each call, the dominant kernel's roofline from the stage
events of an equal region (recorded inside the replayed CUDA graph), its own clock record, and
end-to-end figures.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--workloads all|none|a,b]
                    [--calls C] [--impl colibri|reference]

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
# T up to which int4 weights take the GEMV kernels (d and f multiples of 1024): dp4a up to 2 tokens,
# warp-level MMA beyond
GEMV4_MAX_T = 16


def kernels_per_step(wl):
    """Kernels one forward launches, following the library's launch sequence."""
    if wl.wdt == 3:  # int4: router, Scatter, gate/up (stream or GEMV), H planes, down, combine
        return 1 + (1 if wl.T <= FUSED_ROUTE_MAX_T else 3) + 4
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
    ("mixtral_prefill_bf16", "tc2_ffn"): 1.9466e9 + 0.2246e9,      # launches_mixtral_prefill_bf16.md
    ("fine_grained_shared_bf16", "tc2_ffn"): 1.0012e9 + 0.0707e9,  # launches_fine_grained_shared_bf16.md
    ("skewed_bf16", "tc2_ffn"): 2.2216e9 + 0.0584e9,               # tc_ffn_traffic_skewed_bf16.md
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
    ap.add_argument("--workloads", default="all",
                    help="workloads measured in the line's `workloads` object: all, none, or a comma list")
    ap.add_argument("--calls", type=int, default=100, help="minimum calls per `workloads` entry")
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
    wsize = {0: 4, 1: 2, 2: 1, 3: 0.5}[wl.wdt]
    touched = sum(1 for c in counts if c > 0)
    flops_gateup = 2.0 * rows * d * 2 * f + 2.0 * wl.T * d * 2 * fs
    flops_down = 2.0 * rows * f * d + 2.0 * wl.T * fs * d
    flops_router = 2.0 * wl.T * d * wl.E
    w13_bytes = touched * 2 * f * d * wsize + (2 * fs * d * wsize if fs else 0)
    w2_bytes = touched * d * f * wsize + (fs * d * wsize if fs else 0)
    scale_bytes = touched * (2 * f + d) * 4 if wl.wdt == 2 else 0
    if wl.wdt == 3:  # one fp32 scale per output channel and group of 128 inputs
        scale_bytes = touched * 3 * d * f // 128 * 4
    return dict(flops_gateup=flops_gateup, flops_down=flops_down, flops_router=flops_router,
                flops=flops_gateup + flops_down + flops_router, w13_bytes=w13_bytes, w2_bytes=w2_bytes,
                scale_bytes=scale_bytes, touched=touched)


class ClockSampler:
    """Samples the SM clock and clock-event reasons through NVML (read-only queries) every
    10 ms on a background thread during the timed region."""

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
        while not self.stop.wait(0.01):
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
                "reasons": active, "samples": len(mhz), "source": "NVML, 10 ms"}


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
           "act_dtype": {0: "f32", 1: "bf16"}[wl.act],
           "weight_dtype": {0: "f32", 1: "bf16", 2: "i8", 3: "i4 (groups of 128)"}[wl.wdt]}
    if wl.fs:
        cfg["shared_d_ff"] = wl.fs
    if wl.bias:
        cfg["router_bias"] = {str(e): v for e, v in wl.bias}
    return cfg


L2_BYTES = 126 * 1024 * 1024
FLUSH_BYTES = 256 * 1024 * 1024  # one write larger than L2 evicts what the previous call left there
STAGES = ("gate", "scatter", "expert_gateup", "expert_down", "gather")
ENTRY_WORKLOADS = ("tiny_f32", "mixtral_prefill_bf16", "fine_grained_shared_bf16", "skewed_bf16",
                   "decode_int8_T1", "decode_int8_T8", "decode_int8_T32", "decode_int4_T1", "decode_int4_T8",
                   "decode_int4_T32")


def median(v):
    return statistics.median(v) if v else None


def percentile(v, q):
    if not v:
        return None
    s = sorted(v)
    return s[min(len(s) - 1, max(0, int(round(q * (len(s) - 1)))))]


class Runner:
    """One workload on one GPU: inputs resident in HBM, one layer context, a dedicated stream.

    Every timed call goes through colibri_moe_forward (the library replays its captured CUDA
    graph of the call).  Per-call device times come from CUDA events recorded on the forward's
    stream between calls; stage times from the library's stage events, which sit inside the
    replayed graph (colibri_profile_begin), so the timed launch sequence is the same."""

    def __init__(self, wl, seed, local, world, pin=False):
        import torch

        import inputgen
        import sparse_expert_ffn_router_b200 as colibri

        self.torch, self.colibri, self.wl, self.world = torch, colibri, wl, world
        self.dev = torch.device("cuda", local)
        self.p = p = inputgen.make_problem(wl, seed=seed, pin=pin)
        dev = self.dev
        self.x = p.x.to(dev)
        self.rw = p.router_w.to(dev)
        self.rb = None if p.router_b is None else p.router_b.to(dev)
        self.ew = p.expert_w.to(dev)
        self.sc = None if p.expert_scales is None else p.expert_scales.to(dev)
        self.sw = None if p.shared_w is None else p.shared_w.to(dev)
        self.y = torch.empty(wl.T, wl.d, dtype=self.x.dtype, device=dev)
        self.layer = colibri.MoELayer(wl.d, wl.f, wl.E, wl.k, wl.fs, wl.act, wl.wdt, max_tokens=wl.T,
                                      device_id=local)
        assert self.layer.expert_stride == p.expert_stride
        self.stream = torch.cuda.Stream(device=dev)
        self.flush_buf = None
        props = torch.cuda.get_device_properties(dev)
        self.pci = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"

    def step(self, xin=None, yout=None, ctx=None, stream=None):
        self.colibri.colibri_moe_forward(ctx or self.layer.ctx, self.x if xin is None else xin, self.wl.T, self.rw,
                                         self.rb, self.ew, self.sc, self.sw, self.y if yout is None else yout,
                                         stream or self.stream)

    def flush(self):
        if self.flush_buf is None:
            self.flush_buf = self.torch.empty(FLUSH_BYTES, dtype=self.torch.uint8, device=self.dev)
        with self.torch.cuda.stream(self.stream):
            self.flush_buf.zero_()

    def barrier(self):
        import torch.distributed as dist

        if self.world > 1:
            dist.barrier()
        self.torch.cuda.synchronize(self.dev)

    def counts(self):
        torch = self.torch
        c = torch.empty(self.wl.E, dtype=torch.int32, device=self.dev)
        self.colibri.colibri_get_routing(self.layer.ctx, counts=c, stream=self.stream)
        self.stream.synchronize()
        return c.cpu().tolist()

    def timed(self, n, flush):
        """n calls, an event pair around each (L2 flushed before each call if `flush`).
        Returns (per-call ms list, ms from the first call's start to the last call's end, clocks)."""
        torch = self.torch
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * n)]
        self.barrier()
        with ClockSampler(self.pci) as clk:
            for i in range(n):
                if flush:
                    self.flush()
                ev[2 * i].record(self.stream)
                self.step()
                ev[2 * i + 1].record(self.stream)
            self.barrier()
        self.layer.sync_status()
        per = [ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(n)]
        return per, ev[0].elapsed_time(ev[-1]), clk.summary()

    def profiled(self, n, flush):
        """n calls with the library's stage events (inside the replayed graph).  Returns the
        per-call stage dicts and the clock summary of the region."""
        colibri = self.colibri
        colibri.colibri_profile_begin(self.layer.ctx, n)
        self.barrier()
        with ClockSampler(self.pci) as clk:
            for _ in range(n):
                if flush:
                    self.flush()
                self.step()
            self.barrier()
        _, ncalls = colibri.colibri_profile_end(self.layer.ctx)
        calls = colibri.colibri_profile_calls(self.layer.ctx, ncalls)
        self.layer.sync_status()
        return calls, clk.summary()

    def e2e(self, n):
        """End to end through the same call with pinned host x and y: every call copies its x in
        and its y out inside the call.  Serial: one context on one stream (the reported value).
        Pipelined: two contexts on two streams taking alternate calls."""
        torch, colibri, wl = self.torch, self.colibri, self.wl
        x_host = self.p.x if self.p.x.is_pinned() else self.p.x.pin_memory()
        y_hosts = [torch.empty(wl.T, wl.d, dtype=self.x.dtype).pin_memory() for _ in range(2)]
        for _ in range(2):
            self.step(x_host, y_hosts[0])
        self.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(self.stream)
        for _ in range(n):
            self.step(x_host, y_hosts[0])
        e1.record(self.stream)
        self.barrier()
        serial_ms = max_over_ranks(e0.elapsed_time(e1), self.world, self.dev)
        layer2 = colibri.MoELayer(wl.d, wl.f, wl.E, wl.k, wl.fs, wl.act, wl.wdt, max_tokens=wl.T,
                                  device_id=self.dev.index)
        stream2 = torch.cuda.Stream(device=self.dev)
        ctxs, streams = (self.layer.ctx, layer2.ctx), (self.stream, stream2)
        for i in range(4):
            self.step(x_host, y_hosts[i & 1], ctxs[i & 1], streams[i & 1])
        self.barrier()
        f0, f1, fj = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
                      torch.cuda.Event())
        f0.record(self.stream)
        stream2.wait_event(f0)
        for i in range(n):
            self.step(x_host, y_hosts[i & 1], ctxs[i & 1], streams[i & 1])
        fj.record(stream2)
        self.stream.wait_event(fj)
        f1.record(self.stream)
        self.barrier()
        layer2.sync_status()
        layer2.close()
        pipe_ms = max_over_ranks(f0.elapsed_time(f1), self.world, self.dev)
        row_bytes = wl.d * (4 if wl.act == 0 else 2)
        return {"value": job_throughput(self.world, wl.T, n, serial_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": wl.T * row_bytes, "d2h_bytes_per_step": wl.T * row_bytes,
                "us_per_call": serial_ms / n * 1e3,
                "pipelined_value": job_throughput(self.world, wl.T, n, pipe_ms),
                "how": "colibri_moe_forward with pinned host x and y (the call copies x in and y out, every "
                       "call); value: one context on one stream (calls in sequence); pipelined_value: two "
                       "contexts on two streams taking alternate calls"}

    def close(self):
        self.layer.close()


def roofline(wl, wk, stage_ms, pk):
    """Roofline of the dominant kernel from its per-launch duration (ms)."""
    if wl.wdt == 3:
        wbytes = wk["w13_bytes"] + wk["w2_bytes"] + wk["scale_bytes"]
        ms = stage_ms["expert_gateup"] + stage_ms["expert_down"] + stage_ms["gather"]
        achieved = wbytes / (ms / 1e3) / 1e9
        gemv = (wl.T <= GEMV4_MAX_T and wl.d % 1024 == 0 and wl.f % 1024 == 0
                and os.environ.get("COLIBRI_I4_GEMV", "1") != "0")
        gk = "gemv4_kernel" if wl.T <= 2 else "gemv4m_kernel"
        how = ("dp4a on the CUDA cores" if wl.T <= 2 else "mma.sync m16n8k32 s8, up to 8 tokens per instruction")
        roof = {"kernel": (f"{gk}<gate/up> + dec_finish_h_kernel + {gk}<down> + combine_split_kernel "
                           f"({how}, packed int4 weights read straight into registers, group scales)") if gemv else
                          ("dec_stream4_kernel<gate/up> + dec_finish_h_kernel + dec_stream4_kernel<down> + "
                           "combine_split_kernel (packed int4 tiles widened to int8 in shared memory, tcgen05 "
                           "kind::i8, group scales per K block)"),
                "bound": "hbm", "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s",
                "frac": achieved / pk["hbm"], "algorithmic_bytes_per_launch": wbytes}
    elif wl.wdt == 2:
        # the expert stage and the combine: one fused launch (or, with COLIBRI_DEC_FUSED=0, the
        # gate/up stream, H planes, down stream and combine launches), all touched weights
        wbytes = wk["w13_bytes"] + wk["w2_bytes"] + wk["scale_bytes"]
        ms = stage_ms["expert_gateup"] + stage_ms["expert_down"] + stage_ms["gather"]
        achieved = wbytes / (ms / 1e3) / 1e9
        fused = os.environ.get("COLIBRI_DEC_FUSED", "1") != "0"
        roof = {"kernel": ("dec_fused_kernel (one cooperative launch: tcgen05 kind::i8 gate/up stream, H planes, "
                           "down stream, combine" + (", and for T <= 64 routing" if wl.T <= 64 else "") + ")")
                if fused else ("dec_stream_kernel<gate/up> + dec_finish_h_kernel + dec_stream_kernel<down> + "
                               "combine_split_kernel (tcgen05 kind::i8 weight streams)"),
                "bound": "hbm", "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s",
                "frac": achieved / pk["hbm"], "algorithmic_bytes_per_launch": wbytes}
    elif wl.wdt == 1:
        ms = stage_ms["expert_gateup"]
        achieved = wk["flops_gateup"] / (ms / 1e3) / 1e12
        mode = "1" if os.environ.get("COLIBRI_GEMM_CTA", "")[:1] == "1" else "2"
        name = {"1": "tc_ffn_kernel<gate/up> (tcgen05, 128x256 tiles)",
                "2": "tc2_ffn_kernel<gate/up> (tcgen05, 2-CTA 256x256 pair tiles)"}[mode]
        roof = {"kernel": name, "bound": "tensor", "achieved": achieved, "peak": pk["bf16"], "unit": "TFLOP/s",
                "frac": achieved / pk["bf16"], "algorithmic_flops_per_launch": wk["flops_gateup"]}
    else:
        ms = stage_ms["expert_gateup"]
        achieved = wk["flops_gateup"] / (ms / 1e3) / 1e12
        roof = {"kernel": "simt_ffn_kernel<gate/up> (fp32 FMA)", "bound": "alu", "achieved": achieved,
                "peak": FP32_SIMT_TFLOPS, "unit": "TFLOP/s", "frac": achieved / FP32_SIMT_TFLOPS,
                "algorithmic_flops_per_launch": wk["flops_gateup"]}
    roof["kernel_ms"] = ms
    roof["peak_source"] = pk["source"] + (" burst" if roof["bound"] == "tensor" else "")
    tag = {"dec_fused_kernel": "dec_fused", "tc_ffn_kernel<": "tc_ffn", "tc2_ffn_kernel<": "tc2_ffn"}
    ktag = next((v for k, v in tag.items() if roof["kernel"].startswith(k)), None)
    roof["traffic"] = NCU_TRAFFIC.get((wl.name, ktag))
    return roof


def stage_summary(calls, agg):
    """Per-stage aggregate (median or mean) over the recorded calls, and the per-call total."""
    out = {s: agg([c[s] for c in calls]) for s in STAGES}
    out["total"] = agg([sum(c[s] for s in STAGES) for c in calls])
    return out


def measure_entry(wl, a, local, world, pk):
    """One entry of the `workloads` object: median us per call over >= a.calls calls, the
    dominant kernel's roofline from stage events of an equal region, and e2e.  A workload whose
    touched weights exceed twice the L2 runs its calls back to back (inputs larger than L2, as
    the headline); a smaller one (the tiny fp32 layer) has L2 flushed before every call.  The
    other kind of region is reported beside it."""
    r = Runner(wl, a.seed, local, world)
    try:
        for _ in range(10):
            r.step()
        r.layer.sync_status()
        counts = r.counts()
        wk = work(wl, counts)
        flush = wk["w13_bytes"] + wk["w2_bytes"] < 2 * L2_BYTES
        # size the regions: at least a.calls calls and about 0.2 s of calls
        per, _, _ = r.timed(5, flush=flush)
        n = int(max(a.calls, min(4000, 0.2 / max(median(per) / 1e3, 1e-6))))
        per, _, clk = r.timed(n, flush=flush)
        med = max_over_ranks(median(per), world, r.dev)
        alt_per, alt_total, alt_clk = r.timed(n, flush=not flush)
        calls, pclk = r.profiled(n, flush=flush)
        st_med = stage_summary(calls, median)
        roof = roofline(wl, wk, st_med, pk)
        region = ("L2 flushed (256 MB write) before each call" if flush else
                  "calls back to back, inputs larger than L2 (%.2f GB of expert weights per call)" %
                  ((wk["w13_bytes"] + wk["w2_bytes"]) / 1e9))
        roof["timing"] = (f"median over {n} calls of the kernel's stage events, recorded inside the replayed CUDA "
                          f"graph; {region}")
        e2e = r.e2e(max(20, min(n, 200)))
        entry = {
            "us_per_call": med * 1e3, "tokens_per_s": job_throughput(world, wl.T, 1, med),
            "calls": n, "stat": f"median of per-call CUDA-event times; {region}",
            "us_p10": percentile(per, 0.1) * 1e3, "us_p90": percentile(per, 0.9) * 1e3,
            ("back_to_back_median_us" if flush else "l2_flushed_median_us"): median(alt_per) * 1e3,
            "roofline": roof,
            "stage_us_median": {k: v * 1e3 for k, v in st_med.items()},
            "profiled_over_timed": st_med["total"] / median(per),
            "e2e": e2e,
            "kernels_per_call": kernels_per_step(wl),
            "clocks": clk, ("clocks_back_to_back" if flush else "clocks_l2_flushed"): alt_clk,
            "clocks_profiled": pclk,
            "routing_counts": counts,
            "config": config_of(wl),
        }
        return entry
    finally:
        r.close()


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

    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    wl = inputgen.WORKLOADS[a.workload]
    pk = peaks()
    r = Runner(wl, a.seed, local, world)
    for _ in range(a.warmup):
        r.step()
    r.layer.sync_status()
    counts = r.counts()
    wk = work(wl, counts)
    touched = wk["w13_bytes"] + wk["w2_bytes"]
    flush = touched < 2 * L2_BYTES

    # ---- device-resident timed region: exactly a.steps calls (graph replay of each forward),
    # an event pair around each, bracketed by a barrier and a device synchronisation
    per, total_ms, clk = r.timed(a.steps, flush=flush)
    ms_sum = sum(per) if flush else total_ms
    ms_max = max_over_ranks(ms_sum, world, r.dev)
    value = job_throughput(world, wl.T, a.steps, ms_max)

    # ---- the dominant kernel: an equal region with the stage events inside the replayed graph
    calls, pclk = r.profiled(a.steps, flush=flush)
    st_mean = stage_summary(calls, statistics.fmean)
    roof = roofline(wl, wk, st_mean, pk)
    roof["timing"] = (f"mean over the {a.steps} calls of an equal region of the kernel's stage events, recorded "
                      "inside the replayed CUDA graph")
    e2e = r.e2e(a.steps)
    r.close()
    problem = r.p
    del r
    torch.cuda.empty_cache()

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": ms_max / a.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": {0: "f32", 1: "bf16", 2: "bf16"}[wl.act],
        "data": "synthetic (seeded SplitMix64 + Box-Muller inputs, random-init weights)",
        "config": dict(config_of(wl), l2=("L2 flushed (256 MB write) before every call" if flush else
                                          "inputs larger than L2: %.2f GB of expert weights per step" %
                                          (touched / 1e9)), parallelism=f"replicas x{world}"),
        "roofline": roof,
        "e2e": e2e,
        "gpu_launches": kernels_per_step(wl) * a.steps,
        "clocks": clk,
        "clocks_profiled": pclk,
        "stage_ms_per_call": {k: v for k, v in st_mean.items() if k != "total"},
        "profiled_over_timed": st_mean["total"] / (ms_sum / a.steps),
        "stage_timing": "per-stage CUDA events recorded inside the replayed graph, equal region after the timed one",
        "median_ms_per_step": median(per),
        "tflops_per_gpu_layer": wk["flops"] * a.steps / (ms_max / 1e3) / 1e12,
        "routing_counts": counts,
    }
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        n = a.cpu_sample_tokens or default_sample(wl)
        line["cpu_baseline"] = cpu_baseline(problem, n)
    del problem

    # ---- every workload of the metric (prefill and decode), each in its own regions
    names = ENTRY_WORKLOADS if a.workloads == "all" else tuple(x for x in a.workloads.split(",") if x and x != "none")
    if names:
        entries = {}
        for name in names:
            entries[name] = measure_entry(inputgen.WORKLOADS[name], a, local, world, pk)
            torch.cuda.empty_cache()
        line["workloads"] = entries
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
