"""The measurement arithmetic of bench.py, pinned to values worked out by hand from the
workloads' shapes (no GPU): the algorithmic work per call, the roofline fraction of the dominant
kernel, the whole-job throughput and the number of kernels a forward launches."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import inputgen  # noqa: E402

W = inputgen.WORKLOADS
PK = dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


def all_touched(wl):
    return [1] * wl.E


def test_mixtral_prefill_work():
    # 4096 tokens x top-2 = 8192 routed rows; gate/up 2 FLOP x rows x d x 2f, down 2 x rows x f x d
    wk = bench.work(W["mixtral_prefill_bf16"], all_touched(W["mixtral_prefill_bf16"]))
    assert wk["flops_gateup"] == 2 * 8192 * 4096 * 2 * 14336  # 1.924 TFLOP
    assert wk["flops_down"] == 2 * 8192 * 14336 * 4096        # 0.962 TFLOP
    assert wk["flops_router"] == 2 * 4096 * 4096 * 8
    assert wk["w13_bytes"] == 8 * 2 * 14336 * 4096 * 2        # 1.879 GB of bf16 W1 | W3
    assert wk["w2_bytes"] == 8 * 14336 * 4096 * 2             # 0.940 GB of bf16 W2
    assert wk["scale_bytes"] == 0


def test_shared_expert_work():
    # the shared expert adds its FLOPs for every token and its weights once
    wl = W["fine_grained_shared_bf16"]
    wk = bench.work(wl, all_touched(wl))
    assert wk["flops_gateup"] == 2 * 8192 * 4 * 2048 * 2 * 768 + 2 * 8192 * 2048 * 2 * 3072
    assert wk["flops_down"] == 2 * 8192 * 4 * 768 * 2048 + 2 * 8192 * 3072 * 2048
    assert wk["w13_bytes"] == 128 * 2 * 768 * 2048 * 2 + 2 * 3072 * 2048 * 2


def test_int8_decode_one_token_bytes():
    # one token touches two experts: 3 d f int8 bytes each, plus fp32 scales s1[f] | s3[f] | s2[d]
    wl = W["decode_int8_T1"]
    counts = [1, 1] + [0] * 6
    wk = bench.work(wl, counts)
    total = wk["w13_bytes"] + wk["w2_bytes"] + wk["scale_bytes"]
    assert wk["touched"] == 2
    assert total == 2 * 3 * 14336 * 4096 + 2 * (2 * 14336 + 4096) * 4 == 352_583_680


def test_int4_decode_one_token_bytes():
    # packed nibbles: half a byte per weight; one fp32 scale per output channel and 128 inputs
    wl = W["decode_int4_T1"]
    wk = bench.work(wl, [1, 1] + [0] * 6)
    assert wk["w13_bytes"] + wk["w2_bytes"] == 2 * 3 * 14336 * 4096 // 2      # 176.2 MB
    assert wk["scale_bytes"] == 2 * 3 * 4096 * 14336 // 128 * 4             # 11.0 MB


def test_untouched_experts_cost_no_bytes():
    wl = W["skewed_empty_bf16"]
    counts = [1000, 1000] + [4] * 10 + [0] * 4
    wk = bench.work(wl, counts)
    assert wk["touched"] == 12
    assert wk["w13_bytes"] == 12 * 2 * 8192 * 4096 * 2


def test_roofline_fraction_of_the_gate_up_gemm():
    wl = W["mixtral_prefill_bf16"]
    wk = bench.work(wl, all_touched(wl))
    stage = {"gate": 0.015, "scatter": 0.03, "expert_gateup": 1.2, "expert_down": 0.75, "gather": 0.02}
    roof = bench.roofline(wl, wk, stage, PK)
    assert roof["bound"] == "tensor" and roof["unit"] == "TFLOP/s"
    assert roof["achieved"] == pytest.approx(2 * 8192 * 4096 * 2 * 14336 / 1.2e-3 / 1e12)
    assert roof["frac"] == pytest.approx(roof["achieved"] / 1590.0)
    assert roof["kernel_ms"] == 1.2


def test_roofline_of_the_int8_decode_launch():
    # the fused launch holds both weight streams, the H planes and the combine: all touched
    # weights and scales over the three stages' summed duration
    wl = W["decode_int8_T1"]
    wk = bench.work(wl, [1, 1] + [0] * 6)
    stage = {"gate": 0.001, "scatter": 0.001, "expert_gateup": 0.075, "expert_down": 0.001, "gather": 0.001}
    roof = bench.roofline(wl, wk, stage, PK)
    assert roof["bound"] == "hbm"
    assert roof["kernel_ms"] == pytest.approx(0.077)
    assert roof["achieved"] == pytest.approx(352_583_680 / 0.077e-3 / 1e9)
    assert roof["frac"] == pytest.approx(roof["achieved"] / 6650.0)


def test_whole_job_throughput():
    # every rank ran `steps` batches in the slowest rank's time
    assert bench.job_throughput(1, 4096, 50, 119.65) == pytest.approx(4096 * 50 / 0.11965)
    assert bench.job_throughput(8, 4096, 50, 119.65) == pytest.approx(8 * 4096 * 50 / 0.11965)


@pytest.mark.parametrize("name,n", [("mixtral_prefill_bf16", 7),       # router, count, scan, scatter, 2 GEMMs, combine
                                    ("fine_grained_shared_bf16", 7),   # the shared expert rides in the GEMM launches
                                    ("tiny_f32", 5),                   # router, fused grouping, 2 GEMMs, combine
                                    ("decode_int8_T1", 1),             # one cooperative launch
                                    ("decode_int8_T32", 1),
                                    ("decode_int4_T1", 6),             # router, grouping, 2 GEMVs, H, combine
                                    ("decode_int4_T32", 6)])
def test_kernels_per_forward(name, n, monkeypatch):
    for var in ("COLIBRI_DEC_FUSED", "COLIBRI_DEC_ROUTE"):
        monkeypatch.delenv(var, raising=False)
    assert bench.kernels_per_step(W[name]) == n
