"""The shared seeded generator: published SplitMix64 vector, determinism, distributions."""
import math
import os

import numpy as np
import pytest
import torch

import inputgen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_ints(name):
    with open(os.path.join(GOLDEN, name)) as fh:
        return [int(l) for l in fh if l.strip() and not l.startswith("#")]


def test_splitmix64_reference_vector():
    # raw(key, i) is the i-th output of a SplitMix64 stream whose state starts at key.
    want = _golden_ints("splitmix64_seed1234567.txt")
    assert [inputgen.raw(1234567, i) for i in range(len(want))] == want


def test_streams_are_deterministic_and_distinct():
    a = inputgen.fill_normal(torch.empty(4096), 0, 7, 1.0)
    b = inputgen.fill_normal(torch.empty(4096), 0, 7, 1.0)
    c = inputgen.fill_normal(torch.empty(4096), 0, 8, 1.0)
    d = inputgen.fill_normal(torch.empty(4096), 1, 7, 1.0)
    assert torch.equal(a, b)
    assert not torch.equal(a, c) and not torch.equal(a, d)


def test_counter_based_prefix_property():
    # element i does not depend on how many elements are drawn
    long = inputgen.fill_normal(torch.empty(1001), 3, 11, 2.0)
    short = inputgen.fill_normal(torch.empty(17), 3, 11, 2.0)
    assert torch.equal(long[:17], short)


def test_normal_moments():
    n = 1 << 20
    v = inputgen.fill_normal(torch.empty(n), 0, 1, 0.5).double()
    # mean within 6 standard errors, std within 1 %
    assert abs(v.mean().item()) < 6 * 0.5 / math.sqrt(n)
    assert abs(v.std().item() / 0.5 - 1) < 0.01
    # fourth moment of a normal is 3 sigma^4
    k4 = ((v / 0.5) ** 4).mean().item()
    assert abs(k4 - 3.0) < 0.05


def test_bf16_is_round_to_nearest_even_of_f32():
    n = 1 << 16
    f = inputgen.fill_normal(torch.empty(n, dtype=torch.float32), 5, 9, 3.0)
    h = inputgen.fill_normal(torch.empty(n, dtype=torch.bfloat16), 5, 9, 3.0)
    # torch's float32 -> bfloat16 conversion rounds to nearest even
    assert torch.equal(h, f.to(torch.bfloat16))


def test_int8_uniform_range():
    n = 255 * 4000
    q = inputgen.fill_int(torch.empty(n, dtype=torch.int8), 0, 3, -127, 127)
    assert int(q.min()) == -127 and int(q.max()) == 127
    counts = np.bincount(q.numpy().astype(np.int64) + 127, minlength=255)
    exp = n / 255
    chi2 = ((counts - exp) ** 2 / exp).sum()
    assert chi2 < 254 + 6 * math.sqrt(2 * 254)


def test_uniform_range_and_mean():
    n = 1 << 18
    u = inputgen.fill_uniform(torch.empty(n), 0, 4, 0.5, 1.5).double()
    assert u.min().item() >= 0.5 and u.max().item() <= 1.5
    assert abs(u.mean().item() - 1.0) < 6 * (1 / math.sqrt(12)) / math.sqrt(n)


def test_problem_layout_small():
    wl = inputgen.custom("t", T=5, d=16, E=3, k=2, f=24, fs=8, act=inputgen.BF16, wdt=inputgen.BF16)
    p = inputgen.make_problem(wl, seed=0)
    assert p.x.shape == (5, 16) and p.x.dtype == torch.bfloat16
    assert p.router_w.shape == (3, 16)
    assert p.expert_stride == inputgen.expert_stride_elems(16, 24) and p.expert_stride % 128 == 0
    assert p.expert_w.numel() == 3 * p.expert_stride
    # padding between experts is zero, W2 std is 1/sqrt(f)
    e0 = p.expert_w[: p.expert_stride]
    assert torch.count_nonzero(e0[3 * 16 * 24:]) == 0
    assert p.shared_w.numel() == 3 * 8 * 16


def test_int8_problem_scales():
    wl = inputgen.custom("q", T=2, d=32, E=2, k=1, f=64, act=inputgen.BF16, wdt=inputgen.I8)
    p = inputgen.make_problem(wl, seed=0)
    assert p.expert_w.dtype == torch.int8
    s = p.expert_scales.view(2, 2 * 64 + 32)
    lo1, hi1 = 0.5 / (127 * math.sqrt(32)), 1.5 / (127 * math.sqrt(32))
    lo2, hi2 = 0.5 / (127 * math.sqrt(64)), 1.5 / (127 * math.sqrt(64))
    assert s[:, :128].min() >= lo1 and s[:, :128].max() <= hi1
    assert s[:, 128:].min() >= lo2 and s[:, 128:].max() <= hi2


def test_int4_problem_packing_and_scales():
    wl = inputgen.custom("i4", T=2, d=256, E=2, k=1, f=128, act=inputgen.BF16, wdt=inputgen.I4)
    p = inputgen.make_problem(wl, seed=5)
    assert p.expert_w.dtype == torch.uint8
    assert p.expert_stride % 256 == 0 and p.expert_w.numel() == wl.E * p.expert_stride // 2
    lo = (p.expert_w.to(torch.int16) & 0xF)
    hi = (p.expert_w.to(torch.int16) >> 4)
    for nib in (lo, hi):  # values in [-7, 7]: nibble 8 (-8) never occurs
        assert not torch.any(nib == 8)
    assert p.expert_scales.numel() == wl.E * 3 * wl.d * wl.f // 128
    f, d = wl.f, wl.d
    s = p.expert_scales.view(wl.E, -1)
    s13 = s[:, : 2 * f * d // 128]
    s2 = s[:, 2 * f * d // 128:]
    assert torch.all(s13 > 0.5 / (7 * d ** 0.5) * 0.999) and torch.all(s13 < 1.5 / (7 * d ** 0.5) * 1.001)
    assert torch.all(s2 > 0.5 / (7 * f ** 0.5) * 0.999) and torch.all(s2 < 1.5 / (7 * f ** 0.5) * 1.001)
