"""Pins of the CPU oracle to things other than itself.

The pages print no worked numeric example of the layer, so the oracle is pinned by
(a) the hand-stepped tie rule of the routing scan printed on www.mhpq.cn/news/563172 §3.2
(tests/golden/topk_tie_rule.txt), (b) closed forms (k = 2 weights are a logistic of the
logit gap; k = E weights are the textbook softmax), (c) library routines on special cases
(float64 matmul for the router, float64 torch SwiGLU for E = k = 1, a stable sort for the
grouping permutation), (d) a brute-force dense "run every expert on every token, then mask"
restatement of the whole layer, and (e) invariants (k distinct experts per token, weights
non-negative summing to one, the permutation a bijection matching the histogram).
Each is chosen so that a dropped term, a wrong sign or index, or a transposed operand in
the oracle fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as F

import inputgen
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------------- helpers


def _f64(t):
    return t.to(torch.float64).numpy()


def _ref_select(logits, k):
    """Brute force: sort every row by (value descending, index ascending)."""
    T, E = logits.shape
    out = np.empty((T, k), dtype=np.int64)
    for t in range(T):
        order = np.lexsort((np.arange(E), -logits[t].astype(np.float64)))
        out[t] = order[:k]
    return out


def _unpack_int4(packed: torch.Tensor) -> torch.Tensor:
    """Packed bytes -> int8 elements (low nibble first), nibbles 8..15 read as -8..-1."""
    b = packed.to(torch.int16)
    q = torch.stack([b & 0xF, b >> 4], dim=-1).reshape(-1)
    return torch.where(q >= 8, q - 16, q).to(torch.int8)


def _int4_mats(p, e):
    """W1, W3, W2 of an int4 expert dequantised as float32 s[o][i // 128] * q[o][i]."""
    wl = p.wl
    d, f = wl.d, wl.f
    base = e * p.expert_stride
    q = _unpack_int4(p.expert_w[base // 2: (base + 3 * f * d) // 2]).to(torch.float32)
    s = p.expert_scales[e * 3 * d * f // 128:(e + 1) * 3 * d * f // 128]
    # group-major scales: [inputs / 128][outputs] per matrix
    s1 = s[: f * d // 128].view(d // 128, f).t().repeat_interleave(128, dim=1)
    s3 = s[f * d // 128: 2 * f * d // 128].view(d // 128, f).t().repeat_interleave(128, dim=1)
    s2 = s[2 * f * d // 128:].view(f // 128, d).t().repeat_interleave(128, dim=1)
    return (s1 * q[: f * d].view(f, d), s3 * q[f * d: 2 * f * d].view(f, d), s2 * q[2 * f * d:].view(d, f))


def _expert_mats(p, e):
    """W1, W3, W2 of expert e as float64 numpy (int8 / int4 dequantised as float32 s*q)."""
    wl = p.wl
    d, f = wl.d, wl.f
    base = e * p.expert_stride
    if wl.wdt == inputgen.I4:
        return tuple(_f64(m) for m in _int4_mats(p, e))
    raw = p.expert_w[base: base + 3 * f * d]
    if wl.wdt == inputgen.I8:
        s = p.expert_scales[e * (2 * f + d):(e + 1) * (2 * f + d)]
        q = raw.to(torch.float32)
        w1 = (s[:f, None] * q[: f * d].view(f, d))
        w3 = (s[f:2 * f, None] * q[f * d: 2 * f * d].view(f, d))
        w2 = (s[2 * f:, None] * q[2 * f * d:].view(d, f))
    else:
        w1 = raw[: f * d].view(f, d)
        w3 = raw[f * d: 2 * f * d].view(f, d)
        w2 = raw[2 * f * d:].view(d, f)
    return _f64(w1), _f64(w3), _f64(w2)


def _swiglu(x, w1, w3, w2):
    g = x @ w1.T
    u = x @ w3.T
    return (g / (1.0 + np.exp(-g)) * u) @ w2.T


def _dense_layer(p, flags=0):
    """Every expert on every token, combined through a masked [T, E] weight matrix.
    ``flags``: oracle.ROUTER_CLAMP clips the logits to [-50, 50]; oracle.ROUTER_RAW uses the
    chosen logits as the weights."""
    wl = p.wl
    x = _f64(p.x)
    wr = _f64(p.router_w)
    logits = x @ wr.T
    if p.router_b is not None:
        logits = logits + _f64(p.router_b)
    if flags & oracle.ROUTER_CLAMP:
        logits = np.clip(logits, -50.0, 50.0)
    sel = _ref_select(logits.astype(np.float32), wl.k)
    mask = np.zeros((wl.T, wl.E))
    for t in range(wl.T):
        ls = logits[t, sel[t]]
        if flags & oracle.ROUTER_RAW:
            mask[t, sel[t]] = ls
        else:
            mask[t, sel[t]] = np.exp(ls - ls.max()) / np.exp(ls - ls.max()).sum()
    y = np.zeros((wl.T, wl.d))
    for e in range(wl.E):
        y += mask[:, e:e + 1] * _swiglu(x, *_expert_mats(p, e))
    if wl.fs:
        fs, d = wl.fs, wl.d
        sw = p.shared_w
        y += _swiglu(x, _f64(sw[: fs * d].view(fs, d)), _f64(sw[fs * d: 2 * fs * d].view(fs, d)),
                     _f64(sw[2 * fs * d:].view(d, fs)))
    return y, sel, mask


def _rel_err(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return np.abs(a - b).max() / max(np.abs(b).max(), 1e-30)


# ------------------------------------------------------------------------- top-k


def test_topk_tie_rule_golden():
    with open(os.path.join(GOLDEN, "topk_tie_rule.txt")) as fh:
        rows = [l.strip() for l in fh if l.strip() and not l.startswith("#")]
    for row in rows:
        lhs, rhs = row.split("|")
        logits = torch.tensor([[float(v) for v in lhs.split()]], dtype=torch.float32)
        want = [int(v) for v in rhs.split()]
        idx, _, _ = oracle.topk(logits, 2)
        assert idx[0].tolist() == want, row


@pytest.mark.parametrize("E,k", [(8, 2), (16, 4), (128, 8), (5, 5), (64, 1)])
def test_topk_brute_force_with_ties(E, k):
    T = 257
    v = inputgen.fill_normal(torch.empty(T * E), 0, 40 + E, 1.0)
    logits = (torch.round(v * 4) / 4).view(T, E)  # coarse grid: many exact ties
    idx, _, gap = oracle.topk(logits, k)
    assert np.array_equal(idx.numpy(), _ref_select(logits.numpy(), k))
    # each token has k distinct experts
    for t in range(T):
        assert len(set(idx[t].tolist())) == k
    if k < E:
        srt = -np.sort(-logits.numpy(), axis=1)
        assert np.allclose(gap.numpy(), srt[:, k - 1] - srt[:, k])


# ------------------------------------------------------------------------- weights


def test_weights_k_equals_E_is_textbook_softmax():
    T, E = 33, 6
    logits = inputgen.fill_normal(torch.empty(T * E), 1, 5, 2.0).view(T, E)
    idx, w, _ = oracle.topk(logits, E)
    sm = scipy.special.softmax(logits.numpy().astype(np.float64), axis=1)
    assert np.allclose(w.numpy(), np.take_along_axis(sm, idx.numpy().astype(np.int64), 1), rtol=1e-6, atol=0)


def test_weights_k2_closed_form_logistic():
    T, E = 100, 8
    logits = inputgen.fill_normal(torch.empty(T * E), 2, 6, 1.5).view(T, E)
    idx, w, _ = oracle.topk(logits, 2)
    l = logits.numpy().astype(np.float64)
    l0 = l[np.arange(T), idx[:, 0].numpy()]
    l1 = l[np.arange(T), idx[:, 1].numpy()]
    assert np.allclose(w[:, 0].numpy(), 1.0 / (1.0 + np.exp(l1 - l0)), rtol=1e-6, atol=0)
    assert np.allclose(w[:, 1].numpy(), 1.0 / (1.0 + np.exp(l0 - l1)), rtol=1e-6, atol=0)


def test_weights_k1_is_one_and_invariants():
    T, E = 50, 16
    logits = inputgen.fill_normal(torch.empty(T * E), 3, 7, 3.0).view(T, E)
    _, w1, _ = oracle.topk(logits, 1)
    assert torch.all(w1 == 1.0)
    for k in (2, 3, 8):
        _, w, _ = oracle.topk(logits, k)
        assert torch.all(w >= 0)
        assert torch.all((w.double().sum(1) - 1).abs() <= 1e-6)
        assert torch.all(w[:, :-1] >= w[:, 1:])  # slot order follows the logits


def test_weights_for_other_selection_matches_softmax_subset():
    T, E, k = 20, 8, 3
    logits = inputgen.fill_normal(torch.empty(T * E), 4, 8, 1.0).view(T, E)
    idx = torch.tensor([[(t + j * 3) % E for j in range(k)] for t in range(T)], dtype=torch.int32)
    w = oracle.weights_for(logits, idx)
    l = logits.numpy().astype(np.float64)
    for t in range(T):
        sub = scipy.special.softmax(l[t, idx[t].numpy()])
        assert np.allclose(w[t].numpy(), sub, rtol=1e-6, atol=0)


# ------------------------------------------------------------------------- router


@pytest.mark.parametrize("act", [inputgen.F32, inputgen.BF16])
def test_router_logits_vs_float64_matmul(act):
    wl = inputgen.custom("r", T=37, d=96, E=12, k=2, f=8, act=act, wdt=act)
    p = inputgen.make_problem(wl, seed=1)
    b = inputgen.fill_normal(torch.empty(12), 1, 77, 0.3)
    got = oracle.router_logits(p.x, p.router_w, b)
    want = _f64(p.x) @ _f64(p.router_w).T + _f64(b)
    assert got.shape == (37, 12)
    assert _rel_err(got.numpy(), want) < 1e-6
    # without bias
    got0 = oracle.router_logits(p.x, p.router_w, None)
    assert _rel_err(got0.numpy(), _f64(p.x) @ _f64(p.router_w).T) < 1e-6


@pytest.mark.parametrize("act", [inputgen.F32, inputgen.BF16])
def test_router_clamp_vs_clipped_float64_matmul(act):
    # biases far outside [-50, 50] on some experts: the clamped logits are the float64 matmul
    # clipped to [-50, 50], exactly +-50 where it bites and untouched elsewhere
    wl = inputgen.custom("rc", T=29, d=64, E=10, k=2, f=8, act=act, wdt=act)
    p = inputgen.make_problem(wl, seed=5)
    b = torch.zeros(10)
    b[2], b[7], b[9] = 80.0, -90.0, 49.5
    got = oracle.router_logits(p.x, p.router_w, b, oracle.ROUTER_CLAMP).numpy()
    raw = _f64(p.x) @ _f64(p.router_w).T + _f64(b)
    assert _rel_err(got, np.clip(raw, -50.0, 50.0)) < 1e-6
    assert np.all(got[:, 2] == 50.0) and np.all(got[:, 7] == -50.0)
    assert np.all(got <= 50.0) and np.all(got >= -50.0)
    # some tokens push expert 9 over 50 and some do not (both sides of the clip are exercised)
    assert 0 < int((got[:, 9] == 50.0).sum()) < 29
    unclipped = np.abs(raw) < 50.0
    assert _rel_err(got[unclipped], raw[unclipped]) < 1e-6
    assert np.array_equal(oracle.router_logits(p.x, p.router_w, b).numpy() == 50.0, np.zeros_like(got, bool))


def test_clamp_makes_large_logits_tie_and_lower_index_wins():
    # logits 70, 60, 55 on experts 5, 3, 1: unclamped the order is 5, 3; clamped all three are
    # 50 and the tie rule keeps the two lowest indices, 1 then 3
    wl = inputgen.custom("rt", T=4, d=64, E=8, k=2, f=8, act=inputgen.F32, wdt=inputgen.F32)
    p = inputgen.make_problem(wl, seed=6)
    x = torch.zeros_like(p.x)  # logits = bias exactly
    b = torch.zeros(8)
    b[5], b[3], b[1] = 70.0, 60.0, 55.0
    l0 = oracle.router_logits(x, p.router_w, b)
    l1 = oracle.router_logits(x, p.router_w, b, oracle.ROUTER_CLAMP)
    i0, w0, _ = oracle.topk(l0, 2)
    i1, w1, _ = oracle.topk(l1, 2, oracle.ROUTER_CLAMP)
    assert i0.tolist() == [[5, 3]] * 4
    assert i1.tolist() == [[1, 3]] * 4
    assert torch.allclose(w0, torch.tensor([[1 / (1 + math.exp(-10)), 1 / (1 + math.exp(10))]] * 4))
    assert torch.all(w1 == 0.5)  # equal logits, equal weights
    _, w3, _ = oracle.topk(l1, 2, oracle.ROUTER_CLAMP | oracle.ROUTER_RAW)
    assert torch.all(w3 == 50.0)


@pytest.mark.parametrize("k", [1, 2, 4])
def test_raw_weights_are_the_chosen_logits(k):
    T, E = 40, 12
    logits = inputgen.fill_normal(torch.empty(T * E), 9, 11, 2.0).view(T, E)
    idx0, w0, gap0 = oracle.topk(logits, k)
    idx, w, gap = oracle.topk(logits, k, oracle.ROUTER_RAW)
    assert torch.equal(idx, idx0) and torch.equal(gap, gap0)  # selection unchanged
    assert torch.equal(w, torch.gather(logits, 1, idx.long()))
    assert torch.all(w[:, :-1] >= w[:, 1:])
    # weights_for on an arbitrary selection agrees
    other = torch.tensor([[(t + 5 * j) % E for j in range(k)] for t in range(T)], dtype=torch.int32)
    assert torch.equal(oracle.weights_for(logits, other, oracle.ROUTER_RAW), torch.gather(logits, 1, other.long()))
    with pytest.raises(RuntimeError):
        oracle.topk(logits, k, 4)  # unknown variant bit


# ------------------------------------------------------------------------- grouping


@pytest.mark.parametrize("T,E,k", [(1, 4, 2), (300, 8, 2), (129, 128, 4), (64, 3, 3)])
def test_group_is_stable_counting_sort(T, E, k):
    logits = inputgen.fill_normal(torch.empty(T * E), 5, T + E, 1.0).view(T, E)
    idx, _, _ = oracle.topk(logits, k)
    counts, offsets, src, dst = oracle.group(idx, E)
    flat = idx.numpy().reshape(-1).astype(np.int64)
    assert np.array_equal(counts.numpy(), np.bincount(flat, minlength=E))
    assert offsets[0] == 0 and offsets[-1] == T * k
    assert np.all(np.diff(offsets.numpy()) == counts.numpy())
    # a stable sort of the flattened (t, j) assignments by expert gives the same rows
    perm = np.argsort(flat, kind="stable")
    assert np.array_equal(src.numpy(), perm // k)
    # dst is the inverse permutation and lands inside the right expert's range
    assert np.array_equal(np.sort(dst.numpy().reshape(-1)), np.arange(T * k))
    for t in range(T):
        for j in range(k):
            r = int(dst[t, j])
            e = int(idx[t, j])
            assert src[r] == t and offsets[e] <= r < offsets[e + 1]
    # each token appears exactly k times
    assert np.array_equal(np.bincount(src.numpy(), minlength=T), np.full(T, k))


# ------------------------------------------------------------------------- expert FFN / layer


@pytest.mark.parametrize("act", [inputgen.F32, inputgen.BF16])
def test_single_expert_is_dense_swiglu(act):
    # E = 1, k = 1: the layer is one dense SwiGLU FFN (torch float64, F.silu)
    wl = inputgen.custom("dense", T=9, d=48, E=1, k=1, f=80, act=act, wdt=act)
    p = inputgen.make_problem(wl, seed=2)
    out = oracle.moe_forward(p.x, p.router_w, p.router_b, 1, p.expert_w, p.expert_stride, wl.f)
    assert torch.all(out["w"] == 1.0) and torch.all(out["idx"] == 0)
    x = p.x.to(torch.float64)
    w = p.expert_w.to(torch.float64)
    f, d = wl.f, wl.d
    w1, w3, w2 = w[: f * d].view(f, d), w[f * d: 2 * f * d].view(f, d), w[2 * f * d: 3 * f * d].view(d, f)
    want = (F.silu(x @ w1.T) * (x @ w3.T)) @ w2.T
    assert _rel_err(out["y"].numpy(), want.numpy()) < 2e-6


@pytest.mark.parametrize("case", ["f32", "bf16", "bf16_shared", "bf16_bias", "i8", "bf16_clamp", "f32_raw",
                                  "i8_clamp_raw", "i4"])
def test_layer_equals_brute_force_dense(case):
    kw = dict(T=23, d=64, E=6, k=2, f=96)
    flags = 0
    if case == "bf16_clamp":
        # three experts beyond 50: clamped, they tie and the two lowest indices win
        wl = inputgen.custom(case, bias=((5, 70.0), (3, 60.0), (1, 55.0)), **kw)
        flags = oracle.ROUTER_CLAMP
    elif case == "f32_raw":
        wl = inputgen.custom(case, act=inputgen.F32, wdt=inputgen.F32, **dict(kw, k=3))
        flags = oracle.ROUTER_RAW
    elif case == "i8_clamp_raw":
        wl = inputgen.custom(case, act=inputgen.BF16, wdt=inputgen.I8, bias=((4, 49.5),), **kw)
        flags = oracle.ROUTER_CLAMP | oracle.ROUTER_RAW
    elif case == "f32":
        wl = inputgen.custom(case, act=inputgen.F32, wdt=inputgen.F32, **kw)
    elif case == "bf16":
        wl = inputgen.custom(case, **kw)
    elif case == "bf16_shared":
        wl = inputgen.custom(case, fs=40, **dict(kw, k=3))
    elif case == "bf16_bias":
        wl = inputgen.custom(case, bias=((1, 2.0), (4, -1.0)), **kw)
    elif case == "i4":  # int4 needs d and f multiples of the 128-wide scale group
        wl = inputgen.custom(case, act=inputgen.BF16, wdt=inputgen.I4, **dict(kw, d=256, f=128))
    else:
        wl = inputgen.custom(case, act=inputgen.BF16, wdt=inputgen.I8, **kw)
    p = inputgen.make_problem(wl, seed=3)
    out = oracle.moe_forward(p.x, p.router_w, p.router_b, wl.k, p.expert_w, p.expert_stride, wl.f,
                             p.expert_scales, p.shared_w, wl.fs, flags)
    y, sel, mask = _dense_layer(p, flags)
    assert np.array_equal(out["idx"].numpy(), sel)
    if case == "bf16_clamp":
        assert out["idx"].tolist() == [[1, 3]] * wl.T
    if case == "i8_clamp_raw":
        assert torch.all(out["idx"][:, 0] == 4) and torch.all(out["w"][:, 0] <= 50.0)
        assert 0 < int((out["w"][:, 0] == 50.0).sum()) < wl.T
    assert _rel_err(out["y"].numpy(), y) < 2e-6
    # the sampled path agrees bit for bit with the whole-layer path
    toks = [0, 5, 22, 11]
    ys = oracle.combine(p.x, out["idx"], out["w"], p.expert_w, p.expert_stride, wl.f, p.expert_scales,
                        p.shared_w, wl.fs, toks)
    assert torch.equal(ys, out["y"][toks])


def test_int8_dequant_identity():
    # the oracle on (s, q) equals the oracle on float32 weights s[o] * q[o][i]
    wl = inputgen.custom("i8", T=11, d=32, E=3, k=2, f=48, act=inputgen.BF16, wdt=inputgen.I8)
    p = inputgen.make_problem(wl, seed=4)
    f, d = wl.f, wl.d
    deq = torch.zeros(3 * p.expert_stride, dtype=torch.float32)
    for e in range(3):
        s = p.expert_scales[e * (2 * f + d):(e + 1) * (2 * f + d)]
        q = p.expert_w[e * p.expert_stride: e * p.expert_stride + 3 * f * d].to(torch.float32)
        rows = torch.cat([s[:f].repeat_interleave(d), s[f:2 * f].repeat_interleave(d), s[2 * f:].repeat_interleave(f)])
        deq[e * p.expert_stride: e * p.expert_stride + 3 * f * d] = rows * q
    a = oracle.moe_forward(p.x, p.router_w, None, 2, p.expert_w, p.expert_stride, f, p.expert_scales)
    b = oracle.moe_forward(p.x, p.router_w, None, 2, deq, p.expert_stride, f)
    assert torch.equal(a["y"], b["y"])


def _golden_int4():
    rows = []
    with open(os.path.join(GOLDEN, "int4_packing.txt")) as fh:
        for line in fh:
            line = line.split("#")[0].strip()
            if line:
                word, *vals = line.split()
                rows.append((int(word, 16), [int(v) for v in vals]))
    return rows


def test_int4_packing_golden():
    # the hand-worked words of tests/golden/int4_packing.txt, read back element by element by the
    # oracle (one 128-element row, unit scale), and written by the generator's packer
    rows = _golden_int4()
    assert len(rows) >= 4
    for word, vals in rows:
        buf = torch.zeros(64, dtype=torch.uint8)
        buf[:4] = torch.tensor(list(word.to_bytes(4, "little")), dtype=torch.uint8)
        one = torch.ones(1, dtype=torch.float32)
        got = [oracle.weight_element(buf, 0, 1, 128, 0, i, one) for i in range(8)]
        assert got == [float(v) for v in vals], hex(word)
        assert all(oracle.weight_element(buf, 0, 1, 128, 0, i, one) == 0.0 for i in range(8, 128))
        packed = inputgen.pack_int4(torch.tensor(vals, dtype=torch.int8))
        assert packed.tolist() == list(word.to_bytes(4, "little")), hex(word)
        assert _unpack_int4(packed).tolist() == vals


def test_int4_group_scales_apply_per_128_inputs():
    # W[o][i] = s[i // 128][o] * q[o][i] (group-major scales): distinct power-of-two scales per
    # (group, row) show which one applies
    rows, cols = 3, 384
    q = torch.tensor([((o * 7 + i) % 15) - 7 for o in range(rows) for i in range(cols)], dtype=torch.int8)
    buf = inputgen.pack_int4(q)
    s = torch.tensor([2.0 ** -(o * 3 + g) for g in range(cols // 128) for o in range(rows)], dtype=torch.float32)
    for o in range(rows):
        for i in (0, 1, 127, 128, 255, 256, 383):
            want = float(q[o * cols + i]) * 2.0 ** -(o * 3 + i // 128)
            assert oracle.weight_element(buf, 0, rows, cols, o, i, s) == want
    # an offset base (the second matrix of an expert) shifts the element index, not the scales
    assert oracle.weight_element(buf, cols, 2, cols, 1, 5, s[:2]) == float(q[2 * cols + 5]) * 2.0 ** -(3 + 0)


def test_int4_dequant_identity():
    # the oracle on (s, q) equals the oracle on float32 weights s[o][i // 128] * q[o][i]
    wl = inputgen.custom("i4", T=7, d=256, E=3, k=2, f=256, act=inputgen.BF16, wdt=inputgen.I4)
    p = inputgen.make_problem(wl, seed=6)
    f, d = wl.f, wl.d
    deq = torch.zeros(3 * p.expert_stride, dtype=torch.float32)
    for e in range(3):
        w1, w3, w2 = _int4_mats(p, e)
        deq[e * p.expert_stride: e * p.expert_stride + 3 * f * d] = torch.cat([w1.reshape(-1), w3.reshape(-1),
                                                                             w2.reshape(-1)])
    a = oracle.moe_forward(p.x, p.router_w, None, 2, p.expert_w, p.expert_stride, f, p.expert_scales)
    b = oracle.moe_forward(p.x, p.router_w, None, 2, deq, p.expert_stride, f)
    assert torch.equal(a["y"], b["y"])
    assert torch.equal(a["idx"], b["idx"])


def test_tiny_f32_workload_float64_restatement():
    # the full 64-token fp32 workload against an independent float64 torch restatement
    wl = inputgen.WORKLOADS["tiny_f32"]
    p = inputgen.make_problem(wl, seed=0)
    out = oracle.problem_forward(p)
    y, sel, _ = _dense_layer(p)
    assert np.array_equal(out["idx"].numpy(), sel)
    assert _rel_err(out["y"].numpy(), y) < 2e-6


def test_empty_and_nonfinite():
    wl = inputgen.custom("z", T=0, d=16, E=4, k=2, f=16)
    p = inputgen.make_problem(wl, seed=0)
    out = oracle.moe_forward(p.x, p.router_w, None, 2, p.expert_w, p.expert_stride, 16)
    assert out["y"].numel() == 0
    wl = inputgen.custom("nf", T=3, d=16, E=4, k=2, f=16, act=inputgen.F32, wdt=inputgen.F32)
    p = inputgen.make_problem(wl, seed=0)
    p.x[1, 3] = float("nan")
    with pytest.raises(RuntimeError):
        oracle.moe_forward(p.x, p.router_w, None, 2, p.expert_w, p.expert_stride, 16)


def test_bad_arguments_rejected():
    logits = torch.zeros(2, 4)
    with pytest.raises(RuntimeError):
        oracle.topk(logits, 5)  # k > E
    with pytest.raises(RuntimeError):
        oracle.group(torch.tensor([[0, 7]], dtype=torch.int32), 4)  # expert id out of range


@pytest.mark.slow
def test_skewed_workload_histogram():
    # +4 bias on experts 0/1 concentrates almost every assignment there; the variant with
    # -30 on experts 12..15 leaves those four experts with exactly zero rows.
    for name in ("skewed_bf16", "skewed_empty_bf16"):
        wl = inputgen.WORKLOADS[name]
        p = inputgen.make_problem(wl, seed=0)
        logits = oracle.router_logits(p.x, p.router_w, p.router_b)
        idx, _, _ = oracle.topk(logits, wl.k)
        counts, _, _, _ = oracle.group(idx, wl.E)
        frac01 = (counts[0] + counts[1]).item() / (wl.T * wl.k)
        assert frac01 > 0.9
        if name == "skewed_empty_bf16":
            assert counts[12:].sum().item() == 0
