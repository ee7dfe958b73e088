"""Helpers for the GPU parity tests: run the C ABI on a generated problem and compare it
with the oracle under the near-tie protocol.

Near-tie protocol: a token is near-tied when the oracle's k-th and (k+1)-th logits, or two
consecutive chosen logits, differ by less than 1e-4.  Top-k ids must match bit for bit on
every other token.  On near-tied tokens the GPU's choice is accepted if it is a valid top-k
under a 1e-4 slack; the oracle is then re-run with the GPU's ids substituted on exactly those
tokens, after which counts, offsets and the permutation must match bit for bit and y within
the tolerance of the dtype.
"""
from __future__ import annotations

import numpy as np
import torch

import inputgen
import oracle
import sparse_expert_ffn_router_b200 as colibri

NEAR_TIE = 1e-4
TOL = {inputgen.F32: 1e-4, inputgen.BF16: 2e-2, inputgen.I8: 5e-2, inputgen.I4: 5e-2}


def tolerance(wl) -> float:
    if wl.wdt in (inputgen.I8, inputgen.I4):  # quantised-weight configs
        return TOL[wl.wdt]
    return TOL[wl.act]


def to_device(p, dev="cuda"):
    return dict(
        x=p.x.to(dev), router_w=p.router_w.to(dev),
        router_b=None if p.router_b is None else p.router_b.to(dev),
        expert_w=p.expert_w.to(dev),
        expert_scales=None if p.expert_scales is None else p.expert_scales.to(dev),
        shared_w=None if p.shared_w is None else p.shared_w.to(dev))


def make_layer(wl, max_tokens=None, router_flags=0):
    return colibri.MoELayer(wl.d, wl.f, wl.E, wl.k, wl.fs, wl.act, wl.wdt,
                            max_tokens=max_tokens or max(wl.T, 1), device_id=0, router_flags=router_flags)


def run_gpu(p, layer=None, dev_inputs=None, routed=None, router_flags=0):
    """Run one forward through the C ABI; returns y (host, float32) and the routing state."""
    wl = p.wl
    own = layer is None
    layer = layer or make_layer(wl, router_flags=router_flags)
    assert layer.expert_stride == p.expert_stride
    t = dev_inputs or to_device(p)
    y = torch.empty(wl.T, wl.d, dtype=p.x.dtype, device="cuda")
    if routed is None:
        layer.forward(t["x"], t["router_w"], t["router_b"], t["expert_w"], y, t["expert_scales"], t["shared_w"])
    else:
        idx, w = routed
        layer.forward_routed(t["x"], idx.cuda(), w.cuda(), t["expert_w"], y, t["expert_scales"], t["shared_w"])
    r = dict(
        idx=torch.empty(wl.T, wl.k, dtype=torch.int32, device="cuda"),
        w=torch.empty(wl.T, wl.k, dtype=torch.float32, device="cuda"),
        counts=torch.empty(wl.E, dtype=torch.int32, device="cuda"),
        offsets=torch.empty(wl.E + 1, dtype=torch.int32, device="cuda"),
        src_row=torch.empty(wl.T * wl.k, dtype=torch.int32, device="cuda"),
        dst_row=torch.empty(wl.T, wl.k, dtype=torch.int32, device="cuda"))
    if wl.T > 0:
        layer.routing(topk_idx=r["idx"], topk_w=r["w"], counts=r["counts"], offsets=r["offsets"],
                      src_row=r["src_row"], dst_row=r["dst_row"])
    layer.sync_status()
    out = {k: v.cpu() for k, v in r.items()}
    out["y"] = y.float().cpu()
    if own:
        layer.close()
    return out


def near_tie_tokens(logits: torch.Tensor, idx: torch.Tensor, gap: torch.Tensor):
    """Tokens whose selection or slot order is decided by a logit difference < 1e-4."""
    T, k = idx.shape
    l = logits.numpy().astype(np.float64)
    sel = np.take_along_axis(l, idx.numpy().astype(np.int64), 1)
    slot_gap = (sel[:, :-1] - sel[:, 1:]).min(axis=1) if k > 1 else np.full(T, np.inf)
    return np.nonzero((gap.numpy() < NEAR_TIE) | (slot_gap < NEAR_TIE))[0]


def valid_topk_under_slack(logits_row: np.ndarray, chosen: np.ndarray, k: int) -> bool:
    """The chosen ids are distinct and no unchosen logit beats a chosen one by >= 1e-4."""
    if len(set(chosen.tolist())) != k:
        return False
    mask = np.ones(len(logits_row), bool)
    mask[chosen] = False
    if not mask.any():
        return True
    return logits_row[mask].max() - logits_row[chosen].min() < NEAR_TIE


def compare_routing(p, ref, gpu, flags=0):
    """Apply the near-tie protocol; returns (routing used for the oracle y, n_near_tie).
    ``flags``: the router variant both sides ran (the oracle's logits are already clamped)."""
    wl = p.wl
    logits, idx_o = ref["logits"], ref["idx"]
    near = near_tie_tokens(logits, idx_o, ref["gap"])
    idx_g = gpu["idx"]
    far = np.ones(wl.T, bool)
    far[near] = False
    assert torch.equal(idx_g[torch.from_numpy(far)], idx_o[torch.from_numpy(far)]), "top-k ids differ on a clear token"
    idx_use = idx_o.clone()
    for t in near:
        g = idx_g[t].numpy().astype(np.int64)
        assert valid_topk_under_slack(logits[t].numpy().astype(np.float64), g, wl.k), f"token {t}"
        idx_use[t] = idx_g[t]
    w_use = oracle.weights_for(logits, idx_use, flags)
    # softmax weights lie in [0, 1]; raw-logit weights are compared relative to their size
    assert ((gpu["w"] - w_use).abs() <= 2e-5 * w_use.abs().clamp(min=1.0)).all(), "routing weights differ"
    counts, offsets, src, dst = oracle.group(idx_use, wl.E)
    assert torch.equal(gpu["counts"], counts)
    assert torch.equal(gpu["offsets"], offsets)
    assert torch.equal(gpu["src_row"], src)
    assert torch.equal(gpu["dst_row"], dst)
    return idx_use, w_use, len(near)


def check_y(p, y_gpu_rows, y_ref_rows, tol=None):
    tol = tolerance(p.wl) if tol is None else tol
    ref = y_ref_rows.double()
    err = (y_gpu_rows.double() - ref).abs().max().item()
    scale = ref.abs().max().item()
    assert np.isfinite(err)
    assert err <= tol * scale, f"max abs err {err:.3e} > {tol} x max|ref| {scale:.3e}"
    return err / max(scale, 1e-30)


def parity(p, tokens=None, layer=None, dev_inputs=None, flags=0):
    """Full protocol: routing on every token, y on `tokens` (default all).  ``flags`` selects
    the router variant on both sides."""
    wl = p.wl
    logits = oracle.router_logits(p.x, p.router_w, p.router_b, flags)
    idx, w, gap = oracle.topk(logits, wl.k, flags)
    ref = dict(logits=logits, idx=idx, w=w, gap=gap)
    gpu = run_gpu(p, layer=layer, dev_inputs=dev_inputs, router_flags=flags)
    idx_use, w_use, n_near = compare_routing(p, ref, gpu, flags)
    toks = list(range(wl.T)) if tokens is None else list(tokens)
    y_ref = oracle.combine(p.x, idx_use, w_use, p.expert_w, p.expert_stride, wl.f, p.expert_scales, p.shared_w,
                           wl.fs, toks)
    rel = check_y(p, gpu["y"][toks], y_ref)
    return dict(rel_err=rel, near_ties=n_near, counts=gpu["counts"], idx=gpu["idx"], ref_idx=idx)


def sample_tokens(T: int, n: int):
    return inputgen.sample_tokens(T, n)
