"""colibri_route_noalloc: the Gate and Scatter stages with no device allocation.

Some callers cannot call cudaMalloc -- an engine whose device memory is entirely reserved by its
own allocator, or a latency-critical loop that cannot afford cudaMalloc's implicit
synchronisation.  This entry point serves them: the caller passes every input and output and the
only scratch (per-block expert counts, their bases and an error word) is a file-scope device
array inside the library.

The GPU tests check it, through the C ABI, against the existing entry point (colibri_moe_forward
followed by colibri_get_routing) on calls in a row that reuse the same scratch array with
different sizes, including the largest size the array admits.  The first call of the first test
runs before any context exists in a fresh process, so the entry point must set up everything it
needs by itself.  The file is named to be collected last.
"""
import pytest
import torch

import inputgen
import sparse_expert_ffn_router_b200 as colibri
from tests import gpu_harness as H

W_TOL = 2e-5  # routing-weight tolerance used by the parity tests
LIMIT = 32768  # ceil(T / 256) * E the scratch array admits


def test_route_noalloc_rejects_sizes_beyond_its_scratch():
    # ceil(T / 256) * E > 32768 is refused before anything touches the device
    for T, E in ((256 * 129, 256), (256 * 128 + 1, 256), (256 * 2049, 16)):
        with pytest.raises(colibri.ColibriError) as ei:
            colibri.colibri_route_noalloc(16, colibri.COLIBRI_BF16, T, 256, 16, None, E, 2,
                                          16, 16, 16, 16, 16, 16, 16)
        assert ei.value.status == -1
        assert "32768" in colibri.colibri_last_error()


def _noalloc(p):
    wl = p.wl
    dev = "cuda"
    x = p.x.to(dev)
    rw = p.router_w.to(dev)
    rb = None if p.router_b is None else p.router_b.to(dev)
    i32 = dict(dtype=torch.int32, device=dev)
    out = dict(
        idx=torch.full((wl.T, wl.k), -7, **i32),
        w=torch.full((wl.T, wl.k), -7.0, dtype=torch.float32, device=dev),
        counts=torch.full((wl.E,), -7, **i32),
        offsets=torch.full((wl.E + 1,), -7, **i32),
        src_row=torch.full((wl.T * wl.k,), -7, **i32),
        dst_row=torch.full((wl.T, wl.k), -7, **i32),
        Xp=torch.full((wl.T * wl.k, wl.d), -7.0, dtype=x.dtype, device=dev),
    )
    colibri.colibri_route_noalloc(x, wl.act, wl.T, wl.d, rw, rb, wl.E, wl.k, out["idx"], out["w"], out["counts"],
                                  out["offsets"], out["src_row"], out["dst_row"], out["Xp"])
    colibri.colibri_route_noalloc_check()  # synchronises; raises if a device wait gave up
    return {k: v.cpu() for k, v in out.items()}


def _check_against_existing(p, got):
    ref = H.run_gpu(p)  # existing entry point: colibri_moe_forward + colibri_get_routing
    assert torch.equal(got["idx"], ref["idx"])
    assert (got["w"] - ref["w"]).abs().max().item() <= W_TOL
    for k in ("counts", "offsets", "src_row", "dst_row"):
        assert torch.equal(got[k], ref[k]), k
    # grouped rows are the token rows in the existing entry point's order
    assert torch.equal(got["Xp"], p.x[ref["src_row"].long()])


@pytest.mark.gpu
def test_route_noalloc_matches_existing_entry_point_twice():
    cases = [
        # fp32 with E = 256 and T > 64: the router needs ~70 KB of shared memory, which this call
        # must enable by itself (it runs first, before any context exists in a fresh process)
        inputgen.custom("noalloc_f32_maxE", T=100, d=64, E=256, k=8, f=64, act=inputgen.F32, wdt=inputgen.F32),
        inputgen.custom("noalloc_bf16", T=1000, d=256, E=16, k=4, f=64),
        inputgen.custom("noalloc_f32", T=77, d=128, E=8, k=2, f=64, act=inputgen.F32, wdt=inputgen.F32,
                        bias=((3, 1.5),)),
    ]
    probs = [inputgen.make_problem(wl, seed=seed) for seed, wl in enumerate(cases)]
    got = [_noalloc(p) for p in probs]  # calls in a row over the same scratch array
    for p, g in zip(probs, got):
        _check_against_existing(p, g)


@pytest.mark.gpu
def test_route_noalloc_at_its_size_limit():
    # ceil(T / 256) * E == 32768 exactly: every entry of the scratch array's count and base
    # blocks is used; then a smaller call over the same (now dirty) array
    big = inputgen.custom("noalloc_limit", T=256 * 128, d=64, E=256, k=2, f=64)
    assert ((big.T + 255) // 256) * big.E == LIMIT
    small = inputgen.custom("noalloc_after_limit", T=300, d=64, E=256, k=2, f=64)
    for wl, seed in ((big, 3), (small, 4)):
        p = inputgen.make_problem(wl, seed=seed)
        _check_against_existing(p, _noalloc(p))
