"""Python marshalling for the CPU oracle (``colibri_oracle.cpp``).

TEST INFRASTRUCTURE ONLY: imported by the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg.  The product library never imports or links this module.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

F32, BF16, I8, I4 = 0, 1, 2, 3
# int4 weights travel as packed bytes (two elements per uint8)
_CODE = {torch.float32: F32, torch.bfloat16: BF16, torch.int8: I8, torch.uint8: I4}


def build() -> str:
    """Compile liboracle.so in place: plain g++, single-threaded, no fast-math, no FMA contraction."""
    src = os.path.join(_HERE, "colibri_oracle.cpp")
    if (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-o", _LIB_PATH, src])
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            build()
        lib = ctypes.CDLL(_LIB_PATH)
        vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        lib.oracle_router_logits.argtypes = [vp, i32, i32, i32, vp, vp, i32, i32, vp]
        lib.oracle_weights_for.argtypes = [vp, i32, i32, i32, vp, i32, vp]
        lib.oracle_topk.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp]
        lib.oracle_group.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp]
        lib.oracle_expert_row.argtypes = [vp, i32, i32, i32, vp, i32, i64, i32, vp, i32, vp]
        lib.oracle_combine.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, i32, i64, i32, vp, vp,
                                       i32, vp, i32, vp]
        lib.oracle_moe_forward.argtypes = [vp, i32, i32, i32, vp, vp, i32, i32, i32, vp, i32, i64, i32,
                                           vp, vp, i32] + [vp] * 8
        lib.oracle_weight_element.argtypes = [vp, i32, i64, i64, i64, i64, i64, vp, vp]
        for n in ("oracle_router_logits", "oracle_weights_for", "oracle_topk", "oracle_group",
                  "oracle_expert_row", "oracle_combine", "oracle_moe_forward", "oracle_weight_element"):
            getattr(lib, n).restype = ctypes.c_int
        _lib = lib
    return _lib


ROUTER_CLAMP, ROUTER_RAW = 1, 2  # router variants (logit clamp to [-50, 50]; raw-logit weights)


def _ptr(t):
    if t is None:
        return None
    assert t.device.type == "cpu" and t.is_contiguous(), "oracle takes contiguous host tensors"
    return t.data_ptr()


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def router_logits(x: torch.Tensor, router_w: torch.Tensor, router_b: Optional[torch.Tensor],
                  flags: int = 0) -> torch.Tensor:
    """Logits [T, E] float32; ``flags`` & ROUTER_CLAMP limits them to [-50, 50]."""
    T, d = x.shape
    E = router_w.shape[0]
    out = torch.empty(T, E, dtype=torch.float32)
    _check(_load().oracle_router_logits(_ptr(x), _CODE[x.dtype], T, d, _ptr(router_w), _ptr(router_b), E,
                                        flags, _ptr(out)), "router_logits")
    return out


def topk(logits: torch.Tensor, k: int, flags: int = 0):
    """(idx [T,k] int32, w [T,k] f32, gap [T] f32) with the oracle's selection rule; ``flags`` &
    ROUTER_RAW makes the weights the chosen logits."""
    T, E = logits.shape
    idx = torch.empty(T, k, dtype=torch.int32)
    w = torch.empty(T, k, dtype=torch.float32)
    gap = torch.empty(T, dtype=torch.float32)
    _check(_load().oracle_topk(_ptr(logits.contiguous()), T, E, k, flags, _ptr(idx), _ptr(w), _ptr(gap)),
           "topk")
    return idx, w, gap


def weights_for(logits: torch.Tensor, idx: torch.Tensor, flags: int = 0) -> torch.Tensor:
    T, E = logits.shape
    k = idx.shape[1]
    w = torch.empty(T, k, dtype=torch.float32)
    _check(_load().oracle_weights_for(_ptr(logits.contiguous()), T, E, k, _ptr(idx.contiguous()), flags,
                                      _ptr(w)), "weights_for")
    return w


def group(idx: torch.Tensor, E: int):
    """(counts [E], offsets [E+1], src_row [T*k], dst_row [T,k]) all int32."""
    T, k = idx.shape
    counts = torch.empty(E, dtype=torch.int32)
    offsets = torch.empty(E + 1, dtype=torch.int32)
    src = torch.empty(T * k, dtype=torch.int32)
    dst = torch.empty(T, k, dtype=torch.int32)
    _check(_load().oracle_group(_ptr(idx.contiguous()), T, k, E, _ptr(counts), _ptr(offsets), _ptr(src),
                                _ptr(dst)), "group")
    return counts, offsets, src, dst


def expert_row(x: torch.Tensor, t: int, expert_w: torch.Tensor, stride: int, f: int,
               scales: Optional[torch.Tensor], e: int) -> torch.Tensor:
    d = x.shape[1]
    y = torch.empty(d, dtype=torch.float32)
    _check(_load().oracle_expert_row(_ptr(x), _CODE[x.dtype], d, t, _ptr(expert_w), _CODE[expert_w.dtype],
                                     stride, f, _ptr(scales), e, _ptr(y)), "expert_row")
    return y


def combine(x: torch.Tensor, idx: torch.Tensor, w: torch.Tensor, expert_w: torch.Tensor, stride: int, f: int,
            scales: Optional[torch.Tensor], shared_w: Optional[torch.Tensor], fs: int,
            tokens: Sequence[int]) -> torch.Tensor:
    """Layer output rows y[tokens] (float32 [len(tokens), d]) for the given routing."""
    T, d = x.shape
    k = idx.shape[1]
    tok = torch.tensor(list(tokens), dtype=torch.int32)
    y = torch.empty(len(tok), d, dtype=torch.float32)
    _check(_load().oracle_combine(_ptr(x), _CODE[x.dtype], T, d, k, _ptr(idx.contiguous()), _ptr(w.contiguous()),
                                  _ptr(expert_w), _CODE[expert_w.dtype], stride, f, _ptr(scales),
                                  _ptr(shared_w), fs, _ptr(tok), len(tok), _ptr(y)), "combine")
    return y


def moe_forward(x, router_w, router_b, k, expert_w, stride, f, scales=None, shared_w=None, fs=0, flags=0):
    """Whole layer on the host.  Returns a dict of every intermediate the GPU path exposes."""
    T, d = x.shape
    E = router_w.shape[0]
    out = dict(
        logits=torch.empty(T, E, dtype=torch.float32),
        idx=torch.empty(T, k, dtype=torch.int32),
        w=torch.empty(T, k, dtype=torch.float32),
        counts=torch.empty(E, dtype=torch.int32),
        offsets=torch.empty(E + 1, dtype=torch.int32),
        src_row=torch.empty(T * k, dtype=torch.int32),
        dst_row=torch.empty(T, k, dtype=torch.int32),
        y=torch.empty(T, d, dtype=torch.float32),
    )
    rc = _load().oracle_moe_forward(
        _ptr(x), _CODE[x.dtype], T, d, _ptr(router_w), _ptr(router_b), E, k, flags, _ptr(expert_w),
        _CODE[expert_w.dtype], stride, f, _ptr(scales), _ptr(shared_w), fs,
        *[_ptr(out[n]) for n in ("logits", "idx", "w", "counts", "offsets", "src_row", "dst_row", "y")])
    _check(rc, "moe_forward")
    return out


def weight_element(w: torch.Tensor, base: int, rows: int, cols: int, o: int, i: int,
                   scale: Optional[torch.Tensor] = None) -> float:
    """W[o][i] of the [rows, cols] matrix at element offset `base` of buffer `w` as the oracle
    reads it (int8 / int4: dequantised with the matrix's scales)."""
    out = ctypes.c_double()
    _check(_load().oracle_weight_element(_ptr(w), _CODE[w.dtype], base, rows, cols, o, i, _ptr(scale),
                                         ctypes.byref(out)), "weight_element")
    return out.value


def problem_forward(p, tokens: Optional[Sequence[int]] = None, flags: int = 0):
    """Oracle on an ``inputgen.Problem``: routing for all tokens, y for `tokens` (default: all)."""
    wl = p.wl
    logits = router_logits(p.x, p.router_w, p.router_b, flags)
    idx, w, gap = topk(logits, wl.k, flags)
    counts, offsets, src, dst = group(idx, wl.E)
    toks = list(range(wl.T)) if tokens is None else list(tokens)
    y = combine(p.x, idx, w, p.expert_w, p.expert_stride, wl.f, p.expert_scales, p.shared_w, wl.fs, toks)
    return dict(logits=logits, idx=idx, w=w, gap=gap, counts=counts, offsets=offsets, src_row=src,
                dst_row=dst, y=y, tokens=toks)
