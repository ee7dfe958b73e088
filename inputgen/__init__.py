"""Seeded synthetic inputs for the MoE layer forward (shared by tests, bench, smoke).

This module holds no arithmetic of the MoE layer.  It turns (seed, tensor id,
element index) into numbers with the distributions the workloads state, through
the counter-based SplitMix64 + Box-Muller generator in ``inputgen.c`` (see the
header of that file for the exact definition), and lays them out in the buffers
the C ABI expects:

* ``x``          [T, d] row-major, activation dtype
* ``router_w``   [E, d] row-major, activation dtype
* ``router_b``   [E] float32 or None
* ``expert_w``   one buffer; expert e starts at element ``e * expert_stride`` and
                 holds W1[f, d] | W3[f, d] | W2[d, f] (rows are [out, in])
* ``expert_scales`` int8 weights: per expert [f | f | d] float32 (one per output channel);
                 int4 weights: per expert s1[d/128, f] | s3[d/128, f] | s2[f/128, d] float32
                 (one per group of 128 consecutive inputs and output channel, group-major)
* ``shared_w``   W1s[fs, d] | W3s[fs, d] | W2s[d, fs] or None

int4 weights are stored packed, two per byte along the input dimension: element 2j of a row in
the low nibble of byte j, element 2j + 1 in the high nibble, each a two's-complement 4-bit
integer; the buffer is a uint8 tensor and ``expert_stride`` still counts elements (nibbles).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libinputgen.so")
_lib = None

F32, BF16, I8, I4 = 0, 1, 2, 3
_TORCH_DTYPE = {F32: torch.float32, BF16: torch.bfloat16, I8: torch.int8, I4: torch.uint8}
DTYPE_NAMES = {F32: "f32", BF16: "bf16", I8: "i8", I4: "i4"}
I4_GROUP = 128  # inputs per int4 scale group


def build() -> str:
    """Compile libinputgen.so in place (gcc, OpenMP)."""
    src = os.path.join(_HERE, "inputgen.c")
    if (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-o", _LIB_PATH, src, "-lm"])
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            build()
        lib = ctypes.CDLL(_LIB_PATH)
        u64, i64, dbl, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        lib.ig_key.restype = u64
        lib.ig_key.argtypes = [u64, u64]
        lib.ig_raw.restype = u64
        lib.ig_raw.argtypes = [u64, u64]
        for name in ("ig_fill_normal_f32", "ig_fill_normal_bf16"):
            getattr(lib, name).argtypes = [vp, i64, u64, u64, dbl]
            getattr(lib, name).restype = None
        lib.ig_fill_uniform_f32.argtypes = [vp, i64, u64, u64, dbl, dbl]
        lib.ig_fill_uniform_f32.restype = None
        lib.ig_fill_int8.argtypes = [vp, i64, u64, u64, ctypes.c_int, ctypes.c_int]
        lib.ig_fill_int8.restype = None
        lib.ig_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def raw(key: int, i: int) -> int:
    return int(_load().ig_raw(key, i))


def key(seed: int, tensor_id: int) -> int:
    return int(_load().ig_key(seed, tensor_id))


def fill_normal(t: torch.Tensor, seed: int, tensor_id: int, std: float) -> torch.Tensor:
    """Fill a contiguous CPU float32/bfloat16 tensor with std * N(0, 1)."""
    assert t.is_contiguous() and t.device.type == "cpu"
    if t.dtype == torch.float32:
        _load().ig_fill_normal_f32(t.data_ptr(), t.numel(), seed, tensor_id, std)
    elif t.dtype == torch.bfloat16:
        _load().ig_fill_normal_bf16(t.data_ptr(), t.numel(), seed, tensor_id, std)
    else:
        raise TypeError(t.dtype)
    return t


def fill_uniform(t: torch.Tensor, seed: int, tensor_id: int, lo: float, hi: float) -> torch.Tensor:
    assert t.is_contiguous() and t.device.type == "cpu" and t.dtype == torch.float32
    _load().ig_fill_uniform_f32(t.data_ptr(), t.numel(), seed, tensor_id, lo, hi)
    return t


def fill_int(t: torch.Tensor, seed: int, tensor_id: int, lo: int, hi: int) -> torch.Tensor:
    assert t.is_contiguous() and t.device.type == "cpu" and t.dtype == torch.int8
    _load().ig_fill_int8(t.data_ptr(), t.numel(), seed, tensor_id, lo, hi)
    return t


def max_threads() -> int:
    return int(_load().ig_max_threads())


# ----------------------------------------------------------------------------------------
# Workloads: sizes and distributions only.
# ----------------------------------------------------------------------------------------


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    E: int
    k: int
    f: int
    fs: int = 0  # shared expert d_ff; 0 = none
    act: int = BF16
    wdt: int = BF16
    # router bias: dict expert -> value (others 0); None = no bias at all
    bias: Optional[tuple] = None
    x_std: float = 1.0
    note: str = ""

    @property
    def rows(self) -> int:
        return self.T * self.k

    def with_tokens(self, T: int) -> "Workload":
        return Workload(self.name + f"_T{T}", T, self.d, self.E, self.k, self.f, self.fs, self.act,
                        self.wdt, self.bias, self.x_std, self.note)


WORKLOADS = {
    # T=64, d=256, E=8, top-2, d_ff=512, fp32 throughout
    "tiny_f32": Workload("tiny_f32", 64, 256, 8, 2, 512, act=F32, wdt=F32,
                         note="tiny fp32 layer, seed 0"),
    # Mixtral-8x7B-shaped prefill layer
    "mixtral_prefill_bf16": Workload("mixtral_prefill_bf16", 4096, 4096, 8, 2, 14336,
                                     note="Mixtral-shaped prefill, bf16"),
    # 128 fine-grained experts, top-4, plus one always-on shared expert
    "fine_grained_shared_bf16": Workload("fine_grained_shared_bf16", 8192, 2048, 128, 4, 768,
                                         fs=3072, note="128 experts top-4 + shared expert"),
    # router bias +4 on experts 0 and 1
    "skewed_bf16": Workload("skewed_bf16", 2048, 4096, 16, 2, 8192, bias=((0, 4.0), (1, 4.0)),
                            note="skewed routing, +4 bias on experts 0/1"),
    # the same plus -30 on experts 12..15 so that they receive exactly zero tokens
    "skewed_empty_bf16": Workload("skewed_empty_bf16", 2048, 4096, 16, 2, 8192,
                                  bias=((0, 4.0), (1, 4.0), (12, -30.0), (13, -30.0), (14, -30.0),
                                        (15, -30.0)),
                                  note="skewed routing with four experts forced empty"),
    # the Mixtral-shaped layer with 4 experts and 1024 tokens: the same kernels and tile shapes
    # on ~1.5 GB of device memory (still far larger than L2), sized for ncu captures
    "mixtral_prefill_bf16_small": Workload("mixtral_prefill_bf16_small", 1024, 4096, 4, 2, 14336,
                                           note="profiling-size Mixtral-shaped layer"),
    # routing-dominated layer for profiling the router: 16384 tokens (x = 134 MB, larger than
    # L2) over 8 experts with a tiny d_ff, ~0.2 GB on the device
    "router_profile_bf16": Workload("router_profile_bf16", 16384, 4096, 8, 2, 64,
                                    note="router profiling case"),
    # decode, int8 weights with per-output-channel scales
    "decode_int8_T1": Workload("decode_int8_T1", 1, 4096, 8, 2, 14336, act=BF16, wdt=I8),
    "decode_int8_T8": Workload("decode_int8_T8", 8, 4096, 8, 2, 14336, act=BF16, wdt=I8),
    "decode_int8_T32": Workload("decode_int8_T32", 32, 4096, 8, 2, 14336, act=BF16, wdt=I8),
    # decode, int4 weights with one fp32 scale per output channel and group of 128 inputs
    "decode_int4_T1": Workload("decode_int4_T1", 1, 4096, 8, 2, 14336, act=BF16, wdt=I4),
    "decode_int4_T8": Workload("decode_int4_T8", 8, 4096, 8, 2, 14336, act=BF16, wdt=I4),
    "decode_int4_T32": Workload("decode_int4_T32", 32, 4096, 8, 2, 14336, act=BF16, wdt=I4),
}


def expert_stride_elems(d: int, f: int, wdt: int = BF16) -> int:
    """Elements between consecutive experts: 3*d*f rounded up to a multiple of 128 (of 256 for
    int4, so that every expert still starts on a 128-byte boundary)."""
    n = 3 * d * f
    m = 256 if wdt == I4 else 128
    return (n + m - 1) // m * m


def pack_int4(q: torch.Tensor) -> torch.Tensor:
    """Pack int8 values in [-8, 7] two per byte: element 2j in the low nibble of byte j."""
    assert q.dtype == torch.int8 and q.numel() % 2 == 0
    u = (q.to(torch.int16) & 0xF).to(torch.uint8).view(-1, 2)
    return (u[:, 0] | (u[:, 1] << 4)).contiguous()


# tensor ids of the seeded streams
TID_X, TID_ROUTER_W = 1, 2
TID_EXPERT_BASE, TID_SCALE_BASE, TID_SHARED_BASE = 1000, 500000, 900000


@dataclass
class Problem:
    wl: Workload
    seed: int
    x: torch.Tensor
    router_w: torch.Tensor
    router_b: Optional[torch.Tensor]
    expert_w: torch.Tensor
    expert_scales: Optional[torch.Tensor]
    shared_w: Optional[torch.Tensor]
    expert_stride: int
    extra: dict = field(default_factory=dict)


def _empty(n, dtype, pin):
    return torch.empty(n, dtype=dtype, pin_memory=pin)


def make_x(wl: Workload, seed: int, pin: bool = False) -> torch.Tensor:
    x = _empty(wl.T * wl.d, _TORCH_DTYPE[wl.act], pin)
    fill_normal(x, seed, TID_X, wl.x_std)
    return x.view(wl.T, wl.d)


def make_problem(wl: Workload, seed: int = 0, pin: bool = False, expert_stride: Optional[int] = None,
                 x: bool = True) -> Problem:
    """Generate every input of one layer call on the host.

    Distributions: x ~ N(0, 1); router W ~ N(0, 1/d); expert W ~ N(0, 1/d_in) with d_in = d for
    W1/W3 and f for W2 (bf16/fp32 weights); int8 weights uniform on [-127, 127] with scales
    U(0.5, 1.5) / (127 sqrt(d_in)); int4 weights uniform on [-7, 7] with group scales
    U(0.5, 1.5) / (7 sqrt(d_in)); router bias as the workload states (else none).
    """
    T, d, E, f, fs = wl.T, wl.d, wl.E, wl.f, wl.fs
    adt = _TORCH_DTYPE[wl.act]
    stride = expert_stride if expert_stride is not None else expert_stride_elems(d, f, wl.wdt)
    if wl.wdt == I4:
        assert d % I4_GROUP == 0 and f % I4_GROUP == 0, "int4 weights need d and f multiples of 128"
        assert stride % 2 == 0
    xt = make_x(wl, seed, pin) if x else None
    rw = _empty(E * d, adt, pin)
    fill_normal(rw, seed, TID_ROUTER_W, 1.0 / math.sqrt(d))
    rb = None
    if wl.bias is not None:
        rb = torch.zeros(E, dtype=torch.float32)
        for e, v in wl.bias:
            rb[e] = v
        if pin:
            rb = rb.pin_memory()
    wdt = _TORCH_DTYPE[wl.wdt]
    i4 = wl.wdt == I4
    ew = _empty(E * stride // 2 if i4 else E * stride, wdt, pin)
    ew.zero_() if stride != 3 * d * f else None
    scales = _empty(E * (2 * f + d), torch.float32, pin) if wl.wdt == I8 else None
    if i4:
        scales = _empty(E * 3 * d * f // I4_GROUP, torch.float32, pin)
    for e in range(E):
        base = e * stride
        segs = ((0, f * d, d), (f * d, f * d, d), (2 * f * d, d * f, f))  # W1, W3, W2
        for m, (off, n, d_in) in enumerate(segs):
            tid = TID_EXPERT_BASE + 3 * e + m
            if i4:
                q = fill_int(torch.empty(n, dtype=torch.int8), seed, tid, -7, 7)
                ew[(base + off) // 2: (base + off + n) // 2] = pack_int4(q)
                continue
            view = ew[base + off: base + off + n]
            if wl.wdt == I8:
                fill_int(view, seed, tid, -127, 127)
            else:
                fill_normal(view, seed, tid, 1.0 / math.sqrt(d_in))
        if i4:
            sbase = e * 3 * d * f // I4_GROUP
            for m, (off, n, d_in) in enumerate(segs):
                lo = 0.5 / (7.0 * math.sqrt(d_in))
                hi = 1.5 / (7.0 * math.sqrt(d_in))
                fill_uniform(scales[sbase + off // I4_GROUP: sbase + (off + n) // I4_GROUP], seed,
                             TID_SCALE_BASE + 3 * e + m, lo, hi)
        elif scales is not None:
            sbase = e * (2 * f + d)
            for m, (off, n, d_in) in enumerate(((0, f, d), (f, f, d), (2 * f, d, f))):
                lo = 0.5 / (127.0 * math.sqrt(d_in))
                hi = 1.5 / (127.0 * math.sqrt(d_in))
                fill_uniform(scales[sbase + off: sbase + off + n], seed, TID_SCALE_BASE + 3 * e + m, lo, hi)
    sw = None
    if fs:
        assert wl.wdt not in (I8, I4), "shared expert is defined for bf16/fp32 weights"
        sw = _empty(3 * fs * d, wdt, pin)
        for m, (off, n, d_in) in enumerate(((0, fs * d, d), (fs * d, fs * d, d), (2 * fs * d, d * fs, fs))):
            fill_normal(sw[off: off + n], seed, TID_SHARED_BASE + m, 1.0 / math.sqrt(d_in))
    return Problem(wl, seed, xt, rw.view(E, d), rb, ew, scales, sw, stride)


def sample_tokens(T: int, n: int):
    """n token indices spread evenly over [0, T), always including the first and the last."""
    if n >= T:
        return list(range(T))
    if n <= 1:
        return [0]
    return sorted({round(i * (T - 1) / (n - 1)) for i in range(n)})


def custom(name: str, T: int, d: int, E: int, k: int, f: int, fs: int = 0, act: int = BF16,
           wdt: int = BF16, bias=None) -> Workload:
    """A workload with explicit sizes (for parity cases at oracle-friendly sizes)."""
    return Workload(name, T, d, E, k, f, fs, act, wdt, bias)
