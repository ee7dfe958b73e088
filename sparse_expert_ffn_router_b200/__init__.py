"""Python binding of the B200 MoE layer forward (C ABI in include/colibri.h).

Argument marshalling only: every step of the layer runs in the CUDA kernels of
``libcolibri.so``.  The functions carry the C names; tensors may be passed as torch
tensors (their ``data_ptr()`` is used) or as integer addresses.  A non-OK status raises
:class:`ColibriError`.  Importing works without a GPU; loading the library requires it to
have been built (``python -m sparse_expert_ffn_router_b200.build``) and fails loudly
otherwise -- there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libcolibri.so")

COLIBRI_F32, COLIBRI_BF16, COLIBRI_I8, COLIBRI_I4 = 0, 1, 2, 3
COLIBRI_ROUTER_CLAMP, COLIBRI_ROUTER_RAW_WEIGHTS = 1, 2
COLIBRI_SCALE_PER_CHANNEL, COLIBRI_SCALE_PER_MATRIX = 0, 1

STATUS = {
    0: "COLIBRI_OK",
    -1: "COLIBRI_ERR_INVALID_ARG",
    -2: "COLIBRI_ERR_ALIGNMENT",
    -3: "COLIBRI_ERR_UNSUPPORTED",
    -4: "COLIBRI_ERR_OOM",
    -5: "COLIBRI_ERR_CUDA",
    -6: "COLIBRI_ERR_TIMEOUT",
}

# every symbol include/colibri.h declares
EXPORTS = (
    "colibri_init",
    "colibri_expert_stride",
    "colibri_moe_forward",
    "colibri_moe_forward_routed",
    "colibri_get_routing",
    "colibri_combine",
    "colibri_sync_status",
    "colibri_profile_begin",
    "colibri_profile_end",
    "colibri_profile_calls",
    "colibri_route_noalloc",
    "colibri_route_noalloc_check",
    "colibri_selftest_wait_timeout",
    "colibri_status_string",
    "colibri_last_error",
    "colibri_free",
)


class colibri_desc(ctypes.Structure):
    _fields_ = [
        ("d_model", ctypes.c_int32),
        ("d_ff", ctypes.c_int32),
        ("num_experts", ctypes.c_int32),
        ("top_k", ctypes.c_int32),
        ("shared_d_ff", ctypes.c_int32),
        ("act_dtype", ctypes.c_int32),
        ("weight_dtype", ctypes.c_int32),
        ("max_tokens", ctypes.c_int32),
        ("device_id", ctypes.c_int32),
        ("router_flags", ctypes.c_int32),
        ("weight_scale_mode", ctypes.c_int32),
    ]


class ColibriError(RuntimeError):
    def __init__(self, status: int, what: str, detail: str = ""):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}" + (f" ({detail})" if detail else ""))


_lib = None


def load() -> ctypes.CDLL:
    """Load libcolibri.so (built in place).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build the CUDA library first "
                          "(python -m sparse_expert_ffn_router_b200.build)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    lib.colibri_init.argtypes = [ctypes.POINTER(colibri_desc), ctypes.POINTER(vp)]
    lib.colibri_init.restype = ctypes.c_int
    lib.colibri_expert_stride.argtypes = [vp]
    lib.colibri_expert_stride.restype = i64
    lib.colibri_moe_forward.argtypes = [vp, vp, i32, vp, vp, vp, vp, vp, vp, vp]
    lib.colibri_moe_forward.restype = ctypes.c_int
    lib.colibri_moe_forward_routed.argtypes = [vp, vp, i32, vp, vp, vp, vp, vp, vp, vp]
    lib.colibri_moe_forward_routed.restype = ctypes.c_int
    lib.colibri_get_routing.argtypes = [vp] * 8
    lib.colibri_get_routing.restype = ctypes.c_int
    lib.colibri_combine.argtypes = [vp, i32, vp, vp, i32, i32, i32, vp, vp]
    lib.colibri_combine.restype = ctypes.c_int
    lib.colibri_sync_status.argtypes = [vp, vp]
    lib.colibri_sync_status.restype = ctypes.c_int
    lib.colibri_profile_begin.argtypes = [vp, i32]
    lib.colibri_profile_begin.restype = ctypes.c_int
    lib.colibri_profile_end.argtypes = [vp, vp, vp]
    lib.colibri_profile_end.restype = ctypes.c_int
    lib.colibri_profile_calls.argtypes = [vp, vp, i32]
    lib.colibri_profile_calls.restype = ctypes.c_int
    lib.colibri_route_noalloc.argtypes = [vp, i32, i32, i32, vp, vp, i32, i32] + [vp] * 8
    lib.colibri_route_noalloc.restype = ctypes.c_int
    lib.colibri_route_noalloc_check.argtypes = [vp]
    lib.colibri_route_noalloc_check.restype = ctypes.c_int
    lib.colibri_selftest_wait_timeout.argtypes = [vp, i32, vp]
    lib.colibri_selftest_wait_timeout.restype = ctypes.c_int
    lib.colibri_status_string.argtypes = [ctypes.c_int]
    lib.colibri_status_string.restype = ctypes.c_char_p
    lib.colibri_last_error.argtypes = [vp]
    lib.colibri_last_error.restype = ctypes.c_char_p
    lib.colibri_free.argtypes = [vp]
    lib.colibri_free.restype = None
    _lib = lib
    return lib


def _addr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t or None
    return t.data_ptr() or None


def _stream(stream) -> Optional[int]:
    if stream is None:
        return None
    if isinstance(stream, int):
        return stream or None
    return stream.cuda_stream or None


def _check(rc: int, what: str, ctx=None):
    if rc != 0:
        detail = load().colibri_last_error(ctx)
        raise ColibriError(rc, what, detail.decode() if detail else "")


def colibri_status_string(status: int) -> str:
    return load().colibri_status_string(status).decode()


def colibri_last_error(ctx=None) -> str:
    s = load().colibri_last_error(ctx)
    return s.decode() if s else ""


def colibri_init(d_model: int, d_ff: int, num_experts: int, top_k: int, shared_d_ff: int = 0,
                 act_dtype: int = COLIBRI_BF16, weight_dtype: int = COLIBRI_BF16, max_tokens: int = 1,
                 device_id: int = 0, router_flags: int = 0, weight_scale_mode: int = 0) -> int:
    """Returns the opaque context handle (an address)."""
    desc = colibri_desc(d_model, d_ff, num_experts, top_k, shared_d_ff, act_dtype, weight_dtype,
                        max_tokens, device_id, router_flags, weight_scale_mode)
    out = ctypes.c_void_p()
    _check(load().colibri_init(ctypes.byref(desc), ctypes.byref(out)), "colibri_init")
    return out.value


def colibri_expert_stride(ctx: int) -> int:
    return int(load().colibri_expert_stride(ctx))


def colibri_moe_forward(ctx: int, x, T: int, router_w, router_b, expert_w, expert_scales, shared_w, y,
                        stream=None) -> None:
    _check(load().colibri_moe_forward(ctx, _addr(x), T, _addr(router_w), _addr(router_b), _addr(expert_w),
                                      _addr(expert_scales), _addr(shared_w), _addr(y), _stream(stream)),
           "colibri_moe_forward", ctx)


def colibri_moe_forward_routed(ctx: int, x, T: int, topk_idx, topk_w, expert_w, expert_scales, shared_w, y,
                               stream=None) -> None:
    _check(load().colibri_moe_forward_routed(ctx, _addr(x), T, _addr(topk_idx), _addr(topk_w), _addr(expert_w),
                                             _addr(expert_scales), _addr(shared_w), _addr(y), _stream(stream)),
           "colibri_moe_forward_routed", ctx)


def colibri_get_routing(ctx: int, topk_idx=None, topk_w=None, counts=None, offsets=None, src_row=None,
                        dst_row=None, stream=None) -> None:
    _check(load().colibri_get_routing(ctx, _addr(topk_idx), _addr(topk_w), _addr(counts), _addr(offsets),
                                      _addr(src_row), _addr(dst_row), _stream(stream)),
           "colibri_get_routing", ctx)


def colibri_combine(Yp, act_dtype: int, dst_row, topk_w, T: int, top_k: int, d_model: int, y, stream=None) -> None:
    """Gather stage alone: y[t] = sum_j topk_w[t][j] * Yp[dst_row[t][j]] (see include/colibri.h)."""
    _check(load().colibri_combine(_addr(Yp), act_dtype, _addr(dst_row), _addr(topk_w), T, top_k, d_model, _addr(y),
                                  _stream(stream)), "colibri_combine")


def colibri_sync_status(ctx: int, stream=None) -> None:
    _check(load().colibri_sync_status(ctx, _stream(stream)), "colibri_sync_status", ctx)


def colibri_selftest_wait_timeout(ctx: int, timeout_us: int, stream=None) -> None:
    _check(load().colibri_selftest_wait_timeout(ctx, timeout_us, _stream(stream)),
           "colibri_selftest_wait_timeout", ctx)


NUM_STAGES = 5
STAGE_NAMES = ("gate", "scatter", "expert_gateup", "expert_down", "gather")


def colibri_profile_begin(ctx: int, max_calls: int) -> None:
    _check(load().colibri_profile_begin(ctx, max_calls), "colibri_profile_begin", ctx)


def colibri_profile_end(ctx: int):
    """Returns (per-stage total milliseconds as a dict, number of calls recorded)."""
    ms = (ctypes.c_float * NUM_STAGES)()
    n = ctypes.c_int32()
    _check(load().colibri_profile_end(ctx, ms, ctypes.byref(n)), "colibri_profile_end", ctx)
    return dict(zip(STAGE_NAMES, [float(v) for v in ms])), int(n.value)


def colibri_profile_calls(ctx: int, ncalls: int):
    """Per-call stage milliseconds of the last profiling region: a list of dicts."""
    buf = (ctypes.c_float * (NUM_STAGES * max(ncalls, 1)))()
    _check(load().colibri_profile_calls(ctx, buf, ncalls), "colibri_profile_calls", ctx)
    return [dict(zip(STAGE_NAMES, [float(buf[c * NUM_STAGES + i]) for i in range(NUM_STAGES)]))
            for c in range(ncalls)]


def colibri_route_noalloc(x, act_dtype: int, T: int, d_model: int, router_w, router_b, num_experts: int,
                          top_k: int, topk_idx, topk_w, counts, offsets, src_row, dst_row, Xp, stream=None) -> None:
    """Gate + Scatter without a context or any device allocation (see include/colibri.h)."""
    _check(load().colibri_route_noalloc(_addr(x), act_dtype, T, d_model, _addr(router_w), _addr(router_b),
                                        num_experts, top_k, _addr(topk_idx), _addr(topk_w), _addr(counts),
                                        _addr(offsets), _addr(src_row), _addr(dst_row), _addr(Xp),
                                        _stream(stream)),
           "colibri_route_noalloc")


def colibri_route_noalloc_check(stream=None) -> None:
    """Raises ColibriError(TIMEOUT) if a device wait of the last colibri_route_noalloc gave up."""
    _check(load().colibri_route_noalloc_check(_stream(stream)), "colibri_route_noalloc_check")


def colibri_free(ctx: int) -> None:
    if ctx:
        load().colibri_free(ctx)


class MoELayer:
    """Owns one context; forwards tensors to the C ABI (no computation in Python)."""

    def __init__(self, d_model, d_ff, num_experts, top_k, shared_d_ff=0, act_dtype=COLIBRI_BF16,
                 weight_dtype=COLIBRI_BF16, max_tokens=1, device_id=0, router_flags=0, weight_scale_mode=0):
        self.desc = dict(d_model=d_model, d_ff=d_ff, num_experts=num_experts, top_k=top_k,
                         shared_d_ff=shared_d_ff, act_dtype=act_dtype, weight_dtype=weight_dtype,
                         max_tokens=max_tokens, device_id=device_id, router_flags=router_flags,
                         weight_scale_mode=weight_scale_mode)
        self.ctx = colibri_init(**self.desc)

    @property
    def expert_stride(self) -> int:
        return colibri_expert_stride(self.ctx)

    def forward(self, x, router_w, router_b, expert_w, y, expert_scales=None, shared_w=None, stream=None,
                T=None):
        T = x.shape[0] if T is None else T
        colibri_moe_forward(self.ctx, x, T, router_w, router_b, expert_w, expert_scales, shared_w, y, stream)
        return y

    def forward_routed(self, x, topk_idx, topk_w, expert_w, y, expert_scales=None, shared_w=None, stream=None):
        colibri_moe_forward_routed(self.ctx, x, x.shape[0], topk_idx, topk_w, expert_w, expert_scales, shared_w,
                                   y, stream)
        return y

    def routing(self, **bufs):
        colibri_get_routing(self.ctx, **bufs)

    def sync_status(self, stream=None):
        colibri_sync_status(self.ctx, stream)

    def close(self):
        if self.ctx:
            colibri_free(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
