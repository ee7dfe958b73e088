"""The C-ABI library: it loads, exports every declared symbol, and validates on the host.

These run without a GPU: argument validation happens before any CUDA call, so an invalid
description is rejected with INVALID_ARG / UNSUPPORTED on any machine.
"""
import ctypes
import os
import re
import subprocess

import pytest
import torch

import sparse_expert_ffn_router_b200 as colibri

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "colibri.h")


@pytest.fixture(scope="module")
def lib():
    from sparse_expert_ffn_router_b200 import build

    build.build()
    return colibri.load()


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(colibri_[a-z_]+)\s*\(", src)))


def test_header_declares_the_bound_names():
    assert _declared() == sorted(colibri.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", colibri.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\s[TW]\s+(colibri_\w+)", out))
    for name in _declared():
        assert name in exported, name
        assert getattr(lib, name) is not None


def test_descriptor_layout_matches_the_header(tmp_path):
    # the binding's ctypes struct must have the C struct's size and field offsets
    fields = [name for name, _ in colibri.colibri_desc._fields_]
    src = tmp_path / "layout.c"
    body = "".join(f'  printf("%zu\\n", offsetof(colibri_desc, {n}));\n' for n in fields)
    src.write_text('#include <stddef.h>\n#include <stdio.h>\n#include "colibri.h"\nint main(void) {\n'
                   '  printf("%zu\\n", sizeof(colibri_desc));\n' + body + "  return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    assert got[0] == ctypes.sizeof(colibri.colibri_desc)
    assert got[1:] == [getattr(colibri.colibri_desc, n).offset for n in fields]


def test_status_strings(lib):
    for code, name in colibri.STATUS.items():
        assert colibri.colibri_status_string(code).startswith(name)


def _desc(**kw):
    base = dict(d_model=256, d_ff=512, num_experts=8, top_k=2, shared_d_ff=0, act_dtype=colibri.COLIBRI_BF16,
                weight_dtype=colibri.COLIBRI_BF16, max_tokens=64, device_id=0)
    base.update(kw)
    return base


@pytest.mark.parametrize("kw,code", [
    (dict(d_model=100), -1),           # not a multiple of 64
    (dict(d_model=0), -1),
    (dict(d_ff=96), -1),
    (dict(shared_d_ff=-64), -1),
    (dict(num_experts=0), -1),
    (dict(num_experts=300), -1),
    (dict(top_k=0), -1),
    (dict(top_k=9, num_experts=16), -1),  # k > 8
    (dict(top_k=5, num_experts=4), -1),   # k > E
    (dict(max_tokens=0), -1),
    (dict(act_dtype=7), -1),
    (dict(act_dtype=colibri.COLIBRI_F32, weight_dtype=colibri.COLIBRI_BF16), -3),
    (dict(act_dtype=colibri.COLIBRI_I8, weight_dtype=colibri.COLIBRI_I8), -3),
    (dict(weight_dtype=colibri.COLIBRI_I8, shared_d_ff=64), -3),
    (dict(router_flags=4), -1),        # unknown router variant bit
    (dict(router_flags=-1), -1),
    (dict(weight_scale_mode=1), -1),   # per-matrix scales with bf16 weights
    (dict(weight_scale_mode=2, weight_dtype=colibri.COLIBRI_I8), -1),
])
def test_init_rejects_bad_descriptions(lib, kw, code):
    with pytest.raises(colibri.ColibriError) as ei:
        colibri.colibri_init(**_desc(**kw))
    assert ei.value.status == code
    assert colibri.colibri_last_error()  # a one-line reason is recorded


def test_null_arguments(lib):
    assert lib.colibri_init(None, None) == -1
    out = ctypes.c_void_p(123)
    assert lib.colibri_init(None, ctypes.byref(out)) == -1
    assert out.value is None
    assert lib.colibri_moe_forward(None, None, 0, None, None, None, None, None, None, None) == -1
    assert lib.colibri_get_routing(None, None, None, None, None, None, None, None) == -1
    assert lib.colibri_expert_stride(None) == -1
    lib.colibri_free(None)  # ignored


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_description_without_device_reports_cuda_error(lib):
    with pytest.raises(colibri.ColibriError) as ei:
        colibri.colibri_init(**_desc())
    assert ei.value.status == -5


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(colibri, "_lib", None)
    monkeypatch.setattr(colibri, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        colibri.load()
