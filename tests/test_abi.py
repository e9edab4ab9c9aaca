"""The C ABI on the host: the library loads, exports what include/moe.h
declares, sizes workspaces, and rejects bad arguments before touching a GPU."""
import ctypes
import os
import re

import pytest

import mixture_experts_histogram_b200 as m
from mixture_experts_histogram_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return m.load()


def _declared():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            names |= set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src))
    return names


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert {"moe_forward", "moe_workspace_bytes", "moe_route", "moe_permute", "moe_experts", "moe_combine",
            "moe_quantize_act", "moe_forward_host", "moe_read_status"} <= names
    for n in names:
        assert hasattr(lib, n), n


def test_workspace_bytes_scales_with_tokens(lib):
    cfg = m.make_config(4096, 352, 8, 1, 1536, m.MOE_WDTYPE_FP8_E4M3)
    a, b = m.moe_workspace_bytes(cfg, 64), m.moe_workspace_bytes(cfg, 8192)
    assert 0 < a < b
    # y (9T x H bf16) dominates at T = 8192
    assert b > 9 * 8192 * 4096 * 2
    assert m.moe_workspace_bytes(cfg, 0) > 0


@pytest.mark.parametrize("field,value,code", [
    ("hidden", 100, m.MOE_ERR_UNSUPPORTED_SHAPE),
    ("inter", 200, m.MOE_ERR_UNSUPPORTED_SHAPE),
    ("n_experts", 513, m.MOE_ERR_UNSUPPORTED_SHAPE),
    ("top_k", 17, m.MOE_ERR_UNSUPPORTED_SHAPE),
    ("top_k", 0, m.MOE_ERR_INVALID_ARG),
    ("n_shared", 2, m.MOE_ERR_UNSUPPORTED_SHAPE),
    ("wdtype", 7, m.MOE_ERR_INVALID_ARG),
])
def test_bad_config_is_rejected(lib, field, value, code):
    cfg = m.make_config(4096, 352, 8, 1, 1536, 0)
    setattr(cfg, field, value)
    n = ctypes.c_size_t(0)
    assert lib.moe_workspace_bytes(ctypes.byref(cfg), 64, ctypes.byref(n)) == code


def test_argument_errors_need_no_device(lib):
    cfg = m.make_config(256, 16, 2, 1, 128, 0)
    w = m.moe_weights()
    # missing weights
    assert lib.moe_forward(ctypes.byref(cfg), 4, 1024, ctypes.byref(w), 2048, None, None, 4096, 1 << 20, None) == \
        m.MOE_ERR_INVALID_ARG
    fake = {k: 1 << 20 for k in m.WEIGHT_FIELDS}
    w = m.moe_weights(*[fake[k] for k in m.WEIGHT_FIELDS])
    # misaligned x
    assert lib.moe_forward(ctypes.byref(cfg), 4, 1030, ctypes.byref(w), 2048, None, None, 4096, 1 << 20, None) == \
        m.MOE_ERR_MISALIGNED
    # workspace too small / misaligned
    assert lib.moe_forward(ctypes.byref(cfg), 4, 1024, ctypes.byref(w), 2048, None, None, 4096, 16, None) == \
        m.MOE_ERR_WORKSPACE_TOO_SMALL
    assert lib.moe_forward(ctypes.byref(cfg), 4, 1024, ctypes.byref(w), 2048, None, None, 4352 + 64, 1 << 30, None) == \
        m.MOE_ERR_MISALIGNED
    # only one of topk_idx / topk_w
    assert lib.moe_forward(ctypes.byref(cfg), 4, 1024, ctypes.byref(w), 2048, 4096, None, 8192, 1 << 30, None) == \
        m.MOE_ERR_INVALID_ARG
    # negative T
    assert lib.moe_forward(ctypes.byref(cfg), -1, 1024, ctypes.byref(w), 2048, None, None, 4096, 1 << 30, None) == \
        m.MOE_ERR_INVALID_ARG
    # T = 0 is a no-op
    assert lib.moe_forward(ctypes.byref(cfg), 0, 1024, ctypes.byref(w), 2048, None, None, 4096, 1 << 30, None) == \
        m.MOE_OK


def test_residual_stream_argument_errors_need_no_device(lib):
    # moe_rmsnorm(T, hidden, residual, weight, eps, x, stream)
    # (Every call below returns before any launch: these are host addresses.)
    assert lib.moe_rmsnorm(4, 100, 1024, 2048, 1e-6, 4096, None) == m.MOE_ERR_INVALID_ARG   # H not a multiple of 128
    assert lib.moe_rmsnorm(4, 256, 1024, 2048, -1.0, 4096, None) == m.MOE_ERR_INVALID_ARG   # negative eps
    assert lib.moe_rmsnorm(-1, 256, 1024, 2048, 1e-6, 4096, None) == m.MOE_ERR_INVALID_ARG
    assert lib.moe_rmsnorm(4, 256, None, 2048, 1e-6, 4096, None) == m.MOE_ERR_INVALID_ARG
    assert lib.moe_rmsnorm(4, 256, 1028, 2048, 1e-6, 4096, None) == m.MOE_ERR_MISALIGNED
    assert lib.moe_rmsnorm(0, 256, None, None, 1e-6, None, None) == m.MOE_OK               # T = 0: no-op
    # moe_combine_residual(cfg, T, y, pos, residual, residual_out, stream)
    cfg = m.make_config(256, 16, 2, 1, 128, 0)
    assert lib.moe_combine_residual(ctypes.byref(cfg), 4, 1024, 2048, 4096, 8192 + 4, None) == m.MOE_ERR_MISALIGNED
    assert lib.moe_combine_residual(ctypes.byref(cfg), 4, 1024, None, 4096, 8192, None) == m.MOE_ERR_INVALID_ARG
    bad = m.make_config(200, 16, 2, 1, 128, 0)
    assert lib.moe_combine_residual(ctypes.byref(bad), 4, 1024, 2048, 4096, 8192, None) == m.MOE_ERR_INVALID_ARG
    assert lib.moe_combine_residual(ctypes.byref(cfg), 0, None, None, None, None, None) == m.MOE_OK


def test_status_strings(lib):
    for c in range(8):
        assert m.moe_status_string(c) not in ("", "unknown status")
    assert m.moe_status_string(99) == "unknown status"
    assert m.load().moe_profile_kernel_name(6).decode() == "gemm1_gate_up_swiglu"


def test_product_path_does_not_touch_the_oracle():
    """The binding and the CUDA sources never import, link or name the oracle."""
    pkg = os.path.join(ROOT, "mixture_experts_histogram_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in src and "from oracle" not in src and "orc_" not in src, f
