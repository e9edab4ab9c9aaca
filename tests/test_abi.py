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


def test_grouped_gemm_and_hooks_argument_errors_need_no_device(lib):
    cfg = m.make_config(256, 16, 2, 1, 128, m.MOE_WDTYPE_FP8_E4M3)
    fake = {k: 1 << 20 for k in m.WEIGHT_FIELDS}
    w = m.moe_weights(*[fake[k] for k in m.WEIGHT_FIELDS])
    g = lib.moe_grouped_gemm
    # moe_grouped_gemm(cfg, stage, R, offsets, a, a_scale, w, row_gate, out, out_scale, ws, ws_bytes, stream)
    assert g(ctypes.byref(cfg), 0, 4, 1024, 2048, 4096, ctypes.byref(w), None, 8192, 8192, 16384, 1 << 20, None) == \
        m.MOE_ERR_INVALID_ARG                                                              # bad stage
    assert g(ctypes.byref(cfg), m.MOE_STAGE_DOWN, -1, 1024, 2048, 4096, ctypes.byref(w), None, 8192, None, 16384,
             1 << 20, None) == m.MOE_ERR_INVALID_ARG                                       # negative R
    assert g(ctypes.byref(cfg), m.MOE_STAGE_DOWN, 4, 1024, 2048, None, ctypes.byref(w), None, 8192, None, 16384,
             1 << 20, None) == m.MOE_ERR_INVALID_ARG                                       # FP8 without scales
    assert g(ctypes.byref(cfg), m.MOE_STAGE_GATE_UP, 4, 1024, 2048, 4096, ctypes.byref(w), None, 8192, None,
             16384, 1 << 20, None) == m.MOE_ERR_INVALID_ARG                                # FP8 h without out_scale
    assert g(ctypes.byref(cfg), m.MOE_STAGE_DOWN, 4, 1024, 2056, 4096, ctypes.byref(w), None, 8192, None, 16384,
             1 << 20, None) == m.MOE_ERR_MISALIGNED                                        # A not 16-byte aligned
    assert g(ctypes.byref(cfg), m.MOE_STAGE_DOWN, 4, 1024, 2048, 4096, ctypes.byref(w), None, 8192, None, 16384,
             16, None) == m.MOE_ERR_WORKSPACE_TOO_SMALL
    assert g(ctypes.byref(cfg), m.MOE_STAGE_DOWN, 0, 1024, 2048, 4096, ctypes.byref(w), None, 8192, None, 16384,
             1 << 20, None) == m.MOE_OK                                                    # R = 0: no-op
    assert lib.moe_debug_inject(7, 0) == m.MOE_ERR_INVALID_ARG
    assert lib.moe_debug_inject(m.MOE_INJECT_NONE, 0) == m.MOE_OK
    for v in (m.MOE_GEMM_SINGLE, m.MOE_GEMM_PAIR, m.MOE_GEMM_SWAP, m.MOE_GEMM_AUTO):
        assert lib.moe_set_gemm_variant(v) == m.MOE_OK
    assert lib.moe_set_gemm_variant(4) == m.MOE_ERR_INVALID_ARG
    assert lib.moe_set_gemm_variant(-1) == m.MOE_ERR_INVALID_ARG


def test_expert_parallel_argument_errors_need_no_device(lib):
    arr = (ctypes.c_void_p * 17)(*([1 << 20] * 17))
    r = lib.moe_ep_reduce
    # moe_ep_reduce(n_ranks, partials, T, hidden, t0, t1, out, stream)
    assert r(0, arr, 8, 256, 0, 8, 4096, None) == m.MOE_ERR_INVALID_ARG
    assert r(17, arr, 8, 256, 0, 8, 4096, None) == m.MOE_ERR_UNSUPPORTED_SHAPE
    assert r(2, arr, 8, 100, 0, 8, 4096, None) == m.MOE_ERR_INVALID_ARG
    assert r(2, arr, 8, 256, 4, 9, 4096, None) == m.MOE_ERR_INVALID_ARG
    assert r(2, arr, 8, 256, 0, 8, 4100, None) == m.MOE_ERR_MISALIGNED
    assert r(2, arr, 8, 256, 3, 3, 4096, None) == m.MOE_OK  # empty range: no launch
    cfg = m.make_config(256, 16, 2, 1, 128, 0)
    fake = {k: 1 << 20 for k in m.WEIGHT_FIELDS}
    w = m.moe_weights(*[fake[k] for k in m.WEIGHT_FIELDS])
    f = lib.moe_forward_ep_partial
    # moe_forward_ep_partial(cfg, T, x, w, e0, e1, t0, t1, partial, idx, gate, ws, ws_bytes, stream)
    assert f(ctypes.byref(cfg), 8, 4096, ctypes.byref(w), 4, 4, 0, 8, 8192, None, None, 16384, 1 << 30, None) == \
        m.MOE_ERR_INVALID_ARG
    assert f(ctypes.byref(cfg), 8, 4096, ctypes.byref(w), 0, 4, 0, 9, 8192, None, None, 16384, 1 << 30, None) == \
        m.MOE_ERR_INVALID_ARG
    assert f(ctypes.byref(cfg), 8, 4096, ctypes.byref(w), 0, 4, 0, 8, 8196, None, None, 16384, 1 << 30, None) == \
        m.MOE_ERR_MISALIGNED
    assert f(ctypes.byref(cfg), 0, 4096, ctypes.byref(w), 0, 4, 0, 0, 8192, None, None, 16384, 1 << 30, None) == \
        m.MOE_OK


def test_nvfp4_config_and_weight_checks_need_no_device(lib):
    n = ctypes.c_size_t(0)
    ok = m.make_config(4096, 352, 8, 1, 1536, m.MOE_WDTYPE_NVFP4)
    assert lib.moe_workspace_bytes(ctypes.byref(ok), 64, ctypes.byref(n)) == m.MOE_OK
    odd = m.make_config(384, 16, 2, 1, 256, m.MOE_WDTYPE_NVFP4)   # H not a multiple of 256
    assert lib.moe_workspace_bytes(ctypes.byref(odd), 64, ctypes.byref(n)) == m.MOE_ERR_UNSUPPORTED_SHAPE
    cfg = m.make_config(256, 16, 2, 1, 256, m.MOE_WDTYPE_NVFP4)
    fake = {k: 1 << 20 for k in m.WEIGHT_FIELDS}
    fake["router_bias"] = None
    for missing in ("s2", "g1", "sg2"):
        w = m.moe_weights(*[None if k == missing else fake[k] for k in m.WEIGHT_FIELDS])
        assert lib.moe_forward(ctypes.byref(cfg), 4, 1024, ctypes.byref(w), 2048, None, None, 4096, 1 << 30,
                               None) == m.MOE_ERR_INVALID_ARG, missing
    w = m.moe_weights(*[(fake[k] + 8 if k == "s1" else fake[k]) for k in m.WEIGHT_FIELDS])
    assert lib.moe_forward(ctypes.byref(cfg), 4, 1024, ctypes.byref(w), 2048, None, None, 4096, 1 << 30, None) == \
        m.MOE_ERR_MISALIGNED


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


def test_traffic_hash_covers_every_grouped_gemm_source():
    """bench.py drops a stored DRAM-traffic figure once the sources it was taken on
    change; every file the grouped-GEMM sources include (and the launch code that
    builds their tensor maps) must be part of that hash."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    csrc = os.path.join(ROOT, "mixture_experts_histogram_b200", "csrc")
    gemm = [f for f in os.listdir(csrc) if f.endswith(".cu") and "gemm" in f]
    assert gemm and set(gemm) <= set(bench.GEMM_SOURCES)
    todo, seen = list(gemm), set()
    while todo:
        f = todo.pop()
        if f in seen:
            continue
        seen.add(f)
        for inc in re.findall(r'#include\s+"([^"]+)"', open(os.path.join(csrc, f)).read()):
            if os.path.exists(os.path.join(csrc, inc)):
                todo.append(inc)
    assert seen <= set(bench.GEMM_SOURCES), sorted(seen - set(bench.GEMM_SOURCES))
    assert "abi.cu" in bench.GEMM_SOURCES
