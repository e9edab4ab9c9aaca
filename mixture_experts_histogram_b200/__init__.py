"""Python binding of libmoe_b200.so, the B200 routed-MoE layer forward.

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels (include/moe.h is the contract). PyTorch supplies device memory and
streams. The binding fails loudly when the library is missing or when a call
returns an error; there is no fallback.

The functions carry the names of the C entry points:
  moe_workspace_bytes, moe_forward, moe_forward_host, moe_forward_host_async, moe_route,
  moe_quantize_act, moe_permute, moe_experts, moe_combine, moe_read_status,
  moe_status_string, moe_profile_enable, moe_profile_read, moe_device_sm_count,
  moe_set_gemm_variant, moe_permute_noalloc, moe_rmsnorm, moe_combine_residual,
  moe_grouped_gemm, moe_read_status_detail, moe_debug_inject, moe_launch_count,
  moe_forward_ep_partial, moe_ep_reduce.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libmoe_b200.so")

MOE_WDTYPE_BF16, MOE_WDTYPE_FP8_E4M3, MOE_WDTYPE_NVFP4 = 0, 1, 2
MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED_SHAPE = 2
MOE_ERR_WORKSPACE_TOO_SMALL = 3
MOE_ERR_CUDA = 4
MOE_ERR_BAD_INDEX = 5
MOE_ERR_DEVICE_TIMEOUT = 6
MOE_ERR_MISALIGNED = 7
MOE_GEMM_AUTO, MOE_GEMM_SINGLE, MOE_GEMM_PAIR, MOE_GEMM_SWAP = 0, 1, 2, 3
MOE_STAGE_GATE_UP, MOE_STAGE_GATE_UP_RAW, MOE_STAGE_DOWN = 1, 2, 3
MOE_INJECT_NONE, MOE_INJECT_GEMM_NO_LOADS = 0, 1

_lib = None


class MoeError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {moe_status_string(code)} (status {code})")
        self.code = code


class moe_config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("n_experts", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("n_shared", ctypes.c_int32), ("inter", ctypes.c_int32), ("wdtype", ctypes.c_int32)]


WEIGHT_FIELDS = ("router_w", "router_bias", "w1", "w3", "w2", "s1", "s3", "s2",
                 "sw1", "sw3", "sw2", "ss1", "ss3", "ss2", "g1", "g3", "g2", "sg1", "sg3", "sg2")


class moe_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in WEIGHT_FIELDS]


def load():
    """Load the in-tree library (build it first with build.build())."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: run mixture_experts_histogram_b200.build.build() first")
    lib = ctypes.CDLL(LIB_PATH)
    i32, i64, vp, sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t
    cfgp, wp = ctypes.POINTER(moe_config), ctypes.POINTER(moe_weights)
    sig = {
        "moe_workspace_bytes": [cfgp, i64, ctypes.POINTER(sz)],
        "moe_forward": [cfgp, i64, vp, wp, vp, vp, vp, vp, sz, vp],
        "moe_forward_host": [cfgp, i64, vp, wp, vp, vp, sz, vp],
        "moe_forward_host_async": [cfgp, i64, vp, wp, vp, vp, sz, vp],
        "moe_route": [cfgp, i64, vp, vp, vp, vp, vp, vp, vp, sz, vp],
        "moe_quantize_act": [i64, i32, vp, vp, vp, vp],
        "moe_permute": [cfgp, i64, vp, vp, vp, vp, vp, vp, sz, vp],
        "moe_experts": [cfgp, i64, vp, vp, vp, wp, vp, vp, vp, sz, vp],
        "moe_combine": [cfgp, i64, vp, vp, vp, vp],
        "moe_read_status": [vp, vp, ctypes.POINTER(ctypes.c_int)],
        "moe_status_string": [ctypes.c_int],
        "moe_profile_enable": [ctypes.c_int],
        "moe_profile_read": [ctypes.POINTER(ctypes.c_float), ctypes.c_int, ctypes.POINTER(ctypes.c_int)],
        "moe_profile_kernel_name": [ctypes.c_int],
        "moe_device_sm_count": [ctypes.POINTER(ctypes.c_int)],
        "moe_set_gemm_variant": [ctypes.c_int],
        "moe_permute_noalloc": [cfgp, i64, vp, vp, vp, vp, vp, vp, vp],
        "moe_rmsnorm": [i64, i32, vp, vp, ctypes.c_float, vp, vp],
        "moe_combine_residual": [cfgp, i64, vp, vp, vp, vp, vp],
        "moe_grouped_gemm": [cfgp, ctypes.c_int, i64, vp, vp, vp, wp, vp, vp, vp, vp, sz, vp],
        "moe_read_status_detail": [vp, vp, ctypes.POINTER(ctypes.c_int)],
        "moe_debug_inject": [ctypes.c_int, ctypes.c_uint64],
        "moe_launch_count": [ctypes.POINTER(ctypes.c_uint64)],
        "moe_forward_ep_partial": [cfgp, i64, vp, wp, i32, i32, i64, i64, vp, vp, vp, vp, sz, vp],
        "moe_ep_reduce": [i32, ctypes.POINTER(ctypes.c_void_p), i64, i32, i64, i64, vp, vp],
    }
    for name, args in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_char_p if name in ("moe_status_string", "moe_profile_kernel_name") else ctypes.c_int
    _lib = lib
    return lib


def _ptr(t) -> Optional[int]:
    """Device (or host) address of a tensor/array, None for None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if hasattr(t, "data_ptr"):
        if not t.is_contiguous():
            raise ValueError("tensors passed to the library must be contiguous")
        return t.data_ptr()
    return t.ctypes.data  # numpy


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _check(rc: int, where: str):
    if rc != MOE_OK:
        raise MoeError(rc, where)


def make_config(hidden, n_experts, top_k, n_shared, inter, wdtype) -> moe_config:
    return moe_config(hidden, n_experts, top_k, n_shared, inter, wdtype)


def make_weights(w: dict) -> moe_weights:
    """moe_weights from a dict of device tensors keyed by the C field names."""
    return moe_weights(*[_ptr(w.get(n)) for n in WEIGHT_FIELDS])


def moe_status_string(code: int) -> str:
    return load().moe_status_string(code).decode()


def moe_workspace_bytes(cfg: moe_config, T: int) -> int:
    n = ctypes.c_size_t(0)
    _check(load().moe_workspace_bytes(ctypes.byref(cfg), T, ctypes.byref(n)), "moe_workspace_bytes")
    return n.value


def moe_forward(cfg, T, x, w: moe_weights, out, workspace, topk_idx=None, topk_w=None, stream=None,
                workspace_bytes=None):
    nb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check(load().moe_forward(ctypes.byref(cfg), T, _ptr(x), ctypes.byref(w), _ptr(out), _ptr(topk_idx),
                              _ptr(topk_w), _ptr(workspace), nb, _stream(stream)), "moe_forward")


def moe_forward_host(cfg, T, x_host, w: moe_weights, out_host, workspace, stream=None):
    nb = workspace.numel() * workspace.element_size()
    _check(load().moe_forward_host(ctypes.byref(cfg), T, _ptr(x_host), ctypes.byref(w), _ptr(out_host),
                                   _ptr(workspace), nb, _stream(stream)), "moe_forward_host")


def moe_forward_host_async(cfg, T, x_host, w: moe_weights, out_host, workspace, stream=None):
    """moe_forward_host queued on `stream` without the final synchronisation."""
    nb = workspace.numel() * workspace.element_size()
    _check(load().moe_forward_host_async(ctypes.byref(cfg), T, _ptr(x_host), ctypes.byref(w), _ptr(out_host),
                                         _ptr(workspace), nb, _stream(stream)), "moe_forward_host_async")


def moe_route(cfg, T, x, router_w, router_bias, topk_idx, topk_w, logits, workspace, stream=None):
    nb = workspace.numel() * workspace.element_size()
    _check(load().moe_route(ctypes.byref(cfg), T, _ptr(x), _ptr(router_w), _ptr(router_bias), _ptr(topk_idx),
                            _ptr(topk_w), _ptr(logits), _ptr(workspace), nb, _stream(stream)), "moe_route")


def moe_quantize_act(T, hidden, x, q, s, stream=None):
    _check(load().moe_quantize_act(T, hidden, _ptr(x), _ptr(q), _ptr(s), _stream(stream)), "moe_quantize_act")


def moe_permute(cfg, T, topk_idx, counts, offsets, perm, pos, workspace, stream=None):
    nb = workspace.numel() * workspace.element_size()
    _check(load().moe_permute(ctypes.byref(cfg), T, _ptr(topk_idx), _ptr(counts), _ptr(offsets), _ptr(perm),
                              _ptr(pos), _ptr(workspace), nb, _stream(stream)), "moe_permute")


def moe_permute_noalloc(cfg, T, topk_idx, counts, offsets, perm, pos, device_status=None, stream=None):
    """moe_permute without a workspace (fixed static scratch inside the library)."""
    _check(load().moe_permute_noalloc(ctypes.byref(cfg), T, _ptr(topk_idx), _ptr(counts), _ptr(offsets),
                                      _ptr(perm), _ptr(pos), _ptr(device_status), _stream(stream)),
           "moe_permute_noalloc")


def moe_experts(cfg, T, x, topk_idx, topk_w, w: moe_weights, y, pos, workspace, stream=None):
    nb = workspace.numel() * workspace.element_size()
    _check(load().moe_experts(ctypes.byref(cfg), T, _ptr(x), _ptr(topk_idx), _ptr(topk_w), ctypes.byref(w),
                              _ptr(y), _ptr(pos), _ptr(workspace), nb, _stream(stream)), "moe_experts")


def moe_forward_ep_partial(cfg, T, x, w: moe_weights, e0, e1, shared_t0, shared_t1, partial, workspace,
                           topk_idx=None, topk_w=None, stream=None):
    """One expert-parallel rank's fp32 partial output (its experts [e0, e1) and
    its shared-expert tokens [shared_t0, shared_t1))."""
    nb = workspace.numel() * workspace.element_size()
    _check(load().moe_forward_ep_partial(ctypes.byref(cfg), T, _ptr(x), ctypes.byref(w), e0, e1, shared_t0,
                                         shared_t1, _ptr(partial), _ptr(topk_idx), _ptr(topk_w), _ptr(workspace),
                                         nb, _stream(stream)), "moe_forward_ep_partial")


def moe_ep_reduce(partials, T, hidden, t0, t1, out, stream=None):
    """out[t0:t1] = bf16 of the fp32 partials added in rank order."""
    arr = (ctypes.c_void_p * len(partials))(*[_ptr(p) for p in partials])
    _check(load().moe_ep_reduce(len(partials), arr, T, hidden, t0, t1, _ptr(out), _stream(stream)),
           "moe_ep_reduce")


def moe_grouped_gemm(cfg, stage, R, offsets, a, a_scale, w: moe_weights, out, workspace, row_gate=None,
                     out_scale=None, stream=None):
    """One grouped expert GEMM over rows grouped by `offsets` (MOE_STAGE_*)."""
    nb = workspace.numel() * workspace.element_size()
    _check(load().moe_grouped_gemm(ctypes.byref(cfg), stage, R, _ptr(offsets), _ptr(a), _ptr(a_scale),
                                   ctypes.byref(w), _ptr(row_gate), _ptr(out), _ptr(out_scale), _ptr(workspace),
                                   nb, _stream(stream)), "moe_grouped_gemm")


def moe_combine(cfg, T, y, pos, out, stream=None):
    _check(load().moe_combine(ctypes.byref(cfg), T, _ptr(y), _ptr(pos), _ptr(out), _stream(stream)),
           "moe_combine")


def moe_rmsnorm(T, hidden, residual, weight, eps, x, stream=None):
    """x = bf16(RMS-normalised fp32 residual * weight): the layer's input."""
    _check(load().moe_rmsnorm(T, hidden, _ptr(residual), _ptr(weight), float(eps), _ptr(x), _stream(stream)),
           "moe_rmsnorm")


def moe_combine_residual(cfg, T, y, pos, residual, residual_out, stream=None):
    """residual_out = residual + fixed-order fp32 sum of the token's expert rows."""
    _check(load().moe_combine_residual(ctypes.byref(cfg), T, _ptr(y), _ptr(pos), _ptr(residual),
                                       _ptr(residual_out), _stream(stream)), "moe_combine_residual")


def moe_read_status(workspace, stream=None) -> int:
    v = ctypes.c_int(0)
    _check(load().moe_read_status(_ptr(workspace), _stream(stream), ctypes.byref(v)), "moe_read_status")
    return v.value


def moe_read_status_detail(workspace, stream=None):
    """(status, wait site, block, progress) of the workspace's status record."""
    v = (ctypes.c_int * 4)()
    _check(load().moe_read_status_detail(_ptr(workspace), _stream(stream), v), "moe_read_status_detail")
    return tuple(int(x) for x in v)


def moe_debug_inject(what: int, wait_limit_ns: int = 0):
    """Test hook of the expert GEMMs' bounded waits (MOE_INJECT_*)."""
    _check(load().moe_debug_inject(what, wait_limit_ns), "moe_debug_inject")


def moe_profile_enable(on: bool):
    _check(load().moe_profile_enable(1 if on else 0), "moe_profile_enable")


def moe_profile_read() -> dict:
    """{kernel name: ms} of the most recent profiled moe_forward."""
    buf = (ctypes.c_float * 16)()
    n = ctypes.c_int(0)
    _check(load().moe_profile_read(buf, 16, ctypes.byref(n)), "moe_profile_read")
    lib = load()
    return {lib.moe_profile_kernel_name(i).decode(): float(buf[i]) for i in range(n.value)}


def moe_set_gemm_variant(variant: int):
    _check(load().moe_set_gemm_variant(variant), "moe_set_gemm_variant")


def moe_launch_count() -> int:
    """Kernels the library has launched in this process so far."""
    v = ctypes.c_uint64(0)
    _check(load().moe_launch_count(ctypes.byref(v)), "moe_launch_count")
    return v.value


def moe_device_sm_count() -> int:
    v = ctypes.c_int(0)
    _check(load().moe_device_sm_count(ctypes.byref(v)), "moe_device_sm_count")
    return v.value


# ---- plumbing: host arrays -> device tensors ----

def to_device(a, device="cuda"):
    """A numpy array (uint16 bf16 bits, uint8 E4M3 codes, int32, fp32) as a device tensor."""
    import numpy as np
    import torch
    if a is None:
        return None
    if a.dtype == np.uint16:
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(a))
    return t.to(device, non_blocking=False)


def upload_weights(w: dict, device="cuda") -> dict:
    """Device copies of a weight dict (keys as in moe_weights); None stays None."""
    return {k: to_device(v, device) for k, v in w.items()}
