"""CPU oracle for the Step-5 routed-MoE layer forward (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this. It is a thin ctypes/numpy wrapper around
``oracle.c`` (plain C, fp64 accumulation), which shares no code with the CUDA
library; the one thing both sides use is the seeded input generator in
``synth``.

Functions and the passages they follow:
  route            learned router + top-k + renormalised gates (NeMo
                   "Step-5-Preview" page, "Model Architecture" table)
  quantize_rows    1x128 E4M3 activation blocks (StepFun "Step-5 minimal
                   inference" README: block-scaled FP8 expert GEMM)
  e2m1_decode, nvfp4_dequantize
                   NVFP4 weights: E2M1 codes two to a byte, an E4M3 scale per
                   16 inputs, an fp32 global scale (TensorFold PR page, the
                   NVFP4 format of its W4A16 linears)
  permute          token->expert histogram, exclusive scan and gather indices
                   (README: the "critical MoE primitives")
  moe_tokens       expert SwiGLU MLPs and the weighted combine, fp64 sums in
                   slot order (README, "Long-output stability": fixed-order
                   accumulation in at least fp32)
  expert_rows      single (token, expert) output rows, the per-row evaluation
                   of moe_tokens (same README row)
  moe_forward      route + moe_tokens for a whole batch (or a token sample)
  ep_partial       one expert-parallel rank's share of the output (README,
                   deployment at TP = EP and "Long-output stability")
  rmsnorm          the fp32 residual stream normalised into the layer's bf16
                   input (NeMo "Step-5-Preview" page, "Full-Depth H100
                   Benchmark" table: FP32 norms and residuals)
  add_residual     the layer output added back into the fp32 residual stream
                   (same table; "Attention and Precision": FP32 residual stream)
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "_oracle.so")
_lib = None

ERR_BAD_INDEX = 5


class _Shape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("H", ctypes.c_int32), ("E", ctypes.c_int32), ("k", ctypes.c_int32),
                ("n_shared", ctypes.c_int32), ("I", ctypes.c_int32), ("wdtype", ctypes.c_int32)]


class _Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("router_w", "router_bias", "w1", "w3", "w2", "s1", "s3", "s2",
                 "sw1", "sw3", "sw2", "ss1", "ss3", "ss2", "g1", "g3", "g2", "sg1", "sg3", "sg2")]


def build(force: bool = False) -> str:
    """Compile oracle.c into _oracle.so (gcc, OpenMP)."""
    src = os.path.join(_HERE, "oracle.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", _SO, src, "-lm"])
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
        lib.orc_num_threads.argtypes = []
        lib.orc_num_threads.restype = ctypes.c_int
        lib.orc_e4m3_value.argtypes = [ctypes.c_uint8]
        lib.orc_e4m3_value.restype = ctypes.c_double
        lib.orc_e2m1_value.argtypes = [ctypes.c_uint8]
        lib.orc_e2m1_value.restype = ctypes.c_double
        lib.orc_e4m3_encode.argtypes = [ctypes.c_float]
        lib.orc_e4m3_encode.restype = ctypes.c_uint8
        lib.orc_e4m3_encode_array.argtypes = [i64, vp, vp]
        lib.orc_e4m3_decode_array.argtypes = [i64, vp, vp]
        lib.orc_quantize_rows.argtypes = [i64, i32, vp, vp, vp]
        lib.orc_route.argtypes = [i64, i32, i32, i32, vp, vp, vp, vp, vp, vp]
        lib.orc_permute.argtypes = [i64, i32, i32, i32, vp, vp, vp, vp, vp]
        lib.orc_permute.restype = ctypes.c_int
        lib.orc_moe_tokens.argtypes = [ctypes.POINTER(_Shape), ctypes.POINTER(_Weights), vp, vp, vp, i64, vp,
                                       vp, vp, vp]
        lib.orc_expert_rows.argtypes = [ctypes.POINTER(_Shape), ctypes.POINTER(_Weights), vp, i64, vp, vp, vp]
        _lib = lib
    return _lib


def _p(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data


# ------------------------------------------------------------------ E4M3 ----

def num_threads() -> int:
    """Threads the oracle's OpenMP loops use (reported beside its timings)."""
    return int(_load().orc_num_threads())


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Exact values (float64) of E4M3 codes (uint8)."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, dtype=np.float64)
    _load().orc_e4m3_decode_array(c.size, _p(c), _p(out))
    return out


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    """Exact values (float64) of 4-bit E2M1 codes (the low nibble of each uint8)."""
    c = np.asarray(codes, dtype=np.uint8) & 15
    lib = _load()
    table = np.array([lib.orc_e2m1_value(i) for i in range(16)], dtype=np.float64)
    return table[c]


def nvfp4_dequantize(codes: np.ndarray, scales: np.ndarray, global_scale: float) -> np.ndarray:
    """One NVFP4 matrix: codes [n, k/2] (input 2j in byte j's low nibble),
    E4M3 scales [n, k/16], global fp32 scale -> float64 [n, k]."""
    lo = e2m1_decode(codes & 15)
    hi = e2m1_decode(codes >> 4)
    v = np.stack([lo, hi], axis=-1).reshape(codes.shape[0], codes.shape[1] * 2)
    s = np.repeat(e4m3_decode(scales), 16, axis=1)
    return v * s * float(global_scale)


def e4m3_encode(values: np.ndarray) -> np.ndarray:
    """E4M3 codes of float32 values: nearest, ties to even, saturating at 448."""
    v = np.ascontiguousarray(values, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    _load().orc_e4m3_encode_array(v.size, _p(v), _p(out))
    return out


def quantize_rows(x_bf16: np.ndarray):
    """x [T, H] bf16 bits -> (codes uint8 [T, H], scales fp32 [T, H/128])."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    T, H = x.shape
    q = np.empty((T, H), dtype=np.uint8)
    s = np.empty((T, H // 128), dtype=np.float32)
    _load().orc_quantize_rows(T, H, _p(x), _p(q), _p(s))
    return q, s


# --------------------------------------------------------------- routing ----

def route(x_bf16: np.ndarray, router_w: np.ndarray, router_bias: Optional[np.ndarray], k: int,
          want_logits: bool = False):
    """Top-k routing. Returns (idx int32 [T,k], gate fp32 [T,k], logits f64 [T,E] or None)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    wr = np.ascontiguousarray(router_w, dtype=np.uint16)
    T, H = x.shape
    E = wr.shape[0]
    b = None if router_bias is None else np.ascontiguousarray(router_bias, dtype=np.float32)
    idx = np.empty((T, k), dtype=np.int32)
    gate = np.empty((T, k), dtype=np.float32)
    logits = np.empty((T, E), dtype=np.float64) if want_logits else None
    _load().orc_route(T, H, E, k, _p(x), _p(wr), _p(b), _p(logits), _p(idx), _p(gate))
    return idx, gate, logits


def permute(idx: np.ndarray, n_experts: int, n_shared: int = 1):
    """Histogram/scan/gather indices: (counts, offsets, perm, pos)."""
    ii = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = ii.shape
    G, S = n_experts + n_shared, k + n_shared
    counts = np.empty(G, dtype=np.int32)
    offsets = np.empty(G + 1, dtype=np.int32)
    perm = np.empty(S * T, dtype=np.int32)
    pos = np.empty((T, S), dtype=np.int32)
    rc = _load().orc_permute(T, n_experts, k, n_shared, _p(ii), _p(counts), _p(offsets), _p(perm), _p(pos))
    if rc != 0:
        raise ValueError(f"oracle permute: status {rc}")
    return counts, offsets, perm, pos


# ---------------------------------------------------------- layer output ----

def _weights_struct(w: dict):
    keep = []

    def q(name):
        a = w.get(name)
        if a is None:
            return None
        a = np.ascontiguousarray(a)
        keep.append(a)
        return a.ctypes.data

    ws = _Weights(*[q(n) for n, _ in _Weights._fields_])
    return ws, keep


def moe_tokens(shape, weights: dict, x_bf16: np.ndarray, idx: np.ndarray, gate: np.ndarray,
               tokens: Optional[Sequence[int]] = None, want_y: bool = False):
    """Layer output for `tokens` (default: all) given the routing.

    Returns (out_f64 [n,H], out_bf16 [n,H] uint16, y_f64 [n, k+S, H] or None).
    """
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    T, H = x.shape
    toks = np.arange(T, dtype=np.int64) if tokens is None else np.ascontiguousarray(tokens, dtype=np.int64)
    n = toks.size
    S = shape.top_k + shape.n_shared
    sh = _Shape(T, shape.hidden, shape.n_experts, shape.top_k, shape.n_shared, shape.inter, shape.wdtype)
    ws, keep = _weights_struct(weights)
    ii = np.ascontiguousarray(idx, dtype=np.int32)
    gg = np.ascontiguousarray(gate, dtype=np.float32)
    out = np.empty((n, H), dtype=np.float64)
    outb = np.empty((n, H), dtype=np.uint16)
    y = np.empty((n, S, H), dtype=np.float64) if want_y else None
    _load().orc_moe_tokens(ctypes.byref(sh), ctypes.byref(ws), _p(x), _p(ii), _p(gg), n, _p(toks), _p(out),
                           _p(outb), _p(y))
    del keep
    return out, outb, y


def expert_rows(shape, weights: dict, x_bf16: np.ndarray, tokens: Sequence[int], groups: Sequence[int]):
    """Ungated output rows y [n, H] (f64) of group groups[i] on token tokens[i].

    Groups 0..E-1 are the routed experts and group E the shared expert; the
    same per-row evaluation as moe_tokens, for chosen rows of a large batch.
    """
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    T, H = x.shape
    toks = np.ascontiguousarray(tokens, dtype=np.int64)
    grp = np.ascontiguousarray(groups, dtype=np.int32)
    assert toks.shape == grp.shape and toks.ndim == 1
    assert np.all((toks >= 0) & (toks < T)) and np.all((grp >= 0) & (grp <= shape.n_experts))
    assert shape.n_shared == 1 or np.all(grp < shape.n_experts)
    sh = _Shape(T, shape.hidden, shape.n_experts, shape.top_k, shape.n_shared, shape.inter, shape.wdtype)
    ws, keep = _weights_struct(weights)
    y = np.empty((toks.size, H), dtype=np.float64)
    _load().orc_expert_rows(ctypes.byref(sh), ctypes.byref(ws), _p(x), toks.size, _p(toks), _p(grp), _p(y))
    del keep
    return y


def moe_forward(shape, weights: dict, x_bf16: np.ndarray, tokens: Optional[Sequence[int]] = None):
    """Whole layer: routing for every token, outputs for `tokens` (default all).

    Returns dict(idx, gate, logits, out_f64, out_bf16).
    """
    idx, gate, logits = route(x_bf16, weights["router_w"], weights.get("router_bias"), shape.top_k,
                              want_logits=True)
    out, outb, _ = moe_tokens(shape, weights, x_bf16, idx, gate, tokens)
    return {"idx": idx, "gate": gate, "logits": logits, "out_f64": out, "out_bf16": outb}


# ------------------------------------------------------ expert parallelism --

def ep_partial(shape, weights: dict, x_bf16: np.ndarray, idx: np.ndarray, gate: np.ndarray, e0: int, e1: int,
               t0: int, t1: int, tokens: Optional[Sequence[int]] = None) -> np.ndarray:
    """One expert-parallel rank's share of the output, fp64 [n, H]: for each
    token, the gate-weighted rows of its routed experts inside [e0, e1), in
    slot order, plus its shared-expert row if the token lies in [t0, t1)
    (StepFun README, deployment at TP = EP: each rank holds a range of the
    routed experts; the ranks' partial results are added in rank order).
    Summed over ranks whose ranges partition the experts and the tokens, the
    partials give moe_tokens' output."""
    toks = np.arange(x_bf16.shape[0], dtype=np.int64) if tokens is None else np.asarray(tokens, dtype=np.int64)
    _, _, y = moe_tokens(shape, weights, x_bf16, idx, gate, tokens=toks, want_y=True)
    k = shape.top_k
    out = np.zeros((toks.size, shape.hidden), dtype=np.float64)
    for n, t in enumerate(toks):
        for j in range(k):
            if e0 <= idx[t, j] < e1:
                out[n] += float(gate[t, j]) * y[n, j]
        if shape.n_shared and t0 <= t < t1:
            out[n] += y[n, k]
    return out


# ---------------------------------------------------------- residual stream --

def rmsnorm(residual: np.ndarray, weight: np.ndarray, eps: float) -> np.ndarray:
    """y = r / sqrt(mean(r^2) + eps) * w per row, in fp64 (r: [T, H] fp32, w: [H]).

    The pages fix only that norms are fp32; the norm type (RMS, no mean
    subtraction, no bias) and eps follow the usual decoder reading.
    """
    r = residual.astype(np.float64)
    ms = np.mean(r * r, axis=1, keepdims=True)
    return r / np.sqrt(ms + eps) * weight.astype(np.float64)[None, :]


def add_residual(residual: np.ndarray, y_rows: np.ndarray, pos: np.ndarray) -> np.ndarray:
    """r_out[t] = r[t] + sum_j y[pos[t, j]] in fp64 (slots in order; pos < 0 skipped)."""
    out = residual.astype(np.float64).copy()
    T, S = pos.shape
    for t in range(T):
        acc = np.zeros(residual.shape[1], np.float64)
        for j in range(S):
            if pos[t, j] >= 0:
                acc += y_rows[pos[t, j]].astype(np.float64)
        out[t] += acc
    return out
