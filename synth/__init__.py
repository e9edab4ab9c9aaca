"""Seeded synthetic inputs for the Step-5 routed-MoE layer.

Shared by the CPU oracle's tests and the benchmark. It only makes inputs (the
counter-based generator in ``synth.c``); none of the layer's forward arithmetic
lives here.

Workloads follow the layer geometry of the NeMo AutoModel "Step-5-Preview"
page ("Model Architecture" table: hidden 4,096, 352 routed experts per MoE
layer, top-8 routing, one shared expert, expert intermediate 1,536) and the
expert storage formats of the StepFun "Step-5 minimal inference" README
(BF16 experts, or block-scaled FP8 E4M3 experts).

Recipe (all seeded; the values never depend on thread count):
  x          ~ N(0, 1)            -> bf16,   [T, H]
  router_w   ~ N(0, 1/H)          -> bf16,   [E, H]
  w1, w3     ~ N(0, 1/H)          -> bf16,   [E, I, H]   (gate, up; nn.Linear [out, in])
  w2         ~ N(0, 1/I)          -> bf16,   [E, H, I]   (down)
  shared sw1, sw3, sw2: same laws, E = 1, their own tensor ids
  FP8 storage: the same bf16 draws quantised per 128x128 block,
               scale = blockmax/448 (fp32), codes E4M3 round-to-nearest-even.
  NVFP4 storage: the same bf16 draws; per matrix a global fp32 scale
               amax/(6*448); per 16 inputs an E4M3 scale of blockmax/(6*global);
               E2M1 codes (nearest, ties to even, saturating), two to a byte.
  Skewed routing: router_bias[e] = -1.1 * alpha * ln(r_e), r a seeded random
               permutation of 1..E (Zipf exponent 1.1 over a random expert
               ranking); alpha = 0.25 makes the hottest expert take about ten
               times the mean load when logits are unit normal.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "_synth.so")
_lib = None

# Tensor ids of the counter-based streams.
ID_X, ID_ROUTER_W, ID_ROUTER_RANK = 1, 2, 3
ID_W1, ID_W3, ID_W2 = 10, 11, 12
ID_SW1, ID_SW3, ID_SW2 = 20, 21, 22

ZIPF_S = 1.1
ZIPF_ALPHA = 0.25

WDTYPE_BF16, WDTYPE_FP8, WDTYPE_NVFP4 = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile synth.c into _synth.so (gcc, OpenMP)."""
    src = os.path.join(_HERE, "synth.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", _SO, src, "-lm"])
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        u64, i64, dbl, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        lib.synth_normal_bf16.argtypes = [u64, u64, i64, dbl, vp]
        lib.synth_normal_f32.argtypes = [u64, u64, i64, dbl, vp]
        lib.synth_u64.argtypes = [u64, u64, i64, vp]
        lib.synth_fp8_blocks.argtypes = [u64, u64, i64, i64, i64, dbl, vp, vp]
        lib.synth_e4m3_value.argtypes = [ctypes.c_uint8]
        lib.synth_e4m3_value.restype = ctypes.c_float
        lib.synth_e2m1_value.argtypes = [ctypes.c_uint8]
        lib.synth_e2m1_value.restype = ctypes.c_float
        lib.synth_nvfp4.argtypes = [u64, u64, i64, i64, i64, dbl, vp, vp, vp]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def normal_bf16(seed: int, tid: int, shape, std: float) -> np.ndarray:
    """bf16 bit patterns (uint16) of std * N(0,1), element-indexed in C order."""
    out = np.empty(shape, dtype=np.uint16)
    _load().synth_normal_bf16(seed, tid, out.size, float(std), _ptr(out))
    return out


def normal_f32(seed: int, tid: int, shape, std: float) -> np.ndarray:
    out = np.empty(shape, dtype=np.float32)
    _load().synth_normal_f32(seed, tid, out.size, float(std), _ptr(out))
    return out


def uniform_u64(seed: int, tid: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    _load().synth_u64(seed, tid, n, _ptr(out))
    return out


def fp8_blocks(seed: int, tid: int, G: int, rows: int, cols: int, std: float):
    """Block-scaled E4M3 version of normal_bf16(seed, tid, (G, rows, cols), std).

    Returns (codes uint8 [G, rows, cols], scales fp32 [G, rows/128, cols/128]).
    """
    assert rows % 128 == 0 and cols % 128 == 0
    codes = np.empty((G, rows, cols), dtype=np.uint8)
    scales = np.empty((G, rows // 128, cols // 128), dtype=np.float32)
    _load().synth_fp8_blocks(seed, tid, G, rows, cols, float(std), _ptr(codes), _ptr(scales))
    return codes, scales


def nvfp4(seed: int, tid: int, G: int, rows: int, cols: int, std: float):
    """NVFP4 version of normal_bf16(seed, tid, (G, rows, cols), std).

    Returns (codes uint8 [G, rows, cols/2], E4M3 scales uint8 [G, rows, cols/16],
    global scales fp32 [G]).
    """
    assert cols % 16 == 0
    codes = np.empty((G, rows, cols // 2), dtype=np.uint8)
    scales = np.empty((G, rows, cols // 16), dtype=np.uint8)
    gs = np.empty(G, dtype=np.float32)
    _load().synth_nvfp4(seed, tid, G, rows, cols, float(std), _ptr(codes), _ptr(scales), _ptr(gs))
    return codes, scales, gs


def e2m1_value_table() -> np.ndarray:
    """The generator's own decoding of all 16 E2M1 codes."""
    lib = _load()
    return np.array([lib.synth_e2m1_value(c) for c in range(16)], dtype=np.float32)


def e4m3_value_table() -> np.ndarray:
    """The generator's own decoding of all 256 E4M3 codes (for input checks)."""
    lib = _load()
    return np.array([lib.synth_e4m3_value(c) for c in range(256)], dtype=np.float32)


@dataclasses.dataclass(frozen=True)
class MoeShape:
    """One workload of the layer: tokens, geometry, storage and seed."""

    name: str
    T: int
    hidden: int = 4096
    n_experts: int = 352
    top_k: int = 8
    n_shared: int = 1
    inter: int = 1536
    wdtype: int = WDTYPE_BF16
    seed: int = 0
    skew: bool = False

    def with_tokens(self, T: int) -> "MoeShape":
        return dataclasses.replace(self, T=T, name=f"{self.name.split('@')[0]}@T={T}")

    @property
    def rows(self) -> int:
        """Expert rows the layer computes: k routed pairs + n_shared per token."""
        return (self.top_k + self.n_shared) * self.T


# The workloads: a tiny correctness case and the Step-5 shapes.
TINY = MoeShape("tiny", T=32, hidden=256, n_experts=16, top_k=2, n_shared=1, inter=128,
                wdtype=WDTYPE_BF16, seed=0)
DECODE_BF16 = MoeShape("step5-decode-bf16", T=64, wdtype=WDTYPE_BF16, seed=1)
PREFILL_FP8 = MoeShape("step5-prefill-fp8", T=8192, wdtype=WDTYPE_FP8, seed=2)
LONG_SKEW_FP8 = MoeShape("step5-long-prefill-zipf-fp8", T=32768, wdtype=WDTYPE_FP8, seed=3, skew=True)
SWEEP_FP8 = MoeShape("step5-decode-sweep-fp8", T=64, wdtype=WDTYPE_FP8, seed=4)
SWEEP_TOKENS = (1, 8, 64, 512, 2048)
# The dense SwiGLU FFN of layers 0-2 and 91 (intermediate 13,824): the same layer
# with one expert, top-1 routing (gate 1) and no shared expert.
DENSE_FFN_FP8 = MoeShape("step5-dense-ffn-fp8", T=8192, n_experts=1, top_k=1, n_shared=0, inter=13824,
                         wdtype=WDTYPE_FP8, seed=5)

# The Step-5 layer with NVFP4 expert storage (W4A16), the storage variant of
# the TensorFold PR page, at the decode shape.
STEP5_NVFP4 = MoeShape("step5-nvfp4-w4a16", T=64, wdtype=WDTYPE_NVFP4, seed=6)

WORKLOADS = {w.name: w for w in (TINY, DECODE_BF16, PREFILL_FP8, LONG_SKEW_FP8, SWEEP_FP8, DENSE_FFN_FP8,
                                 STEP5_NVFP4)}


def zipf_bias(seed: int, E: int, alpha: float = ZIPF_ALPHA) -> np.ndarray:
    """Per-expert router bias -s*alpha*ln(rank) over a seeded random ranking."""
    keys = uniform_u64(seed, ID_ROUTER_RANK, E)
    order = np.argsort(keys, kind="stable")          # expert order[0] gets rank 1
    rank = np.empty(E, dtype=np.float64)
    rank[order] = np.arange(1, E + 1, dtype=np.float64)
    return (-ZIPF_S * alpha * np.log(rank)).astype(np.float32)


def make_x(shape: MoeShape) -> np.ndarray:
    return normal_bf16(shape.seed, ID_X, (shape.T, shape.hidden), 1.0)


def make_weights(shape: MoeShape) -> dict:
    """Router and expert weights for `shape` (numpy, host memory).

    BF16 storage: uint16 bf16 bit patterns. FP8 storage: uint8 E4M3 codes plus
    fp32 block scales. NVFP4 storage: packed E2M1 codes, E4M3 scales per 16
    inputs and fp32 global scales (g1, g3, g2, sg1, sg3, sg2). Keys: router_w,
    router_bias (None unless skewed), w1, w3, w2, s1, s3, s2, sw1, sw3, sw2,
    ss1, ss3, ss2, g1, g3, g2, sg1, sg3, sg2.
    """
    H, E, I, s = shape.hidden, shape.n_experts, shape.inter, shape.seed
    wt = {"router_w": normal_bf16(s, ID_ROUTER_W, (E, H), 1.0 / math.sqrt(H)),
          "router_bias": zipf_bias(s, E) if shape.skew else None}
    specs = [("w1", "s1", ID_W1, E, I, H, H), ("w3", "s3", ID_W3, E, I, H, H), ("w2", "s2", ID_W2, E, H, I, I)]
    if shape.n_shared:
        specs += [("sw1", "ss1", ID_SW1, 1, I, H, H), ("sw3", "ss3", ID_SW3, 1, I, H, H),
                  ("sw2", "ss2", ID_SW2, 1, H, I, I)]
    for wname, sname, tid, G, rows, cols, fan_in in specs:
        std = 1.0 / math.sqrt(fan_in)
        gname = ("s" if wname.startswith("sw") else "") + "g" + wname[-1]
        if shape.wdtype == WDTYPE_FP8:
            wt[wname], wt[sname] = fp8_blocks(s, tid, G, rows, cols, std)
        elif shape.wdtype == WDTYPE_NVFP4:
            wt[wname], wt[sname], wt[gname] = nvfp4(s, tid, G, rows, cols, std)
        else:
            wt[wname], wt[sname] = normal_bf16(s, tid, (G, rows, cols), std), None
    for k in ("sw1", "sw3", "sw2", "ss1", "ss3", "ss2", "g1", "g3", "g2", "sg1", "sg3", "sg2"):
        wt.setdefault(k, None)
    return wt


def bf16_to_f32(a: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float32 exactly."""
    return (a.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 bit patterns, nearest even (finite inputs)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)
