"""The grouped GEMM stage on exact integer inputs, and the bounded-wait error path.

Integer inputs: with E4M3 (or bf16) codes in {-4..4} and unit scales every
product and every partial sum is an integer far below 2^24, so an fp32
accumulation is exact whatever its order, and the grouped GEMMs must return
the integer result bit for bit. The expected values are the plain definition
(an int64 matrix product per group); the gate/up GEMM is read before its
SwiGLU (MOE_STAGE_GATE_UP_RAW), the down GEMM through its bf16 output with
power-of-two row gates (one exact scaling, then one round-to-nearest-even).
Every GEMM variant (single CTAs, 2-SM pairs, and for FP8 the swapped-operand
kernel that runs groups in 32-row chunks) runs the same rows.

Bounded waits: moe_debug_inject(MOE_INJECT_GEMM_NO_LOADS) makes the expert
GEMMs' producer issue no loads, so their consumers' waits run out; the call
must latch MOE_ERR_DEVICE_TIMEOUT with the wait site, every kernel must return,
and the same process must then compute the layer correctly again.
"""
import numpy as np
import pytest

import oracle
import synth
from conftest import cuda_available
from parity import bf16_bits_to_f64, frob_rel, tol_for

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module")
def m():
    import mixture_experts_histogram_b200 as mm
    from mixture_experts_histogram_b200 import build
    build.build()
    mm.load()
    return mm


@pytest.fixture(params=["single", "pair", "swap"])
def variant(request, m):
    m.moe_set_gemm_variant({"single": m.MOE_GEMM_SINGLE, "pair": m.MOE_GEMM_PAIR, "swap": m.MOE_GEMM_SWAP}[request.param])
    yield request.param
    m.moe_set_gemm_variant(m.MOE_GEMM_AUTO)


H, I, E = 512, 256, 5
# Rows per group (routed experts 0..4, then the shared expert): empty, one row,
# one past a 128-row tile, several tiles with a ragged end, a whole tile.
COUNTS = [0, 1, 129, 300, 64, 200]


def _codes(values: np.ndarray, fp8: bool) -> np.ndarray:
    """Exact E4M3 codes (uint8) or bf16 bits (uint16) of small integers."""
    v = values.astype(np.float32)
    return oracle.e4m3_encode(v) if fp8 else synth.f32_to_bf16(v)


def _ints(seed, shape):
    return np.random.default_rng(seed).integers(-4, 5, size=shape).astype(np.int64)


def _setup(m, fp8):
    import torch
    wd = synth.WDTYPE_FP8 if fp8 else synth.WDTYPE_BF16
    cfg = m.make_config(H, E, 2, 1, I, wd)
    w1, w3, w2 = _ints(1, (E + 1, I, H)), _ints(2, (E + 1, I, H)), _ints(3, (E + 1, H, I))
    host = {"router_w": synth.normal_bf16(0, 1, (E, H), 0.05), "router_bias": None,
            "w1": _codes(w1[:E], fp8), "w3": _codes(w3[:E], fp8), "w2": _codes(w2[:E], fp8),
            "sw1": _codes(w1[E:], fp8), "sw3": _codes(w3[E:], fp8), "sw2": _codes(w2[E:], fp8)}
    for k, shp in (("s1", (E, I // 128, H // 128)), ("s3", (E, I // 128, H // 128)), ("s2", (E, H // 128, I // 128)),
                   ("ss1", (1, I // 128, H // 128)), ("ss3", (1, I // 128, H // 128)),
                   ("ss2", (1, H // 128, I // 128))):
        host[k] = np.ones(shp, np.float32) if fp8 else None
    dev = m.upload_weights(host)
    offsets = np.concatenate([[0], np.cumsum(COUNTS)]).astype(np.int32)
    R = int(offsets[-1])
    group = np.repeat(np.arange(E + 1), COUNTS)
    ws = torch.empty(m.moe_workspace_bytes(cfg, -(-R // 3)), dtype=torch.uint8, device="cuda")
    return cfg, dev, (w1, w3, w2), offsets, R, group, ws


@pytest.mark.parametrize("fp8", [True, False], ids=["fp8", "bf16"])
def test_gate_up_integer_inputs_bit_exact(m, fp8, variant):
    import torch
    cfg, dev, (w1, w3, _), offsets, R, group, ws = _setup(m, fp8)
    a = _ints(4, (R, H))
    out = torch.full((R, 2, I), float("nan"), dtype=torch.float32, device="cuda")
    a_scale = m.to_device(np.ones((R, H // 128), np.float32)) if fp8 else None
    m.moe_grouped_gemm(cfg, m.MOE_STAGE_GATE_UP_RAW, R, m.to_device(offsets), m.to_device(_codes(a, fp8)), a_scale,
                       m.make_weights(dev), out, ws)
    assert m.moe_read_status(ws) == 0
    got = out.cpu().numpy()
    ref = np.empty((R, 2, I), np.int64)
    for g in range(E + 1):
        rr = group == g
        ref[rr, 0] = a[rr] @ w1[g].T
        ref[rr, 1] = a[rr] @ w3[g].T
    assert np.abs(ref).max() < 2 ** 24
    bad = np.argwhere(got != ref.astype(np.float32))
    assert bad.size == 0, f"{len(bad)} sums differ, first {bad[:4].tolist()}"


def test_gate_up_h_codes_bit_exact(m, variant):
    """FP8 gate/up GEMM through SwiGLU and the 1x128 quantisation of h, on
    inputs that make every step exact: positive activations and W1 = 1 put each
    gate sum at 512..1024, where exp(-g) underflows and silu(g) = g exactly in
    fp32, and g * u stays an integer below 2^24. The codes then follow from the
    block quantisation alone (scale = amax/448, codes = E4M3 of h * (1/scale),
    ties to even, saturating), for every row position of a tile, including the
    ragged ends of groups."""
    import torch
    cfg, _, _, offsets, R, group, ws = _setup(m, True)
    rng = np.random.default_rng(21)
    a = rng.integers(1, 3, size=(R, H)).astype(np.int64)
    w1 = np.ones((E + 1, I, H), np.int64)
    w3 = rng.integers(-2, 3, size=(E + 1, I, H)).astype(np.int64)
    host = {"router_w": synth.normal_bf16(0, 1, (E, H), 0.05), "router_bias": None,
            "w1": _codes(w1[:E], True), "w3": _codes(w3[:E], True), "w2": _codes(np.ones((E, H, I)), True),
            "sw1": _codes(w1[E:], True), "sw3": _codes(w3[E:], True), "sw2": _codes(np.ones((1, H, I)), True)}
    for k, shp in (("s1", (E, I // 128, H // 128)), ("s3", (E, I // 128, H // 128)), ("s2", (E, H // 128, I // 128)),
                   ("ss1", (1, I // 128, H // 128)), ("ss3", (1, I // 128, H // 128)),
                   ("ss2", (1, H // 128, I // 128))):
        host[k] = np.ones(shp, np.float32)
    dev = m.upload_weights(host)
    h = torch.zeros((R, I), dtype=torch.uint8, device="cuda")
    hs = torch.zeros((R, I // 128), dtype=torch.float32, device="cuda")
    m.moe_grouped_gemm(cfg, m.MOE_STAGE_GATE_UP, R, m.to_device(offsets), m.to_device(_codes(a, True)),
                       m.to_device(np.ones((R, H // 128), np.float32)), m.make_weights(dev), h, ws, out_scale=hs)
    assert m.moe_read_status(ws) == 0
    hv = np.empty((R, I), np.float64)
    for g in range(E + 1):
        rr = group == g
        gs, us = a[rr] @ w1[g].T, a[rr] @ w3[g].T
        assert gs.size == 0 or gs.min() >= 512
        hv[rr] = (gs * us).astype(np.float64)
    assert np.abs(hv).max() < 2 ** 24
    hb = hv.astype(np.float32).reshape(R, I // 128, 128)
    amax = np.abs(hb).max(axis=2)
    scale = np.where(amax > 0, amax / np.float32(448), np.float32(1)).astype(np.float32)
    inv = np.where(amax > 0, np.float32(1) / scale, np.float32(0)).astype(np.float32)
    want = oracle.e4m3_encode((hb * inv[:, :, None]).astype(np.float32)).reshape(R, I)
    got_s = hs.cpu().numpy()
    assert np.array_equal(got_s.view(np.uint32), scale.view(np.uint32))
    got = h.cpu().numpy()
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{len(bad)} codes differ, first {bad[:4].tolist()}"


@pytest.mark.parametrize("fp8", [True, False], ids=["fp8", "bf16"])
def test_down_integer_inputs_bit_exact(m, fp8, variant):
    import torch
    cfg, dev, (_, _, w2), offsets, R, group, ws = _setup(m, fp8)
    a = _ints(5, (R, I))
    gate = np.random.default_rng(6).choice(np.array([0.25, 0.5, 1.0, 2.0], np.float32), size=R)
    y = torch.empty((R, H), dtype=torch.bfloat16, device="cuda")
    a_scale = m.to_device(np.ones((R, I // 128), np.float32)) if fp8 else None
    m.moe_grouped_gemm(cfg, m.MOE_STAGE_DOWN, R, m.to_device(offsets), m.to_device(_codes(a, fp8)), a_scale,
                       m.make_weights(dev), y, ws, row_gate=m.to_device(gate))
    assert m.moe_read_status(ws) == 0
    got = y.view(torch.int16).cpu().numpy().view(np.uint16)
    ref = np.empty((R, H), np.float64)
    for g in range(E + 1):
        rr = group == g
        ref[rr] = (a[rr] @ w2[g].T).astype(np.float64)
    ref *= gate[:, None].astype(np.float64)
    assert np.abs(ref).max() < 2 ** 24
    want = synth.f32_to_bf16(ref.astype(np.float32))  # exact in fp32, one rounding to bf16
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{len(bad)} outputs differ, first {bad[:4].tolist()}"


def test_down_staged_stores_integer_inputs_bit_exact(m, variant):
    """FP8 down GEMM with groups averaging a whole tile, so its y tiles leave
    through shared memory and TMA stores: 32-row quarters wholly inside a group
    are stored as boxes, the quarter straddling a group's end row by row (group
    sizes 1, 300, 129, 256 and 200 put that end at every quarter offset). Rows
    of one group written into the next would break the neighbour's sums."""
    import torch
    counts = [0, 1, 300, 129, 256, 200]
    cfg, dev, (_, _, w2), *_ = _setup(m, True)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R = int(offsets[-1])
    assert R >= 128 * (E + 1)
    group = np.repeat(np.arange(E + 1), counts)
    ws = torch.empty(m.moe_workspace_bytes(cfg, -(-R // 3)), dtype=torch.uint8, device="cuda")
    a = _ints(7, (R, I))
    gate = np.random.default_rng(8).choice(np.array([0.25, 0.5, 1.0, 2.0], np.float32), size=R)
    y = torch.full((R, H), float("nan"), dtype=torch.bfloat16, device="cuda")
    m.moe_grouped_gemm(cfg, m.MOE_STAGE_DOWN, R, m.to_device(offsets), m.to_device(_codes(a, True)),
                       m.to_device(np.ones((R, I // 128), np.float32)), m.make_weights(dev), y, ws,
                       row_gate=m.to_device(gate))
    assert m.moe_read_status(ws) == 0
    got = y.view(torch.int16).cpu().numpy().view(np.uint16)
    ref = np.empty((R, H), np.float64)
    for g in range(E + 1):
        rr = group == g
        ref[rr] = (a[rr] @ w2[g].T).astype(np.float64)
    ref *= gate[:, None].astype(np.float64)
    want = synth.f32_to_bf16(ref.astype(np.float32))
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{len(bad)} outputs differ, first {bad[:4].tolist()}"


@pytest.mark.parametrize("fp8", [True, False], ids=["fp8", "bf16"])
def test_down_split_k_integer_inputs_bit_exact(m, fp8, variant):
    """One group of 50 rows under a 64-row call, K = 2048, H = 512: two output
    tiles for the whole GPU, so the down GEMM splits K (4 pieces FP8, 8 BF16)
    and sums the pieces afterwards; integer sums stay exact in any order, and
    the 14 rows past the group's end are left untouched."""
    import torch
    h, i2, r, valid = 512, 2048, 64, 50
    wd = synth.WDTYPE_FP8 if fp8 else synth.WDTYPE_BF16
    cfg = m.make_config(h, 1, 1, 0, i2, wd)
    w1, w3, w2 = _ints(11, (1, i2, h)), _ints(12, (1, i2, h)), _ints(13, (1, h, i2))
    host = {"router_w": synth.normal_bf16(0, 1, (1, h), 0.05), "router_bias": None,
            "w1": _codes(w1, fp8), "w3": _codes(w3, fp8), "w2": _codes(w2, fp8),
            "s1": np.ones((1, i2 // 128, h // 128), np.float32) if fp8 else None,
            "s3": np.ones((1, i2 // 128, h // 128), np.float32) if fp8 else None,
            "s2": np.ones((1, h // 128, i2 // 128), np.float32) if fp8 else None}
    dev = m.upload_weights(host)
    ws = torch.empty(m.moe_workspace_bytes(cfg, r), dtype=torch.uint8, device="cuda")
    a = _ints(14, (r, i2))
    gate = np.random.default_rng(15).choice(np.array([0.25, 0.5, 1.0, 2.0], np.float32), size=r)
    y = torch.full((r, h), 7.0, dtype=torch.bfloat16, device="cuda")
    a_scale = m.to_device(np.ones((r, i2 // 128), np.float32)) if fp8 else None
    m.moe_grouped_gemm(cfg, m.MOE_STAGE_DOWN, r, m.to_device(np.array([0, valid], np.int32)),
                       m.to_device(_codes(a, fp8)), a_scale, m.make_weights(dev), y, ws, row_gate=m.to_device(gate))
    assert m.moe_read_status(ws) == 0
    got = y.view(torch.int16).cpu().numpy().view(np.uint16)
    ref = (a[:valid] @ w2[0].T).astype(np.float64) * gate[:valid, None].astype(np.float64)
    assert np.abs(ref).max() < 2 ** 24
    bad = np.argwhere(got[:valid] != synth.f32_to_bf16(ref.astype(np.float32)))
    assert bad.size == 0, f"{len(bad)} outputs differ, first {bad[:4].tolist()}"
    assert (got[valid:] == synth.f32_to_bf16(np.float32(7.0))).all()


def test_grouped_gemm_rejects_bad_offsets(m):
    import torch
    cfg, dev, _, offsets, R, _, ws = _setup(m, True)
    bad = offsets.copy()
    bad[3] = bad[2] - 1  # a decreasing offset
    out = torch.zeros((R, 2, I), dtype=torch.float32, device="cuda")
    m.moe_grouped_gemm(cfg, m.MOE_STAGE_GATE_UP_RAW, R, m.to_device(bad), m.to_device(_codes(_ints(4, (R, H)), True)),
                       m.to_device(np.ones((R, H // 128), np.float32)), m.make_weights(dev), out, ws)
    assert m.moe_read_status(ws) == m.MOE_ERR_INVALID_ARG
    assert torch.count_nonzero(out).item() == 0  # nothing computed


# ------------------------------------------------------------ bounded waits --

SHAPE = synth.MoeShape("timeout-fp8", T=300, hidden=512, n_experts=24, top_k=4, n_shared=1, inter=384,
                       wdtype=synth.WDTYPE_FP8, seed=30)


@pytest.mark.parametrize("wdtype", [synth.WDTYPE_FP8, synth.WDTYPE_BF16], ids=["fp8", "bf16"])
def test_timed_out_wait_latches_status_and_the_device_recovers(m, variant, wdtype):
    import dataclasses
    import torch
    shape = dataclasses.replace(SHAPE, wdtype=wdtype)
    x, w = synth.make_x(shape), synth.make_weights(shape)
    idx_r, gate_r, _ = oracle.route(x, w["router_w"], w["router_bias"], shape.top_k)
    cfg = m.make_config(shape.hidden, shape.n_experts, shape.top_k, shape.n_shared, shape.inter, shape.wdtype)
    T, S = shape.T, shape.top_k + shape.n_shared
    wd = m.upload_weights(w)
    args = (m.to_device(x), m.to_device(idx_r), m.to_device(gate_r), m.make_weights(wd))
    y = torch.zeros((S * T, shape.hidden), dtype=torch.bfloat16, device="cuda")
    pos = torch.empty((T, S), dtype=torch.int32, device="cuda")
    ws = torch.empty(m.moe_workspace_bytes(cfg, T), dtype=torch.uint8, device="cuda")
    m.moe_debug_inject(m.MOE_INJECT_GEMM_NO_LOADS, 50_000_000)  # 50 ms
    try:
        m.moe_experts(cfg, T, args[0], args[1], args[2], args[3], y, pos, ws)
        status, site, block, _ = m.moe_read_status_detail(ws)  # synchronises: every kernel returned
    finally:
        m.moe_debug_inject(m.MOE_INJECT_NONE, 0)
    assert status == m.MOE_ERR_DEVICE_TIMEOUT
    fp8_bit = 0x100 if wdtype == synth.WDTYPE_FP8 else 0
    assert (site & 0x300) == (0x200 | fp8_bit), hex(site)  # the gate/up GEMM's wait, first in launch order
    assert (site & 0xF) in (4, 5, 6), hex(site)            # an MMA or epilogue wait on loads that never came
    assert 0 <= block < 1024

    # The same process and device, normal operation: correct results again.
    m.moe_experts(cfg, T, args[0], args[1], args[2], args[3], y, pos, ws)
    assert m.moe_read_status(ws) == 0
    _, _, y_r = oracle.moe_tokens(shape, w, x, idx_r, gate_r, want_y=True)
    gates = np.concatenate([gate_r.astype(np.float64), np.ones((T, shape.n_shared))], axis=1)
    got = bf16_bits_to_f64(y.view(torch.int16).cpu().numpy().view(np.uint16))[pos.cpu().numpy().reshape(-1)]
    assert frob_rel(got.reshape(T, S, -1), y_r * gates[:, :, None]) < tol_for(wdtype)
