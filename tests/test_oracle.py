"""Pins for the CPU oracle: closed forms, library routines, brute force, invariants.

Each check ties the oracle to something other than itself, chosen so that a
plausible slip (a dropped term, a wrong index or sign, a transposed operand, a
wrong rounding rule) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(vals) -> np.ndarray:
    return synth.f32_to_bf16(np.asarray(vals, dtype=np.float32))


# ---------------------------------------------------------------- E4M3 ------

def _torch_e4m3_values() -> np.ndarray:
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_e4m3_decode_closed_forms():
    v = oracle.e4m3_decode(np.array([0x00, 0x01, 0x07, 0x08, 0x38, 0x3C, 0x7E, 0x80, 0xFE, 0x30], np.uint8))
    assert list(v) == [0.0, 2.0 ** -9, 7 * 2.0 ** -9, 2.0 ** -6, 1.0, 1.5, 448.0, -0.0, -448.0, 0.5]
    assert math.isnan(oracle.e4m3_decode(np.array([0x7F], np.uint8))[0])
    assert math.isnan(oracle.e4m3_decode(np.array([0xFF], np.uint8))[0])


def test_e4m3_decode_matches_torch_and_generator_for_all_codes():
    ours = oracle.e4m3_decode(np.arange(256, dtype=np.uint8))
    ref = _torch_e4m3_values()
    gen = synth.e4m3_value_table().astype(np.float64)
    finite = ~np.isnan(ref)
    assert np.array_equal(np.isnan(ours), ~finite)
    assert np.array_equal(ours[finite], ref[finite])
    assert np.array_equal(gen[finite], ref[finite])


def test_e4m3_encode_roundtrip_every_finite_code():
    vals = _torch_e4m3_values()
    for c in range(256):
        if math.isnan(vals[c]):
            continue
        assert oracle.e4m3_encode(np.array([vals[c]], np.float32))[0] == c, hex(c)


def test_e4m3_encode_ties_to_even_at_every_midpoint():
    vals = _torch_e4m3_values()[:127]  # non-negative finite, ascending with the code
    for c in range(126):
        mid = np.float32((vals[c] + vals[c + 1]) / 2)  # exact in fp32
        assert float(mid) == (vals[c] + vals[c + 1]) / 2
        got = int(oracle.e4m3_encode(np.array([mid, -mid], np.float32))[0])
        assert got == (c if c % 2 == 0 else c + 1), (c, mid)
        neg = int(oracle.e4m3_encode(np.array([-mid], np.float32))[0])
        assert neg == (got | 0x80)


def test_e4m3_encode_saturates():
    got = oracle.e4m3_encode(np.array([448.0, 449.0, 463.9, 480.0, 1e6, -1e6, np.inf, -np.inf], np.float32))
    assert list(got) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x7E, 0xFE]


def test_e4m3_encode_matches_torch_cast():
    rng = np.random.default_rng(7)
    v = np.concatenate([rng.standard_normal(200000) * s for s in (1e-3, 0.05, 1.0, 20.0, 150.0)])
    v = np.clip(v, -448, 448).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(v), ref)


# ----------------------------------------------------- activation blocks ----

def test_quantize_rows_matches_torch_and_block_rules():
    x = synth.normal_bf16(11, 1, (37, 512), 1.0)
    x[3, 128:256] = 0                      # an all-zero block: scale 1, codes 0
    q, s = oracle.quantize_rows(x)
    xf = torch.from_numpy(synth.bf16_to_f32(x)).reshape(37, 4, 128)
    amax = xf.abs().amax(dim=2)
    s_ref = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))   # fp32 division
    q_ref = (xf / s_ref[..., None]).to(torch.float8_e4m3fn).view(torch.uint8).reshape(37, 512)
    assert np.array_equal(s, s_ref.numpy())
    assert np.array_equal(q, q_ref.numpy())
    assert s[3, 1] == 1.0 and not q[3, 128:256].any()
    dq = oracle.e4m3_decode(q).reshape(37, 4, 128)
    nz = amax.numpy() > 0
    assert np.all(np.abs(dq).max(axis=2)[nz] == 448.0)  # the block max maps onto the top code
    rel = np.abs(dq * s[..., None] - xf.numpy()) / np.maximum(np.abs(xf.numpy()), 1e-30)
    assert rel[np.abs(dq) >= 2 ** -6].max() <= 2 ** -4 + 1e-7  # half an E4M3 ulp, normal range


# --------------------------------------------------------------- routing ----

def _route_with_logits(logits, k, H=128):
    """Router inputs whose logits are exactly `logits`: one-hot x, column 0 of Wr."""
    E = len(logits)
    x = np.zeros((1, H), np.uint16)
    x[0, 0] = _bf16([1.0])[0]
    wr = np.zeros((E, H), np.uint16)
    wr[:, 0] = _bf16(logits)
    assert np.array_equal(synth.bf16_to_f32(wr[:, 0]), np.asarray(logits, np.float32))
    return oracle.route(x, wr, None, k, want_logits=True)


def test_route_closed_forms():
    cases = json.load(open(os.path.join(GOLDEN, "route_closed_form.json")))["cases"]
    for c in cases:
        idx, gate, logits = _route_with_logits(c["logits"], c["k"])
        assert list(idx[0]) == c["idx"], c
        np.testing.assert_allclose(gate[0], c["gate"], rtol=1e-7)
        np.testing.assert_array_equal(logits[0], c["logits"])


def test_route_bias_enters_selection_and_gates():
    logits = [2.0, 1.0, 0.0, -1.0]
    x = np.zeros((1, 128), np.uint16)
    x[0, 0] = _bf16([1.0])[0]
    wr = np.zeros((4, 128), np.uint16)
    wr[:, 0] = _bf16(logits)
    idx, gate, lg = oracle.route(x, wr, np.array([0.0, 0.0, 3.0, 0.0], np.float32), 2, want_logits=True)
    assert list(idx[0]) == [2, 0]          # 0 + 3 beats 2
    np.testing.assert_allclose(gate[0], [1 / (1 + math.exp(-1)), 1 / (1 + math.exp(1))], rtol=1e-7)


def test_route_zero_input_picks_lowest_indices_with_equal_gates():
    x = np.zeros((5, 256), np.uint16)
    wr = synth.normal_bf16(3, 2, (16, 256), 1 / 16)
    idx, gate, _ = oracle.route(x, wr, None, 4)
    assert (idx == np.arange(4)).all()
    np.testing.assert_allclose(gate, 0.25, rtol=1e-7)


def test_route_k_equals_E_is_the_full_softmax():
    import scipy.special
    x = synth.normal_bf16(5, 1, (9, 256), 1.0)
    wr = synth.normal_bf16(5, 2, (16, 256), 1 / 16)
    idx, gate, logits = oracle.route(x, wr, None, 16, want_logits=True)
    ref_logits = synth.bf16_to_f32(x).astype(np.float64) @ synth.bf16_to_f32(wr).astype(np.float64).T
    np.testing.assert_allclose(logits, ref_logits, rtol=1e-12, atol=1e-12)
    p = scipy.special.softmax(ref_logits, axis=1)
    order = np.argsort(-ref_logits, axis=1, kind="stable")
    assert np.array_equal(idx, order)
    np.testing.assert_allclose(gate, np.take_along_axis(p, order, axis=1), rtol=1e-6)


def test_route_brute_force_topk():
    import scipy.special
    x = synth.normal_bf16(6, 1, (64, 256), 1.0)
    wr = synth.normal_bf16(6, 2, (16, 256), 1 / 16)
    bias = synth.normal_f32(6, 3, (16,), 0.5)
    idx, gate, _ = oracle.route(x, wr, bias, 3)
    L = synth.bf16_to_f32(x).astype(np.float64) @ synth.bf16_to_f32(wr).astype(np.float64).T + bias
    P = scipy.special.softmax(L, axis=1)
    for t in range(64):
        best = sorted(range(16), key=lambda e: (-L[t, e], e))[:3]
        assert list(idx[t]) == best
        np.testing.assert_allclose(gate[t], P[t, best] / P[t, best].sum(), rtol=1e-6)
    np.testing.assert_allclose(gate.sum(axis=1), 1.0, rtol=1e-6)


# ------------------------------------------------------- histogram/permute ----

def test_permute_golden_example():
    g = json.load(open(os.path.join(GOLDEN, "permute_tiny.json")))
    counts, offsets, perm, pos = oracle.permute(np.array(g["idx"], np.int32), g["E"], g["n_shared"])
    assert counts.tolist() == g["counts"]
    assert offsets.tolist() == g["offsets"]
    assert perm.tolist() == g["perm"]
    assert pos.tolist() == g["pos"]


@pytest.mark.parametrize("n_shared", [0, 1])
def test_permute_invariants(n_shared):
    rng = np.random.default_rng(3)
    T, E, k = 333, 40, 6
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    counts, offsets, perm, pos = oracle.permute(idx, E, n_shared)
    S = k + n_shared
    assert counts.sum() == S * T and offsets[-1] == S * T
    assert np.all(np.diff(offsets) == counts)
    assert np.array_equal(np.bincount(idx.ravel(), minlength=E), counts[:E])
    assert sorted(pos.ravel().tolist()) == list(range(S * T))           # a bijection
    assert np.array_equal(np.bincount(perm, minlength=T), np.full(T, S))  # every token S times
    for t in range(T):
        for j in range(S):
            r = pos[t, j]
            assert perm[r] == t
            g = np.searchsorted(offsets, r, side="right") - 1
            assert g == (idx[t, j] if j < k else E)
    for g in range(E + n_shared):
        seg = perm[offsets[g]:offsets[g + 1]]
        assert np.all(np.diff(seg) > 0)                                   # tokens ascend


def test_permute_rejects_bad_index():
    with pytest.raises(ValueError):
        oracle.permute(np.array([[0, 9]], np.int32), 4, 1)


def test_permute_empty():
    counts, offsets, perm, pos = oracle.permute(np.zeros((0, 8), np.int32), 352, 1)
    assert not counts.any() and not offsets.any() and perm.size == 0 and pos.shape == (0, 9)


# ------------------------------------------------------------ expert MLPs ----

def _dense_swiglu_torch(xf, w1, w3, w2, wdtype):
    """One expert by torch CPU matmul (float64), h rounded as the layer defines."""
    g = xf @ w1.T
    u = xf @ w3.T
    h = torch.nn.functional.silu(g) * u
    if wdtype == synth.WDTYPE_BF16:
        h = h.to(torch.float32).to(torch.bfloat16).to(torch.float64)
    else:
        hf = h.to(torch.float32).reshape(h.shape[0], -1, 128)
        amax = hf.abs().amax(dim=2, keepdim=True)
        sc = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
        h = ((hf / sc).to(torch.float8_e4m3fn).to(torch.float64) * sc.to(torch.float64)).reshape(h.shape)
    return h @ w2.T


def _deq(codes_or_bits, scales, wdtype):
    """Dequantised weights [G, R, C] as float64 torch tensors (library decode)."""
    if wdtype == synth.WDTYPE_BF16:
        return torch.from_numpy(synth.bf16_to_f32(codes_or_bits).astype(np.float64))
    v = torch.from_numpy(codes_or_bits).view(torch.float8_e4m3fn).to(torch.float64)
    s = torch.from_numpy(scales).to(torch.float64)
    s = s.repeat_interleave(128, dim=1).repeat_interleave(128, dim=2)
    return v * s


# E2M1 magnitudes by code (OCP MX 4-bit float, written out: codes 0-7 are
# 0, 0.5, 1, 1.5, 2, 3, 4, 6; bit 3 is the sign).
E2M1_CLOSED_FORM = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _deq_nvfp4(codes, scales, gs):
    """[G, R, C] float64 from NVFP4 storage, by the closed-form E2M1 table and
    torch's E4M3 decode (independent of the oracle's decoders)."""
    mag = np.array(E2M1_CLOSED_FORM + [-v for v in E2M1_CLOSED_FORM])
    lo, hi = mag[codes & 15], mag[codes >> 4]
    v = np.stack([lo, hi], axis=-1).reshape(codes.shape[0], codes.shape[1], -1)
    sc = torch.from_numpy(scales).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return torch.from_numpy(v * np.repeat(sc, 16, axis=2) * gs.astype(np.float64)[:, None, None])


def _act(x, wdtype):
    xf = torch.from_numpy(synth.bf16_to_f32(x).astype(np.float64))
    if wdtype in (synth.WDTYPE_BF16, synth.WDTYPE_NVFP4):
        return xf
    xr = xf.to(torch.float32).reshape(x.shape[0], -1, 128)
    amax = xr.abs().amax(dim=2, keepdim=True)
    sc = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    return ((xr / sc).to(torch.float8_e4m3fn).to(torch.float64) * sc.to(torch.float64)).reshape(xf.shape)


@pytest.mark.parametrize("wdtype", [synth.WDTYPE_BF16, synth.WDTYPE_FP8])
def test_single_expert_top1_is_a_dense_swiglu_mlp(wdtype):
    shape = synth.MoeShape("one", T=24, hidden=256, n_experts=1, top_k=1, n_shared=0, inter=256,
                           wdtype=wdtype, seed=21)
    w = synth.make_weights(shape)
    x = synth.make_x(shape)
    r = oracle.moe_forward(shape, w, x)
    assert (r["idx"] == 0).all() and (r["gate"] == 1.0).all()
    W1, W3, W2 = (_deq(w[a], w[b], wdtype)[0] for a, b in (("w1", "s1"), ("w3", "s3"), ("w2", "s2")))
    ref = _dense_swiglu_torch(_act(x, wdtype), W1, W3, W2, wdtype).numpy()
    err = np.linalg.norm(r["out_f64"] - ref) / np.linalg.norm(ref)
    assert err < 1e-6, err


@pytest.mark.parametrize("wdtype", [synth.WDTYPE_BF16, synth.WDTYPE_FP8])
def test_layer_equals_brute_force_over_all_experts(wdtype):
    shape = synth.MoeShape("bf", T=20, hidden=256, n_experts=8, top_k=3, n_shared=1, inter=128,
                           wdtype=wdtype, seed=22)
    w = synth.make_weights(shape)
    x = synth.make_x(shape)
    r = oracle.moe_forward(shape, w, x)
    a = _act(x, wdtype)
    W1, W3, W2 = (_deq(w[p], w[q], wdtype) for p, q in (("w1", "s1"), ("w3", "s3"), ("w2", "s2")))
    SW1, SW3, SW2 = (_deq(w[p], w[q], wdtype)[0] for p, q in (("sw1", "ss1"), ("sw3", "ss3"), ("sw2", "ss2")))
    Y = torch.stack([_dense_swiglu_torch(a, W1[e], W3[e], W2[e], wdtype) for e in range(8)])  # [E, T, H]
    G = torch.zeros(20, 8, dtype=torch.float64)                    # dense gate matrix, zeros off top-k
    for t in range(20):
        for j in range(3):
            G[t, r["idx"][t, j]] = float(r["gate"][t, j])
    ref = torch.einsum("te,eth->th", G, Y) + _dense_swiglu_torch(a, SW1, SW3, SW2, wdtype)
    err = np.linalg.norm(r["out_f64"] - ref.numpy()) / np.linalg.norm(ref.numpy())
    assert err < 1e-6, err
    # the bf16 output is the fp64 sum rounded once
    assert np.array_equal(r["out_bf16"], torch.from_numpy(r["out_f64"]).to(torch.bfloat16).view(torch.int16)
                          .numpy().view(np.uint16))


@pytest.mark.parametrize("wdtype", [synth.WDTYPE_BF16, synth.WDTYPE_FP8])
def test_expert_rows_equal_dense_swiglu_per_expert(wdtype):
    """Single (token, expert) rows, any expert (routed or not, and the shared
    one), against torch's dense SwiGLU of that expert, and against moe_tokens."""
    shape = synth.MoeShape("rows", T=12, hidden=256, n_experts=6, top_k=2, n_shared=1, inter=256,
                           wdtype=wdtype, seed=23)
    w = synth.make_weights(shape)
    x = synth.make_x(shape)
    toks = np.repeat(np.arange(shape.T), shape.n_experts + 1)
    grps = np.tile(np.arange(shape.n_experts + 1), shape.T)
    y = oracle.expert_rows(shape, w, x, toks, grps).reshape(shape.T, shape.n_experts + 1, -1)
    a = _act(x, wdtype)
    W1, W3, W2 = (_deq(w[p], w[q], wdtype) for p, q in (("w1", "s1"), ("w3", "s3"), ("w2", "s2")))
    SW1, SW3, SW2 = (_deq(w[p], w[q], wdtype)[0] for p, q in (("sw1", "ss1"), ("sw3", "ss3"), ("sw2", "ss2")))
    for e in range(shape.n_experts + 1):
        ref = (_dense_swiglu_torch(a, W1[e], W3[e], W2[e], wdtype) if e < shape.n_experts
               else _dense_swiglu_torch(a, SW1, SW3, SW2, wdtype)).numpy()
        err = np.linalg.norm(y[:, e] - ref) / np.linalg.norm(ref)
        assert err < 1e-6, (e, err)
    idx, gate, _ = oracle.route(x, w["router_w"], None, shape.top_k)
    _, _, ys = oracle.moe_tokens(shape, w, x, idx, gate, want_y=True)
    for t in range(shape.T):
        for j in range(shape.top_k):
            assert np.array_equal(ys[t, j], y[t, idx[t, j]])
        assert np.array_equal(ys[t, shape.top_k], y[t, shape.n_experts])


def test_e2m1_decode_every_code():
    got = oracle.e2m1_decode(np.arange(16, dtype=np.uint8))
    want = np.array(E2M1_CLOSED_FORM + [-v for v in E2M1_CLOSED_FORM])
    assert np.array_equal(got, want)
    assert np.all(np.signbit(got[8:]))                       # code 8 is -0
    assert np.array_equal(got, synth.e2m1_value_table().astype(np.float64))  # the generator's own decoder


def test_nvfp4_nibble_order_and_scales():
    # one row of 32 inputs: bytes j hold inputs 2j (low nibble) and 2j+1 (high)
    codes = np.zeros((1, 16), np.uint8)
    codes[0, 0] = 0x7A          # input 0: code 0xA = -1, input 1: code 7 = 6
    codes[0, 9] = 0x21          # input 18: code 1 = 0.5, input 19: code 2 = 1
    scales = np.array([[0x38, 0x40]], np.uint8)  # E4M3 1.0 for inputs 0-15, 2.0 for 16-31
    w = oracle.nvfp4_dequantize(codes, scales, 0.25)
    want = np.zeros(32)
    want[0], want[1], want[18], want[19] = -0.25, 1.5, 0.25, 0.5
    assert np.array_equal(w[0], want)


def test_nvfp4_generator_keeps_values_within_the_format_error():
    """The checkpoint preparation (input side): dequantised NVFP4 weights stay
    within half an E2M1 step (times the block scale) of the bf16 draws."""
    G, R, C, std = 2, 64, 256, 0.05
    codes, scales, gs = synth.nvfp4(3, 99, G, R, C, std)
    ref = synth.bf16_to_f32(synth.normal_bf16(3, 99, (G, R, C), std)).astype(np.float64)
    deq = _deq_nvfp4(codes, scales, gs).numpy()
    assert np.allclose(gs, np.abs(ref).reshape(G, -1).max(axis=1) / (6 * 448), rtol=1e-6)
    step = np.repeat(torch.from_numpy(scales).view(torch.float8_e4m3fn).to(torch.float64).numpy(), 16, axis=2) \
        * gs[:, None, None]
    assert np.all(np.abs(deq - ref) <= step * 1.0 + 1e-12)   # the widest E2M1 gap is 2 (4 -> 6)
    assert np.linalg.norm(deq - ref) / np.linalg.norm(ref) < 0.15


def test_nvfp4_layer_equals_brute_force_over_all_experts():
    shape = synth.MoeShape("bf-nvfp4", T=16, hidden=256, n_experts=6, top_k=2, n_shared=1, inter=256,
                           wdtype=synth.WDTYPE_NVFP4, seed=24)
    w = synth.make_weights(shape)
    x = synth.make_x(shape)
    r = oracle.moe_forward(shape, w, x)
    a = _act(x, shape.wdtype)
    W1, W3, W2 = (_deq_nvfp4(w[p], w[q], w[g]) for p, q, g in (("w1", "s1", "g1"), ("w3", "s3", "g3"),
                                                                ("w2", "s2", "g2")))
    SW1, SW3, SW2 = (_deq_nvfp4(w[p], w[q], w[g])[0] for p, q, g in (("sw1", "ss1", "sg1"), ("sw3", "ss3", "sg3"),
                                                                       ("sw2", "ss2", "sg2")))
    bf = synth.WDTYPE_BF16  # NVFP4 keeps bf16 activations and rounds h to bf16
    Y = torch.stack([_dense_swiglu_torch(a, W1[e], W3[e], W2[e], bf) for e in range(shape.n_experts)])
    G = torch.zeros(shape.T, shape.n_experts, dtype=torch.float64)
    for t in range(shape.T):
        for j in range(shape.top_k):
            G[t, r["idx"][t, j]] = float(r["gate"][t, j])
    ref = torch.einsum("te,eth->th", G, Y) + _dense_swiglu_torch(a, SW1, SW3, SW2, bf)
    err = np.linalg.norm(r["out_f64"] - ref.numpy()) / np.linalg.norm(ref.numpy())
    assert err < 1e-6, err


def test_token_subset_equals_full_run():
    shape = synth.TINY
    w = synth.make_weights(shape)
    x = synth.make_x(shape)
    full = oracle.moe_forward(shape, w, x)
    sub = oracle.moe_forward(shape, w, x, tokens=[5, 0, 31])
    assert np.array_equal(sub["out_f64"], full["out_f64"][[5, 0, 31]])


def test_shared_expert_is_added_with_unit_weight():
    shape = synth.TINY
    w = synth.make_weights(shape)
    x = synth.make_x(shape)
    r = oracle.moe_forward(shape, w, x)
    _, _, y = oracle.moe_tokens(shape, w, x, r["idx"], r["gate"], want_y=True)
    routed = np.einsum("tj,tjh->th", r["gate"].astype(np.float64), y[:, :shape.top_k])
    np.testing.assert_allclose(r["out_f64"] - routed, y[:, shape.top_k], rtol=1e-9, atol=1e-12)


def test_zipf_skew_gives_about_ten_times_the_mean_load():
    shape = synth.LONG_SKEW_FP8
    x = synth.make_x(shape.with_tokens(2048))
    wr = synth.normal_bf16(shape.seed, synth.ID_ROUTER_W, (shape.n_experts, shape.hidden), 1 / 64)
    idx, _, _ = oracle.route(x, wr, synth.zipf_bias(shape.seed, shape.n_experts), shape.top_k)
    cnt = np.bincount(idx.ravel(), minlength=shape.n_experts)
    ratio = cnt.max() / cnt.mean()
    assert 8.0 <= ratio <= 12.5, ratio


# ------------------------------------------------------------ residual stream --

def test_rmsnorm_closed_forms():
    H, eps = 256, 1e-6
    w = np.linspace(0.5, 1.5, H)
    # A constant row c: every element is c / sqrt(c^2 + eps) * w.
    r = np.full((1, H), 3.0, np.float32)
    np.testing.assert_allclose(oracle.rmsnorm(r, w, eps)[0], 3.0 / np.sqrt(9.0 + eps) * w, rtol=1e-14)
    # One non-zero element a: mean(r^2) = a^2 / H.
    r = np.zeros((1, H), np.float32)
    r[0, 7] = -2.0
    y = oracle.rmsnorm(r, w, eps)[0]
    assert y[7] == pytest.approx(-2.0 / np.sqrt(4.0 / H + eps) * w[7], rel=1e-14)
    assert np.count_nonzero(y) == 1


def test_rmsnorm_is_scale_invariant_and_unit_rms():
    rng = np.random.default_rng(3)
    r = rng.standard_normal((5, 384)).astype(np.float32)
    ones = np.ones(384)
    y1 = oracle.rmsnorm(r, ones, 0.0)
    y2 = oracle.rmsnorm(np.float32(8.0) * r, ones, 0.0)
    np.testing.assert_allclose(y1, y2, rtol=1e-12)
    np.testing.assert_allclose(np.sqrt(np.mean(y1 * y1, axis=1)), 1.0, rtol=1e-12)


def test_add_residual_sums_slots_and_skips_negative_positions():
    rng = np.random.default_rng(4)
    r = rng.standard_normal((3, 8)).astype(np.float32)
    y = rng.standard_normal((6, 8)).astype(np.float32)
    pos = np.array([[0, 1], [2, -1], [5, 4]], np.int32)
    out = oracle.add_residual(r, y, pos)
    np.testing.assert_allclose(out[0], r[0].astype(np.float64) + y[0] + y[1], rtol=1e-14)
    np.testing.assert_allclose(out[1], r[1].astype(np.float64) + y[2], rtol=1e-14)
    np.testing.assert_allclose(out[2], r[2].astype(np.float64) + y[5] + y[4], rtol=1e-14)
