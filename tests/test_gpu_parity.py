"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Bars: bit-exact for integer work (activation codes and scales, histogram,
offsets, permutation); routing by the margin rule of tests/parity.py; layer
and expert outputs within relative Frobenius error 1e-2 (BF16 experts) or
2e-2 (FP8 experts). Full-size workloads compare routing in full and outputs on
a seeded sample of tokens whose routing is unique.
"""
import functools

import numpy as np
import pytest

import oracle
import synth
from parity import (bf16_bits_to_f64, check_routing, frob_rel, rows_rel, tol_for, unique_tokens)
from conftest import cuda_available

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module")
def m():
    import mixture_experts_histogram_b200 as mm
    from mixture_experts_histogram_b200 import build
    build.build()
    mm.load()
    return mm


def _cfg(m, s):
    return m.make_config(s.hidden, s.n_experts, s.top_k, s.n_shared, s.inter, s.wdtype)


@functools.lru_cache(maxsize=4)
def _inputs(shape):
    return synth.make_x(shape), synth.make_weights(shape)


def _workspace(m, cfg, T):
    import torch
    nb = m.moe_workspace_bytes(cfg, T)
    return torch.empty(max(nb, 1024), dtype=torch.uint8, device="cuda")


def _forward(m, shape, x_np, wd):
    import torch
    cfg = _cfg(m, shape)
    T = x_np.shape[0]
    x = m.to_device(x_np)
    out = torch.empty((T, shape.hidden), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((T, shape.top_k), dtype=torch.int32, device="cuda")
    gate = torch.empty((T, shape.top_k), dtype=torch.float32, device="cuda")
    ws = _workspace(m, cfg, T)
    m.moe_forward(cfg, T, x, m.make_weights(wd), out, ws, topk_idx=idx, topk_w=gate)
    st = m.moe_read_status(ws)
    assert st == 0, m.moe_status_string(st)
    out_np = out.view(torch.int16).cpu().numpy().view(np.uint16)
    return out_np, idx.cpu().numpy(), gate.cpu().numpy()


# ------------------------------------------------------------- quantisation --

def test_quantize_act_bit_exact(m):
    import torch
    x = synth.normal_bf16(31, 1, (300, 4096), 1.0)
    x[7, 128:256] = 0                                   # all-zero block
    x[8, :128] = synth.f32_to_bf16(np.full(128, -0.0, np.float32))  # negative zeros
    x[9, :128] = synth.f32_to_bf16(np.geomspace(1e-30, 3e4, 128).astype(np.float32))  # wide range
    x[10, 256:384] = synth.f32_to_bf16(np.linspace(-1e-3, 1e-3, 128).astype(np.float32))
    q_ref, s_ref = oracle.quantize_rows(x)
    q = torch.empty((300, 4096), dtype=torch.uint8, device="cuda")
    s = torch.empty((300, 32), dtype=torch.float32, device="cuda")
    m.moe_quantize_act(300, 4096, m.to_device(x), q, s)
    torch.cuda.synchronize()
    assert np.array_equal(s.cpu().numpy(), s_ref)
    qq = q.cpu().numpy()
    bad = np.argwhere(qq != q_ref)
    assert bad.size == 0, f"{len(bad)} codes differ, first {bad[:5].tolist()}"


def _quant_blocks_every_bf16_and_e4m3_tie():
    """Blocks of 128 bf16 values: every finite bf16 bit pattern, in order (blocks
    of one exponent) and shuffled (blocks spanning many exponents); and for block
    maxima 448 * 2^k, the E4M3 midpoints and values times 2^k, so that x / scale
    lands exactly on every rounding tie and representable value."""
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    finite = pats[(pats & 0x7F80) != 0x7F80]
    rng = np.random.default_rng(77)
    blocks = [finite, rng.permutation(finite)]
    vals = np.unique(oracle.e4m3_decode(np.arange(256, dtype=np.uint8)))
    pos = vals[np.isfinite(vals) & (vals > 0)].astype(np.float64)
    mids = (pos[:-1] + pos[1:]) / 2
    cand = np.concatenate([mids, pos, -mids, -pos])
    for k in range(-30, 31):
        xs = cand * 2.0 ** k
        for c0 in range(0, len(xs), 127):
            blk = np.zeros(128, np.float32)
            blk[0] = 448.0 * 2.0 ** k
            chunk = xs[c0:c0 + 127].astype(np.float32)
            blk[1:1 + len(chunk)] = chunk
            b = synth.f32_to_bf16(blk)
            assert np.array_equal((b.astype(np.uint32) << 16).view(np.float32), blk)  # exact in bf16
            blocks.append(b)
    flat = np.concatenate(blocks)
    flat = np.concatenate([flat, np.zeros((-len(flat)) % 4096, np.uint16)])
    return flat.reshape(-1, 4096)


def test_quantize_act_every_bf16_and_e4m3_tie(m):
    """The activation quantisation over every finite bf16 value and every E4M3
    rounding tie (x / scale exactly halfway between two codes), bit-exact against
    the oracle's IEEE division and round-to-nearest-even."""
    import torch
    x = _quant_blocks_every_bf16_and_e4m3_tie()
    T = x.shape[0]
    q_ref, s_ref = oracle.quantize_rows(x)
    q = torch.empty((T, 4096), dtype=torch.uint8, device="cuda")
    s = torch.empty((T, 32), dtype=torch.float32, device="cuda")
    m.moe_quantize_act(T, 4096, m.to_device(x), q, s)
    torch.cuda.synchronize()
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    bad = np.argwhere(q.cpu().numpy() != q_ref)
    assert bad.size == 0, f"{len(bad)} codes differ, first {bad[:5].tolist()}"


# ------------------------------------------------------------------ routing --

ROUTE_CASES = [
    synth.TINY,
    synth.TINY.with_tokens(333),
    synth.DECODE_BF16,
    synth.PREFILL_FP8,
    synth.LONG_SKEW_FP8,
    synth.SWEEP_FP8.with_tokens(1),
    synth.MoeShape("wide-E512-k16", T=1000, hidden=512, n_experts=512, top_k=16, n_shared=1, inter=128, seed=9),
    synth.MoeShape("E300-k5", T=257, hidden=384, n_experts=300, top_k=5, n_shared=0, inter=128, seed=10),
    # One full 128-token tile, one row past it, and a ragged skewed case (the K
    # split changes with the number of token tiles).
    synth.MoeShape("route-T128", T=128, hidden=4096, n_experts=352, top_k=8, n_shared=1, inter=1536, seed=26),
    synth.MoeShape("route-T13-E300-skew", T=13, hidden=1024, n_experts=300, top_k=6, n_shared=0, inter=256,
                   seed=27, skew=True),
    synth.MoeShape("route-T129", T=129, hidden=4096, n_experts=352, top_k=8, n_shared=1, inter=1536, seed=28),
]


@pytest.mark.parametrize("shape", ROUTE_CASES, ids=lambda s: s.name)
def test_route_parity(m, shape):
    import torch
    cfg = _cfg(m, shape)
    x = synth.make_x(shape)
    H, E, k, T = shape.hidden, shape.n_experts, shape.top_k, shape.T
    wr = synth.normal_bf16(shape.seed, synth.ID_ROUTER_W, (E, H), 1 / np.sqrt(H))
    bias = synth.zipf_bias(shape.seed, E) if shape.skew else None
    idx_r, gate_r, logits_r = oracle.route(x, wr, bias, k, want_logits=True)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    gate = torch.empty((T, k), dtype=torch.float32, device="cuda")
    logits = torch.empty((T, E), dtype=torch.float32, device="cuda")
    ws = _workspace(m, cfg, T)
    m.moe_route(cfg, T, m.to_device(x), m.to_device(wr), m.to_device(bias), idx, gate, logits, ws)
    assert m.moe_read_status(ws) == 0
    lg = logits.cpu().numpy().astype(np.float64)
    # The routing comparison is sound while the fp32 logits stay within half the
    # 1e-4 margin of the fp64 ones (fp32 accumulation over H = 4096 products).
    err = np.abs(lg - logits_r).max()
    assert err < 5e-5, f"fp32 logits off by {err}"
    n_u, n_a = check_routing(idx.cpu().numpy(), gate.cpu().numpy(), logits_r, idx_r, gate_r)
    assert n_u >= 0.99 * T


# ------------------------------------------------------- histogram/permute --

# T <= 256 runs the one-launch path (one 256-token chunk), larger T the three
# kernels, whose chunk scan batches its loads up to 32 chunks (T <= 8192) and
# loops over the chunks beyond.
PERMUTE_CASES = [(32, 16, 2, 1), (1000, 352, 8, 1), (8192, 352, 8, 1), (777, 352, 8, 0), (1, 352, 8, 1),
                 (4096, 512, 16, 1), (300, 5, 5, 1), (64, 352, 8, 1), (256, 512, 16, 1), (255, 352, 8, 0),
                 (257, 352, 8, 1), (8193, 352, 8, 1), (12345, 100, 6, 1), (32768, 352, 8, 1), (40000, 352, 8, 1)]


@pytest.mark.parametrize("T,E,k,S", PERMUTE_CASES)
def test_permute_bit_exact(m, T, E, k, S):
    import torch
    rng = np.random.default_rng(T * 131 + E)
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    counts_r, offsets_r, perm_r, pos_r = oracle.permute(idx, E, S)
    shape = synth.MoeShape("perm", T=T, hidden=256, n_experts=E, top_k=k, n_shared=S, inter=128)
    cfg = _cfg(m, shape)
    G = E + S
    counts = torch.empty(G, dtype=torch.int32, device="cuda")
    offsets = torch.empty(G + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty((k + S) * T, dtype=torch.int32, device="cuda")
    pos = torch.empty((T, k + S), dtype=torch.int32, device="cuda")
    ws = _workspace(m, cfg, T)
    m.moe_permute(cfg, T, m.to_device(idx), counts, offsets, perm, pos, ws)
    assert m.moe_read_status(ws) == 0
    assert np.array_equal(counts.cpu().numpy(), counts_r)
    assert np.array_equal(offsets.cpu().numpy(), offsets_r)
    assert np.array_equal(perm.cpu().numpy(), perm_r)
    assert np.array_equal(pos.cpu().numpy(), pos_r)


def test_permute_skewed_routing_bit_exact(m):
    """Zipf-like load: a few experts take most rows (many M tiles, long segments)."""
    import torch
    T, E, k = 20000, 352, 8
    rng = np.random.default_rng(5)
    p = 1.0 / np.arange(1, E + 1) ** 1.1
    idx = np.stack([rng.choice(E, k, replace=False, p=p / p.sum()) for _ in range(T)]).astype(np.int32)
    counts_r, offsets_r, perm_r, pos_r = oracle.permute(idx, E, 1)
    cfg = m.make_config(256, E, k, 1, 128, 0)
    counts = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 2, dtype=torch.int32, device="cuda")
    perm = torch.empty(9 * T, dtype=torch.int32, device="cuda")
    pos = torch.empty((T, 9), dtype=torch.int32, device="cuda")
    ws = _workspace(m, cfg, T)
    m.moe_permute(cfg, T, m.to_device(idx), counts, offsets, perm, pos, ws)
    assert np.array_equal(perm.cpu().numpy(), perm_r) and np.array_equal(pos.cpu().numpy(), pos_r)
    assert np.array_equal(offsets.cpu().numpy(), offsets_r)


def test_permute_bad_index_latches_status(m):
    import torch
    T, E, k = 64, 16, 2
    idx = np.tile(np.array([[0, 1]], np.int32), (T, 1))
    idx[5, 1] = 99
    idx[6, 0] = -3
    cfg = m.make_config(256, E, k, 1, 128, 0)
    counts = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 2, dtype=torch.int32, device="cuda")
    perm = torch.empty(3 * T, dtype=torch.int32, device="cuda")
    pos = torch.empty((T, 3), dtype=torch.int32, device="cuda")
    ws = _workspace(m, cfg, T)
    m.moe_permute(cfg, T, m.to_device(idx), counts, offsets, perm, pos, ws)
    assert m.moe_read_status(ws) == m.MOE_ERR_BAD_INDEX
    c = counts.cpu().numpy()
    assert c[0] == T - 1 and c[1] == T - 1 and c[E] == T
    pp = pos.cpu().numpy()
    assert pp[5, 1] == -1 and pp[6, 0] == -1


# ------------------------------------------------------------------ combine --

def test_combine_fixed_order_sum(m):
    import torch
    T, E, k, S, H = 257, 40, 6, 1, 512
    rng = np.random.default_rng(2)
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    _, _, _, pos = oracle.permute(idx, E, S)
    y = synth.normal_bf16(3, 7, ((k + S) * T, H), 0.5)
    ref = np.zeros((T, H))
    yf = bf16_bits_to_f64(y)
    for j in range(k + S):
        ref += yf[pos[:, j]]
    cfg = m.make_config(H, E, k, S, 128, 0)
    out = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    m.moe_combine(cfg, T, m.to_device(y), m.to_device(pos), out)
    o = bf16_bits_to_f64(out.view(torch.int16).cpu().numpy().view(np.uint16))
    ulp = np.abs(ref) * 2.0 ** -8
    assert np.all(np.abs(o - ref) <= ulp + 1e-30)
    assert np.mean(synth.f32_to_bf16(ref.astype(np.float32)) == out.view(torch.int16).cpu().numpy().view(np.uint16)) > 0.99


def test_permute_then_combine_with_identity_experts_returns_input(m):
    """y rows = gate * x[token] (identity experts, no shared expert) => out == x."""
    import torch
    T, E, k, H = 300, 24, 4, 256
    rng = np.random.default_rng(4)
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    g = rng.dirichlet(np.ones(k), size=T).astype(np.float32)
    x = synth.normal_bf16(4, 1, (T, H), 1.0)
    cfg = m.make_config(H, E, k, 0, 128, 0)
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(k * T, dtype=torch.int32, device="cuda")
    pos = torch.empty((T, k), dtype=torch.int32, device="cuda")
    ws = _workspace(m, cfg, T)
    m.moe_permute(cfg, T, m.to_device(idx), counts, offsets, perm, pos, ws)
    pp, pm = pos.cpu().numpy(), perm.cpu().numpy()
    xf = bf16_bits_to_f64(x)
    y = np.zeros((k * T, H), np.float32)
    for t in range(T):
        for j in range(k):
            y[pp[t, j]] = xf[t] * g[t, j]
    assert np.array_equal(pm[pp[:, 0]], np.arange(T))
    out = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    m.moe_combine(cfg, T, m.to_device(synth.f32_to_bf16(y)), pos, out)
    o = bf16_bits_to_f64(out.view(torch.int16).cpu().numpy().view(np.uint16))
    assert np.all(np.abs(o - xf) <= np.abs(xf) * 2.0 ** -6 + 1e-30)


# ------------------------------------------------------------- expert MLPs --

def _expert_cases():
    import dataclasses
    return [
        synth.TINY,
        dataclasses.replace(synth.TINY, name="tiny-fp8", wdtype=synth.WDTYPE_FP8),
        synth.MoeShape("mid-bf16", T=300, hidden=512, n_experts=24, top_k=4, n_shared=1, inter=384, seed=12),
        synth.MoeShape("mid-fp8", T=300, hidden=512, n_experts=24, top_k=4, n_shared=1, inter=384,
                       wdtype=synth.WDTYPE_FP8, seed=13),
        synth.MoeShape("odd-H-fp8", T=130, hidden=384, n_experts=10, top_k=3, n_shared=0, inter=256,
                       wdtype=synth.WDTYPE_FP8, seed=14),
    ]


@pytest.fixture(params=["single", "pair", "swap"])
def variant(request, m):
    """Run the test under each expert-GEMM variant (same result expected)."""
    m.moe_set_gemm_variant({"single": m.MOE_GEMM_SINGLE, "pair": m.MOE_GEMM_PAIR, "swap": m.MOE_GEMM_SWAP}[request.param])
    yield request.param
    m.moe_set_gemm_variant(m.MOE_GEMM_AUTO)


@pytest.mark.parametrize("shape", _expert_cases(), ids=lambda s: s.name)
def test_experts_parity(m, shape, variant):
    import torch
    x, w = _inputs(shape)
    idx_r, gate_r, _ = oracle.route(x, w["router_w"], w["router_bias"], shape.top_k)
    _, _, y_r = oracle.moe_tokens(shape, w, x, idx_r, gate_r, want_y=True)
    cfg = _cfg(m, shape)
    T, S = shape.T, shape.top_k + shape.n_shared
    wd = m.upload_weights(w)
    y = torch.empty((S * T, shape.hidden), dtype=torch.bfloat16, device="cuda")
    pos = torch.empty((T, S), dtype=torch.int32, device="cuda")
    ws = _workspace(m, cfg, T)
    m.moe_experts(cfg, T, m.to_device(x), m.to_device(idx_r), m.to_device(gate_r), m.make_weights(wd), y, pos, ws)
    assert m.moe_read_status(ws) == 0
    yy = bf16_bits_to_f64(y.view(torch.int16).cpu().numpy().view(np.uint16))
    pp = pos.cpu().numpy()
    gates = np.concatenate([gate_r.astype(np.float64), np.ones((T, shape.n_shared))], axis=1)
    got = yy[pp.reshape(-1)].reshape(T, S, shape.hidden)
    ref = y_r * gates[:, :, None]
    err = frob_rel(got, ref)
    assert err < tol_for(shape.wdtype), err


# ------------------------------------------------------------- whole layer --

def _layer_cases():
    import dataclasses
    return [
        (synth.TINY, None),
        (dataclasses.replace(synth.TINY, name="tiny-fp8", wdtype=synth.WDTYPE_FP8), None),
        (synth.MoeShape("ragged-bf16", T=200, hidden=512, n_experts=24, top_k=4, n_shared=1, inter=256, seed=15),
         None),
        (synth.MoeShape("no-shared-fp8", T=77, hidden=256, n_experts=12, top_k=3, n_shared=0, inter=128,
                        wdtype=synth.WDTYPE_FP8, seed=16), None),
        (synth.MoeShape("E512-k16-fp8", T=160, hidden=256, n_experts=512, top_k=16, n_shared=1, inter=128,
                        wdtype=synth.WDTYPE_FP8, seed=17), None),
        # top_k * T >= 128 * E: the automatic choice runs the gate/up GEMM on 2-SM
        # pairs and the down GEMM on single CTAs.
        (synth.MoeShape("auto-pair-fp8", T=600, hidden=512, n_experts=8, top_k=2, n_shared=1, inter=256,
                        wdtype=synth.WDTYPE_FP8, seed=24), None),
        (synth.MoeShape("auto-pair-bf16", T=520, hidden=384, n_experts=6, top_k=2, n_shared=0, inter=384,
                        seed=25), None),
        # The dense SwiGLU FFN (one expert, top-1, no shared expert, I = 13,824).
        (synth.DENSE_FFN_FP8.with_tokens(300), 12),
        # Few down-GEMM tiles: its K range is split into pieces summed afterwards
        # (dense FFN at T = 64 and 1: 9 pieces; the 5-group case: 2 FP8, 4 BF16).
        (synth.DENSE_FFN_FP8.with_tokens(64), 16),
        (synth.DENSE_FFN_FP8.with_tokens(1), None),
        (synth.MoeShape("split-down-fp8", T=40, hidden=512, n_experts=4, top_k=1, n_shared=1, inter=1024,
                        wdtype=synth.WDTYPE_FP8, seed=26), None),
        (synth.MoeShape("split-down-bf16", T=40, hidden=512, n_experts=4, top_k=1, n_shared=1, inter=1024,
                        seed=27), None),
        (dataclasses.replace(synth.DENSE_FFN_FP8, name="step5-dense-ffn-bf16", wdtype=synth.WDTYPE_BF16)
         .with_tokens(64), 8),
        (synth.DECODE_BF16, None),
        (synth.SWEEP_FP8.with_tokens(1), None),
        (synth.SWEEP_FP8.with_tokens(8), None),
        (synth.SWEEP_FP8.with_tokens(64), 32),
        (synth.SWEEP_FP8.with_tokens(512), 24),
        (synth.SWEEP_FP8.with_tokens(2048), 24),
        (synth.PREFILL_FP8, 32),
        (synth.LONG_SKEW_FP8, 24),
    ]


@pytest.mark.parametrize("shape,n_sample", _layer_cases(), ids=lambda v: getattr(v, "name", str(v)))
def test_forward_parity(m, shape, n_sample):
    """The automatic variant choice (single-CTA GEMMs for FP8 experts)."""
    x = synth.make_x(shape)
    w = synth.make_weights(shape)
    idx_r, gate_r, logits_r = oracle.route(x, w["router_w"], w["router_bias"], shape.top_k, want_logits=True)
    wd = m.upload_weights(w)
    out, idx, gate = _forward(m, shape, x, wd)
    del wd
    check_routing(idx, gate, logits_r, idx_r, gate_r)
    uniq = np.flatnonzero(unique_tokens(logits_r, shape.top_k))
    if n_sample is None or n_sample >= uniq.size:
        toks = uniq
    else:
        toks = np.sort(np.random.default_rng(shape.seed).choice(uniq, n_sample, replace=False))
    ref, _, _ = oracle.moe_tokens(shape, w, x, idx_r, gate_r, tokens=toks)
    got = bf16_bits_to_f64(out[toks])
    err = frob_rel(got, ref)
    per_token = rows_rel(got, ref)
    print(f"{shape.name}: {toks.size} tokens, pooled rel Frobenius {err:.2e}, per-token max {per_token.max():.2e}")
    assert err < tol_for(shape.wdtype), err
    # The stricter reading of the bar: every token's own relative error.
    assert per_token.max() < tol_for(shape.wdtype), (toks[per_token.argmax()], per_token.max())
    assert np.all(np.isfinite(bf16_bits_to_f64(out)))


@pytest.mark.parametrize("shape", [
    synth.MoeShape("pair-big-groups-fp8", T=600, hidden=512, n_experts=8, top_k=2, n_shared=1, inter=256,
                   wdtype=synth.WDTYPE_FP8, seed=20),
    synth.MoeShape("pair-big-groups-bf16", T=600, hidden=512, n_experts=8, top_k=2, n_shared=1, inter=256,
                   wdtype=synth.WDTYPE_BF16, seed=21),
    synth.MoeShape("pair-odd-H-fp8", T=333, hidden=384, n_experts=6, top_k=2, n_shared=0, inter=384,
                   wdtype=synth.WDTYPE_FP8, seed=22),
], ids=lambda s: s.name)
def test_forward_parity_both_variants(m, shape, variant):
    """Groups of several hundred rows: several 256-row pair tiles and ragged ends."""
    x, w = _inputs(shape)
    idx_r, gate_r, logits_r = oracle.route(x, w["router_w"], w["router_bias"], shape.top_k, want_logits=True)
    out, idx, gate = _forward(m, shape, x, m.upload_weights(w))
    check_routing(idx, gate, logits_r, idx_r, gate_r)
    toks = np.flatnonzero(unique_tokens(logits_r, shape.top_k))
    ref, _, _ = oracle.moe_tokens(shape, w, x, idx_r, gate_r, tokens=toks)
    err = frob_rel(bf16_bits_to_f64(out[toks]), ref)
    assert err < tol_for(shape.wdtype), err


def test_variants_agree_on_bf16(m):
    """Both GEMM variants accumulate each K stage in the same order in fp32 TMEM."""
    shape = synth.MoeShape("agree", T=400, hidden=512, n_experts=6, top_k=2, n_shared=1, inter=256, seed=23)
    x, w = _inputs(shape)
    wd = m.upload_weights(w)
    outs = []
    for v in (m.MOE_GEMM_SINGLE, m.MOE_GEMM_PAIR):
        m.moe_set_gemm_variant(v)
        outs.append(_forward(m, shape, x, wd)[0])
    m.moe_set_gemm_variant(m.MOE_GEMM_AUTO)
    assert frob_rel(bf16_bits_to_f64(outs[0]), bf16_bits_to_f64(outs[1])) < 1e-3


def test_forward_zero_tokens_is_a_noop(m):
    import torch
    shape = synth.TINY
    cfg = _cfg(m, shape)
    wd = m.upload_weights(synth.make_weights(shape))
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    x = torch.empty((0, shape.hidden), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((0, shape.hidden), dtype=torch.bfloat16, device="cuda")
    m.moe_forward(cfg, 0, x.data_ptr() or 1024, m.make_weights(wd), out.data_ptr() or 1024, ws)


def test_forward_host_matches_forward(m):
    import torch
    shape = synth.MoeShape("host", T=96, hidden=512, n_experts=24, top_k=4, n_shared=1, inter=256,
                           wdtype=synth.WDTYPE_FP8, seed=18)
    x, w = _inputs(shape)
    wd = m.upload_weights(w)
    out_dev, _, _ = _forward(m, shape, x, wd)
    cfg = _cfg(m, shape)
    xh = torch.from_numpy(x.view(np.int16)).pin_memory()
    oh = torch.empty((shape.T, shape.hidden), dtype=torch.int16).pin_memory()
    ws = _workspace(m, cfg, shape.T)
    m.moe_forward_host(cfg, shape.T, xh, m.make_weights(wd), oh, ws)
    assert np.array_equal(oh.numpy().view(np.uint16), out_dev)


def test_forward_is_deterministic(m):
    shape = synth.MoeShape("det", T=500, hidden=512, n_experts=32, top_k=4, n_shared=1, inter=256,
                           wdtype=synth.WDTYPE_FP8, seed=19)
    x, w = _inputs(shape)
    wd = m.upload_weights(w)
    a = _forward(m, shape, x, wd)
    b = _forward(m, shape, x, wd)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


def test_profile_reports_every_kernel(m):
    shape = synth.TINY
    x, w = _inputs(shape)
    wd = m.upload_weights(w)
    m.moe_profile_enable(True)
    try:
        _forward(m, shape, x, wd)
        prof = m.moe_profile_read()
    finally:
        m.moe_profile_enable(False)
    assert list(prof) == ["router_gemm", "router_topk", "histogram", "scan", "scatter", "gather",
                          "gemm1_gate_up_swiglu", "gemm2_down", "combine"]
    assert all(v > 0 for v in prof.values())
