"""NVFP4 expert storage (W4A16) on the GPU against the oracle.

Exact cases first: E2M1 codes with power-of-two E4M3 block scales and global
scales make every weight a small dyadic number, and bf16 activations in
{-4..4} make every product and partial sum exact in fp32, so the gate/up sums
(read before the SwiGLU) and the down GEMM's bf16 output must equal the plain
definition bit for bit; this pins the codes' nibble order, the scale indexing,
the shared-memory layout the converter warps write and the global scales.
Then the whole layer against the oracle on seeded NVFP4 weights, within the
BF16 tolerance 1e-2 (relative Frobenius, pooled and per token). Every case runs
both NVFP4 kernels (128-row tiles, and weight rows as the MMA's M side with the
weights expanded into tensor memory).
"""
import numpy as np
import pytest

import oracle
import synth
from conftest import cuda_available
from parity import bf16_bits_to_f64, check_routing, frob_rel, rows_rel, tol_for, unique_tokens

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]

NV = synth.WDTYPE_NVFP4


@pytest.fixture(scope="module")
def m():
    import mixture_experts_histogram_b200 as mm
    from mixture_experts_histogram_b200 import build
    build.build()
    mm.load()
    return mm


@pytest.fixture(params=["single", "swap"])
def variant(request, m):
    """The NVFP4 GEMM kernels: tiles of 128 rows, or weight rows as the MMA's M side
    expanded into tensor memory (same results expected)."""
    m.moe_set_gemm_variant(m.MOE_GEMM_SINGLE if request.param == "single" else m.MOE_GEMM_SWAP)
    yield request.param
    m.moe_set_gemm_variant(m.MOE_GEMM_AUTO)


H, I, E = 512, 256, 5
COUNTS = [0, 1, 129, 300, 64, 200]
POW2_SCALES = np.array([0x30, 0x38, 0x40], np.uint8)   # E4M3 0.5, 1, 2


def _nvfp4_exact(seed, G, rows, cols):
    """Random E2M1 codes, power-of-two E4M3 scales and global scales, and the
    matrices they define (float64, by the closed-form E2M1 table)."""
    rng = np.random.default_rng(seed)
    nib = rng.integers(0, 16, size=(G, rows, cols), dtype=np.uint8)
    codes = (nib[..., 0::2] | (nib[..., 1::2] << 4)).astype(np.uint8)
    scales = rng.choice(POW2_SCALES, size=(G, rows, cols // 16))
    gs = rng.choice(np.array([0.25, 0.5, 1.0], np.float32), size=G)
    mag = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    val = np.where(nib & 8, -1.0, 1.0) * mag[nib & 7]
    sv = {0x30: 0.5, 0x38: 1.0, 0x40: 2.0}
    sval = np.vectorize(sv.get)(scales).astype(np.float64)
    w = val * np.repeat(sval, 16, axis=2) * gs.astype(np.float64)[:, None, None]
    return codes, scales, gs, w


def _setup(m):
    import torch
    cfg = m.make_config(H, E, 2, 1, I, NV)
    c1, s1, g1, w1 = _nvfp4_exact(1, E + 1, I, H)
    c3, s3, g3, w3 = _nvfp4_exact(2, E + 1, I, H)
    c2, s2, g2, w2 = _nvfp4_exact(3, E + 1, H, I)
    host = {"router_w": synth.normal_bf16(0, 1, (E, H), 0.05), "router_bias": None,
            "w1": c1[:E], "w3": c3[:E], "w2": c2[:E], "s1": s1[:E], "s3": s3[:E], "s2": s2[:E],
            "g1": g1[:E], "g3": g3[:E], "g2": g2[:E],
            "sw1": c1[E:], "sw3": c3[E:], "sw2": c2[E:], "ss1": s1[E:], "ss3": s3[E:], "ss2": s2[E:],
            "sg1": g1[E:], "sg3": g3[E:], "sg2": g2[E:]}
    dev = m.upload_weights({k: (np.ascontiguousarray(v) if v is not None else None) for k, v in host.items()})
    offsets = np.concatenate([[0], np.cumsum(COUNTS)]).astype(np.int32)
    R = int(offsets[-1])
    group = np.repeat(np.arange(E + 1), COUNTS)
    ws = torch.empty(m.moe_workspace_bytes(cfg, -(-R // 3)), dtype=torch.uint8, device="cuda")
    return cfg, dev, (w1, w3, w2), offsets, R, group, ws


def test_nvfp4_gate_up_exact(m, variant):
    import torch
    cfg, dev, (w1, w3, _), offsets, R, group, ws = _setup(m)
    a = np.random.default_rng(4).integers(-4, 5, size=(R, H)).astype(np.float64)
    out = torch.full((R, 2, I), float("nan"), dtype=torch.float32, device="cuda")
    m.moe_grouped_gemm(cfg, m.MOE_STAGE_GATE_UP_RAW, R, m.to_device(offsets),
                       m.to_device(synth.f32_to_bf16(a.astype(np.float32))), None, m.make_weights(dev), out, ws)
    assert m.moe_read_status(ws) == 0
    ref = np.empty((R, 2, I))
    for g in range(E + 1):
        rr = group == g
        ref[rr, 0] = a[rr] @ w1[g].T
        ref[rr, 1] = a[rr] @ w3[g].T
    assert np.array_equal(ref, ref.astype(np.float32).astype(np.float64))  # exact in fp32
    got = out.cpu().numpy().astype(np.float64)
    bad = np.argwhere(got != ref)
    assert bad.size == 0, f"{len(bad)} sums differ, first {bad[:4].tolist()}"


def test_nvfp4_down_exact(m, variant):
    import torch
    cfg, dev, (_, _, w2), offsets, R, group, ws = _setup(m)
    a = np.random.default_rng(5).integers(-4, 5, size=(R, I)).astype(np.float64)
    gate = np.random.default_rng(6).choice(np.array([0.5, 1.0, 2.0], np.float32), size=R)
    y = torch.empty((R, H), dtype=torch.bfloat16, device="cuda")
    m.moe_grouped_gemm(cfg, m.MOE_STAGE_DOWN, R, m.to_device(offsets),
                       m.to_device(synth.f32_to_bf16(a.astype(np.float32))), None, m.make_weights(dev), y, ws,
                       row_gate=m.to_device(gate))
    assert m.moe_read_status(ws) == 0
    ref = np.empty((R, H))
    for g in range(E + 1):
        rr = group == g
        ref[rr] = a[rr] @ w2[g].T
    ref *= gate[:, None].astype(np.float64)
    assert np.array_equal(ref, ref.astype(np.float32).astype(np.float64))
    want = synth.f32_to_bf16(ref.astype(np.float32))
    got = y.view(torch.int16).cpu().numpy().view(np.uint16)
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{len(bad)} outputs differ, first {bad[:4].tolist()}"


LAYER_CASES = [
    (synth.MoeShape("nvfp4-small", T=40, hidden=256, n_experts=16, top_k=2, n_shared=1, inter=256, wdtype=NV,
                    seed=50), None),
    (synth.MoeShape("nvfp4-mid", T=300, hidden=512, n_experts=24, top_k=4, n_shared=1, inter=512, wdtype=NV,
                    seed=51), None),
    (synth.MoeShape("nvfp4-noshared", T=77, hidden=256, n_experts=12, top_k=3, n_shared=0, inter=256, wdtype=NV,
                    seed=52), None),
    (synth.MoeShape("step5-decode-nvfp4", T=64, wdtype=NV, seed=53), 24),
    (synth.MoeShape("step5-nvfp4-T1024", T=1024, wdtype=NV, seed=54), 24),
]


@pytest.mark.parametrize("shape,n_sample", LAYER_CASES, ids=lambda v: getattr(v, "name", str(v)))
def test_nvfp4_layer_parity(m, shape, n_sample, variant):
    import torch
    x, w = synth.make_x(shape), synth.make_weights(shape)
    idx_r, gate_r, logits_r = oracle.route(x, w["router_w"], w["router_bias"], shape.top_k, want_logits=True)
    cfg = m.make_config(shape.hidden, shape.n_experts, shape.top_k, shape.n_shared, shape.inter, shape.wdtype)
    wd = m.upload_weights(w)
    T = shape.T
    out = torch.empty((T, shape.hidden), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((T, shape.top_k), dtype=torch.int32, device="cuda")
    gate = torch.empty((T, shape.top_k), dtype=torch.float32, device="cuda")
    ws = torch.empty(m.moe_workspace_bytes(cfg, T), dtype=torch.uint8, device="cuda")
    m.moe_forward(cfg, T, m.to_device(x), m.make_weights(wd), out, ws, topk_idx=idx, topk_w=gate)
    assert m.moe_read_status(ws) == 0
    check_routing(idx.cpu().numpy(), gate.cpu().numpy(), logits_r, idx_r, gate_r)
    uniq = np.flatnonzero(unique_tokens(logits_r, shape.top_k))
    toks = uniq if n_sample is None else np.sort(np.random.default_rng(shape.seed).choice(uniq, n_sample, False))
    ref, _, _ = oracle.moe_tokens(shape, w, x, idx_r, gate_r, tokens=toks)
    got = bf16_bits_to_f64(out.view(torch.int16).cpu().numpy().view(np.uint16)[toks])
    err, per_tok = frob_rel(got, ref), rows_rel(got, ref)
    print(f"{shape.name}: {toks.size} tokens, rel Frobenius {err:.2e}, per-token max {per_tok.max():.2e}")
    assert err < tol_for(shape.wdtype) and per_tok.max() < tol_for(shape.wdtype)
