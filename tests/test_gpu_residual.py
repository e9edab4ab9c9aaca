"""The fp32 residual stream around the layer: RMSNorm into the layer's input and
the combine that adds the layer's output back, against the oracle."""
import numpy as np
import pytest

import oracle
import synth
from parity import bf16_bits_to_f64, frob_rel, tol_for

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def m():
    import mixture_experts_histogram_b200 as mm
    from mixture_experts_histogram_b200 import build
    build.build()
    mm.load()
    return mm


@pytest.mark.parametrize("T,H", [(1, 4096), (333, 4096), (77, 384)])
def test_rmsnorm_matches_the_oracle_to_bf16_rounding(m, T, H):
    import torch
    rng = np.random.default_rng(T + H)
    r = (rng.standard_normal((T, H)) * 3.0).astype(np.float32)
    w = rng.uniform(0.5, 1.5, H).astype(np.float32)
    x = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    m.moe_rmsnorm(T, H, m.to_device(r), m.to_device(w), 1e-6, x)
    got = bf16_bits_to_f64(x.view(torch.int16).cpu().numpy().view(np.uint16))
    ref = oracle.rmsnorm(r, w, 1e-6)
    # One bf16 rounding of a value whose fp32 computation is off by a few fp32 ulps.
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 * 1.001 + 1e-30)
    ref_bf16 = bf16_bits_to_f64(synth.f32_to_bf16(ref.astype(np.float32)))
    assert np.mean(got == ref_bf16) > 0.99


@pytest.mark.parametrize("in_place", [False, True])
def test_combine_residual_is_the_fixed_order_fp32_sum_plus_residual(m, in_place):
    import torch
    T, H, k, S = 200, 512, 4, 1
    rng = np.random.default_rng(7 + in_place)
    rows = (k + S) * T
    y_bits = synth.f32_to_bf16((rng.standard_normal((rows, H)) * 0.5).astype(np.float32))
    pos = rng.permutation(rows).reshape(T, k + S).astype(np.int32)
    pos[3, 1] = -1  # a skipped pair
    r = (rng.standard_normal((T, H)) * 4.0).astype(np.float32)
    cfg = m.make_config(H, 16, k, S, 128, 0)
    rd = m.to_device(r)
    out = rd if in_place else torch.empty((T, H), dtype=torch.float32, device="cuda")
    m.moe_combine_residual(cfg, T, m.to_device(y_bits), m.to_device(pos), rd, out)
    got = out.cpu().numpy().astype(np.float64)
    y = bf16_bits_to_f64(y_bits)
    ref = oracle.add_residual(r, y, pos)
    mag = np.abs(r).astype(np.float64) + sum(np.abs(y[np.maximum(pos[:, j], 0)]) * (pos[:, j:j + 1] >= 0)
                                             for j in range(k + S))
    assert np.all(np.abs(got - ref) <= mag * 2e-6)


@pytest.mark.parametrize("wdtype", [synth.WDTYPE_BF16, synth.WDTYPE_FP8])
def test_norm_layer_residual_against_the_oracle(m, wdtype):
    """RMSNorm -> route -> experts -> combine with the residual add, end to end."""
    import dataclasses
    import torch
    shape = dataclasses.replace(synth.TINY, wdtype=wdtype, name=f"tiny-residual-{wdtype}")
    T, H, k, S = shape.T, shape.hidden, shape.top_k, shape.n_shared
    rng = np.random.default_rng(11)
    r = (rng.standard_normal((T, H)) * 2.0).astype(np.float32)
    nw = rng.uniform(0.8, 1.2, H).astype(np.float32)
    w = synth.make_weights(shape)
    x_ref = synth.f32_to_bf16(oracle.rmsnorm(r, nw, 1e-6).astype(np.float32))
    # CUDA path through the C ABI.
    cfg = m.make_config(H, shape.n_experts, k, S, shape.inter, wdtype)
    wd = m.upload_weights(w)
    rd = m.to_device(r)
    x = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    m.moe_rmsnorm(T, H, rd, m.to_device(nw), 1e-6, x)
    nb = m.moe_workspace_bytes(cfg, T)
    ws = torch.empty(max(nb, 1024), dtype=torch.uint8, device="cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    gate = torch.empty((T, k), dtype=torch.float32, device="cuda")
    m.moe_route(cfg, T, x, wd["router_w"], wd["router_bias"], idx, gate, None, ws)
    y = torch.empty(((k + S) * T, H), dtype=torch.bfloat16, device="cuda")
    pos = torch.empty((T, k + S), dtype=torch.int32, device="cuda")
    m.moe_experts(cfg, T, x, idx, gate, m.make_weights(wd), y, pos, ws)
    r_out = torch.empty((T, H), dtype=torch.float32, device="cuda")
    m.moe_combine_residual(cfg, T, y, pos, rd, r_out)
    assert m.moe_read_status(ws) == 0
    x_bits = x.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.mean(x_bits == x_ref) > 0.99  # the norm itself: see the test above
    # Oracle layer on the same bf16 input, then the residual add in fp64.
    ref = oracle.moe_forward(shape, w, x_bits)
    ref_r = r.astype(np.float64) + ref["out_f64"]
    got = r_out.cpu().numpy().astype(np.float64)
    # The layer's part of the result carries the layer's tolerance.
    assert frob_rel(got - r, ref_r - r) < tol_for(wdtype)
