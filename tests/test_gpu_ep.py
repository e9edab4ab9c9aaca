"""Expert parallelism on one GPU: every rank's share computed in turn.

moe_forward_ep_partial runs one rank's experts and shared-expert tokens; the
ranks are run one after another on the same GPU (no kernel of one waits for
another), each into its own fp32 buffer, and moe_ep_reduce adds the buffers in
rank order. Checks:
  - one rank's partial (the pages' 44-expert share of 352 at TP = EP = 8)
    against the oracle's partial for that rank, token by token;
  - moe_ep_reduce bit for bit against torch's fp32 sum in rank order with one
    bf16 rounding;
  - the reduced layer output against the oracle (the layer's tolerance).
"""
import numpy as np
import pytest

import oracle
import synth
from conftest import cuda_available
from parity import bf16_bits_to_f64, frob_rel, rows_rel, tol_for, unique_tokens

from mixture_experts_histogram_b200 import ep

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module")
def m():
    import mixture_experts_histogram_b200 as mm
    from mixture_experts_histogram_b200 import build
    build.build()
    mm.load()
    return mm


def _rank_weights(wd: dict, e0: int, e1: int) -> dict:
    """This rank's expert slices (views) and the shared/router weights whole."""
    out = dict(wd)
    for k in ("w1", "w3", "w2", "s1", "s3", "s2"):
        if wd.get(k) is not None:
            out[k] = wd[k][e0:e1]
    return out


CASES = [
    (synth.MoeShape("ep8-step5-fp8", T=1024, wdtype=synth.WDTYPE_FP8, seed=31), 8, 24),
    (synth.MoeShape("ep3-bf16", T=300, hidden=512, n_experts=24, top_k=4, n_shared=1, inter=256, seed=32), 3, None),
    (synth.MoeShape("ep4-fp8-noshared", T=200, hidden=256, n_experts=16, top_k=2, n_shared=0, inter=128,
                    wdtype=synth.WDTYPE_FP8, seed=33), 4, None),
]


@pytest.mark.parametrize("shape,world,n_sample", CASES, ids=lambda v: getattr(v, "name", str(v)))
def test_ranks_partials_and_rank_ordered_reduce(m, shape, world, n_sample):
    import torch
    x, w = synth.make_x(shape), synth.make_weights(shape)
    idx_r, gate_r, logits_r = oracle.route(x, w["router_w"], w["router_bias"], shape.top_k, want_logits=True)
    T, H = shape.T, shape.hidden
    cfg = m.make_config(H, shape.n_experts, shape.top_k, shape.n_shared, shape.inter, shape.wdtype)
    wd = m.upload_weights(w)
    xd = m.to_device(x)
    ws = torch.empty(m.moe_workspace_bytes(cfg, T), dtype=torch.uint8, device="cuda")
    ranges, slices = ep.expert_ranges(shape.n_experts, world), ep.token_slices(T, world)
    partials = []
    for r in range(world):
        (e0, e1), (t0, t1) = ranges[r], slices[r]
        p = torch.empty((T, H), dtype=torch.float32, device="cuda")
        rw = _rank_weights(wd, e0, e1)
        m.moe_forward_ep_partial(cfg, T, xd, m.make_weights(rw), e0, e1, t0, t1, p, ws)
        assert m.moe_read_status(ws) == 0
        partials.append(p)

    # Rank 0's partial against the oracle's, on tokens with unique routing.
    uniq = np.flatnonzero(unique_tokens(logits_r, shape.top_k))
    toks = uniq if n_sample is None else np.sort(np.random.default_rng(shape.seed).choice(uniq, n_sample, False))
    (e0, e1), (t0, t1) = ranges[0], slices[0]
    toks = np.union1d(toks, [t0, max(t0, t1 - 1)])  # tokens of rank 0's shared slice
    toks = toks[np.isin(toks, uniq)]
    ref0 = oracle.ep_partial(shape, w, x, idx_r, gate_r, e0, e1, t0, t1, tokens=toks)
    got0 = partials[0].cpu().numpy()[toks].astype(np.float64)
    nz = np.linalg.norm(ref0, axis=1) > 0
    assert np.all(np.linalg.norm(got0[~nz], axis=1) == 0)  # tokens with no row on this rank stay zero
    if nz.any():
        err = rows_rel(got0[nz], ref0[nz])
        print(f"{shape.name}: rank 0 partial, {nz.sum()} tokens, max per-token rel error {err.max():.2e}")
        assert err.max() < tol_for(shape.wdtype)

    # The reduce kernel: torch's fp32 sum in rank order, one bf16 rounding.
    out = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    m.moe_ep_reduce(partials, T, H, 0, T, out)
    acc = torch.zeros((T, H), dtype=torch.float32, device="cuda")
    for p in partials:
        acc = acc + p
    assert torch.equal(out.view(torch.int16), acc.to(torch.bfloat16).view(torch.int16))
    # A token range only: rows outside it untouched.
    part = torch.full((T, H), 7.0, dtype=torch.bfloat16, device="cuda")
    lo, hi = T // 3, T // 3 + max(1, T // 5)
    m.moe_ep_reduce(partials, T, H, lo, hi, part)
    assert torch.equal(part[lo:hi], out[lo:hi]) and bool((part[:lo] == 7.0).all()) and bool((part[hi:] == 7.0).all())

    # The layer output against the oracle.
    toks_all = uniq if n_sample is None else np.sort(np.random.default_rng(shape.seed + 1).choice(uniq, n_sample, False))
    ref, _, _ = oracle.moe_tokens(shape, w, x, idx_r, gate_r, tokens=toks_all)
    got = bf16_bits_to_f64(out.view(torch.int16).cpu().numpy().view(np.uint16)[toks_all])
    assert frob_rel(got, ref) < tol_for(shape.wdtype)
    assert rows_rel(got, ref).max() < tol_for(shape.wdtype)


def test_ep_partial_argument_errors(m):
    import torch
    shape = synth.TINY
    cfg = m.make_config(shape.hidden, shape.n_experts, shape.top_k, shape.n_shared, shape.inter, shape.wdtype)
    wd = m.upload_weights(synth.make_weights(shape))
    ws = torch.empty(m.moe_workspace_bytes(cfg, shape.T), dtype=torch.uint8, device="cuda")
    x = m.to_device(synth.make_x(shape))
    p = torch.empty((shape.T, shape.hidden), dtype=torch.float32, device="cuda")
    for e0, e1, t0, t1 in [(3, 3, 0, 1), (-1, 4, 0, 1), (0, 17, 0, 1), (0, 4, 5, 2), (0, 4, 0, shape.T + 1)]:
        with pytest.raises(m.MoeError) as e:
            m.moe_forward_ep_partial(cfg, shape.T, x, m.make_weights(_rank_weights(wd, 0, 4)), e0, e1, t0, t1, p, ws)
        assert e.value.code == m.MOE_ERR_INVALID_ARG
    with pytest.raises(m.MoeError) as e:
        m.moe_ep_reduce([p] * 17, shape.T, shape.hidden, 0, shape.T, x)
    assert e.value.code == m.MOE_ERR_UNSUPPORTED_SHAPE
