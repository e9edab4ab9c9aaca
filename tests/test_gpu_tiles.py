"""Full-size expert rows, element by element, over every tile of the grouped GEMMs.

At the workloads' own sizes (T = 8192 uniform prefill, T = 32768 Zipf-skewed
long prefill, FP8 experts) the routing decision of the oracle goes through
moe_experts, the launch sequence the layer uses, and rows of its output y are
compared one by one with the oracle's evaluation of the same (token, expert)
pair. The rows are chosen so that every 128-row tile of every group (routed
experts and the shared expert) is looked at: its first and last rows at
T = 8192, one of them (alternating) at T = 32768, and always each group's
last row, the ragged tail of its last tile. A 256-row pair tile is two such
128-row tiles, so pair tiles are covered too. Bar: each row's relative
Frobenius error against the oracle within the FP8 tolerance 2e-2.
"""
import numpy as np
import pytest

import oracle
import synth
from conftest import cuda_available
from parity import bf16_bits_to_f64, rows_rel, tol_for

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module")
def m():
    import mixture_experts_histogram_b200 as mm
    from mixture_experts_histogram_b200 import build
    build.build()
    mm.load()
    return mm


def tile_rows(offsets: np.ndarray, both_ends: bool) -> np.ndarray:
    """Rows that touch every 128-row tile of every group, plus each group's last row."""
    rows = []
    for g in range(offsets.size - 1):
        lo, hi = int(offsets[g]), int(offsets[g + 1])
        for i, r0 in enumerate(range(lo, hi, 128)):
            r1 = min(r0 + 127, hi - 1)
            if both_ends:
                rows += [r0, r1]
            else:
                rows.append(r0 if i % 2 == 0 else r1)
        if hi > lo:
            rows.append(hi - 1)
    return np.unique(np.array(rows, dtype=np.int64))


@pytest.mark.parametrize("shape,both_ends", [(synth.PREFILL_FP8, True), (synth.LONG_SKEW_FP8, False)],
                         ids=["prefill-T8192", "long-skew-T32768"])
def test_expert_rows_cover_every_tile(m, shape, both_ends):
    import torch
    x = synth.make_x(shape)
    w = synth.make_weights(shape)
    idx_r, gate_r, _ = oracle.route(x, w["router_w"], w["router_bias"], shape.top_k)
    T, k, S, E = shape.T, shape.top_k, shape.top_k + shape.n_shared, shape.n_experts
    counts, offsets, perm, pos_r = oracle.permute(idx_r, E, shape.n_shared)

    cfg = m.make_config(shape.hidden, E, k, shape.n_shared, shape.inter, shape.wdtype)
    wd = m.upload_weights(w)
    y = torch.empty((S * T, shape.hidden), dtype=torch.bfloat16, device="cuda")
    pos = torch.empty((T, S), dtype=torch.int32, device="cuda")
    ws = torch.empty(m.moe_workspace_bytes(cfg, T), dtype=torch.uint8, device="cuda")
    m.moe_experts(cfg, T, m.to_device(x), m.to_device(idx_r), m.to_device(gate_r), m.make_weights(wd), y, pos, ws)
    assert m.moe_read_status(ws) == 0
    assert np.array_equal(pos.cpu().numpy(), pos_r)

    rows = tile_rows(offsets, both_ends)
    # Every tile of every group is hit.
    n_tiles = int(sum((int(c) + 127) // 128 for c in counts))
    assert n_tiles > 0 and rows.size >= n_tiles
    group = np.searchsorted(offsets, rows, side="right") - 1
    tok = perm[rows]
    slot = np.array([int(np.flatnonzero(pos_r[t] == r)[0]) for t, r in zip(tok, rows)])
    gates = np.where(slot < k, gate_r[tok, np.minimum(slot, k - 1)].astype(np.float64), 1.0)
    assert np.all(np.where(slot < k, idx_r[tok, np.minimum(slot, k - 1)], E) == group)

    got_t = y.index_select(0, torch.from_numpy(rows).to("cuda"))
    got = bf16_bits_to_f64(got_t.view(torch.int16).cpu().numpy().view(np.uint16))
    del y, ws, wd
    ref = oracle.expert_rows(shape, w, x, tok, group) * gates[:, None]
    err = rows_rel(got, ref)
    worst = int(err.argmax())
    print(f"{shape.name}: {rows.size} rows over {n_tiles} tiles of {offsets.size - 1} groups; "
          f"max per-row rel error {err.max():.2e} (row {rows[worst]}, group {group[worst]}), "
          f"mean {err.mean():.2e}; hottest group {counts[:E].max()} rows, mean {counts[:E].mean():.1f}")
    assert err.max() < tol_for(shape.wdtype), (rows[worst], group[worst], err.max())
