"""Expert parallelism on CPU ranks (gloo): the partition, the exchange and the
rank-ordered reduction of mixture_experts_histogram_b200.ep, with the oracle's
per-rank partials standing in for the GPU kernels.

Bar: with world_size 2 and 8, the ranks' oracle partials, exchanged and summed
in rank order, give every rank the full oracle output (fp64, up to summation
order), and the bf16 output equals the oracle's one rounding of the fp64 sum.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from mixture_experts_histogram_b200 import ep

SHAPE_ARGS = dict(name="ep-cpu", T=37, hidden=256, n_experts=24, top_k=4, n_shared=1, inter=128, seed=41)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_partition_covers_every_expert_and_token_once():
    assert ep.expert_ranges(352, 8) == [(44 * r, 44 * (r + 1)) for r in range(8)]
    for n, w in [(352, 3), (24, 8), (37, 8), (5, 5), (0, 4)]:
        rs = ep.even_split(n, w)
        assert rs[0][0] == 0 and rs[-1][1] == n and len(rs) == w
        assert all(a[1] == b[0] for a, b in zip(rs, rs[1:]))
        sizes = [hi - lo for lo, hi in rs]
        assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)
    with pytest.raises(ValueError):
        ep.expert_ranges(4, 8)


def _worker(rank, world, port, q, wdtype):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import sys
        sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
        import oracle
        import synth
        shape = synth.MoeShape(wdtype=wdtype, **SHAPE_ARGS)
        x, w = synth.make_x(shape), synth.make_weights(shape)
        idx, gate, _ = oracle.route(x, w["router_w"], w["router_bias"], shape.top_k)
        seen = {}

        def partial_fn(e0, e1, t0, t1):
            seen["range"] = (e0, e1, t0, t1)
            return torch.from_numpy(oracle.ep_partial(shape, w, x, idx, gate, e0, e1, t0, t1))

        def reduce_f64(blocks, t0, t1):
            acc = torch.zeros_like(blocks[0])
            for b in blocks:  # rank order
                acc += b
            return acc

        out = ep.ep_forward(shape.T, rank, world, shape.n_experts, partial_fn, reduce_f64)

        def reduce_bf16(blocks, t0, t1):
            acc = torch.zeros_like(blocks[0])
            for b in blocks:
                acc += b
            return torch.from_numpy(synth.f32_to_bf16(acc.numpy().astype(np.float32)).view(np.int16))

        out_b = ep.ep_forward(shape.T, rank, world, shape.n_experts, partial_fn, reduce_bf16)
        q.put((rank, seen["range"], out.numpy(), out_b.numpy().view(np.uint16)))
    except Exception:
        import traceback
        q.put((rank, "error", traceback.format_exc(), None))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 8])
@pytest.mark.parametrize("wdtype", [0, 1], ids=["bf16", "fp8"])
def test_ep_ranks_sum_to_the_whole_layer(world, wdtype):
    import oracle
    import synth
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, wdtype)) for r in range(world)]
    for p in procs:
        p.start()
    got = []
    for _ in range(world):
        item = q.get(timeout=240)
        assert item[1] != "error", item[2]
        got.append(item)
    got.sort(key=lambda v: v[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    shape = synth.MoeShape(wdtype=wdtype, **SHAPE_ARGS)
    x, w = synth.make_x(shape), synth.make_weights(shape)
    ref = oracle.moe_forward(shape, w, x)
    # the ranks' ranges partition the experts and the shared expert's tokens
    ranges = [g[1] for g in got]
    assert [r[:2] for r in ranges] == ep.expert_ranges(shape.n_experts, world)
    assert [r[2:] for r in ranges] == ep.token_slices(shape.T, world)
    for rank, _, out, out_b in got:
        err = np.linalg.norm(out - ref["out_f64"]) / np.linalg.norm(ref["out_f64"])
        assert err < 1e-12, (rank, err)
        # one rounding of (a different fp64 association of) the same sum
        diff = np.abs(out_b.astype(np.int32) - ref["out_bf16"].astype(np.int32))
        assert diff.max() <= 1 and np.mean(diff == 0) > 0.999, (rank, diff.max())
