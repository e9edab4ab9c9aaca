"""Expert parallelism of the layer over one process per GPU (torch.distributed).

The pages deploy Step-5's MoE layers at TP = EP = 8: 44 of the 352 routed
experts on each of 8 GPUs, tokens replicated over the group (StepFun "Step-5
minimal inference" README, deployment section), and add the ranks' partial
results in rank order with FP32 accumulation (same README, "Long-output
stability"). One layer forward here, on every rank r of W:

  1. partial_r = moe_forward_ep_partial: routing over all experts, then rank
     r's routed experts expert_ranges(E, W)[r] and the shared expert for its
     tokens token_slices(T, W)[r]; fp32 [T, H], not rounded.
  2. exchange: rank r receives every rank's partial rows of its own token
     slice, in rank order (an all-to-all over the group).
  3. reduce: out[t] = bf16(sum over ranks in rank order, fp32) for the rank's
     token slice (moe_ep_reduce, one kernel).
  4. gather: every rank receives every slice of the bf16 output.

Steps 2-4 are a reduce-scatter whose sum order is fixed (a collective's own
reduction order is not) followed by an all-gather. With transport "p2p" the
partials live in symmetric memory and step 2 disappears: moe_ep_reduce reads
the peers' buffers directly over NVLink (plain loads; no TMA, no multicast).

The compute steps are passed in (`partial_fn`, `reduce_fn`), so the same
driver runs the CUDA library on GPUs and the oracle on CPU ranks (gloo) in the
tests.
"""
from __future__ import annotations

from typing import Callable, List, Sequence, Tuple


def even_split(n: int, parts: int) -> List[Tuple[int, int]]:
    """[lo, hi) ranges of n items over `parts`, in order, sizes differing by at
    most one (the first n % parts ranges one larger)."""
    if parts < 1 or n < 0:
        raise ValueError("need parts >= 1 and n >= 0")
    base, extra = divmod(n, parts)
    out, lo = [], 0
    for r in range(parts):
        hi = lo + base + (1 if r < extra else 0)
        out.append((lo, hi))
        lo = hi
    return out


def expert_ranges(n_experts: int, world: int) -> List[Tuple[int, int]]:
    """Routed experts [e0, e1) of each rank: 352 over 8 ranks is 44 each."""
    if world > n_experts:
        raise ValueError("every rank needs at least one routed expert")
    return even_split(n_experts, world)


def token_slices(T: int, world: int) -> List[Tuple[int, int]]:
    """Tokens [t0, t1) whose shared-expert rows (and output slice) each rank owns."""
    return even_split(T, world)


def exchange_token_slices(partial, slices: Sequence[Tuple[int, int]], rank: int, group=None):
    """All-to-all: rank r sends rows [t0_s, t1_s) of its partial to rank s and
    receives, from every rank in rank order, the rows of its own slice.
    Returns [world, n_rank, H] (block q = rank q's partial rows)."""
    import torch
    import torch.distributed as dist
    world = len(slices)
    n_me = slices[rank][1] - slices[rank][0]
    H = partial.shape[1]
    out = torch.empty((world * n_me, H), dtype=partial.dtype, device=partial.device)
    dist.all_to_all_single(out, partial.contiguous(), [n_me] * world, [hi - lo for lo, hi in slices], group=group)
    return out.view(world, n_me, H)


def gather_token_slices(mine, slices: Sequence[Tuple[int, int]], group=None):
    """All-gather of every rank's output slice into [T, H] (slices padded to the
    longest one for the collective, then trimmed)."""
    import torch
    import torch.distributed as dist
    world = len(slices)
    n_max = max(hi - lo for lo, hi in slices)
    H = mine.shape[1]
    pad = torch.zeros((n_max, H), dtype=mine.dtype, device=mine.device)
    pad[: mine.shape[0]] = mine
    # A pure copy: 2-byte types (bf16 bits) travel as float16 words, which
    # every backend moves bit for bit.
    wire = pad.view(torch.float16) if pad.element_size() == 2 else pad
    parts = [torch.empty_like(wire) for _ in range(world)]
    dist.all_gather(parts, wire, group=group)
    return torch.cat([p.view(mine.dtype)[: hi - lo] for p, (lo, hi) in zip(parts, slices)], dim=0)


def ep_forward(T: int, rank: int, world: int, n_experts: int,
               partial_fn: Callable[[int, int, int, int], "object"],
               reduce_fn: Callable[[list, int, int], "object"], group=None):
    """One expert-parallel layer forward on this rank (every rank calls it, in
    the same order). partial_fn(e0, e1, t0, t1) -> [T, H] fp32 partial;
    reduce_fn(blocks, t0, t1) -> the rank-ordered sum of `blocks` (one [n, H]
    block per rank, in rank order) for tokens [t0, t1), rounded to the output
    type. Returns the whole output [T, H] (identical on every rank)."""
    e0, e1 = expert_ranges(n_experts, world)[rank]
    slices = token_slices(T, world)
    t0, t1 = slices[rank]
    partial = partial_fn(e0, e1, t0, t1)
    blocks = exchange_token_slices(partial, slices, rank, group)
    mine = reduce_fn([blocks[q] for q in range(world)], t0, t1)
    return gather_token_slices(mine, slices, group)


class ExpertParallelLayer:
    """The CUDA path of one rank: this rank's expert weights on its GPU, the
    library's kernels for the compute steps and NCCL (or peer loads) between.

    weights: device tensors keyed like moe_weights, with w1/w3/w2 (and their
    FP8 scales) holding only this rank's experts expert_ranges(E, W)[rank].
    transport: "nccl" (all-to-all, then moe_ep_reduce on local memory) or
    "p2p" (partials in symmetric memory; moe_ep_reduce reads the peers'
    buffers over NVLink, after a barrier that orders their writes).
    """

    def __init__(self, cfg, weights: dict, T: int, rank: int, world: int, group=None, transport: str = "nccl"):
        import torch
        import mixture_experts_histogram_b200 as m
        if transport not in ("nccl", "p2p"):
            raise ValueError(transport)
        self.m, self.cfg, self.T, self.rank, self.world, self.group = m, cfg, T, rank, world, group
        self.transport = transport
        self.dev = torch.device("cuda", torch.cuda.current_device())
        self.w = m.make_weights(weights)
        self._keep = weights
        self.ws = torch.empty(m.moe_workspace_bytes(cfg, T), dtype=torch.uint8, device=self.dev)
        shape = (T, cfg.hidden)
        if transport == "p2p":
            import torch.distributed._symmetric_memory as symm
            import torch.distributed as dist
            self.partial = symm.empty(shape, dtype=torch.float32, device=self.dev)
            name = (group or dist.group.WORLD).group_name
            self.handle = symm.rendezvous(self.partial, name)
            self.peers = [self.handle.get_buffer(q, shape, torch.float32) for q in range(world)]
        else:
            self.partial = torch.empty(shape, dtype=torch.float32, device=self.dev)

    def forward(self, x):
        import torch
        m, cfg, T = self.m, self.cfg, self.T

        def partial_fn(e0, e1, t0, t1):
            m.moe_forward_ep_partial(cfg, T, x, self.w, e0, e1, t0, t1, self.partial, self.ws)
            return self.partial

        def reduce_fn(blocks, t0, t1):
            out = torch.empty((t1 - t0, cfg.hidden), dtype=torch.bfloat16, device=self.dev)
            m.moe_ep_reduce(blocks, t1 - t0, cfg.hidden, 0, t1 - t0, out)
            return out

        if self.transport == "nccl":
            return ep_forward(T, self.rank, self.world, cfg.n_experts, partial_fn, reduce_fn, self.group)
        # p2p: every rank writes its partial, a barrier orders those writes
        # before the peers' reads, and each rank reduces its own token slice
        # straight from the peers' buffers.
        e0, e1 = expert_ranges(cfg.n_experts, self.world)[self.rank]
        slices = token_slices(T, self.world)
        t0, t1 = slices[self.rank]
        partial_fn(e0, e1, t0, t1)
        self.handle.barrier(channel=0)
        out = torch.empty((T, cfg.hidden), dtype=torch.bfloat16, device=self.dev)
        m.moe_ep_reduce(self.peers, T, cfg.hidden, t0, t1, out)
        self.handle.barrier(channel=0)  # peers may overwrite their partials after this
        return gather_token_slices(out[t0:t1], slices, self.group)
