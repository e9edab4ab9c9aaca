"""moe_permute_noalloc: the permutation for callers that cannot allocate.

Some callers cannot allocate device memory at all (a plugin inside a framework
that owns the device memory, a serving loop with memory reserved up front, a
latency-critical path where an allocation would stall the device), so they
cannot hand moe_permute a workspace. moe_permute_noalloc keeps its scratch in
a fixed device array inside the library instead. This file checks, through the
C ABI, that it gives exactly moe_permute's results on two calls in a row (the
scratch array is shared and keeps the previous call's contents), and that
sizes beyond the array are refused. It is named so that pytest collects it
last; it passes on its own and after the other tests.
"""
import numpy as np
import pytest

from conftest import cuda_available

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module", autouse=True)
def _library():
    from mixture_experts_histogram_b200 import build
    build.build()


def _routing(T, E, k, seed):
    rng = np.random.default_rng(seed)
    return np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)


def test_noalloc_permute_matches_moe_permute_on_two_calls():
    import torch
    import mixture_experts_histogram_b200 as m
    E, k, S = 352, 8, 1
    G = E + S
    for call, (T, seed) in enumerate([(8192, 1), (3000, 2)]):  # a large call, then a smaller one
        cfg = m.make_config(4096, E, k, S, 1536, 1)
        idx = m.to_device(_routing(T, E, k, seed))
        ref = [torch.empty(G, dtype=torch.int32, device="cuda"), torch.empty(G + 1, dtype=torch.int32, device="cuda"),
               torch.empty((k + S) * T, dtype=torch.int32, device="cuda"),
               torch.empty((T, k + S), dtype=torch.int32, device="cuda")]
        ws = torch.empty(m.moe_workspace_bytes(cfg, T), dtype=torch.uint8, device="cuda")
        m.moe_permute(cfg, T, idx, *ref, ws)
        got = [torch.full_like(t, -7) for t in ref]
        status = torch.full((1,), 99, dtype=torch.int32, device="cuda")
        m.moe_permute_noalloc(cfg, T, idx, *got, device_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, f"call {call}"
        for name, a, b in zip(("counts", "offsets", "perm", "pos"), ref, got):
            assert torch.equal(a, b), f"call {call}: {name} differs"


@pytest.mark.parametrize("T", [1, 64, 256, 257])
def test_noalloc_permute_matches_the_one_chunk_path(T):
    """T <= 256: moe_permute takes its one-launch path, this entry point the
    three-kernel one; both must give the same rows."""
    import torch
    import mixture_experts_histogram_b200 as m
    E, k, S = 352, 8, 1
    G = E + S
    cfg = m.make_config(4096, E, k, S, 1536, 1)
    idx = m.to_device(_routing(T, E, k, 40 + T))
    ref = [torch.empty(G, dtype=torch.int32, device="cuda"), torch.empty(G + 1, dtype=torch.int32, device="cuda"),
           torch.empty((k + S) * T, dtype=torch.int32, device="cuda"),
           torch.empty((T, k + S), dtype=torch.int32, device="cuda")]
    ws = torch.empty(m.moe_workspace_bytes(cfg, T), dtype=torch.uint8, device="cuda")
    m.moe_permute(cfg, T, idx, *ref, ws)
    got = [torch.full_like(t, -7) for t in ref]
    status = torch.full((1,), 99, dtype=torch.int32, device="cuda")
    m.moe_permute_noalloc(cfg, T, idx, *got, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for name, a, b in zip(("counts", "offsets", "perm", "pos"), ref, got):
        assert torch.equal(a, b), f"T={T}: {name} differs"


def test_noalloc_permute_zero_tokens_and_bad_index():
    import torch
    import mixture_experts_histogram_b200 as m
    E, k, S = 16, 2, 1
    cfg = m.make_config(256, E, k, S, 128, 0)
    counts = torch.full((E + S,), 5, dtype=torch.int32, device="cuda")
    offsets = torch.full((E + S + 1,), 5, dtype=torch.int32, device="cuda")
    status = torch.full((1,), 99, dtype=torch.int32, device="cuda")
    m.moe_permute_noalloc(cfg, 0, 1024, counts, offsets, 1024, 1024, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.count_nonzero(counts).item() == 0 and torch.count_nonzero(offsets).item() == 0
    T = 300
    idx_np = np.tile(np.array([[0, 1]], np.int32), (T, 1))
    idx_np[5, 1] = 99
    perm = torch.empty((k + S) * T, dtype=torch.int32, device="cuda")
    pos = torch.empty((T, k + S), dtype=torch.int32, device="cuda")
    m.moe_permute_noalloc(cfg, T, m.to_device(idx_np), counts, offsets, perm, pos, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == m.MOE_ERR_BAD_INDEX
    assert pos[5, 1].item() == -1 and counts[1].item() == T - 1


def test_noalloc_permute_refuses_sizes_beyond_its_scratch():
    import mixture_experts_histogram_b200 as m
    cfg = m.make_config(4096, 352, 8, 1, 1536, 1)
    T = 256 * 800  # 352 experts x 800 chunks of 256 tokens > 260,032 scratch ints
    with pytest.raises(m.MoeError) as e:
        m.moe_permute_noalloc(cfg, T, 1024, 1024, 1024, 1024, 1024, stream=0)
    assert e.value.code == m.MOE_ERR_UNSUPPORTED_SHAPE
