"""Comparison rules between the CUDA path and the oracle (test infrastructure).

Routing: the expert set of a token is unique wherever the gap between its k-th
and (k+1)-th largest oracle logits exceeds MARGIN; there the GPU must pick the
same experts, in an order consistent with the oracle logits (adjacent picks may
swap only when their logits are within MARGIN). Where the gap is smaller, any
k experts whose logits are all within MARGIN of the k-th largest are a correct
answer, and the check is that the GPU's set is such a set.

Outputs: relative Frobenius error ||out - ref|| / ||ref|| against the oracle's
fp64 result, at most 1e-2 for BF16 experts and 2e-2 for FP8 experts, both
pooled over the compared tokens and for every token (or expert row) on its own.
"""
import numpy as np

MARGIN = 1e-4
TOL_BF16 = 1e-2
TOL_FP8 = 2e-2


def tol_for(wdtype: int) -> float:
    return TOL_FP8 if wdtype == 1 else TOL_BF16


def check_routing(idx_gpu: np.ndarray, gate_gpu: np.ndarray, logits_ref: np.ndarray, idx_ref: np.ndarray,
                  gate_ref: np.ndarray, gate_rtol: float = 2e-5, gate_atol: float = 1e-6):
    """Returns (n_unique, n_ambiguous); raises AssertionError on a mismatch."""
    T, k = idx_ref.shape
    E = logits_ref.shape[1]
    srt = -np.sort(-logits_ref, axis=1)
    kth = srt[:, k - 1]
    nxt = srt[:, k] if k < E else np.full(T, -np.inf)
    unique = (kth - nxt) > MARGIN
    assert idx_gpu.shape == (T, k)
    assert np.all((idx_gpu >= 0) & (idx_gpu < E)), "expert index out of range"
    for t in range(T):
        g = idx_gpu[t]
        assert len(set(g.tolist())) == k, f"token {t}: repeated expert {g}"
        lg = logits_ref[t, g]
        assert np.all(np.diff(lg) <= MARGIN), f"token {t}: order {g} inconsistent with logits {lg}"
        if unique[t]:
            assert sorted(g.tolist()) == sorted(idx_ref[t].tolist()), f"token {t}: {g} vs {idx_ref[t]}"
            if np.all(np.abs(np.diff(logits_ref[t, idx_ref[t]])) > MARGIN):
                assert np.array_equal(g, idx_ref[t]), f"token {t}: order {g} vs {idx_ref[t]}"
            order = {e: j for j, e in enumerate(idx_ref[t].tolist())}
            ref = np.array([gate_ref[t, order[e]] for e in g.tolist()])
            np.testing.assert_allclose(gate_gpu[t], ref, rtol=gate_rtol, atol=gate_atol,
                                       err_msg=f"token {t} gates")
        else:
            assert np.all(lg >= kth[t] - MARGIN), f"token {t}: {g} not a top-{k} set within the margin"
        assert abs(float(gate_gpu[t].sum()) - 1.0) < 1e-5
    return int(unique.sum()), int((~unique).sum())


def unique_tokens(logits_ref: np.ndarray, k: int) -> np.ndarray:
    """Mask of tokens whose top-k expert set is unique under MARGIN."""
    srt = -np.sort(-logits_ref, axis=1)
    nxt = srt[:, k] if k < logits_ref.shape[1] else np.full(logits_ref.shape[0], -np.inf)
    return (srt[:, k - 1] - nxt) > MARGIN


def frob_rel(out: np.ndarray, ref: np.ndarray) -> float:
    out = out.astype(np.float64)
    ref = ref.astype(np.float64)
    return float(np.linalg.norm(out - ref) / max(np.linalg.norm(ref), 1e-300))


def rows_rel(out: np.ndarray, ref: np.ndarray) -> np.ndarray:
    """Relative Frobenius error of each row (last axis) on its own."""
    out = out.astype(np.float64).reshape(-1, out.shape[-1])
    ref = ref.astype(np.float64).reshape(-1, ref.shape[-1])
    return np.linalg.norm(out - ref, axis=1) / np.maximum(np.linalg.norm(ref, axis=1), 1e-300)


def bf16_bits_to_f64(a: np.ndarray) -> np.ndarray:
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
