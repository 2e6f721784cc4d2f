"""Shared helpers of the GPU parity tests (tolerances and comparisons)."""
import numpy as np
import torch

import oracle as O

# Output tolerances: bf16 / fp8-cache paths: max-abs 2e-2 and mean-abs 2e-3;
# fp32 paths: relative 1e-4 per element (with a 1e-5 absolute floor for
# outputs near zero, where a relative bound has no meaning).
BF16_MAX_ABS, BF16_MEAN_ABS = 2e-2, 2e-3
F32_REL, F32_ABS_FLOOR = 1e-4, 1e-5
# Top-k sets are compared exactly wherever the oracle's k-th / (k+1)-th gap
# exceeds this; elsewhere the GPU set must still be a valid top-k up to it.
TOPK_GAP = 1e-3


def host(t):
    return t.detach().to("cpu")


def check_close(gpu, ref, dtype, what=""):
    g = O.f64(host(gpu))
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.all(np.isfinite(g)), what
    err = np.abs(g - r)
    if dtype == torch.float32:
        bad = err > F32_REL * np.abs(r) + F32_ABS_FLOOR
        assert not bad.any(), f"{what}: {bad.sum()} elements beyond 1e-4 rel, max err " \
                              f"{err.max():.3e}"
    else:
        assert err.max() <= BF16_MAX_ABS, f"{what}: max abs err {err.max():.3e}"
        assert err.mean() <= BF16_MEAN_ABS, f"{what}: mean abs err {err.mean():.3e}"
    return float(err.max())


def check_topk_row(gpu_row, scores, k, what=""):
    """gpu_row: int array [k]; scores: oracle fp64 scores of the V visible entries."""
    V = scores.shape[0]
    g = [int(s) for s in gpu_row]
    chosen = [s for s in g if s >= 0]
    # structure: ascending, unique, in range, -1 padding after them
    assert chosen == sorted(set(chosen)), (what, g[:8])
    assert all(0 <= s < V for s in chosen), what
    assert len(chosen) == min(k, V), (what, len(chosen), min(k, V))
    assert all(s == -1 for s in g[len(chosen):]), what
    if V <= k:
        return True
    order = np.sort(scores)[::-1]
    kth, nxt = order[k - 1], order[k]
    # validity: every chosen entry scores at least the k-th score (minus the gap)
    assert scores[chosen].min() >= kth - TOPK_GAP, (what, scores[chosen].min(), kth)
    if kth - nxt > TOPK_GAP:
        ref = O.topk_row(scores, k)
        assert np.array_equal(np.asarray(g), ref), what
        return True
    return False
