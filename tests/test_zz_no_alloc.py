"""The indexer + top-k entry point for callers that cannot allocate.

Some callers cannot call cudaMalloc: their device memory belongs to another
framework's caching allocator, or they run inside a plugin hook that forbids
allocation at enqueue time.  csa_index_topk_noalloc serves them from a fixed
scratch array inside the library instead of a caller workspace.

Checked through the C ABI: on two calls in a row (different inputs, so stale
scratch contents would show) it returns exactly the indices that
csa_index_topk returns with a caller-provided workspace (top-k sets are
compared bit-exactly, as in the other top-k tests), and its rows are also
checked against the fp64 oracle's top-k.  The edges of its size check are
covered: a call that needs exactly the scratch's 2^21 score slots runs, one
that needs a little more is refused with a clear error before any launch,
and a sequence shorter than one block (no visible entry) gives all -1.

This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import compressed_sparse_attention_11_b200 as csa
import csa_inputs as G
import oracle as O
from _util import check_topk_row

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _inputs(B, n, H, ci, m, dt, seed):
    q = G.normal((B, n, H, ci), seed, 15, dtype=dt).to(DEV)
    w = G.uniform((B, n, H), seed, 16).to(DEV)
    kk = G.normal((B, n // m, ci), seed, 21, dtype=dt).to(DEV)
    return q, w, kk


def _noalloc_via_abi(q, w, kk, m, k):
    B, n, H, ci = q.shape
    out = torch.full((B, n, k), -7, dtype=torch.int32, device=DEV)
    dt = csa.CSA_BF16 if q.dtype == torch.bfloat16 else csa.CSA_F32
    st = csa.lib().csa_index_topk_noalloc(q.data_ptr(), w.data_ptr(), kk.data_ptr(), B, n, H, ci,
                                          m, k, dt, out.data_ptr(),
                                          torch.cuda.current_stream().cuda_stream)
    assert st == csa.CSA_OK, csa.lib().csa_last_error().decode()
    return out


@pytest.mark.parametrize("dt,B,n,H,ci,m,k", [
    (torch.bfloat16, 1, 2048, 64, 128, 4, 64),
    (torch.float32, 2, 1030, 4, 64, 4, 32),
])
def test_noalloc_matches_workspace_entry_point_on_two_calls(dt, B, n, H, ci, m, k):
    first = _inputs(B, n, H, ci, m, dt, seed=31)
    second = _inputs(B, n, H, ci, m, dt, seed=32)
    for inp in (first, second):
        ref = csa.csa_index_topk(*inp, m, k)          # caller-provided workspace
        got = _noalloc_via_abi(*inp, m, k)
        torch.cuda.synchronize()
        assert torch.equal(got, ref)
        _check_against_oracle(got, *inp, m, k)


def _check_against_oracle(got, q, w, kk, m, k, rows_per_seq=24):
    """Sampled rows of the no-allocation output against the oracle's top-k
    (exact where the k-th gap exceeds the tolerance, a valid top-k elsewhere)."""
    g = got.cpu().numpy()
    qh, wh, kh = q.cpu(), w.cpu(), kk.cpu()
    B, n = g.shape[0], g.shape[1]
    rows = sorted(set([0, 1, m - 1, m, n - 1] + list(range(5, n, max(1, n // rows_per_seq)))))
    exact = 0
    for b in range(B):
        for t in rows:
            V = O.visible(t, m)
            sc = O.index_scores_row(qh[b, t], wh[b, t], kh[b], V)
            exact += check_topk_row(g[b, t], sc, k, f"b={b} t={t}")
    assert exact > 0.9 * B * len(rows)


def test_noalloc_at_exactly_its_scratch_size():
    B, n, H, ci, m, k = 1, 2048, 16, 64, 2, 40      # 2048 * 1024 = 2^21 score slots
    inp = _inputs(B, n, H, ci, m, torch.bfloat16, seed=34)
    ref = csa.csa_index_topk(*inp, m, k)
    got = _noalloc_via_abi(*inp, m, k)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)
    _check_against_oracle(got, *inp, m, k, rows_per_seq=12)


def test_noalloc_short_sequence_has_no_entries():
    B, n, H, ci, m, k = 2, 3, 16, 64, 4, 8          # n < m: nothing is visible
    inp = _inputs(B, n, H, ci, m, torch.bfloat16, seed=35)
    got = _noalloc_via_abi(*inp, m, k)
    torch.cuda.synchronize()
    assert bool((got == -1).all())


@pytest.mark.parametrize("B,n,m", [(1, 8192, 4), (1, 2050, 2)])
def test_noalloc_rejects_work_beyond_its_scratch(B, n, m):
    H, ci, k = 4, 64, 32                             # n * floor(n/m) > 2^21
    q, w, kk = _inputs(B, n, H, ci, m, torch.bfloat16, seed=33)
    out = torch.zeros((B, n, k), dtype=torch.int32, device=DEV)
    st = csa.lib().csa_index_topk_noalloc(q.data_ptr(), w.data_ptr(), kk.data_ptr(), B, n, H, ci,
                                          m, k, csa.CSA_BF16, out.data_ptr(), None)
    assert st == csa.CSA_ERR_UNSUPPORTED
    assert "built-in scratch" in csa.lib().csa_last_error().decode()
    torch.cuda.synchronize()
    assert int(out.abs().sum()) == 0                 # nothing was launched
