"""Host logic of bench.py: the algorithmic work that the roofline divides by,
and the roofline and traffic bookkeeping.

The work counts are pinned three ways: against entry sets built row by row
by the oracle on small inputs (with a top-k that really selects), against
the closed forms of the sums, and at the full workloads against the figures
the design states (41,410,112 entries for CSA prefill n = 65536, k = 512,
W = 128; 3,129,536 for HCA prefill n = 16384, m' = 128; 536,854,528
visible (query, key) pairs for the indexer at n = 65536, m = 4).
"""
import os

import numpy as np
import pytest
import torch

import bench
import oracle


def _brute_entry_count(n, m, k, window, seed=0):
    rng = np.random.default_rng(seed)
    E = n // m
    kv_comp = rng.standard_normal((max(E, 1), 4))
    kv_win = rng.standard_normal((n, 4))
    tot = 0
    for t in range(n):
        if k is None:
            rows = oracle.dense_entry_set(kv_comp[:E], kv_win, t, m, window)
        else:
            V = oracle.visible(t, m)
            # a real selection: the k best of random scores over the visible
            # entries, padded with -1 like the library's output
            sel = oracle.topk_row(rng.standard_normal(V), k) if V > 0 else np.array([], int)
            idx_row = np.full(k, -1, dtype=np.int64)
            idx_row[:len(sel)] = sel
            rows = oracle.sparse_entry_set(kv_comp[:E], idx_row, kv_win, t, m, window)
        tot += rows.shape[0]
    return tot


@pytest.mark.parametrize("n,m,k,window", [
    (64, 4, 3, 5), (200, 4, 7, 16), (96, 8, 2, 1), (300, 128, None, 128), (257, 16, None, 7)])
def test_entry_set_sum_matches_built_sets(n, m, k, window):
    assert bench.sum_entry_sets(n, m, k, window) == _brute_entry_count(n, m, k, window)


@pytest.mark.parametrize("n,m", [(64, 4), (1000, 4), (513, 128)])
def test_visible_sum_matches_definition(n, m):
    # the indexer scores every visible key of every query: count the pairs
    pairs = sum(len(range(oracle.visible(t, m))) for t in range(n))
    assert bench.sum_visible(n, m) == pairs


def test_visible_sum_closed_form():
    # sum_{t<n} floor((t+1)/m) with n a multiple of m: each value v in
    # 1 .. n/m - 1 occurs m times, n/m occurs once, 0 occurs m - 1 times
    for n, m in [(65536, 4), (16384, 128), (4096, 64)]:
        q = n // m
        assert bench.sum_visible(n, m) == m * (q - 1) * q // 2 + q


def test_workload_figures():
    assert bench.sum_visible(65536, 4) == 536_854_528
    assert bench.sum_entry_sets(65536, 4, 512, 128) == 41_410_112
    assert bench.sum_entry_sets(16384, 128, None, 128) == 3_129_536


def test_roofline_arithmetic():
    peaks = {"hbm_gbs": 5000.0, "bf16": 1000.0, "bf16_sustained": 800.0, "source": "measured"}
    r = bench.roofline("flops", 2e12, 4.0, peaks)      # 2 TFLOP in 4 ms
    assert r["bound"] == "tensor" and r["achieved"] == pytest.approx(500.0)
    assert r["frac"] == pytest.approx(0.5)
    r = bench.roofline("bytes", 1e9, 0.5, peaks)       # 1 GB in 0.5 ms
    assert r["bound"] == "hbm" and r["achieved"] == pytest.approx(2000.0)
    assert r["frac"] == pytest.approx(0.4)


def test_measured_traffic_follows_sources(monkeypatch):
    # a figure is reported exactly while every source it was measured on is
    # unchanged (a changed kernel reports null until it is measured again)
    import hashlib
    for call, entry in bench.MEASURED_TRAFFIC.items():
        fresh = all(hashlib.sha256(open(os.path.join(bench.ROOT, p), "rb").read()).hexdigest()[:16]
                    == d for p, d in entry["sources"].items())
        assert bench.measured_traffic(call) == (entry["bytes"] if fresh else None), call
    assert bench.measured_traffic("no_such_call") is None
    call, entry = next(iter(bench.MEASURED_TRAFFIC.items()))
    path = next(iter(entry["sources"]))
    stale = dict(entry, sources=dict(entry["sources"], **{path: "0" * 16}))
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, call, stale)
    assert bench.measured_traffic(call) is None


@pytest.mark.parametrize("batch,cap,m", [(64, 32770, 4), (3, 1, 4), (2, 300, 128), (5, 97, 1)])
def test_paged_block_table_is_a_partial_permutation(batch, cap, m):
    """The paged decode workload's table: enough blocks per sequence for the
    capacity, every physical block inside the pool and used at most once."""
    bt, pool = bench.paged_block_table(batch, cap, m)
    assert bt.dtype == torch.int32 and bt.shape[0] == batch
    assert bt.shape[1] * (128 // m) >= cap > (bt.shape[1] - 1) * (128 // m)
    flat = bt.flatten().tolist()
    assert len(set(flat)) == len(flat)
    assert min(flat) >= 0 and max(flat) < pool
    assert pool == batch * bt.shape[1] + 7
