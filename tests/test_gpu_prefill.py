"""GPU parity of the prefill entry points (through the C ABI) against the oracle.

Inputs come from the seeded generator; the oracle reads the same host bits.
Sizes span several tiles and a ragged tail; full-size workloads are in
test_gpu_workloads.py.
"""
import math

import numpy as np
import pytest
import torch

import compressed_sparse_attention_11_b200 as csa
import csa_inputs as G
import oracle as O
from _util import check_close, check_topk_row, host

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _streams(B, n, c, m, dt, seed, overlap=True):
    t = dict(ca=G.normal((B, n, c), seed, 1, dtype=dt), za=G.normal((B, n, c), seed, 3, dtype=dt),
             ba=G.normal((m, c), seed, 5, std=0.1, dtype=torch.float32))
    if overlap:
        t.update(cb=G.normal((B, n, c), seed, 2, dtype=dt), zb=G.normal((B, n, c), seed, 4, dtype=dt),
                 bb=G.normal((m, c), seed, 6, std=0.1, dtype=torch.float32))
    return t


@pytest.mark.parametrize("B,n,c,m,dt", [
    (2, 1030, 128, 4, torch.float32),     # ragged tail (1030 = 257*4 + 2)
    (1, 4100, 512, 4, torch.bfloat16),
    (3, 64, 8, 4, torch.float32),         # narrowest dim
    (1, 7, 16, 4, torch.bfloat16),        # one entry + tail
    (1, 1030, 136, 8, torch.bfloat16),    # 16 rows per entry: rows split over thread groups
    (2, 2048 + 64, 512, 64, torch.bfloat16),  # 128 rows: two rounds per thread
    (1, 512, 40, 16, torch.float32),      # fp32, 32 rows, 5 chunks
    # bf16, one thread per (entry, 4 dims): entries across warps and blocks
    (2, 1030, 128, 4, torch.bfloat16),    # 32 threads an entry, ragged tail rows
    (3, 200, 64, 2, torch.bfloat16),      # 16 threads an entry, three sequences
    (1, 777, 256, 1, torch.bfloat16),     # m = 1 (DSA), two rows per entry
    (2, 12, 512, 4, torch.bfloat16),      # fewer entries than a block holds
])
def test_csa_compress_parity(B, n, c, m, dt):
    s = _streams(B, n, c, m, dt, seed=11)
    d = {k: v.to(DEV) for k, v in s.items()}
    out = csa.csa_compress(d["ca"], d["cb"], d["za"], d["zb"], d["ba"], d["bb"], m)
    torch.cuda.synchronize()
    assert out.shape == (B, n // m, c)
    for b in range(B):
        ref = O.csa_compress(s["ca"][b], s["cb"][b], s["za"][b], s["zb"][b], s["ba"], s["bb"], m)
        check_close(out[b], ref, dt, f"csa compress b={b}")


@pytest.mark.parametrize("B,n,c,m,dt", [
    (2, 1024 + 77, 512, 128, torch.bfloat16),
    (1, 640, 64, 128, torch.float32),
    (1, 300, 32, 1, torch.float32),       # m = 1: identity
    (1, 96, 16, 32, torch.bfloat16),
    (1, 2048 + 5, 264, 512, torch.bfloat16),  # 512 rows: eight rounds per thread, 33 chunks
    (2, 40, 24, 5, torch.bfloat16),       # odd m within one round
    (2, 1000, 128, 8, torch.bfloat16),    # eight own rows per entry, one thread each
    (1, 130, 64, 1, torch.bfloat16),      # m = 1 through the per-thread rows: identity
])
def test_hca_compress_parity(B, n, c, m, dt):
    s = _streams(B, n, c, m, dt, seed=12, overlap=False)
    d = {k: v.to(DEV) for k, v in s.items()}
    out = csa.csa_compress(d["ca"], None, d["za"], None, d["ba"], None, m)
    torch.cuda.synchronize()
    for b in range(B):
        ref = O.hca_compress(s["ca"][b], s["za"][b], s["ba"], m)
        check_close(out[b], ref, dt, f"hca compress b={b}")
    if m == 1:
        assert torch.equal(host(out), s["ca"])


@pytest.mark.parametrize("overlap,m,c", [(True, 4, 512), (False, 128, 512), (True, 64, 136)])
def test_compress_single_infinite_logit_copies_its_row(overlap, m, c):
    """One logit at +inf (every dim of one own-block row per entry) takes all
    the weight: the entry is that row of C, bit for bit."""
    n = 64 * m
    s = _streams(1, n, c, m, torch.bfloat16, seed=14, overlap=overlap)
    E = n // m
    pick = np.random.default_rng(14).integers(0, m, E)
    rows = np.arange(E) * m + pick
    s["za"][0, rows] = float("inf")
    d = {k: v.to(DEV) for k, v in s.items()}
    if overlap:
        out = csa.csa_compress(d["ca"], d["cb"], d["za"], d["zb"], d["ba"], d["bb"], m)
    else:
        out = csa.csa_compress(d["ca"], None, d["za"], None, d["ba"], None, m)
    torch.cuda.synchronize()
    assert torch.equal(host(out)[0], s["ca"][0, rows])


def test_compress_empty_and_short():
    s = _streams(1, 3, 16, 4, torch.float32, seed=13)
    d = {k: v.to(DEV) for k, v in s.items()}
    out = csa.csa_compress(d["ca"], d["cb"], d["za"], d["zb"], d["ba"], d["bb"], 4)
    assert out.shape == (1, 0, 16)


# ------------------------------------------------------------------ indexer ---

def _index_inputs(B, n, H, ci, m, dt, seed):
    q = G.normal((B, n, H, ci), seed, 15, dtype=dt)
    w = G.uniform((B, n, H), seed, 16)
    k = G.normal((B, n // m, ci), seed, 21, dtype=dt)
    return q, w, k


@pytest.mark.parametrize("B,n,H,ci,m,k,dt,rows", [
    (1, 1024, 4, 64, 4, 32, torch.float32, None),          # tiny workload, every row
    (2, 1030, 4, 64, 4, 32, torch.float32, None),          # ragged, batch 2
    (1, 4096, 64, 128, 4, 512, torch.bfloat16, "sample"),  # V up to 1024 > k
    (1, 300, 3, 24, 4, 5, torch.bfloat16, None),           # odd head count and dim
    # tensor-core indexer shapes (bf16, c_i in {64, 128}, nh_i in {16..128})
    (2, 1000, 64, 128, 4, 64, torch.bfloat16, "sample"),   # ragged query tile, batch 2
    (1, 2100, 16, 64, 4, 100, torch.bfloat16, "sample"),
    (1, 1500, 32, 128, 4, 33, torch.bfloat16, "sample"),
    (1, 1100, 128, 64, 4, 20, torch.bfloat16, "sample"),
    (1, 600, 64, 128, 1, 200, torch.bfloat16, "sample"),   # m = 1 (token-level selection)
])
def test_index_topk_parity(B, n, H, ci, m, k, dt, rows):
    q, w, kk = _index_inputs(B, n, H, ci, m, dt, seed=17)
    idx = csa.csa_index_topk(q.to(DEV), w.to(DEV), kk.to(DEV), m, k)
    csa.csa_check()
    g = host(idx).numpy()
    rr = range(n) if rows is None else sorted(set(list(range(0, 12)) + list(range(n - 40, n)) +
                                                 list(range(3, n, 97))))
    exact = 0
    for b in range(B):
        for t in rr:
            V = O.visible(t, m)
            sc = O.index_scores_row(q[b, t], w[b, t], kk[b], V)
            exact += check_topk_row(g[b, t], sc, k, f"b={b} t={t}")
    assert exact > 0.9 * B * len(rr)


@pytest.mark.parametrize("dt,H,ci", [(torch.float32, 1, 16), (torch.bfloat16, 1, 16),
                                     (torch.bfloat16, 16, 64), (torch.bfloat16, 64, 128)])
def test_index_topk_integer_scores_bit_exact(dt, H, ci):
    """Head 0 has q = (256, 1, 0..) and w = 1, the other heads q = 0; key s is
    (hi_s, lo_s, 0..): every score is the integer 256*hi + lo, exact in bf16
    inputs and fp32 sums, with deliberate ties (repeated pairs) that must
    resolve to the smaller index.  H > 1 runs the tensor-core indexer."""
    n, m, k = 2048, 4, 37
    E = n // m
    r = np.random.default_rng(3)
    hi = r.integers(0, 200, E)
    lo = r.integers(0, 256, E)
    dup = r.choice(E, 60, replace=False)
    hi[dup[:30]], lo[dup[:30]] = hi[dup[30:]], lo[dup[30:]]
    keys = np.zeros((1, E, ci))
    keys[0, :, 0], keys[0, :, 1] = hi, lo
    q = np.zeros((1, n, H, ci))
    q[:, :, 0, 0], q[:, :, 0, 1] = 256.0, 1.0
    w = np.ones((1, n, H), dtype=np.float32)
    qt, kt = torch.tensor(q, dtype=dt), torch.tensor(keys, dtype=dt)
    idx = host(csa.csa_index_topk(qt.to(DEV), torch.tensor(w).to(DEV), kt.to(DEV), m, k)).numpy()
    csa.csa_check()
    scores = 256.0 * hi + lo
    for t in range(n):
        V = O.visible(t, m)
        assert np.array_equal(idx[0, t], O.topk_row(scores[:V], k)), t


# ---------------------------------------------------------------- attention ---

def _attn_inputs(B, n, nh, c, m, dt, seed, sink_scalar=None):
    q = G.normal((B, n, nh, c), seed, 14, dtype=dt)
    kv = G.normal((B, n // m, c), seed, 22, dtype=dt)
    win = G.normal((B, n, c), seed, 13, dtype=dt)
    sink = torch.full((nh,), float(sink_scalar)) if sink_scalar is not None else \
        G.normal((nh,), seed, 17, dtype=torch.float32)
    return q, kv, win, sink


def _random_selection(B, n, m, k, seed):
    r = np.random.default_rng(seed)
    idx = np.full((B, n, k), -1, dtype=np.int32)
    for b in range(B):
        for t in range(n):
            V = O.visible(t, m)
            ch = np.sort(r.choice(V, size=min(k, V), replace=False)) if V else []
            idx[b, t, :len(ch)] = ch
    return idx


@pytest.mark.parametrize("B,n,nh,c,m,k,W,dt,rows", [
    (1, 1024, 16, 128, 4, 32, 128, torch.float32, None),
    (2, 777, 8, 64, 4, 16, 40, torch.float32, None),
    (1, 2048, 64, 512, 4, 512, 128, torch.bfloat16, "sample"),
    (1, 200, 12, 96, 4, 7, 9, torch.bfloat16, None),
])
def test_sparse_attn_parity(B, n, nh, c, m, k, W, dt, rows):
    q, kv, win, sink = _attn_inputs(B, n, nh, c, m, dt, seed=19)
    idx = _random_selection(B, n, m, k, seed=5)
    out = csa.csa_sparse_attn(q.to(DEV), kv.to(DEV), torch.tensor(idx).to(DEV), win.to(DEV), W,
                              sink.to(DEV), 1 / math.sqrt(c), m)
    csa.csa_check()
    g = host(out)
    rr = list(range(n)) if rows is None else sorted(set(list(range(0, 8)) + list(range(n - 8, n)) +
                                                        list(range(5, n, 61))))
    for b in range(B):
        ref = O.sparse_attn(q[b], kv[b], idx[b], win[b], W, sink, 1 / math.sqrt(c), m, rows=rr)
        check_close(g[b, rr], ref, dt, f"sparse attn b={b}")


def _messy_selection(B, n, m, k, seed):
    """Valid entries in ascending order with -1, negative and future (>= V)
    indices sprinkled between them; only the valid ones may be attended."""
    r = np.random.default_rng(seed)
    idx = np.full((B, n, k), -1, dtype=np.int32)
    for b in range(B):
        for t in range(n):
            V = O.visible(t, m)
            cnt = int(r.integers(0, min(k, V) + 1)) if V else 0
            ch = np.sort(r.choice(V, size=cnt, replace=False)) if cnt else np.zeros(0, int)
            slots = np.sort(r.choice(k, size=cnt, replace=False))
            row = r.choice([-1, -5, V, V + 3, 10 ** 6], size=k).astype(np.int32)
            row[slots] = ch
            idx[b, t] = row
    return idx


@pytest.mark.parametrize("B,n,k,W,sink_none", [
    (2, 700, 96, 200, False),    # window longer than a tile boundary, batch 2
    (1, 300, 2048, 7, True),     # the largest selection, tiny window, no sink
])
def test_sparse_attn_tensor_core_messy_selection(B, n, k, W, sink_none):
    nh, c, m = 64, 512, 4
    q, kv, win, sink = _attn_inputs(B, n, nh, c, m, torch.bfloat16, seed=41)
    idx = _messy_selection(B, n, m, k, seed=6)
    s_dev = None if sink_none else sink.to(DEV)
    out = csa.csa_sparse_attn(q.to(DEV), kv.to(DEV), torch.tensor(idx).to(DEV), win.to(DEV), W,
                              s_dev, 1 / math.sqrt(c), m)
    csa.csa_check()
    g = host(out)
    rr = sorted(set(list(range(0, 12)) + list(range(n - 12, n)) + list(range(5, n, 23))))
    for b in range(B):
        ref = O.sparse_attn(q[b], kv[b], idx[b], win[b], W, None if sink_none else sink,
                            1 / math.sqrt(c), m, rows=rr)
        check_close(g[b, rr], ref, torch.bfloat16, f"sparse attn b={b}")


@pytest.mark.parametrize("B,n,k,W", [
    (1, 3, 4, 128),      # fewer queries than SMs, no compressed entry visible yet
    (2, 300, 130, 64),   # selection rows not whole 16-byte units: read in place
    (1, 150, 1, 5),      # a single selection, a short window
])
def test_sparse_attn_tensor_core_edge_shapes(B, n, k, W):
    nh, c, m = 64, 512, 4
    q, kv, win, sink = _attn_inputs(B, n, nh, c, m, torch.bfloat16, seed=47)
    idx = _random_selection(B, n, m, k, seed=8)
    out = csa.csa_sparse_attn(q.to(DEV), kv.to(DEV), torch.tensor(idx).to(DEV), win.to(DEV), W,
                              sink.to(DEV), 1 / math.sqrt(c), m)
    csa.csa_check()
    g = host(out)
    rr = sorted(set(list(range(0, min(n, 12))) + list(range(max(0, n - 12), n)) +
                    list(range(5, n, 29))))
    for b in range(B):
        ref = O.sparse_attn(q[b], kv[b], idx[b], win[b], W, sink, 1 / math.sqrt(c), m, rows=rr)
        check_close(g[b, rr], ref, torch.bfloat16, f"sparse attn b={b}")


@pytest.mark.parametrize("B,n,nh,c,m,W,dt,rows", [
    (1, 2048, 64, 512, 128, 128, torch.bfloat16, "sample"),
    (1, 5, 64, 512, 128, 128, torch.bfloat16, None),        # window only, 5 queries
    (2, 1100, 64, 512, 16, 64, torch.bfloat16, "sample"),   # more entries than a tile
    (2, 700, 16, 128, 32, 50, torch.float32, None),
    (1, 64, 4, 32, 128, 128, torch.float32, None),    # no entry complete: window only
])
def test_hca_attn_parity(B, n, nh, c, m, W, dt, rows):
    q, kv, win, sink = _attn_inputs(B, n, nh, c, m, dt, seed=23)
    out = csa.hca_attn(q.to(DEV), kv.to(DEV), win.to(DEV), W, sink.to(DEV), 1 / math.sqrt(c), m)
    csa.csa_check()
    g = host(out)
    rr = list(range(n)) if rows is None else sorted(set(list(range(0, 8)) + list(range(n - 8, n)) +
                                                        list(range(120, 140)) +
                                                        list(range(3, n, 53))))
    for b in range(B):
        ref = O.hca_attn(q[b], kv[b], win[b], W, sink, 1 / math.sqrt(c), m, rows=rr)
        check_close(g[b, rr], ref, dt, f"hca attn b={b}")


def test_sink_limits_on_gpu():
    """sink -> -inf equals no sink (plain softmax); a very large sink drives o to 0."""
    B, n, nh, c, m, W = 1, 300, 8, 64, 4, 32
    q, kv, win, _ = _attn_inputs(B, n, nh, c, m, torch.float32, seed=29)
    d = [x.to(DEV) for x in (q, kv, win)]
    idx = torch.tensor(_random_selection(B, n, m, 6, seed=2)).to(DEV)
    none = csa.csa_sparse_attn(d[0], d[1], idx, d[2], W, None, 0.125, m)
    neg = csa.csa_sparse_attn(d[0], d[1], idx, d[2], W, torch.full((nh,), -1e30, device=DEV),
                              0.125, m)
    big = csa.csa_sparse_attn(d[0], d[1], idx, d[2], W, torch.full((nh,), 60.0, device=DEV),
                              0.125, m)
    assert torch.equal(none, neg)
    assert host(big).abs().max() < 1e-20
    ref = O.sparse_attn(q[0], kv[0], host(idx)[0].numpy(), win[0], W, None, 0.125, m)
    check_close(host(none)[0], ref, torch.float32, "no sink")


# ------------------------------------------------------------ whole layer ----

def _run_layer(inp, w, dev=DEV):
    d = {k: v.to(dev) for k, v in inp.items()}
    kv = csa.csa_compress(d["ca"], d["cb"], d["za"], d["zb"], d["ba"], d["bb"], w.m)
    ki = csa.csa_compress(d["ica"], d["icb"], d["iza"], d["izb"], d["iba"], d["ibb"], w.m)
    idx = csa.csa_index_topk(d["q_i"], d["w_i"], ki, w.m, w.k)
    out = csa.csa_sparse_attn(d["q"], kv, idx, d["kv_win"], w.window, d["sink"], w.scale, w.m)
    torch.cuda.synchronize()
    return kv, ki, idx, out


def test_tiny_layer_end_to_end_against_oracle():
    """The fp32 tiny CSA workload (n=1024): compressor, indexer, top-k and
    attention each against the oracle, with the oracle fed the oracle's own
    upstream results."""
    w = G.TINY_CSA_PREFILL
    inp = G.prefill_inputs(w)
    kv, ki, idx, out = _run_layer(inp, w)
    b = 0
    kv_ref = O.csa_compress(inp["ca"][b], inp["cb"][b], inp["za"][b], inp["zb"][b], inp["ba"],
                            inp["bb"], w.m)
    ki_ref = O.csa_compress(inp["ica"][b], inp["icb"][b], inp["iza"][b], inp["izb"][b],
                            inp["iba"], inp["ibb"], w.m)
    check_close(host(kv)[b], kv_ref, torch.float32, "kv")
    check_close(host(ki)[b], ki_ref, torch.float32, "index keys")
    gi = host(idx)[b].numpy()
    same = 0
    for t in range(w.n):
        sc = O.index_scores_row(inp["q_i"][b, t], inp["w_i"][b, t], ki_ref, O.visible(t, w.m))
        same += check_topk_row(gi[t], sc, w.k, f"t={t}")
    assert same > 0.95 * w.n
    ref_idx = O.index_topk(inp["q_i"][b], inp["w_i"][b], ki_ref, w.m, w.k)
    rows = [t for t in range(w.n) if np.array_equal(gi[t], ref_idx[t])]
    ref = O.sparse_attn(inp["q"][b], kv_ref, ref_idx, inp["kv_win"][b], w.window, inp["sink"],
                        w.scale, w.m, rows=rows)
    check_close(host(out)[b, rows], ref, torch.float32, "attention")


def test_future_perturbation_leaves_past_unchanged_on_gpu():
    """Completion rule on the GPU path: changing every input at positions > t
    leaves outputs at positions <= t bit-identical (boundaries 3, 4, 7, 8)."""
    w = G.TINY_CSA_PREFILL
    inp = G.prefill_inputs(w, n=64)
    _, _, idx0, out0 = _run_layer(inp, w)
    for t in (3, 4, 7, 8, 37):
        pert = {}
        for key, v in inp.items():
            v = v.clone()
            if v.dim() >= 3:   # per-token tensors [B, n, ...]; biases and sinks are 1-2 D
                v[:, t + 1:] += 3.0
            pert[key] = v
        _, _, idx1, out1 = _run_layer(pert, w)
        assert torch.equal(host(out1)[:, :t + 1], host(out0)[:, :t + 1]), t
        assert torch.equal(host(idx1)[:, :t + 1], host(idx0)[:, :t + 1]), t
        assert not torch.equal(host(out1)[:, t + 1:], host(out0)[:, t + 1:])
