"""The full-size workloads, in the launch configuration bench.py times,
against the oracle on sampled outputs.

The GPU runs every call on the whole workload; the oracle recomputes what it
can one by one: the compressed entries (all of them, vectorised fp64), the
index scores and top-k sets of sampled query rows, and the attention output
of sampled rows (prefill) or sampled sequences (decode).  Sampled rows cover
the first position, the completion boundaries, the end and seeded random
positions.
"""
import numpy as np
import pytest
import torch

import bench
import compressed_sparse_attention_11_b200 as csa
import csa_inputs as G
import oracle as O
from _util import check_close, check_topk_row, host

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _sample_rows(n, m, count, seed):
    fixed = [0, m - 2, m - 1, m, 2 * m - 1, 127, 128, n // 2 - 1, n - 2, n - 1]
    rnd = np.random.default_rng(seed).integers(0, n, count).tolist()
    return sorted({r for r in fixed + rnd if 0 <= r < n})


def test_hca_prefill_full_size_sampled():
    """HCA prefill, n = 16384, m' = 128, 64 heads x 512, bf16."""
    w = G.HCA_PREFILL
    inp = G.prefill_inputs(w)
    d = {k: v.to(DEV) for k, v in inp.items()}
    kv = csa.csa_compress(d["ca"], None, d["za"], None, d["ba"], None, w.m)
    out = csa.hca_attn(d["q"], kv, d["kv_win"], w.window, d["sink"], w.scale, w.m)
    torch.cuda.synchronize()
    csa.csa_check()
    ref_kv = O.hca_compress(inp["ca"][0], inp["za"][0], inp["ba"], w.m)
    check_close(kv[0], ref_kv, torch.bfloat16, "hca entries")
    rows = _sample_rows(w.n, w.m, 12, 21)
    # the attention is checked on the GPU's own entries (bf16, as stored)
    kv_h = O.f64(host(kv)[0])
    ref = O.hca_attn(inp["q"][0], kv_h, O.f64(inp["kv_win"][0]), w.window, inp["sink"], w.scale,
                     w.m, rows=rows)
    got = host(out)[0, rows]
    for i, t in enumerate(rows):
        check_close(got[i], ref[i], torch.bfloat16, f"hca row {t}")


def test_csa_prefill_full_size_sampled():
    """CSA prefill, n = 65536, m = 4, indexer 64 x 128, top-k 512, 64 heads x 512."""
    w = G.CSA_PREFILL
    run = bench.CsaPrefill(w, torch.device(DEV))
    run.step()
    torch.cuda.synchronize()
    csa.csa_check()
    inp = run.host
    ref_kv = O.csa_compress(inp["ca"][0], inp["cb"][0], inp["za"][0], inp["zb"][0], inp["ba"],
                            inp["bb"], w.m)
    check_close(run.kv[0], ref_kv, torch.bfloat16, "csa entries")
    ref_ki = O.csa_compress(inp["ica"][0], inp["icb"][0], inp["iza"][0], inp["izb"][0],
                            inp["iba"], inp["ibb"], w.m)
    check_close(run.ki[0], ref_ki, torch.bfloat16, "index keys")
    rows = _sample_rows(w.n, w.m, 6, 22)
    idx = host(run.idx)[0]
    ki_h = O.f64(host(run.ki)[0])   # the indexer reads the stored bf16 keys
    exact = 0
    for t in rows:
        V = O.visible(t, w.m)
        scores = O.index_scores_row(inp["q_i"][0, t], inp["w_i"][0, t], ki_h, V)
        exact += check_topk_row(idx[t].numpy(), scores, w.k, f"top-k row {t}")
    assert exact >= len(rows) // 2, "too few rows with a clear k-th gap"
    # attention on the GPU's selection and entries
    kv_h = O.f64(host(run.kv)[0])
    ref = O.sparse_attn(inp["q"][0], kv_h, idx.numpy(), O.f64(inp["kv_win"][0]), w.window,
                        inp["sink"], w.scale, w.m, rows=rows)
    got = host(run.out)[0, rows]
    for i, t in enumerate(rows):
        check_close(got[i], ref[i], torch.bfloat16, f"csa row {t}")


# ------------------------------------------------------------------- decode ---

def _decode_run(w):
    """The cache as bench.py builds it, one decode step at t = w.t (no emission
    at that position), with the selection captured.  Returns host inputs,
    output and selection."""
    inp = G.decode_inputs(w, steps=1)
    E = w.t // w.m
    cache = csa.CsaCache(w.batch, E + 2, w.c, w.rope_dims, w.m, w.window, w.nh, w.is_hca,
                         c_i=w.c_i, nh_i=w.nh_i, k=w.k, device=DEV)
    cache.store_entries(0, inp["cache_kv"].to(DEV),
                        None if w.is_hca else inp["cache_ikey"].to(DEV))
    names = ("ca", "za", "kv_win") if w.is_hca else \
        ("ca", "cb", "za", "zb", "ica", "icb", "iza", "izb", "kv_win")
    tail = w.window + 2 * w.m
    cache.write_rows(w.t - tail, {nm: inp["rows_" + nm][:, :tail].contiguous().to(DEV)
                                  for nm in names})
    rows = {nm: inp["rows_" + nm][:, tail].contiguous().to(DEV) for nm in names}
    keys = ("ba",) if w.is_hca else ("ba", "bb", "iba", "ibb")
    biases = {k: inp[k].to(DEV) for k in keys}
    pos = torch.full((w.batch,), w.t, dtype=torch.int64, device=DEV)
    sel = None if w.is_hca else torch.empty((w.batch, w.k), dtype=torch.int32, device=DEV)
    out = cache.decode_step(pos, rows, biases, inp["sink"].to(DEV), w.scale, inp["q"][0].to(DEV),
                            None if w.is_hca else inp["q_i"][0].to(DEV),
                            None if w.is_hca else inp["w_i"][0].to(DEV), sel_out=sel)
    torch.cuda.synchronize()
    csa.csa_check()
    return inp, host(out), None if sel is None else host(sel)


def _check_decode_sequence(w, inp, out, sel, b):
    t, E = w.t, w.t // w.m
    assert (t + 1) % w.m != 0  # nothing is emitted at this position
    V = min(O.visible(t, w.m), E)
    X = O.dequantize_entries(*O.quantize_entries(inp["cache_kv"][b].numpy(), w.rope_dims))
    first = int(inp["first_pos"])
    win = np.stack([O.f64(inp["rows_kv_win"][b, u - first]) for u in O.window_rows(t, w.window)])
    if w.is_hca:
        chosen = list(range(V))
    else:
        K = O.dequantize_entries(*O.quantize_entries(inp["cache_ikey"][b].numpy(), 0))
        scores = O.index_scores_row(inp["q_i"][0, b], inp["w_i"][0, b], K, V)
        check_topk_row(sel[b].numpy(), scores, w.k, f"{w.name} selection b={b}")
        chosen = [int(s) for s in sel[b] if 0 <= int(s) < V]
    Et = np.concatenate([X[chosen], win], axis=0)
    ref = O.attend(inp["q"][0, b], Et, inp["sink"], w.scale)
    check_close(out[b], ref, torch.bfloat16, f"{w.name} b={b}")


def test_csa_decode_full_size_sampled():
    """CSA decode, batch 64 at context 131072 (32768 entries), top-k 512."""
    w = G.CSA_DECODE
    inp, out, sel = _decode_run(w)
    for b in (0, 29, 63):
        _check_decode_sequence(w, inp, out, sel, b)


def test_mixed_decode_full_size_sampled():
    """Long-context mixed decode, batch 4 at context 1048576: the CSA layer
    (262144 entries, top-k 512) and the HCA layer (8192 entries, dense)."""
    for w, seqs in ((G.MIXED_DECODE_CSA, (3,)), (G.MIXED_DECODE_HCA, (0, 3))):
        inp, out, sel = _decode_run(w)
        for b in seqs:
            _check_decode_sequence(w, inp, out, sel, b)
        del inp
