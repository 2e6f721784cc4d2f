"""GPU parity of the decode entry points (cache store, row hand-off, decode
step) against the oracle's incremental decode sequence."""
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
CSA_STREAMS = ("ca", "cb", "za", "zb", "ica", "icb", "iza", "izb", "kv_win")
HCA_STREAMS = ("ca", "za", "kv_win")


def _quantize_all(x, rope):
    """Oracle cache form of every entry in x [E, c] (fp32)."""
    q = [O.quantize_entry(np.asarray(x[e], dtype=np.float32), rope) for e in range(x.shape[0])]
    return q


def code_distance(a, b):
    """|ordinal distance| between E4M3 codes of the same sign (sign flips count large)."""
    a = a.astype(np.int64)
    b = b.astype(np.int64)
    same_sign = (a & 0x80) == (b & 0x80)
    return np.where(same_sign, np.abs((a & 0x7F) - (b & 0x7F)), 1000)


@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
def test_store_entries_bit_exact(dt):
    B, E, c, rope, ci = 3, 50, 128, 32, 64
    kv = G.normal((B, E, c), 5, 20, dtype=dt)
    ik = G.normal((B, E, ci), 5, 21, dtype=dt)
    kv[0, 3] = 0.0                                   # amax 0: scale 1, codes 0
    kv[1, 4, 7] = 1e4                                # one huge element
    cache = csa.CsaCache(B, E + 5, c, rope, 4, 16, 8, False, c_i=ci, nh_i=4, k=8)
    cache.store_entries(2, kv.to(DEV), ik.to(DEV))
    torch.cuda.synchronize()
    got = {k: host(v) for k, v in cache.entries().items()}
    for b in range(B):
        for e in range(E):
            codes, scale, rp = O.quantize_entry(kv[b, e].float().numpy(), rope)
            assert np.array_equal(got["codes"][b, 2 + e].numpy(), codes), (b, e)
            assert got["scale"][b, 2 + e].item() == scale, (b, e)
            assert np.array_equal(got["rope"][b, 2 + e].double().numpy(), rp), (b, e)
            icodes, iscale, _ = O.quantize_entry(ik[b, e].float().numpy(), 0)
            assert np.array_equal(got["icodes"][b, 2 + e].numpy(), icodes), (b, e)
            assert got["iscale"][b, 2 + e].item() == iscale


def _block_table(B, cap, epb, seed):
    """A block table covering `cap` entries per sequence in a pool with a few
    spare blocks, the physical blocks in a random order."""
    nb = (cap + epb - 1) // epb
    pool = B * nb + 7
    perm = np.random.default_rng(seed).permutation(pool)[:B * nb]
    return torch.tensor(perm.reshape(B, nb), dtype=torch.int32, device=DEV), pool


def _setup(w, B, E, steps, seed, edit=None, paged=False):
    """Cache with E stored entries and raw rows up to position t0-1 (t0 = m*E).
    ``edit(inp)`` may change the host inputs in place before anything uses them.
    ``paged``: the entries in a pool of 128-token blocks behind a block table."""
    t0 = w.m * E
    inp = G.decode_inputs(w, entries=E, batch=B, t=t0, steps=steps, seed=seed)
    if edit is not None:
        edit(inp)
    first = int(inp["first_pos"])
    cap = E + steps // w.m + 2
    if paged:
        epb = 128 // w.m
        bt, pool = _block_table(B, cap, epb, seed)
        cache = csa.CsaCache(B, cap, w.c, w.rope_dims, w.m, w.window, w.nh, w.is_hca,
                             c_i=w.c_i, nh_i=w.nh_i, k=w.k, block_table=bt, block_tokens=128,
                             num_blocks=pool)
    else:
        cache = csa.CsaCache(B, cap, w.c, w.rope_dims, w.m, w.window, w.nh, w.is_hca,
                             c_i=w.c_i, nh_i=w.nh_i, k=w.k)
    cache.store_entries(0, inp["cache_kv"].to(DEV),
                        None if w.is_hca else inp["cache_ikey"].to(DEV))
    tail = w.window + 2 * w.m
    skip = max(0, -first)             # short histories start at position 0
    names = HCA_STREAMS if w.is_hca else CSA_STREAMS
    cache.write_rows(first + skip, {nm: inp["rows_" + nm][:, skip:tail].contiguous().to(DEV)
                                    for nm in names})
    return inp, cache, t0, first, tail, names


def _oracle_sequence(w, inp, b, E, first, tail, names):
    seq = O.DecodeSequence(w.c, w.rope_dims, w.m, w.window, w.is_hca, w.c_i)
    for e in range(E):
        seq.store_entry(inp["cache_kv"][b, e].numpy(),
                        None if w.is_hca else inp["cache_ikey"][b, e].numpy())
    for r in range(max(0, -first), tail):
        for nm in names:
            seq.put_row(nm, first + r, inp["rows_" + nm][b, r])
    return seq


def _biases(inp, w):
    keys = ("ba",) if w.is_hca else ("ba", "bb", "iba", "ibb")
    return {k: inp[k] for k in keys}


def _run_and_compare(w, B, E, steps, seed, check_seqs=None, edit=None, sel_exact=False,
                     paged=False):
    inp, cache, t0, first, tail, names = _setup(w, B, E, steps, seed, edit, paged)
    biases = _biases(inp, w)
    dbias = {k: v.to(DEV) for k, v in biases.items()}
    sink = inp["sink"].to(DEV)
    check_seqs = range(B) if check_seqs is None else check_seqs
    seqs = {b: _oracle_sequence(w, inp, b, E, first, tail, names) for b in check_seqs}
    for s in range(steps):
        t = t0 + s
        r = tail + s
        rows = {nm: inp["rows_" + nm][:, r].contiguous().to(DEV) for nm in names}
        pos = torch.full((B,), t, dtype=torch.int64, device=DEV)
        q = inp["q"][s].to(DEV)
        qi = None if w.is_hca else inp["q_i"][s].to(DEV)
        wi = None if w.is_hca else inp["w_i"][s].to(DEV)
        sel = None if w.is_hca else torch.empty((B, w.k), dtype=torch.int32, device=DEV)
        out = host(cache.decode_step(pos, rows, dbias, sink, w.scale, q, qi, wi, sel_out=sel))
        csa.csa_check()
        for b in check_seqs:
            ref, ref_sel = seqs[b].step(t, {nm: inp["rows_" + nm][b, r] for nm in names}, biases,
                                        inp["q"][s, b], None if w.is_hca else inp["q_i"][s, b],
                                        None if w.is_hca else inp["w_i"][s, b], inp["sink"],
                                        w.scale, w.k)
            check_close(out[b], ref, torch.bfloat16, f"step t={t} b={b}")
            if w.is_hca:
                continue
            if sel_exact:
                assert np.array_equal(host(sel)[b].numpy(), np.asarray(ref_sel, dtype=np.int32)), \
                    f"selection t={t} b={b}"
            else:  # exact wherever the k-th gap exceeds the tolerance, else a valid top-k
                V = min(O.visible(t, w.m), len(seqs[b].ikeys))
                K = np.stack([O.dequantize_entry(*e) for e in seqs[b].ikeys[:V]])
                scores = O.index_scores_row(inp["q_i"][s, b], inp["w_i"][s, b], K, V)
                check_topk_row(host(sel)[b].numpy(), scores, w.k, f"selection t={t} b={b}")
    # emitted entries agree with the oracle's from-scratch compression
    got = {k: host(v) for k, v in cache.entries().items()}
    n_emit = (t0 + steps) // w.m - E
    for b in check_seqs:
        for i in range(E, E + n_emit):
            codes, scale, rope = seqs[b].entries[i]
            assert abs(got["scale"][b, i].item() / scale - 1) < 1e-5
            dist = code_distance(got["codes"][b, i].numpy(), codes)
            assert dist.max() <= 1 and (dist > 0).mean() < 0.02, (b, i, dist.max())
            assert np.abs(got["rope"][b, i].double().numpy() - rope).max() <= \
                np.abs(rope).max() * 2 ** -7
            if not w.is_hca:
                icodes, iscale, _ = seqs[b].ikeys[i]
                assert abs(got["iscale"][b, i].item() / iscale - 1) < 1e-5
                assert code_distance(got["icodes"][b, i].numpy(), icodes).max() <= 1
    return cache


SMALL_CSA = G.Decode("small_csa_decode", 3, 0, 128, 32, 4, 8, 16, False, nh_i=4, c_i=64, k=12,
                     seed=101)
SMALL_HCA = G.Decode("small_hca_decode", 2, 0, 128, 32, 16, 8, 16, True, seed=102)


def test_decode_csa_small_crosses_emissions():
    _run_and_compare(SMALL_CSA, B=3, E=100, steps=9, seed=7)


def test_decode_csa_fewer_entries_than_k():
    _run_and_compare(SMALL_CSA, B=2, E=5, steps=6, seed=8)    # V <= k: every entry selected


def test_decode_hca_small_crosses_emission():
    _run_and_compare(SMALL_HCA, B=2, E=20, steps=18, seed=9)


def test_decode_csa_realistic_dims_two_chunks():
    w = G.Decode("csa_decode_dims", 2, 0, 512, 64, 4, 64, 128, False, nh_i=64, c_i=128, k=512,
                 seed=103)
    _run_and_compare(w, B=2, E=2500, steps=4, seed=10)


def test_decode_csa_128_index_heads():
    """128 indexer heads: the query operand fills N = 256 of the keys-on-M
    indexer form (64 heads use the heads-on-M form)."""
    w = G.Decode("csa_decode_h128", 3, 0, 512, 64, 4, 64, 128, False, nh_i=128, c_i=128, k=256,
                 seed=109)
    _run_and_compare(w, B=3, E=1300, steps=3, seed=16)


def test_decode_hca_realistic_dims_split_k():
    """64 heads x 512, FP8/bf16 cache, dense over ~300 entries: the tensor-core
    attention splits the entry set over several CTAs and a combine kernel."""
    w = G.Decode("hca_decode_dims", 2, 0, 512, 64, 128, 64, 128, True, seed=104)
    _run_and_compare(w, B=2, E=300, steps=2, seed=11)


def test_decode_csa_many_sequences_one_split():
    """Enough sequences that each gets a single attention CTA (no combine)."""
    w = G.Decode("csa_decode_many", 80, 0, 512, 64, 4, 64, 128, False, nh_i=64, c_i=128, k=64,
                 seed=105)
    _run_and_compare(w, B=80, E=40, steps=5, seed=12, check_seqs=[0, 37, 79])


def _csa_dims(name, seed, k=512):
    return G.Decode(name, 2, 0, 512, 64, 4, 64, 128, False, nh_i=64, c_i=128, k=k, seed=seed)


def test_decode_csa_topk_many_slices():
    """~36000 visible entries: the selection spreads each sequence over nine
    4096-score slices, the last of which resolves the threshold bin."""
    _run_and_compare(_csa_dims("csa_decode_cluster", 106), B=2, E=36000, steps=2, seed=13)


def test_decode_csa_all_scores_tied():
    """q_i = 0 makes every score 0: the selection is entries 0..k-1 (ties go to
    the smaller index): every score falls in the threshold bin, so the exact
    step ranks all 20000 of them, gathered from five slices."""
    def edit(inp):
        inp["q_i"].zero_()
    _run_and_compare(_csa_dims("csa_decode_ties", 107), B=2, E=20000, steps=2, seed=14, edit=edit,
                     sel_exact=True)


def test_decode_csa_topk_integer_scores_with_ties():
    """Scores in {0, 1, 2, 3}, computed exactly on both sides: one index-key dim
    holds the integer, one dim holds 448 (entry scale exactly 1), and one
    query head reads the integer dim with weight 1.  The k-th largest score
    sits inside a large tied group that spans several slices, so the
    selection is fixed by the smaller-index rule alone."""
    def edit(inp):
        B, E, ci = inp["cache_ikey"].shape
        gen = torch.Generator().manual_seed(15)
        ik = torch.zeros(B, E, ci)
        ik[:, :, 0] = torch.randint(0, 4, (B, E), generator=gen).float()
        ik[:, :, ci - 1] = 448.0
        inp["cache_ikey"].copy_(ik)
        inp["q_i"].zero_()
        inp["q_i"][:, :, 0, 0] = 1.0
        inp["w_i"].fill_(0.5)
        inp["w_i"][:, :, 0] = 1.0
    _run_and_compare(_csa_dims("csa_decode_int", 108), B=2, E=20000, steps=2, seed=15, edit=edit,
                     sel_exact=True)


def test_write_rows_fills_ring_and_state():
    w = SMALL_CSA
    B, E = 2, 10
    inp, cache, t0, first, tail, names = _setup(w, B, E, 1, seed=4)
    win = cache.region("window", torch.bfloat16, (B, w.window, w.c))
    st = cache.region("state", torch.bfloat16, (B, 2, 4, w.m, w.c))
    for u in range(t0 - w.window, t0):
        assert torch.equal(host(win)[:, u % w.window], inp["rows_kv_win"][:, u - first])
    for u in range(t0 - 2 * w.m, t0):
        par, row = (u // w.m) % 2, u % w.m
        for si, nm in enumerate(("ca", "cb", "za", "zb")):
            assert torch.equal(host(st)[:, par, si, row], inp["rows_" + nm][:, u - first])


def test_decode_index_scores_match_oracle_elementwise():
    """The decode indexer's scores themselves, element by element.  The GPU
    feeds the bf16 query to the FP8 tensor-core MMA as hi + lo E4M3 halves
    times a per-head power of two s_h >= max|q_h| / 448; that pair equals the
    bf16 value except for elements below 2^-2 s_h, whose error is at most
    2^-10 s_h.  So |I_gpu[s] - I[s]| <= sum_h w_h 2^-10 s_h sum_d |k_sd|, plus
    fp32 accumulation, bounded here by 2^-16 sum_h w_h sum_d |q_hd k_sd|."""
    w = _csa_dims("csa_decode_scores", 110)
    B, E = 2, 3000
    inp, cache, t0, first, tail, names = _setup(w, B, E, 1, seed=17)
    biases = {k: v.to(DEV) for k, v in _biases(inp, w).items()}
    rows = {nm: inp["rows_" + nm][:, tail].contiguous().to(DEV) for nm in names}
    pos = torch.full((B,), t0, dtype=torch.int64, device=DEV)
    scores = torch.full((B, cache.desc.capacity), float("nan"), dtype=torch.float32, device=DEV)
    cache.decode_step(pos, rows, biases, inp["sink"].to(DEV), w.scale, inp["q"][0].to(DEV),
                      inp["q_i"][0].to(DEV), inp["w_i"][0].to(DEV), scores_out=scores)
    csa.csa_check()
    got = host(scores).double().numpy()
    for b in range(B):
        seq = _oracle_sequence(w, inp, b, E, first, tail, names)
        seq.step(t0, {nm: inp["rows_" + nm][b, tail] for nm in names}, _biases(inp, w),
                 inp["q"][0, b], inp["q_i"][0, b], inp["w_i"][0, b], inp["sink"], w.scale, w.k)
        V = O.visible(t0, w.m)
        K = np.stack([O.dequantize_entry(*e) for e in seq.ikeys[:V]])
        q = O.f64(inp["q_i"][0, b])
        wt = O.f64(inp["w_i"][0, b])
        ref = O.index_scores_row(q, wt, K, V)
        s_h = 2.0 ** np.ceil(np.log2(np.abs(q).max(axis=1) / 448.0))
        kabs = np.abs(K).sum(axis=1)                                  # [V]
        bound = (wt * s_h).sum() * 2.0 ** -10 * kabs + \
            2.0 ** -16 * (np.abs(K) @ np.abs(q).T @ np.abs(wt))
        err = np.abs(got[b, :V] - ref)
        assert np.all(np.isfinite(got[b, :V]))
        assert np.all(err <= bound), (b, float(err.max()), float((err / bound).max()))
        assert np.isnan(got[b, V:]).all()             # nothing past the visible entries


# ----------------------------------------------------------- paged cache ---
# The classical cache in 128-token blocks behind a block table ([Analysis]
# "Inference KV Cache"): 32 CSA entries or 1 HCA entry per block (m = 4, 128).

def test_paged_decode_csa_realistic_dims():
    w = G.Decode("csa_decode_paged", 2, 0, 512, 64, 4, 64, 128, False, nh_i=64, c_i=128, k=512,
                 seed=111)
    _run_and_compare(w, B=2, E=2500, steps=4, seed=18, paged=True)


def test_paged_decode_csa_128_index_heads():
    w = G.Decode("csa_decode_paged_h128", 2, 0, 512, 64, 4, 64, 128, False, nh_i=128, c_i=128,
                 k=256, seed=112)
    _run_and_compare(w, B=2, E=1300, steps=3, seed=19, paged=True)


def test_paged_decode_hca_split_k():
    w = G.Decode("hca_decode_paged", 2, 0, 512, 64, 128, 64, 128, True, seed=113)
    _run_and_compare(w, B=2, E=300, steps=2, seed=20, paged=True)


def test_dsa_decode_is_csa_with_m1():
    """m = 1: every token is an entry and the indexer picks the top k among all
    of them (the fine-grained token selection of DSA), here in 128-entry
    blocks of the paged cache and in the contiguous cache."""
    w = G.Decode("dsa_decode", 2, 0, 512, 64, 1, 64, 128, False, nh_i=64, c_i=128, k=256,
                 seed=114)
    _run_and_compare(w, B=2, E=3000, steps=3, seed=21, paged=True)
    _run_and_compare(w, B=2, E=700, steps=2, seed=22)


def test_paged_decode_bit_identical_to_contiguous():
    """Same inputs through the contiguous and the paged cache: the same
    arithmetic on the same values, only the entry addresses differ."""
    w = G.Decode("csa_decode_pair", 3, 0, 512, 64, 4, 64, 128, False, nh_i=64, c_i=128, k=512,
                 seed=115)
    B, E, steps = 3, 2300, 5
    outs = []
    for paged in (False, True):
        inp, cache, t0, first, tail, names = _setup(w, B, E, steps, 23, paged=paged)
        biases = {k: v.to(DEV) for k, v in _biases(inp, w).items()}
        res = []
        for s_ in range(steps):
            rows = {nm: inp["rows_" + nm][:, tail + s_].contiguous().to(DEV) for nm in names}
            pos = torch.full((B,), t0 + s_, dtype=torch.int64, device=DEV)
            sel = torch.empty((B, w.k), dtype=torch.int32, device=DEV)
            o = cache.decode_step(pos, rows, biases, inp["sink"].to(DEV), w.scale,
                                  inp["q"][s_].to(DEV), inp["q_i"][s_].to(DEV),
                                  inp["w_i"][s_].to(DEV), sel_out=sel)
            res.append((host(o), host(sel)))
        csa.csa_check()
        outs.append(res)
    for (o1, s1), (o2, s2) in zip(*outs):
        assert torch.equal(s1, s2)
        assert torch.equal(o1, o2)


@pytest.mark.parametrize("is_hca", [False, True])
def test_decode_step_replays_in_a_cuda_graph(is_hca):
    """A decode step captured in a CUDA graph (the launches of every kernel of
    the step, with their programmatic dependencies) replays bit-identically
    to the same step launched directly; the step is idempotent at a fixed
    position, so the replay recomputes exactly what was computed."""
    w = G.Decode("graph_decode", 2, 0, 512, 64, 128 if is_hca else 4, 64, 128, is_hca, nh_i=64,
                 c_i=128, k=512, seed=117)
    B, E, steps = 2, 40 if is_hca else 2100, 1
    inp, cache, t0, first, tail, names = _setup(w, B, E, steps, 29)
    biases = {k: v.to(DEV) for k, v in _biases(inp, w).items()}
    rows = {nm: inp["rows_" + nm][:, tail].contiguous().to(DEV) for nm in names}
    pos = torch.full((B,), t0, dtype=torch.int64, device=DEV)
    sink, q = inp["sink"].to(DEV), inp["q"][0].to(DEV)
    qi = None if is_hca else inp["q_i"][0].to(DEV)
    wi = None if is_hca else inp["w_i"][0].to(DEV)
    out = torch.empty_like(q)

    def step():
        cache.decode_step(pos, rows, biases, sink, w.scale, q, qi, wi, out=out)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    eager = host(out)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    out.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    csa.csa_check()
    assert torch.equal(host(out), eager)
    del g
