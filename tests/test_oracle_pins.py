"""Pins of the fp64 oracle against facts fixed outside the oracle itself.

Each test checks the oracle against one of: a value the pages print (golden
fixtures under tests/golden, each citing its page), a closed form, an
invariant, a special case that reduces to a library routine (scipy / torch),
or brute force written independently on tiny inputs.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------- ledger ---

def test_ledger_golden():
    g = _golden("ledger.json")
    for case in g["cases"]:
        got = O.attention_ledger(*case["args"])
        for key, val in case["expect"].items():
            assert got[key] == val, (case, key, got[key])


def test_ledger_value_errors():
    g = _golden("ledger.json")
    for args in g["value_errors"]["args"]:
        with pytest.raises(ValueError):
            O.attention_ledger(*args)


def test_read_count_estimates():
    g = _golden("read_counts.json")
    t = g["history"] - 1
    assert O.reads_per_query(t, g["csa"]["m"], g["csa"]["k"], g["window"]) == g["csa"]["reads"]
    assert O.reads_per_query(t, g["hca"]["m"], None, g["window"]) == g["hca"]["reads"]


def test_completion_boundary_golden():
    g = _golden("completion_boundary.json")
    got = [O.visible(t, g["m"]) for t in g["positions"]]
    assert got == g["visible_entries"]
    # the stricter floor(t/m) reading differs exactly at t = m-1 (mod m)
    for t in range(64):
        diff = O.visible(t, 4) != O.visible(t, 4, strict=True)
        assert diff == (t % 4 == 3)


def test_read_counts_equal_entry_sets():
    """reads_per_query counts exactly the rows of the sets the oracle attends."""
    n, c, m, W, k = 40, 4, 4, 8, 3
    kv = rng.standard_normal((n // m, c))
    win = rng.standard_normal((n, c))
    idx = np.array([np.arange(k) for _ in range(n)])
    for t in range(n):
        Et = O.sparse_entry_set(kv, idx[t], win, t, m, W)
        assert Et.shape[0] == O.reads_per_query(t, m, k, W)
        Ed = O.dense_entry_set(kv, win, t, m, W)
        assert Ed.shape[0] == O.reads_per_query(t, m, None, W)


# ------------------------------------------------------------- compressor ---

def _csa_streams(n, c, m, seed=0):
    r = np.random.default_rng(seed)
    return [r.standard_normal((n, c)) for _ in range(4)] + \
        [0.1 * r.standard_normal((m, c)) for _ in range(2)]


def test_csa_weights_sum_to_one_and_first_entry_padding():
    n, c, m = 40, 6, 4
    Ca, Cb, Za, Zb, Ba, Bb = _csa_streams(n, c, m)
    Sa, Sb = O.csa_compress_weights(Za, Zb, Ba, Bb, m)
    tot = Sa.sum(axis=1) + Sb.sum(axis=1)
    assert np.abs(tot - 1).max() < 1e-12
    assert np.all(Sb[0] == 0.0)           # i = 0: previous block padded with -inf
    assert np.all(Sb[1:] > 0.0)


def test_csa_weights_match_library_softmax():
    n, c, m = 24, 5, 4
    _, _, Za, Zb, Ba, Bb = _csa_streams(n, c, m, seed=3)
    Sa, Sb = O.csa_compress_weights(Za, Zb, Ba, Bb, m)
    for i in range(1, n // m):
        for d in range(c):
            logits = np.concatenate([Za[m * i:m * i + m, d] + Ba[:, d],
                                     Zb[m * (i - 1):m * i, d] + Bb[:, d]])
            ref = scipy.special.softmax(logits)
            assert np.allclose(np.concatenate([Sa[i, :, d], Sb[i, :, d]]), ref,
                               rtol=1e-13, atol=1e-15)
    for d in range(c):   # first entry: softmax over the m own-block logits only
        ref = scipy.special.softmax(Za[:m, d] + Ba[:, d])
        assert np.allclose(Sa[0, :, d], ref, rtol=1e-13, atol=1e-15)


def test_csa_constant_logits_give_block_means():
    n, c, m = 32, 5, 4
    Ca, Cb, _, _, _, _ = _csa_streams(n, c, m, seed=5)
    Z = np.full((n, c), 0.7)
    B0 = np.zeros((m, c))
    out = O.csa_compress(Ca, Cb, Z, Z, B0, B0, m)
    assert np.allclose(out[0], Ca[:m].mean(axis=0), atol=1e-14)
    for i in range(1, n // m):
        ref = (Ca[m * i:m * i + m].sum(axis=0) + Cb[m * (i - 1):m * i].sum(axis=0)) / (2 * m)
        assert np.allclose(out[i], ref, atol=1e-14)


def test_csa_dominant_logit_copies_its_row():
    n, c, m = 32, 4, 4
    Ca, Cb, Za, Zb, Ba, Bb = _csa_streams(n, c, m, seed=7)
    Za2, Zb2 = Za.copy(), Zb.copy()
    Za2[4 * 3 + 2, 1] = 1e4          # entry 3, own block row 2, dim 1
    Zb2[4 * 4 + 1, 2] = 1e4          # entry 5 draws Cb row 4*4+1 in dim 2
    out = O.csa_compress(Ca, Cb, Za2, Zb2, Ba, Bb, m)
    assert out[3, 1] == pytest.approx(Ca[14, 1], abs=1e-12)
    assert out[5, 2] == pytest.approx(Cb[17, 2], abs=1e-12)


def test_csa_bias_only_weights():
    """Z = 0: every entry (i > 0) weights its 2m rows by softmax(B) per dim."""
    n, c, m = 16, 3, 4
    Ca, Cb, _, _, Ba, Bb = _csa_streams(n, c, m, seed=9)
    Z = np.zeros((n, c))
    out = O.csa_compress(Ca, Cb, Z, Z, Ba, Bb, m)
    w = scipy.special.softmax(np.concatenate([Ba, Bb], axis=0), axis=0)   # [2m, c]
    for i in range(1, n // m):
        ref = (w[:m] * Ca[m * i:m * i + m]).sum(0) + (w[m:] * Cb[m * (i - 1):m * i]).sum(0)
        assert np.allclose(out[i], ref, atol=1e-13)


def test_csa_dependency_structure():
    """Entry i reads Ca/Za block i and Cb/Zb block i-1, nothing else."""
    n, c, m = 36, 3, 4          # 9 entries, no partial tail
    base = _csa_streams(n + 3, c, m, seed=11)   # 3 trailing rows form a partial block
    ref = O.csa_compress(*base[:6], m)
    E = ref.shape[0]
    assert E == n // m
    for stream in range(4):
        for blk in range(E + 1):
            pert = [x.copy() for x in base]
            rows = slice(m * blk, min(m * blk + m, n + 3))
            pert[stream][rows] += 3.0
            out = O.csa_compress(*pert[:6], m)
            changed = {i for i in range(E) if not np.array_equal(out[i], ref[i])}
            if stream in (0, 2):      # Ca, Za: own block
                expect = {blk} if blk < E else set()
            else:                     # Cb, Zb: next entry
                expect = {blk + 1} if blk + 1 < E else set()
            assert changed == expect, (stream, blk, changed)


def test_hca_m1_is_identity_and_constant_logits_mean():
    n, c = 12, 5
    C = rng.standard_normal((n, c))
    Z = rng.standard_normal((n, c))
    assert np.allclose(O.hca_compress(C, Z, np.zeros((1, c)), 1), C, atol=1e-15)
    m = 4
    out = O.hca_compress(C, np.full((n, c), -2.0), np.zeros((m, c)), m)
    assert np.allclose(out, C.reshape(n // m, m, c).mean(axis=1), atol=1e-14)
    S = O.hca_compress_weights(Z, 0.1 * rng.standard_normal((m, c)), m)
    assert np.abs(S.sum(axis=1) - 1).max() < 1e-12


def test_hca_weights_match_library_softmax():
    n, c, m = 16, 3, 8
    Z = rng.standard_normal((n, c))
    B = 0.1 * rng.standard_normal((m, c))
    S = O.hca_compress_weights(Z, B, m)
    for i in range(n // m):
        for d in range(c):
            assert np.allclose(S[i, :, d], scipy.special.softmax(Z[m * i:m * i + m, d] + B[:, d]),
                               rtol=1e-13)


# ---------------------------------------------------------------- indexer ---

def test_index_scores_all_positive_dots_reduce_to_matvec():
    """When every q.k >= 0, ReLU is the identity and I = K (sum_h w_h q_h)."""
    H, ci, E = 5, 7, 11
    q = np.abs(rng.standard_normal((H, ci)))
    K = np.abs(rng.standard_normal((E, ci)))
    w = rng.uniform(0, 1, H)
    got = O.index_scores_row(q, w, K, E)
    ref = K @ (w @ q)
    assert np.allclose(got, ref, rtol=1e-13)


def test_index_scores_relu_and_head_weights():
    H, ci, E = 3, 4, 6
    K = rng.standard_normal((E, ci))
    q = rng.standard_normal((H, ci))
    # all-negative dots contribute nothing
    neg = O.index_scores_row(-np.abs(q), np.ones(H), np.abs(K), E)
    assert np.all(neg == 0.0)
    # one head, unit weight: max(0, q.k) against a direct numpy dot
    for h in range(H):
        w = np.zeros(H)
        w[h] = 1.0
        got = O.index_scores_row(q, w, K, E)
        assert np.allclose(got, np.maximum(0.0, np.dot(K, q[h])), rtol=1e-14)
    # linear in the head weights
    w1, w2 = rng.uniform(0, 1, H), rng.uniform(0, 1, H)
    s12 = O.index_scores_row(q, w1 + w2, K, E)
    assert np.allclose(s12, O.index_scores_row(q, w1, K, E) + O.index_scores_row(q, w2, K, E))
    # only the first V entries are scored
    assert O.index_scores_row(q, w1, K, 2).shape == (2,)


def test_topk_against_bruteforce_integer_scores():
    r = np.random.default_rng(5)
    for trial in range(200):
        V = int(r.integers(0, 40))
        k = int(r.integers(1, 12))
        scores = r.integers(-4, 5, size=V).astype(np.float64)   # many ties
        got = O.topk_row(scores, k)
        ranked = sorted(range(V), key=lambda s: (-scores[s], s))[:k]
        expect = sorted(ranked) + [-1] * (k - min(k, V))
        assert list(got) == expect


def test_index_topk_respects_visibility():
    n, H, ci, m, k = 30, 2, 4, 4, 3
    q = rng.standard_normal((n, H, ci))
    w = rng.uniform(0, 1, (n, H))
    K = rng.standard_normal((n // m, ci))
    idx = O.index_topk(q, w, K, m, k)
    for t in range(n):
        V = O.visible(t, m)
        sel = [s for s in idx[t] if s >= 0]
        assert len(sel) == min(k, V)
        assert all(s < V for s in sel)


# -------------------------------------------------------------- attention ---

def test_attend_without_sink_is_library_softmax():
    nh, c, N = 3, 5, 9
    q = rng.standard_normal((nh, c))
    E = rng.standard_normal((N, c))
    scale = 0.37
    got = O.attend(q, E, None, scale)
    P = scipy.special.softmax(scale * q @ E.T, axis=1)
    assert np.allclose(got, P @ E, rtol=1e-13, atol=1e-15)
    # a sink at -inf is the same
    assert np.allclose(O.attend(q, E, np.full(nh, -np.inf), scale), got, rtol=1e-14)


def test_attend_sink_limits_and_logistic():
    nh, c = 2, 4
    q = rng.standard_normal((nh, c))
    E = rng.standard_normal((6, c))
    assert np.abs(O.attend(q, E, np.full(nh, 800.0), 1.0)).max() < 1e-300
    one = rng.standard_normal((1, c))
    z = np.array([0.0, 1.3])
    got = O.attend(q, one, z, 0.5)
    logit = 0.5 * q @ one[0]
    wgt = scipy.special.expit(logit - z)     # e^l / (e^z + e^l)
    assert np.allclose(got, wgt[:, None] * one, rtol=1e-13)
    # the sink shares the denominator: weights sum to 1 - p_sink (< 1)
    s = O.attend(q, np.eye(c), np.zeros(nh), 1.0).sum(axis=1)
    ref = 1.0 - 1.0 / (1.0 + np.exp(q).sum(axis=1))
    assert np.allclose(s, ref, rtol=1e-13)


def test_attend_entry_order_invariant():
    nh, c, N = 4, 6, 10
    q = rng.standard_normal((nh, c))
    E = rng.standard_normal((N, c))
    z = rng.standard_normal(nh)
    perm = rng.permutation(N)
    assert np.allclose(O.attend(q, E, z, 0.3), O.attend(q, E[perm], z, 0.3), rtol=1e-13)


def _masked_dense_reference(q, kv_comp, kv_win, sel_sets, window, sink, scale):
    """Independent formulation: one masked row over [compressed ; raw] keys
    with an extra sink column, normalised by scipy's softmax."""
    n, nh, c = q.shape
    E = kv_comp.shape[0]
    keys = np.concatenate([kv_comp, kv_win], axis=0)        # [E + n, c]
    out = np.zeros((n, nh, c))
    for t in range(n):
        mask = np.zeros(E + n, dtype=bool)
        for s in sel_sets[t]:
            mask[s] = True
        for u in range(n):
            if t - window < u <= t:
                mask[E + u] = True
        logits = scale * q[t] @ keys.T                       # [nh, E + n]
        logits[:, ~mask] = -np.inf
        ext = np.concatenate([logits, np.asarray(sink).reshape(-1, 1) * np.ones((nh, 1))], axis=1)
        P = scipy.special.softmax(ext, axis=1)[:, :-1]
        out[t] = P @ keys
    return out


def test_sparse_and_dense_attention_match_masked_bruteforce():
    n, c, nh, m, W, k = 37, 6, 3, 4, 8, 3
    q = rng.standard_normal((n, nh, c))
    kv = rng.standard_normal((n // m, c))
    win = rng.standard_normal((n, c))
    z = rng.standard_normal(nh)
    scale = 1 / math.sqrt(c)
    # arbitrary valid selections: random subsets of the visible entries
    idx = np.full((n, k), -1)
    sets = []
    for t in range(n):
        V = (t + 1) // m
        chosen = sorted(rng.choice(V, size=min(k, V), replace=False)) if V else []
        idx[t, :len(chosen)] = chosen
        sets.append(chosen)
    got = O.sparse_attn(q, kv, idx, win, W, z, scale, m)
    assert np.allclose(got, _masked_dense_reference(q, kv, win, sets, W, z, scale),
                       rtol=1e-12, atol=1e-14)
    dense_sets = [list(range((t + 1) // m)) for t in range(n)]
    got = O.hca_attn(q, kv, win, W, z, scale, m)
    assert np.allclose(got, _masked_dense_reference(q, kv, win, dense_sets, W, z, scale),
                       rtol=1e-12, atol=1e-14)


def test_selection_with_k_at_least_visible_equals_dense():
    n, c, nh, m, W = 45, 5, 2, 4, 6
    q = rng.standard_normal((n, nh, c))
    kv = rng.standard_normal((n // m, c))
    win = rng.standard_normal((n, c))
    q_i = rng.standard_normal((n, 2, 3))
    w_i = rng.uniform(0, 1, (n, 2))
    K_i = rng.standard_normal((n // m, 3))
    k = n // m
    idx = O.index_topk(q_i, w_i, K_i, m, k)
    z = rng.standard_normal(nh)
    a = O.sparse_attn(q, kv, idx, win, W, z, 0.4, m)
    b = O.hca_attn(q, kv, win, W, z, 0.4, m)
    assert np.allclose(a, b, rtol=1e-13, atol=1e-15)


def test_future_perturbation_leaves_past_outputs_unchanged():
    """Full CSA pipeline (compress, index, top-k, attend) in the oracle."""
    n, c, nh, m, W, k, ci, H = 33, 4, 2, 4, 6, 2, 3, 2
    r = np.random.default_rng(21)
    base = dict(Ca=r.standard_normal((n, c)), Cb=r.standard_normal((n, c)),
                Za=r.standard_normal((n, c)), Zb=r.standard_normal((n, c)),
                iCa=r.standard_normal((n, ci)), iCb=r.standard_normal((n, ci)),
                iZa=r.standard_normal((n, ci)), iZb=r.standard_normal((n, ci)),
                win=r.standard_normal((n, c)), q=r.standard_normal((n, nh, c)),
                q_i=r.standard_normal((n, H, ci)), w_i=r.uniform(0, 1, (n, H)))
    Ba, Bb = 0.1 * r.standard_normal((m, c)), 0.1 * r.standard_normal((m, c))
    iBa, iBb = 0.1 * r.standard_normal((m, ci)), 0.1 * r.standard_normal((m, ci))
    z = r.standard_normal(nh)

    def run(d):
        kv = O.csa_compress(d["Ca"], d["Cb"], d["Za"], d["Zb"], Ba, Bb, m)
        K = O.csa_compress(d["iCa"], d["iCb"], d["iZa"], d["iZb"], iBa, iBb, m)
        idx = O.index_topk(d["q_i"], d["w_i"], K, m, k)
        return O.sparse_attn(d["q"], kv, idx, d["win"], W, z, 0.5, m)

    ref = run(base)
    for t in (3, 4, 7, 8, 20):
        pert = {key: v.copy() for key, v in base.items()}
        for v in pert.values():
            v[t + 1:] += 5.0
        out = run(pert)
        assert np.array_equal(out[:t + 1], ref[:t + 1]), t
        assert not np.array_equal(out[t + 1:], ref[t + 1:])


# ----------------------------------------------------------- fp8 / bf16 ---

def test_e4m3_codes_round_trip_and_table():
    # a few values fixed by the format: max 448, min normal 2^-6, min subnormal 2^-9
    assert O.e4m3_value(0x7E) == 448.0
    assert O.e4m3_value(0x08) == 2.0 ** -6
    assert O.e4m3_value(0x01) == 2.0 ** -9
    assert math.isnan(O.e4m3_value(0x7F))
    for code in range(256):
        if code in (0x7F, 0xFF, 0x80):
            continue
        assert O.e4m3_encode(O.e4m3_value(code)) == code
    # the table agrees with torch's float8_e4m3fn decoding
    raw = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    ours = O.e4m3_decode(np.arange(256))
    fin = ~np.isnan(ours)
    assert np.array_equal(raw.numpy()[fin], ours[fin])


def test_e4m3_rounding_matches_torch_cast_in_range():
    r = np.random.default_rng(8)
    vals = np.concatenate([
        r.uniform(-448, 448, 20000), r.standard_normal(20000) * 0.01,
        # exact midpoints between neighbouring codes (ties to even)
        (O.e4m3_decode(np.arange(0, 0x7E)) + O.e4m3_decode(np.arange(1, 0x7F))) / 2,
    ]).astype(np.float32)
    ours = O.e4m3_decode(O.e4m3_encode(vals))
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_saturates():
    assert O.e4m3_encode(1000.0) == 0x7E
    assert O.e4m3_encode(-1e30) == 0xFE


def test_bf16_round_matches_torch():
    r = np.random.default_rng(9)
    x = np.concatenate([r.standard_normal(50000).astype(np.float32),
                        # exact ties: low half 0x8000
                        (np.arange(1, 2000, dtype=np.uint32) << 16 | 0x8000).view(np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.bf16_round(x), ref)


def test_quantize_entry_properties():
    r = np.random.default_rng(10)
    x = r.standard_normal(64).astype(np.float32)
    codes, scale, rope = O.quantize_entry(x, 16)
    body = x[:48]
    j = int(np.argmax(np.abs(body)))
    assert abs(O.e4m3_value(codes[j])) == 448.0          # amax maps to the top code
    xhat = O.dequantize_entry(codes, scale, rope)
    # E4M3 keeps 3 fraction bits: relative error <= 2^-4 for normal codes
    big = np.abs(body) > 2.0 ** -6 * scale
    assert np.all(np.abs(xhat[:48] - body)[big] <= np.abs(body)[big] * 2.0 ** -4)
    assert np.array_equal(xhat[48:], O.bf16_round(x[48:]))
    zc, zs, _ = O.quantize_entry(np.zeros(8, dtype=np.float32), 0)
    assert zs == 1.0 and np.all(zc == 0)


def test_quantize_entries_equals_row_by_row():
    """The block form used at full workload sizes gives the per-entry results
    bit for bit (blocks smaller than the row count, a zero row, a huge value)."""
    r = np.random.default_rng(11)
    X = r.standard_normal((37, 40)).astype(np.float32)
    X[5] = 0.0
    X[9, 3] = 1e5
    codes, scales, rope = O.quantize_entries(X, 8, rows_per_pass=10)
    deq = O.dequantize_entries(codes, scales, rope)
    for e in range(X.shape[0]):
        c1, s1, r1 = O.quantize_entry(X[e], 8)
        assert np.array_equal(codes[e], c1) and scales[e] == s1 and np.array_equal(rope[e], r1)
        assert np.array_equal(deq[e], O.dequantize_entry(c1, s1, r1))


# ----------------------------------------------------------------- decode ---

def test_decode_sequence_matches_prefill_pipeline():
    """Incremental decode (emission from raw rows, FP8 cache) equals the
    prefill compressor and attention over the same dequantised entries."""
    m, c, rope, ci, nh, H, W, k = 4, 16, 4, 8, 2, 2, 6, 3
    T = 27
    r = np.random.default_rng(33)
    rows = {nm: r.standard_normal((T, c)) for nm in ("ca", "cb", "za", "zb", "kv_win")}
    rows.update({nm: r.standard_normal((T, ci)) for nm in ("ica", "icb", "iza", "izb")})
    bias = dict(ba=0.1 * r.standard_normal((m, c)), bb=0.1 * r.standard_normal((m, c)),
                iba=0.1 * r.standard_normal((m, ci)), ibb=0.1 * r.standard_normal((m, ci)))
    z = r.standard_normal(nh)
    seq = O.DecodeSequence(c, rope, m, W, False, ci)
    kv_all = O.csa_compress(rows["ca"], rows["cb"], rows["za"], rows["zb"],
                            bias["ba"], bias["bb"], m)
    ik_all = O.csa_compress(rows["ica"], rows["icb"], rows["iza"], rows["izb"],
                            bias["iba"], bias["ibb"], m)
    for t in range(T):
        q = r.standard_normal((nh, c))
        q_i = r.standard_normal((H, ci))
        w_i = r.uniform(0, 1, H)
        out, sel = seq.step(t, {nm: rows[nm][t] for nm in rows}, bias, q, q_i, w_i, z, 0.3, k)
        V = O.visible(t, m)
        assert len(seq.entries) == V
        X = np.stack([O.dequantize_entry(*e) for e in seq.entries]) if V else np.zeros((0, c))
        # emitted entries equal the quantised prefill compressor output
        for i in range(V):
            codes, scale, rp = O.quantize_entry(np.float32(kv_all[i]), rope)
            assert np.array_equal(seq.entries[i][0], codes) and seq.entries[i][1] == scale
        Kd = np.stack([O.dequantize_entry(*e) for e in seq.ikeys]) if V else np.zeros((0, ci))
        ref_sel = O.topk_row(O.index_scores_row(q_i, w_i, Kd, V), k)
        assert np.array_equal(sel, ref_sel)
        Et = O.sparse_entry_set(X, ref_sel, rows["kv_win"], t, m, W)
        assert np.allclose(out, O.attend(q, Et, z, 0.3), rtol=1e-13)
    for i, (codes, scale, _) in enumerate(seq.ikeys):
        ref_codes, ref_scale, _ = O.quantize_entry(np.float32(ik_all[i]), 0)
        assert np.array_equal(codes, ref_codes) and scale == ref_scale


# ------------------------------------------- RMSNorm and partial RoPE ---------
# Pins of the norm / rotation applied around core attention ([Walk-through]
# §4.5, §7.1, §7.4): closed forms of RMSNorm, the rotation written a second
# way (complex multiplication), group properties of the rotation, and the
# property the pages give as the reason for the output rotation: with the
# output turned back by -t, the layer depends on relative positions only.

def test_rms_norm_closed_forms():
    x = rng.standard_normal((5, 512)) * 3.0
    y = O.rms_norm(x, np.ones(512), eps=0.0)
    assert np.allclose((y * y).mean(axis=1), 1.0, atol=1e-12)      # unit RMS
    ms = (x * x).mean(axis=1)
    y = O.rms_norm(x, np.ones(512), eps=0.5)
    assert np.allclose((y * y).mean(axis=1), ms / (ms + 0.5), rtol=1e-12)
    g = rng.uniform(0.5, 2.0, 512)
    assert np.allclose(O.rms_norm(x, g, 0.0), O.rms_norm(x, np.ones(512), 0.0) * g)
    assert np.allclose(O.rms_norm(7.0 * x, g, 0.0), O.rms_norm(x, g, 0.0))  # scale-free
    assert np.all(O.rms_norm(np.zeros((2, 8)), np.ones(8)) == 0.0)


def test_rope_matches_complex_multiplication():
    c, R, base = 512, 64, 10000.0
    x = rng.standard_normal((3, c))
    pos = np.array([0, 7, 131071])
    got = O.rope_rotate(x, pos, R, base)
    assert np.array_equal(got[:, :c - R], x[:, :c - R])        # only the last 64 dims
    z = x[:, c - R::2] + 1j * x[:, c - R + 1::2]
    theta = np.array([base ** (-(2.0 * j) / R) for j in range(R // 2)])
    zr = z * np.exp(1j * pos[:, None] * theta[None, :])
    assert np.allclose(got[:, c - R::2], zr.real, atol=1e-12)
    assert np.allclose(got[:, c - R + 1::2], zr.imag, atol=1e-12)
    assert np.array_equal(O.rope_rotate(x, 0, R), x)              # angle 0: identity
    assert O.rope_theta(R)[0] == 1.0                                # the first pair: 1 rad / pos


def test_rope_group_properties():
    R = 64
    x = rng.standard_normal((4, 128))
    a, b = 1234, -987
    assert np.allclose(O.rope_rotate(O.rope_rotate(x, a, R), b, R), O.rope_rotate(x, a + b, R),
                       atol=1e-12)
    assert np.allclose(O.rope_rotate(O.rope_rotate(x, a, R), -a, R), x, atol=1e-12)
    pairs = lambda v: v[:, -R::2] ** 2 + v[:, -R + 1::2] ** 2        # noqa: E731
    assert np.allclose(pairs(O.rope_rotate(x, a, R)), pairs(x), atol=1e-12)
    # relative: <rot(q, a), rot(k, b)> = <rot(q, a - b), k>
    q, k = rng.standard_normal(128), rng.standard_normal(128)
    lhs = O.rope_rotate(q, a, R) @ O.rope_rotate(k, b, R)
    assert np.isclose(lhs, O.rope_rotate(q, a - b, R) @ k, atol=1e-10)


def test_norm_rope_attention_depends_on_relative_positions_only():
    nh, c, N, R = 4, 128, 9, 64
    q = rng.standard_normal((nh, c))
    ents = rng.standard_normal((N, c))
    pos = np.array([0, 4, 8, 20, 21, 22, 23, 24, 25])
    t = 25
    gq, gk = rng.uniform(0.5, 1.5, c), rng.uniform(0.5, 1.5, c)
    sink = rng.standard_normal(nh)
    o1 = O.attend_norm_rope(q, t, ents, pos, sink, c ** -0.5, gq, gk, R)
    o2 = O.attend_norm_rope(q, t + 100003, ents, pos + 100003, sink, c ** -0.5, gq, gk, R)
    assert np.allclose(o1, o2, atol=1e-10)
    # without the output rotation the result would move with the shift
    raw = lambda tt, pp: O.rope_rotate(                                # noqa: E731
        O.attend_norm_rope(q, tt, ents, pp, sink, c ** -0.5, gq, gk, R), tt, R)
    assert not np.allclose(raw(t, pos), raw(t + 100003, pos + 100003), atol=1e-3)


def test_norm_rope_attention_reduces_to_plain_attention():
    nh, c, N = 3, 64, 6
    q = rng.standard_normal((nh, c)) * 5
    ents = rng.standard_normal((N, c)) * 0.2
    pos = np.arange(N)
    ones = np.ones(c)
    # no rotation: plain attention of the normalised vectors, an explicit
    # softmax written out here
    got = O.attend_norm_rope(q, 5, ents, pos, None, 0.125, ones, ones, 0, eps=0.0)
    qn = q / np.sqrt((q * q).mean(axis=1, keepdims=True))
    en = ents / np.sqrt((ents * ents).mean(axis=1, keepdims=True))
    p = scipy.special.softmax(0.125 * qn @ en.T, axis=1)
    assert np.allclose(got, p @ en, atol=1e-12)
    # the norm bounds every logit: |l| <= scale * c * max|gq| * max|gk| (Cauchy-Schwarz)
    gq, gk = rng.uniform(0.5, 2.0, c), rng.uniform(0.5, 2.0, c)
    qq = O.rms_norm(q, gq)
    ee = O.rms_norm(ents, gk)
    assert np.abs(qq @ ee.T).max() <= c * gq.max() * gk.max()


def test_norm_rope_sparse_attn_entry_positions():
    # the per-row set and positions: entry s at m*s, window row u at u,
    # checked against attend_norm_rope on a set assembled by hand
    n, m, c, nh, W, R = 40, 4, 128, 2, 8, 64
    q = rng.standard_normal((n, nh, c))
    kv = rng.standard_normal((n // m, c))
    win = rng.standard_normal((n, c))
    g = np.ones(c)
    t = 37
    idx = np.full((n, 3), -1)
    idx[t] = [2, 8, 5]                  # V(37) = 9: entries 0..8 are visible
    got = O.sparse_attn_norm_rope(q, kv, idx, win, W, None, 0.1, m, g, g, R, rows=[t])[0]
    ents = np.concatenate([kv[[2, 8, 5]], win[t - W + 1:t + 1]])
    pos = np.concatenate([[8, 32, 20], np.arange(t - W + 1, t + 1)])
    assert np.allclose(got, O.attend_norm_rope(q[t], t, ents, pos, None, 0.1, g, g, R),
                       atol=1e-12)
    dense = O.hca_attn_norm_rope(q, kv, win, W, None, 0.1, m, g, g, R, rows=[t])[0]
    ents = np.concatenate([kv[:9], win[t - W + 1:t + 1]])
    pos = np.concatenate([4 * np.arange(9), np.arange(t - W + 1, t + 1)])
    assert np.allclose(dense, O.attend_norm_rope(q[t], t, ents, pos, None, 0.1, g, g, R),
                       atol=1e-12)


# --------------------------------------------- low-precision indexer ---------

def test_fp8_index_scores_exact_when_inputs_are_e4m3_values():
    # vectors whose largest magnitude is 448 get scale 1, and small integers
    # are E4M3 values: the FP8 form is then exact and equals the plain scores
    r = np.random.default_rng(7)
    H, ci, E = 4, 64, 50
    q = r.integers(-8, 9, (H, ci)).astype(np.float64)
    q[:, 0] = 448.0
    K = r.integers(-6, 7, (E, ci)).astype(np.float64)
    K[:, 1] = -448.0
    w = r.uniform(0, 1, H)
    assert np.array_equal(O.index_scores_row_fp8(q, w, K, 40), O.index_scores_row(q, w, K, 40))
    # the same from bf16 torch tensors (how the GPU tests call it)
    qt, Kt = torch.tensor(q, dtype=torch.bfloat16), torch.tensor(K, dtype=torch.bfloat16)
    assert np.array_equal(O.index_scores_row_fp8(qt, torch.tensor(w), Kt, 40),
                          O.index_scores_row(q, w, K, 40))


def test_fp8_index_scores_close_to_plain_on_random_inputs():
    # E4M3 keeps 3 mantissa bits: each product is off by at most ~2^-3 of its
    # size, so scores agree to a few percent and most of the top-k survives
    r = np.random.default_rng(8)
    H, ci, E, k = 8, 128, 2000, 64
    q, K, w = r.standard_normal((H, ci)), r.standard_normal((E, ci)), r.uniform(0, 1, H)
    a = O.index_scores_row(q, w, K, E)
    b = O.index_scores_row_fp8(q, w, K, E)
    assert np.abs(a - b).max() <= 0.1 * np.abs(a).max()
    assert O.selection_recall(O.topk_row(b, k), O.topk_row(a, k)) > 0.8


def test_bf16_score_selection_and_recall():
    # integer scores below 256 are bf16 values: the bf16 selection is exact
    r = np.random.default_rng(9)
    sc = r.integers(0, 256, 1000).astype(np.float64)
    assert np.array_equal(O.topk_row_bf16_scores(sc, 50), O.topk_row(sc, 50))
    # bf16 spacing is 2 in [256, 512): 257 rounds (to even) to 256 and ties
    # with it, and the tie goes to the smaller index
    sc = np.array([256.0, 257.0])
    assert list(O.topk_row_bf16_scores(sc, 1)) == [0]
    assert list(O.topk_row(sc, 1)) == [1]
    assert list(O.bf16_round(np.array([257.0, 259.0]))) == [256.0, 260.0]
    assert O.selection_recall([1, 2, 3, -1], [2, 3, 4, 5]) == 0.5
    assert O.selection_recall([-1], [-1]) == 1.0


# --------------------------------------------- grouped output projection ------

def test_grouped_projection_equals_block_diagonal_dense():
    # the grouped first stage is one dense product with a block-diagonal weight
    r = np.random.default_rng(11)
    n, nh, c, G, dg, d = 5, 8, 6, 4, 3, 7
    o = r.standard_normal((n, nh, c))
    W1 = r.standard_normal((G, dg, nh // G * c))
    W2 = r.standard_normal((d, G * dg))
    blk = np.zeros((G * dg, nh * c))
    for g in range(G):
        blk[g * dg:(g + 1) * dg, g * (nh // G) * c:(g + 1) * (nh // G) * c] = W1[g]
    ref = (o.reshape(n, nh * c) @ blk.T) @ W2.T
    assert np.allclose(O.grouped_output_projection(o, W1, W2), ref, atol=1e-12)


def test_grouped_projection_special_cases():
    r = np.random.default_rng(12)
    n, nh, c = 4, 4, 3
    o = r.standard_normal((n, nh, c))
    # one group with identity weights returns the flattened heads
    eye = np.eye(nh * c)[None]
    assert np.allclose(O.grouped_output_projection(o, eye, np.eye(nh * c)), o.reshape(n, -1))
    # a head outside group g never reaches z_g: zeroing group 1's heads leaves
    # only group 0 in y when W2 reads group 0 alone
    W1 = r.standard_normal((2, 5, 2 * c))
    W2 = np.concatenate([r.standard_normal((3, 5)), np.zeros((3, 5))], axis=1)
    o2 = o.copy()
    o2[:, 2:, :] = r.standard_normal((n, 2, c))
    assert np.allclose(O.grouped_output_projection(o, W1, W2),
                       O.grouped_output_projection(o2, W1, W2), atol=1e-12)
