"""GPU parity of the query / KV-entry RMSNorm and partial RoPE ("DeepSeek-V4:
million-token context" sections 4.5, 7.1, 7.4) against the fp64 oracle:
the row kernel, the compressor with the norm folded into its epilogue, and
core attention with the query norm in its prologue and the output rotation by
-t in its epilogue, end to end on both the tensor-core and CUDA-core paths."""
import numpy as np
import pytest
import torch

import compressed_sparse_attention_11_b200 as csa
import csa_inputs as G
import oracle as O
from _util import check_close, host

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _gamma(c, seed, tid):
    # positive weights around 1 (a learnable RMSNorm weight)
    return (1.0 + 0.25 * G.normal((c,), seed, tid, dtype=torch.float32)).contiguous()


@pytest.mark.parametrize("dt,heads,c,R,pos_mul", [
    (torch.float32, 3, 128, 64, 1),
    (torch.bfloat16, 4, 512, 64, 1),
    (torch.bfloat16, 1, 512, 64, 4),
    (torch.float32, 1, 256, 32, 32768),      # positions up to ~2M: angles reduced in fp64
    (torch.bfloat16, 2, 64, 0, 1),           # norm only
])
def test_norm_rope_rows(dt, heads, c, R, pos_mul):
    B, n = 2, 67
    x = G.normal((B, n, heads, c), 41, 1, dtype=dt) * 3.0
    x = x.to(dt)
    g = _gamma(c, 41, 2)
    out = host(csa.csa_norm_rope_rows(x.to(DEV), g.to(DEV), pos_mul=pos_mul, rope_dims=R))
    pos = (np.arange(n) * pos_mul)[None, :, None]
    ref = O.rope_rotate(O.rms_norm(O.f64(x), O.f64(g)), pos, R)
    check_close(out, ref, dt, f"rows {dt} c={c} R={R}")


def test_norm_rope_rows_in_place():
    x = G.normal((1, 40, 512), 42, 1, dtype=torch.bfloat16).to(DEV)
    g = _gamma(512, 42, 2).to(DEV)
    ref = host(csa.csa_norm_rope_rows(x, g))
    csa.csa_norm_rope_rows(x, g, out=x)
    assert torch.equal(host(x), ref)


@pytest.mark.parametrize("dt,n,c,m,overlap", [
    (torch.bfloat16, 1024, 512, 4, True),     # fused: an entry's 128 threads span four warps
    (torch.float32, 512, 128, 4, True),       # fused: 32 threads per entry, one warp
    (torch.bfloat16, 2048, 512, 128, False),  # HCA split kernel + in-place second pass
    (torch.float32, 96, 40, 4, True),         # 10 chunks per entry: second pass
])
def test_compress_norm_rope(dt, n, c, m, overlap):
    B, R = 2, 64 if c >= 64 else 8
    s = 43
    ca = G.normal((B, n, c), s, 1, dtype=dt)
    za = G.normal((B, n, c), s, 3, dtype=dt)
    ba = G.normal((m, c), s, 5, std=0.1, dtype=torch.float32)
    cb = G.normal((B, n, c), s, 2, dtype=dt) if overlap else None
    zb = G.normal((B, n, c), s, 4, dtype=dt) if overlap else None
    bb = G.normal((m, c), s, 6, std=0.1, dtype=torch.float32) if overlap else None
    g = _gamma(c, s, 7)
    d = lambda t: None if t is None else t.to(DEV)     # noqa: E731
    out = host(csa.csa_compress_norm_rope(d(ca), d(cb), d(za), d(zb), d(ba), d(bb), m, d(g),
                                          rope_dims=R))
    for b in range(B):
        if overlap:
            raw = O.csa_compress(ca[b], cb[b], za[b], zb[b], ba, bb, m)
        else:
            raw = O.hca_compress(ca[b], za[b], ba, m)
        ref = O.rope_rotate(O.rms_norm(raw, O.f64(g)), m * np.arange(raw.shape[0]), R)
        check_close(out[b], ref, dt, f"compress b={b}")


def _random_selection(n, m, k, seed):
    r = np.random.default_rng(seed)
    idx = np.full((1, n, k), -1, dtype=np.int32)
    for t in range(n):
        V = O.visible(t, m)
        if V:
            sel = np.sort(r.choice(V, min(k, V), replace=False))
            idx[0, t, :len(sel)] = sel
    return idx


@pytest.mark.parametrize("dt,n,nh,c,m,k,sparse", [
    (torch.bfloat16, 1536, 64, 512, 4, 160, True),    # tensor-core path
    (torch.bfloat16, 2048, 64, 512, 128, 0, False),   # tensor-core path, HCA
    (torch.float32, 600, 16, 128, 4, 32, True),       # CUDA-core path
    (torch.float32, 700, 8, 128, 16, 0, False),       # CUDA-core path, HCA
])
def test_attention_with_norm_rope_end_to_end(dt, n, nh, c, m, k, sparse):
    """Raw streams -> csa_compress_norm_rope, raw window rows ->
    csa_norm_rope_rows, then csa_sparse_attn_norm_rope / hca_attn_norm_rope,
    against the oracle's attention with the norm and rotation, computed from
    the raw (un-normed) compressed entries and window rows."""
    s, W, R = 44, 128, 64
    ca = G.normal((1, n, c), s, 1, dtype=dt)
    za = G.normal((1, n, c), s, 3, dtype=dt)
    ba = G.normal((m, c), s, 5, std=0.1, dtype=torch.float32)
    cb = G.normal((1, n, c), s, 2, dtype=dt) if sparse else None
    zb = G.normal((1, n, c), s, 4, dtype=dt) if sparse else None
    bb = G.normal((m, c), s, 6, std=0.1, dtype=torch.float32) if sparse else None
    win = G.normal((1, n, c), s, 13, dtype=dt)
    q = G.normal((1, n, nh, c), s, 14, dtype=dt) * 2.0
    q = q.to(dt)
    sink = G.normal((nh,), s, 17, dtype=torch.float32)
    gq, gk = _gamma(c, s, 30), _gamma(c, s, 31)
    scale = c ** -0.5
    d = lambda t: None if t is None else t.to(DEV)     # noqa: E731
    kv = csa.csa_compress_norm_rope(d(ca), d(cb), d(za), d(zb), d(ba), d(bb), m, d(gk),
                                    rope_dims=R)
    wn = csa.csa_norm_rope_rows(d(win), d(gk), rope_dims=R)
    if sparse:
        idx = _random_selection(n, m, k, seed=5)
        out = csa.csa_sparse_attn_norm_rope(d(q), kv, torch.tensor(idx).to(DEV), wn, W, d(sink),
                                            scale, m, d(gq), rope_dims=R)
    else:
        out = csa.hca_attn_norm_rope(d(q), kv, wn, W, d(sink), scale, m, d(gq), rope_dims=R)
    csa.csa_check()
    got = host(out)[0]
    rows = sorted(set([0, 1, m - 1, m, 127, 128, n // 2, n - 1] + list(range(3, n, 61))))
    if sparse:
        raw = O.csa_compress(ca[0], cb[0], za[0], zb[0], ba, bb, m)
        ref = O.sparse_attn_norm_rope(q[0], raw, idx[0], win[0], W, sink, scale, m, O.f64(gq),
                                      O.f64(gk), R, rows=rows)
    else:
        raw = O.hca_compress(ca[0], za[0], ba, m)
        ref = O.hca_attn_norm_rope(q[0], raw, win[0], W, sink, scale, m, O.f64(gq), O.f64(gk), R,
                                   rows=rows)
    check_close(got[rows], ref, dt, f"attention with norm/rope {dt} m={m}")


def test_norm_rope_rejects_bad_parameters():
    x = torch.zeros((1, 4, 64), dtype=torch.float32, device=DEV)
    g = torch.ones(64, dtype=torch.float32, device=DEV)
    for kw in (dict(rope_dims=12), dict(rope_dims=72), dict(rope_base=1.0), dict(eps=-1.0)):
        with pytest.raises(csa.CsaError) as e:
            csa.csa_norm_rope_rows(x, g, **kw)
        assert e.value.status == csa.CSA_ERR_INVALID_ARG
