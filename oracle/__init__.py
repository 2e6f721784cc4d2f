"""Plain, slow fp64 CPU oracle of the CSA / HCA attention layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path (the CUDA library
``libcsa.so`` and its Python binding) imports, calls or links this module.
Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline /
reference arm of ``bench.py`` may use it.  It shares no code with the CUDA
path; the only shared module is the seeded input generator ``csa_inputs``.

Every function below is written from the method's definition, in fp64, with
no blocking, fusion or reordering beyond what the definition states.  Sources
(web pages about DeepSeek-V4's hybrid attention), cited by title and section:

* [Formulas B9]  "Core formulas chapter" (polysight, 06-formulas), section
  B9 "CSA + HCA": the compressor, indexer and HCA equations.
* [Walk-through] "DeepSeek-V4: million-token context" (songhuiming.github.io),
  §4.1 overlapped compression, §4.2 lightning indexer, §4.3 shared-KV MQA,
  §4.5 sliding window and attention sink, §5.1 HCA compression.
* [Analysis]     "DeepSeek paper-feature analysis" (deepseek-paper-analysis.md),
  §7.1 CSA pseudo-code, §7.2 HCA, §7.3 KV mixed-precision storage,
  "Inference KV Cache" (state cache + classical cache).
* [Notes]        "DeepSeek-V4 reader's notes" (cooking-agi, deepseek-v4.html),
  §2 attention ledger, §3 completion rule and boundary tests.

Readings taken where the pages are silent or disagree (each is also listed
with its reason in the design notes of the repository):

* visibility: a query at 0-based position t reads the compressed entries
  s < floor((t+1)/m)  ([Notes] §3; [Formulas B9] prints s < floor(t/m),
  available here as ``strict=True``);
* window: rows u with max(0, t-W+1) <= u <= t (the current token included);
* sink: p_j = exp(l_j) / (exp(z_h) + sum_j exp(l_j)); the sink has no value;
* top-k ties: larger score first, then smaller index; the output lists the
  chosen indices in ascending order, padded with -1;
* index entries outside [0, V(t)) in a selection are ignored (padding);
* FP8 cache: E4M3 with round-to-nearest-even and saturation at +-448, one
  fp32 scale per entry, scale = amax/448 (1.0 when amax is 0), the code of x
  is E4M3(x / scale) with the division in fp32; the trailing ``rope_dims``
  dims are stored as bf16.
"""
from __future__ import annotations

from typing import Optional, Sequence

import numpy as np

NEG_INF = -np.inf


def f64(x) -> np.ndarray:
    """Host tensor / array -> float64 numpy array (exact widening)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", dtype=torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# Visibility ([Notes] §3 completion rule; [Formulas B9] causal constraint)
# ---------------------------------------------------------------------------

def visible(t: int, m: int, strict: bool = False) -> int:
    """Number of compressed entries the query at 0-based position t may read.

    An entry i covers tokens m*i .. m*i+m-1 and is complete once token
    m*i+m-1 has been seen, so after t+1 tokens floor((t+1)/m) entries are
    complete.  ``strict`` gives the variant floor(t/m) printed in B9.
    """
    return (t // m) if strict else ((t + 1) // m)


def window_rows(t: int, window: int) -> range:
    """Raw rows in the causal sliding window of the query at position t."""
    return range(max(0, t - window + 1), t + 1)


# ---------------------------------------------------------------------------
# Compressors ([Formulas B9] CSA / HCA equations; [Walk-through] §4.1, §5.1;
# [Analysis] §7.1, §7.2)
# ---------------------------------------------------------------------------

def csa_entry_weights(Za_cur, Zb_prev, Ba, Bb):
    """Per-dimension softmax weights of one CSA entry.

    The entry joins 2m logits per dimension d: Za_cur[j, d] + Ba[j, d] for the
    m rows of its own block and Zb_prev[j, d] + Bb[j, d] for the m rows of the
    previous block.  ``Zb_prev=None`` (the first entry) pads those logits with
    -inf, so they get weight 0.  Returns (Sa, Sb), each [m, c]; together they
    sum to 1 over the 2m terms of every dimension.
    """
    la = f64(Za_cur) + f64(Ba)                                # [m, c]
    if Zb_prev is None:
        lb = np.full(la.shape, NEG_INF)
    else:
        lb = f64(Zb_prev) + f64(Bb)                           # [m, c]
    logits = np.concatenate([la, lb], axis=0)                 # [2m, c]
    e = np.exp(logits - logits.max(axis=0))
    s = e / e.sum(axis=0)
    m = la.shape[0]
    return s[:m], s[m:]


def csa_entry(Ca_cur, Za_cur, Cb_prev, Zb_prev, Ba, Bb) -> np.ndarray:
    """One CSA entry: sum_j Sa_j * Ca_cur[j] + sum_j Sb_j * Cb_prev[j].

    The products are Hadamard (per dimension).  ``Cb_prev=None`` is the zero
    padding of the first entry.
    """
    Sa, Sb = csa_entry_weights(Za_cur, Zb_prev, Ba, Bb)
    out = (Sa * f64(Ca_cur)).sum(axis=0)
    if Cb_prev is not None:
        out = out + (Sb * f64(Cb_prev)).sum(axis=0)
    return out


def csa_compress_weights(Za, Zb, Ba, Bb, m: int):
    """Weights (Sa, Sb) [E, m, c] of all n//m entries of one sequence."""
    Za, Zb = f64(Za), f64(Zb)
    E = Za.shape[0] // m
    pairs = [csa_entry_weights(Za[m * i:m * i + m],
                               Zb[m * (i - 1):m * i] if i > 0 else None, Ba, Bb)
             for i in range(E)]
    c = Za.shape[1]
    Sa = np.stack([p[0] for p in pairs]) if E else np.zeros((0, m, c))
    Sb = np.stack([p[1] for p in pairs]) if E else np.zeros((0, m, c))
    return Sa, Sb


def csa_compress(Ca, Cb, Za, Zb, Ba, Bb, m: int) -> np.ndarray:
    """CSA overlapped compression of one sequence: [n, c] streams -> [n//m, c].

    Entry i draws on rows m*i .. m*i+m-1 of Ca/Za (its own block) and rows
    m*(i-1) .. m*i-1 of Cb/Zb (the previous block).  Trailing rows past the
    last full block are not compressed.
    """
    Ca, Cb, Za, Zb = f64(Ca), f64(Cb), f64(Za), f64(Zb)
    n, c = Ca.shape
    E = n // m
    out = np.zeros((E, c))
    for i in range(E):
        prev = slice(m * (i - 1), m * i)
        out[i] = csa_entry(Ca[m * i:m * i + m], Za[m * i:m * i + m],
                           Cb[prev] if i > 0 else None, Zb[prev] if i > 0 else None,
                           Ba, Bb)
    return out


def hca_compress_weights(Z, B, m: int) -> np.ndarray:
    """HCA weights [E, m, c]: per-dim softmax of Z[m*i+j] + B[j] over j."""
    Z, B = f64(Z), f64(B)
    n, c = Z.shape
    E = n // m
    S = np.zeros((E, m, c))
    for i in range(E):
        logits = Z[m * i:m * i + m] + B
        e = np.exp(logits - logits.max(axis=0))
        S[i] = e / e.sum(axis=0)
    return S


def hca_compress(C, Z, B, m: int) -> np.ndarray:
    """HCA compression (single stream, no overlap): [n, c] -> [n//m, c]."""
    C = f64(C)
    S = hca_compress_weights(Z, B, m)
    E = S.shape[0]
    return np.stack([(S[i] * C[m * i:m * i + m]).sum(axis=0) for i in range(E)]) \
        if E else np.zeros((0, C.shape[1]))


# ---------------------------------------------------------------------------
# Lightning indexer and top-k ([Formulas B9] I_{t,s}; [Walk-through] §4.2;
# [Analysis] §7.1 "Lightning Indexer")
# ---------------------------------------------------------------------------

def index_scores_row(q_i_t, w_i_t, K_i, V: int) -> np.ndarray:
    """I[t, s] = sum_h w[t,h] * ReLU(q_i[t,h] . K_i[s]) for s < V.

    q_i_t [H, c_i], w_i_t [H], K_i [E, c_i] -> [V].
    """
    q, w, K = f64(q_i_t), f64(w_i_t), f64(K_i)
    dots = K[:V] @ q.T                           # [V, H]
    return (np.maximum(dots, 0.0) * w[None, :]).sum(axis=1)


def topk_row(scores: np.ndarray, k: int) -> np.ndarray:
    """Top-k of one row: larger score first, ties to the smaller index.

    Returns the chosen indices sorted ascending, padded with -1 to length k.
    """
    scores = np.asarray(scores, dtype=np.float64)
    V = scores.shape[0]
    order = np.lexsort((np.arange(V), -scores))      # primary key: -score
    chosen = np.sort(order[:min(k, V)])
    out = np.full(k, -1, dtype=np.int64)
    out[:chosen.shape[0]] = chosen
    return out


def index_topk(q_i, w_i, K_i, m: int, k: int, rows: Optional[Sequence[int]] = None,
               strict: bool = False) -> np.ndarray:
    """Selected entries of one sequence: q_i [n,H,c_i], w_i [n,H], K_i [E,c_i].

    Returns [len(rows), k] int64 (rows default to all positions 0..n-1).
    """
    n = q_i.shape[0]
    rows = range(n) if rows is None else rows
    K = f64(K_i)
    res = []
    for t in rows:
        V = min(visible(t, m, strict), K.shape[0])
        res.append(topk_row(index_scores_row(q_i[t], w_i[t], K, V), k))
    return np.stack(res) if res else np.zeros((0, k), dtype=np.int64)


# ---------------------------------------------------------------------------
# Core attention with sink ([Walk-through] §4.3 shared-KV MQA, §4.5 sliding
# window + attention sink, one softmax; [Formulas B9]; [Notes] §1)
# ---------------------------------------------------------------------------

def attend(q_t, entries, sink, scale: float) -> np.ndarray:
    """Shared-KV MQA of one query over an explicit entry set, with a sink.

    q_t [nh, c], entries [N, c] (each entry is both key and value), sink [nh]
    logits z_h or None.  o_h = sum_j exp(l_hj) e_j / (exp(z_h) + sum_j exp(l_hj))
    with l_hj = scale * q_h . e_j.  Two passes: max, then normalised sums.
    """
    q, Ev = f64(q_t), f64(entries)
    nh = q.shape[0]
    logits = scale * (q @ Ev.T)                                  # [nh, N]
    z = np.full(nh, NEG_INF) if sink is None else f64(sink).reshape(-1) * np.ones(nh)
    mx = np.maximum(logits.max(axis=1) if Ev.shape[0] else np.full(nh, NEG_INF), z)
    num = np.exp(logits - mx[:, None])
    den = num.sum(axis=1) + np.exp(z - mx)
    return (num @ Ev) / den[:, None]


def sparse_entry_set(kv_comp, idx_row, kv_win, t: int, m: int, window: int,
                     strict: bool = False) -> np.ndarray:
    """E_t for CSA: the selected visible compressed entries plus the window."""
    kv_comp, kv_win = f64(kv_comp), f64(kv_win)
    V = min(visible(t, m, strict), kv_comp.shape[0])
    sel = [int(s) for s in idx_row if 0 <= int(s) < V]
    parts = [kv_comp[sel]] if sel else []
    parts.append(kv_win[list(window_rows(t, window))])
    return np.concatenate(parts, axis=0)


def dense_entry_set(kv_comp, kv_win, t: int, m: int, window: int,
                    strict: bool = False) -> np.ndarray:
    """E_t for HCA: every visible compressed entry plus the window."""
    kv_comp, kv_win = f64(kv_comp), f64(kv_win)
    V = min(visible(t, m, strict), kv_comp.shape[0])
    return np.concatenate([kv_comp[:V], kv_win[list(window_rows(t, window))]], axis=0)


def sparse_attn(q, kv_comp, idx, kv_win, window: int, sink, scale: float, m: int,
                rows: Optional[Sequence[int]] = None, strict: bool = False) -> np.ndarray:
    """CSA core attention of one sequence: q [n,nh,c], idx [n,k] -> [len(rows),nh,c]."""
    n = q.shape[0]
    rows = range(n) if rows is None else rows
    out = []
    for t in rows:
        Et = sparse_entry_set(kv_comp, np.asarray(idx[t]), kv_win, t, m, window, strict)
        out.append(attend(q[t], Et, sink, scale))
    return np.stack(out)


def hca_attn(q, kv_comp, kv_win, window: int, sink, scale: float, m: int,
             rows: Optional[Sequence[int]] = None, strict: bool = False) -> np.ndarray:
    """HCA core attention of one sequence (dense over visible entries)."""
    n = q.shape[0]
    rows = range(n) if rows is None else rows
    return np.stack([attend(q[t], dense_entry_set(kv_comp, kv_win, t, m, window, strict),
                            sink, scale) for t in rows])


def reads_per_query(t: int, m: int, k: Optional[int], window: int) -> int:
    """|E_t|: entries the main attention reads for the query at position t.

    k=None means dense (HCA).  This counts the very sets built above.
    """
    V = visible(t, m)
    sel = V if k is None else min(k, V)
    return sel + len(window_rows(t, window))


# ---------------------------------------------------------------------------
# Query / KV-entry RMSNorm and partial RoPE ([Walk-through] §4.5 "other
# details" and §7.1 Partial RoPE, §7.4 Query/KV Entry Normalization).
#
# The pages state: every query head and every KV entry is RMSNorm-ed before
# core attention; RoPE is applied to the last 64 dims of queries and KV
# entries; because each entry is both key and value, the attention output's
# last 64 dims are rotated by position -t so the output carries relative
# position only.  Readings where they are silent (listed in the design notes):
#   * RMSNorm(x) = x / sqrt(mean(x^2) + eps) * gamma over the head dim, one
#     learnable gamma for queries and one for KV entries, eps = 1e-6;
#   * the norm applies to every entry core attention reads (compressed and
#     window rows alike), before the rotation;
#   * RoPE pairs the trailing dims as (2j, 2j+1), j = 0 .. rope_dims/2 - 1,
#     and turns pair j by angle pos * base^(-2j/rope_dims), base = 10000;
#   * a window row sits at its token position u; a compressed entry s at the
#     position of its block's first token, m * s.
# ---------------------------------------------------------------------------

ROPE_BASE = 10000.0
NORM_EPS = 1e-6


def rms_norm(x, gamma, eps: float = NORM_EPS) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * gamma over the last axis (fp64)."""
    x = f64(x)
    ms = (x * x).mean(axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * f64(gamma)


def rope_theta(rope_dims: int, base: float = ROPE_BASE) -> np.ndarray:
    """Angle per unit position of each rotated pair: base^(-2j/rope_dims)."""
    j = np.arange(rope_dims // 2, dtype=np.float64)
    return base ** (-2.0 * j / rope_dims)


def rope_rotate(x, pos, rope_dims: int, base: float = ROPE_BASE) -> np.ndarray:
    """Rotates the last `rope_dims` dims of x in pairs (2j, 2j+1) by pos * theta_j.

    x [..., c]; pos a scalar or an array broadcast against x's leading axes.
    The leading c - rope_dims dims are returned unchanged.
    """
    x = f64(x).copy()
    if rope_dims == 0:
        return x
    c = x.shape[-1]
    ang = np.asarray(pos, dtype=np.float64)[..., None] * rope_theta(rope_dims, base)
    cs, sn = np.cos(ang), np.sin(ang)
    a = x[..., c - rope_dims::2].copy()
    b = x[..., c - rope_dims + 1::2].copy()
    x[..., c - rope_dims::2] = a * cs - b * sn
    x[..., c - rope_dims + 1::2] = a * sn + b * cs
    return x


def entry_position(s, m: int):
    """Position a compressed entry is rotated with: its block's first token."""
    return m * np.asarray(s)


def attend_norm_rope(q_t, t: int, entries, entry_pos, sink, scale: float, q_gamma, kv_gamma,
                     rope_dims: int, eps: float = NORM_EPS,
                     base: float = ROPE_BASE) -> np.ndarray:
    """Core attention of one query with the norm and partial RoPE around it.

    q_t [nh, c] raw query heads at position t; entries [N, c] raw entries at
    positions entry_pos [N].  q' = RoPE_t(RMSNorm(q)), e' = RoPE_p(RMSNorm(e)),
    o = attend(q', e', sink), returned as RoPE_{-t}(o).
    """
    q = rope_rotate(rms_norm(q_t, q_gamma, eps), t, rope_dims, base)
    E = rope_rotate(rms_norm(entries, kv_gamma, eps), np.asarray(entry_pos), rope_dims, base)
    return rope_rotate(attend(q, E, sink, scale), -t, rope_dims, base)


def sparse_attn_norm_rope(q, kv_comp, idx, kv_win, window: int, sink, scale: float, m: int,
                          q_gamma, kv_gamma, rope_dims: int, rows: Optional[Sequence[int]] = None,
                          eps: float = NORM_EPS) -> np.ndarray:
    """CSA core attention with the norm and RoPE, on raw (un-normed) entries
    kv_comp [E, c] and window rows kv_win [n, c]: [len(rows), nh, c]."""
    kv_comp, kv_win = f64(kv_comp), f64(kv_win)
    n = q.shape[0]
    rows = range(n) if rows is None else rows
    out = []
    for t in rows:
        V = min(visible(t, m), kv_comp.shape[0])
        sel = [int(s) for s in np.asarray(idx[t]) if 0 <= int(s) < V]
        win = list(window_rows(t, window))
        ents = np.concatenate([kv_comp[sel], kv_win[win]], axis=0)
        pos = np.concatenate([entry_position(np.asarray(sel, dtype=np.int64), m),
                              np.asarray(win, dtype=np.int64)])
        out.append(attend_norm_rope(q[t], t, ents, pos, sink, scale, q_gamma, kv_gamma,
                                    rope_dims, eps))
    return np.stack(out)


def hca_attn_norm_rope(q, kv_comp, kv_win, window: int, sink, scale: float, m: int, q_gamma,
                       kv_gamma, rope_dims: int, rows: Optional[Sequence[int]] = None,
                       eps: float = NORM_EPS) -> np.ndarray:
    """HCA core attention (every visible entry) with the norm and RoPE."""
    E = f64(kv_comp).shape[0]
    n = q.shape[0]
    idx = [np.arange(min(visible(t, m), E)) for t in range(n)]
    return sparse_attn_norm_rope(q, kv_comp, idx, kv_win, window, sink, scale, m, q_gamma,
                                 kv_gamma, rope_dims, rows, eps)


# ---------------------------------------------------------------------------
# FP8 E4M3 and bf16 storage ([Analysis] §7.3 "KV mixed-precision storage":
# RoPE dims in BF16, the other dims in FP8)
# ---------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3_value(code: int) -> float:
    """Value of an E4M3 byte: 1 sign, 4 exponent (bias 7), 3 mantissa bits.

    Exponent field 0 is subnormal (mantissa/8 * 2^-6); S.1111.111 is NaN;
    there is no infinity.
    """
    code = int(code) & 0xFF
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    f = code & 0x7
    if e == 0xF and f == 0x7:
        return float("nan")
    if e == 0:
        return sign * (f / 8.0) * 2.0 ** -6
    return sign * (1.0 + f / 8.0) * 2.0 ** (e - 7)


_E4M3_POS = np.array([e4m3_value(c) for c in range(0x7F)])  # codes 0x00..0x7E, ascending


def e4m3_encode(x) -> np.ndarray:
    """Round each value to E4M3, nearest with ties to the even code, saturating.

    Works on the exact value of x (float32 inputs widen exactly).  The
    candidates are the 127 finite non-negative codes, whose values increase
    with the code; a tie between two neighbours picks the even code (the one
    whose mantissa ends in 0).  NaN maps to 0x7F.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.searchsorted(_E4M3_POS, a, side="left")           # first code with value >= a
    hi = np.minimum(hi, len(_E4M3_POS) - 1)
    lo = np.maximum(hi - 1, 0)
    dlo = a - _E4M3_POS[lo]
    dhi = _E4M3_POS[hi] - a
    code = np.where(dlo < dhi, lo, hi)
    code = np.where(dlo == dhi, np.where(lo % 2 == 0, lo, hi), code)
    code = np.where(_E4M3_POS[hi] == a, hi, code)             # exact hit
    neg = (x < 0) | ((x == 0) & np.signbit(x))
    out = (code.astype(np.uint8) | np.where(neg, 0x80, 0).astype(np.uint8))
    out = np.where(np.isnan(x), np.uint8(0x7F), out).astype(np.uint8)
    return out


_E4M3_ALL = np.array([e4m3_value(c) for c in range(256)])  # value of every byte


def e4m3_decode(codes) -> np.ndarray:
    return _E4M3_ALL[np.asarray(codes, dtype=np.uint8)]


def bf16_round(x) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returns float64.

    bf16 keeps the top 16 bits of the float32 encoding; the dropped low half
    decides the rounding.
    """
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    low = u & 0xFFFF
    up = u >> 16
    inc = (low > 0x8000) | ((low == 0x8000) & ((up & 1) == 1))
    up = (up + inc.astype(np.uint64)) & 0xFFFF
    return (up.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def quantize_entry(x, rope_dims: int):
    """Cache form of one compressed entry (x taken at fp32).

    Returns (codes uint8 [c-rope], scale float32, rope float64 [rope] of bf16
    values).  scale = amax/448 in fp32 over the FP8 part (1.0 if amax == 0);
    code = E4M3(fp32(x / scale)).
    """
    x32 = np.asarray(x, dtype=np.float32)
    c = x32.shape[0]
    body = x32[:c - rope_dims]
    amax = np.float32(np.abs(body).max()) if body.size else np.float32(0)
    scale = np.float32(amax / np.float32(E4M3_MAX)) if amax > 0 else np.float32(1.0)
    codes = e4m3_encode((body / scale).astype(np.float32))
    rope = bf16_round(x32[c - rope_dims:])
    return codes, scale, rope


def dequantize_entry(codes, scale, rope) -> np.ndarray:
    """x_hat = code value * scale (fp64) followed by the bf16 rope dims."""
    return np.concatenate([e4m3_decode(codes) * float(scale), f64(rope)])


def quantize_entries(X, rope_dims: int, rows_per_pass: int = 4096):
    """quantize_entry of every row of X [E, c], the rows taken a block at a time.

    Returns (codes [E, c-rope] uint8, scales [E] float32, rope [E, rope] float64):
    the same fp32 arithmetic per row as quantize_entry.
    """
    x32 = np.asarray(X, dtype=np.float32)
    E, c = x32.shape
    codes = np.zeros((E, c - rope_dims), dtype=np.uint8)
    scales = np.ones(E, dtype=np.float32)
    for r0 in range(0, E, rows_per_pass):
        body = x32[r0:r0 + rows_per_pass, :c - rope_dims]
        amax = np.abs(body).max(axis=1) if body.shape[1] else np.zeros(body.shape[0], np.float32)
        sc = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
        scales[r0:r0 + rows_per_pass] = sc
        codes[r0:r0 + rows_per_pass] = e4m3_encode((body / sc[:, None]).astype(np.float32))
    return codes, scales, bf16_round(x32[:, c - rope_dims:])


def dequantize_entries(codes, scales, rope) -> np.ndarray:
    """dequantize_entry of every row: [E, c] fp64."""
    return np.concatenate([e4m3_decode(codes) * f64(scales)[:, None], f64(rope)], axis=1)


# ---------------------------------------------------------------------------
# Grouped output projection ([Walk-through] §4.4: the n_h heads are split
# into G groups; each group's concatenated outputs (n_h/G * c values) are
# projected to an intermediate dim d_G, and the G intermediate outputs,
# concatenated, are projected to the model dim d; [Formulas B9] gives
# V4-Flash n_h = 64, g = 8, d = 4096 and d_g = 1024).  Weights are stored
# [out, in]: W1 [G, d_G, (n_h/G) c], W2 [d, G d_G].
# ---------------------------------------------------------------------------

def grouped_output_projection(o, W1, W2) -> np.ndarray:
    """o [n, n_h, c] -> y [n, d]:  z_g = o_g W1[g]^T,  y = [z_1 .. z_G] W2^T."""
    o, W1, W2 = f64(o), f64(W1), f64(W2)
    n, nh, c = o.shape
    G = W1.shape[0]
    hpg = nh // G
    z = [o[:, g * hpg:(g + 1) * hpg, :].reshape(n, hpg * c) @ W1[g].T for g in range(G)]
    return np.concatenate(z, axis=1) @ W2.T


# ---------------------------------------------------------------------------
# Low-precision lightning indexer ([Analysis] "Lightning Indexer": small head
# count + FP8 keep the indexer cheap, the ReLU suits FP8; [Analysis] "FP4
# Quantization-Aware Training": index scores stored in BF16 instead of FP32,
# "2x speed-up, 99.7% recall").  FP8 form read here: each query head's
# vector and each index key is quantised to E4M3 with one fp32 scale
# (the same rule as the cache entries above); the score is the indexer
# formula on the dequantised vectors.  The BF16 form rounds each score to
# bf16 before the selection (ties then go to the smaller index).
# ---------------------------------------------------------------------------

def index_scores_row_fp8(q_i_t, w_i_t, K_i, V: int) -> np.ndarray:
    """index_scores_row with q_i_t [H, c_i] and K_i [E, c_i] first put through
    the FP8 E4M3 form (per-row scale amax/448): scores of the V visible keys."""
    qc, qs, _ = quantize_entries(f64(q_i_t).astype(np.float32), 0)
    kc, ks, _ = quantize_entries(f64(K_i)[:V].astype(np.float32), 0)
    q = e4m3_decode(qc) * qs.astype(np.float64)[:, None]
    K = e4m3_decode(kc) * ks.astype(np.float64)[:, None]
    return index_scores_row(q, w_i_t, K, V)


def topk_row_bf16_scores(scores: np.ndarray, k: int) -> np.ndarray:
    """topk_row on the scores rounded to bf16 (from their fp32 values)."""
    return topk_row(bf16_round(np.asarray(scores, dtype=np.float32)), k)


def selection_recall(sel, ref) -> float:
    """|sel & ref| / |ref| over the valid (>= 0) entries of two selections."""
    a = {int(s) for s in np.asarray(sel).ravel() if s >= 0}
    b = {int(s) for s in np.asarray(ref).ravel() if s >= 0}
    return 1.0 if not b else len(a & b) / len(b)


# ---------------------------------------------------------------------------
# Decode step over a persistent cache ([Analysis] "Inference KV Cache": state
# cache = SWA window + tail waiting for compression, classical cache = the
# compressed entries; [Notes] §2 tail + overlap state, §3 completion rule)
# ---------------------------------------------------------------------------

class DecodeSequence:
    """Decode-time state of one sequence for one layer, kept as plain history.

    ``rows`` maps a stream name to {position: raw row}; ``entries`` holds the
    cache entries as (codes, scale, rope) and ``ikeys`` the index keys as
    (codes, scale, empty).  The compressor of an entry is recomputed from raw
    rows with the prefill compressor above, so an incremental implementation
    must agree with a from-scratch one.
    """

    def __init__(self, c: int, rope_dims: int, m: int, window: int, is_hca: bool,
                 c_i: int = 0):
        self.c, self.rope_dims, self.m, self.window = c, rope_dims, m, window
        self.is_hca, self.c_i = is_hca, c_i
        self.rows = {}
        self.entries = []
        self.ikeys = []

    def store_entry(self, x, ikey=None):
        self.entries.append(quantize_entry(x, self.rope_dims))
        if not self.is_hca:
            self.ikeys.append(quantize_entry(ikey, 0))

    def put_row(self, name: str, pos: int, row):
        self.rows.setdefault(name, {})[pos] = f64(row)

    def _block(self, name: str, first: int, count: int, dim: int) -> np.ndarray:
        if first < 0:
            return np.zeros((count, dim))
        return np.stack([self.rows[name][p] for p in range(first, first + count)])

    def emit_value(self, i: int, biases: dict) -> tuple:
        """fp64 value of entry i (and its index key) from the raw rows."""
        m, c = self.m, self.c
        if self.is_hca:
            C = self._block("ca", m * i, m, c)
            Z = self._block("za", m * i, m, c)
            return hca_compress(C, Z, biases["ba"], m)[0], None

        def one(pre: str, dim: int, ba, bb):
            cur, prev = m * i, m * (i - 1)
            return csa_entry(self._block(pre + "ca", cur, m, dim),
                             self._block(pre + "za", cur, m, dim),
                             self._block(pre + "cb", prev, m, dim) if i > 0 else None,
                             self._block(pre + "zb", prev, m, dim) if i > 0 else None,
                             ba, bb)

        return one("", c, biases["ba"], biases["bb"]), \
            one("i", self.c_i, biases["iba"], biases["ibb"])

    def step(self, t: int, new_rows: dict, biases: dict, q, q_i, w_i, sink,
             scale: float, k: int = 0):
        """One decode token at position t; returns (out [nh, c], selected idx)."""
        for name, row in new_rows.items():
            self.put_row(name, t, row)
        m = self.m
        if (t + 1) % m == 0:
            i = t // m
            assert len(self.entries) == i, "cache must hold entries 0..i-1"
            kv, ik = self.emit_value(i, biases)
            self.store_entry(np.float32(kv), None if ik is None else np.float32(ik))
        V = min(visible(t, m), len(self.entries))
        X = np.stack([dequantize_entry(*e) for e in self.entries[:V]]) if V else \
            np.zeros((0, self.c))
        win = np.stack([self.rows["kv_win"][u] for u in window_rows(t, self.window)])
        if self.is_hca:
            sel = np.arange(V)
        else:
            K = np.stack([dequantize_entry(*e) for e in self.ikeys[:V]]) if V else \
                np.zeros((0, self.c_i))
            sel = topk_row(index_scores_row(q_i, w_i, K, V), k)
        chosen = [int(s) for s in sel if 0 <= s < V]
        Et = np.concatenate([X[chosen], win], axis=0)
        return attend(q, Et, sink, scale), sel


# ---------------------------------------------------------------------------
# Attention ledger ([Notes] §2): entry counts per query for a history length
# ---------------------------------------------------------------------------

def attention_ledger(history: int, light_ratio: int, heavy_ratio: int, selected: int,
                     window: int) -> dict:
    """Stored and read entry counts after ``history`` tokens (current included).

    Argument contract: positive integers, heavy_ratio > light_ratio, else
    ValueError.  Read counts come from the entry sets the oracle attends to at
    position t = history - 1.
    """
    vals = (history, light_ratio, heavy_ratio, selected, window)
    if any(type(v) is not int or v <= 0 for v in vals):
        raise ValueError("counts must be positive integers")
    if heavy_ratio <= light_ratio:
        raise ValueError("heavy ratio must exceed light ratio")
    t = history - 1
    return {
        "light_stored": visible(t, light_ratio),
        "heavy_stored": visible(t, heavy_ratio),
        "light_main_reads": reads_per_query(t, light_ratio, selected, window),
        "heavy_main_reads": reads_per_query(t, heavy_ratio, None, window),
        "light_tail": history - light_ratio * visible(t, light_ratio),
        "heavy_tail": history - heavy_ratio * visible(t, heavy_ratio),
    }
