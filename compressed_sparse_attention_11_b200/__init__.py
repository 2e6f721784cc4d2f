"""Python binding of libcsa.so, the CSA/HCA attention layer for one B200.

Argument marshalling only: every function here checks tensor shapes, dtypes
and devices, passes raw device pointers and the current CUDA stream to the C
ABI declared in ``include/csa.h`` and raises ``CsaError`` on a non-OK status.
All arithmetic runs in the library's CUDA kernels; there is no fallback.

The functions carry the C names: ``csa_compress``, ``csa_index_topk``,
``csa_sparse_attn``, ``hca_attn`` and the decode-cache calls
(``CsaCache`` wraps ``csa_cache_layout`` / ``csa_cache_store_entries`` /
``csa_cache_write_rows`` / ``csa_decode_step``).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa.so")

CSA_OK, CSA_ERR_INVALID_ARG, CSA_ERR_UNSUPPORTED, CSA_ERR_WORKSPACE, CSA_ERR_CUDA, \
    CSA_ERR_TIMEOUT = 0, -1, -2, -3, -4, -5
CSA_F32, CSA_BF16 = 0, 1

EXPORTED = (
    "csa_status_string", "csa_last_error", "csa_abi_version", "csa_check", "csa_selftest_wait",
    "csa_compress",
    "csa_index_topk_workspace", "csa_index_topk", "csa_index_topk_noalloc", "csa_sparse_attn",
    "hca_attn",
    "csa_cache_layout", "csa_cache_store_entries", "csa_cache_write_rows",
    "csa_decode_workspace", "csa_decode_step",
    "csa_norm_rope_rows", "csa_compress_norm_rope", "csa_sparse_attn_norm_rope",
    "hca_attn_norm_rope", "csa_index_topk_lowp_workspace", "csa_index_topk_lowp",
    "csa_grouped_out_proj_workspace", "csa_grouped_out_proj",
    "csa_paged_cache_layout", "csa_paged_cache_store_entries", "csa_paged_cache_write_rows",
    "csa_paged_decode_step",
)
CSA_INDEX_FP8_QK, CSA_INDEX_BF16_SCORES = 1, 2


class CsaError(RuntimeError):
    def __init__(self, status: int, detail: str):
        self.status = status
        super().__init__(f"{status_string(status)}: {detail}")


class CacheDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("capacity", ctypes.c_int64), ("c", ctypes.c_int32),
                ("rope_dims", ctypes.c_int32), ("c_i", ctypes.c_int32), ("m", ctypes.c_int32),
                ("window", ctypes.c_int32), ("nh", ctypes.c_int32), ("nh_i", ctypes.c_int32),
                ("k", ctypes.c_int32), ("is_hca", ctypes.c_int32)]


class CacheLayout(ctypes.Structure):
    _fields_ = [(nm, ctypes.c_size_t) for nm in (
        "entry_fp8", "entry_scale", "entry_rope", "ikey_fp8", "ikey_scale", "window", "state",
        "istate", "total_bytes")]


class Rows(ctypes.Structure):
    _fields_ = [(nm, ctypes.c_void_p) for nm in (
        "ca", "cb", "za", "zb", "ica", "icb", "iza", "izb", "kv_win")]


class DecodeParams(ctypes.Structure):
    _fields_ = [("ba", ctypes.c_void_p), ("bb", ctypes.c_void_p), ("iba", ctypes.c_void_p),
                ("ibb", ctypes.c_void_p), ("sink", ctypes.c_void_p), ("scale", ctypes.c_float),
                ("sel_out", ctypes.c_void_p), ("scores_out", ctypes.c_void_p)]


class Paging(ctypes.Structure):
    _fields_ = [("block_tokens", ctypes.c_int32), ("num_blocks", ctypes.c_int64),
                ("max_blocks", ctypes.c_int64), ("block_table", ctypes.c_void_p)]


class NormRope(ctypes.Structure):
    _fields_ = [("gamma", ctypes.c_void_p), ("eps", ctypes.c_float),
                ("rope_dims", ctypes.c_int32), ("rope_base", ctypes.c_float)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libcsa.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m compressed_sparse_attention_11_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, sz, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, \
        ctypes.c_float
    sig = {
        "csa_status_string": (ctypes.c_char_p, [i32]),
        "csa_last_error": (ctypes.c_char_p, []),
        "csa_abi_version": (i32, []),
        "csa_check": (i32, [vp]),
        "csa_selftest_wait": (i32, [ctypes.c_uint32, i32, vp]),
        "csa_compress": (i32, [vp, vp, vp, vp, vp, vp, i64, i64, i32, i32, i32, i32, vp, vp]),
        "csa_index_topk_workspace": (sz, [i64, i64, i32, i32, i32, i32]),
        "csa_index_topk": (i32, [vp, vp, vp, i64, i64, i32, i32, i32, i32, i32, vp, vp, sz, vp]),
        "csa_index_topk_noalloc": (i32, [vp, vp, vp, i64, i64, i32, i32, i32, i32, i32, vp, vp]),
        "csa_sparse_attn": (i32, [vp, vp, vp, i32, vp, i32, vp, f32, i64, i64, i32, i32, i32,
                                  i32, vp, vp]),
        "hca_attn": (i32, [vp, vp, vp, i32, vp, f32, i64, i64, i32, i32, i32, i32, vp, vp]),
        "csa_cache_layout": (i32, [ctypes.POINTER(CacheDesc), ctypes.POINTER(CacheLayout)]),
        "csa_cache_store_entries": (i32, [ctypes.POINTER(CacheDesc), vp, i64, i64, vp, vp, i32,
                                          vp]),
        "csa_cache_write_rows": (i32, [ctypes.POINTER(CacheDesc), vp, i64, i64,
                                       ctypes.POINTER(Rows), vp]),
        "csa_decode_workspace": (sz, [ctypes.POINTER(CacheDesc)]),
        "csa_decode_step": (i32, [ctypes.POINTER(CacheDesc), vp, vp, ctypes.POINTER(Rows),
                                  ctypes.POINTER(DecodeParams), vp, vp, vp, vp, vp, sz, vp]),
        "csa_norm_rope_rows": (i32, [vp, i64, i64, i32, i32, i64, ctypes.POINTER(NormRope), i32,
                                     vp, vp]),
        "csa_compress_norm_rope": (i32, [vp, vp, vp, vp, vp, vp, i64, i64, i32, i32, i32, i32,
                                         ctypes.POINTER(NormRope), vp, vp]),
        "csa_sparse_attn_norm_rope": (i32, [vp, vp, vp, i32, vp, i32, vp, f32, i64, i64, i32, i32,
                                            i32, i32, ctypes.POINTER(NormRope), vp, vp]),
        "hca_attn_norm_rope": (i32, [vp, vp, vp, i32, vp, f32, i64, i64, i32, i32, i32, i32,
                                     ctypes.POINTER(NormRope), vp, vp]),
        "csa_paged_cache_layout": (i32, [ctypes.POINTER(CacheDesc), ctypes.POINTER(Paging),
                                         ctypes.POINTER(CacheLayout)]),
        "csa_paged_cache_store_entries": (i32, [ctypes.POINTER(CacheDesc), ctypes.POINTER(Paging),
                                                vp, i64, i64, vp, vp, i32, vp]),
        "csa_paged_cache_write_rows": (i32, [ctypes.POINTER(CacheDesc), ctypes.POINTER(Paging), vp,
                                             i64, i64, ctypes.POINTER(Rows), vp]),
        "csa_paged_decode_step": (i32, [ctypes.POINTER(CacheDesc), ctypes.POINTER(Paging), vp, vp,
                                        ctypes.POINTER(Rows), ctypes.POINTER(DecodeParams), vp, vp,
                                        vp, vp, vp, sz, vp]),
        "csa_grouped_out_proj_workspace": (sz, [i64, i32, i32]),
        "csa_grouped_out_proj": (i32, [vp, i64, i32, i32, i32, i32, i32, vp, vp, vp, sz, vp, vp]),
        "csa_index_topk_lowp_workspace": (sz, [i64, i64, i32, i32, i32, i32, i32]),
        "csa_index_topk_lowp": (i32, [vp, vp, vp, i64, i64, i32, i32, i32, i32, i32, i32, vp, vp,
                                      sz, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def status_string(status: int) -> str:
    return lib().csa_status_string(int(status)).decode()


def _check(status: int):
    if status != CSA_OK:
        raise CsaError(status, lib().csa_last_error().decode())


def csa_check(device=None):
    """Synchronises the current stream and raises if a kernel gave up a bounded wait."""
    _check(lib().csa_check(torch.cuda.current_stream(device).cuda_stream))


def selftest_wait(limit_us: int, arrive: bool, device=None) -> int:
    """Runs the library's bounded-wait self-test on the current stream and
    returns the status csa_check reports afterwards (CSA_OK when the barrier
    was completed, CSA_ERR_TIMEOUT when the wait gave up)."""
    L = lib()
    stream = torch.cuda.current_stream(device).cuda_stream
    _check(L.csa_selftest_wait(int(limit_us), 1 if arrive else 0, stream))
    return int(L.csa_check(stream))


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return CSA_F32
    if t.dtype == torch.bfloat16:
        return CSA_BF16
    raise ValueError(f"unsupported dtype {t.dtype}; use float32 or bfloat16")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


# ------------------------------------------------------------------ prefill ---

def csa_compress(ca, cb, za, zb, ba, bb, m: int, out: Optional[torch.Tensor] = None):
    """Compress [B, n, c] streams into [B, n//m, c] entries.

    CSA (overlapped) when ``cb`` is given, HCA (single stream) when ``cb``,
    ``zb`` and ``bb`` are None.
    """
    overlap = 1 if cb is not None else 0
    B, n, c = ca.shape
    if out is None:
        out = torch.empty((B, n // m, c), dtype=ca.dtype, device=ca.device)
    _check(lib().csa_compress(_ptr(ca), _ptr(cb), _ptr(za), _ptr(zb), _ptr(ba), _ptr(bb), B, n,
                              c, m, overlap, _dt(ca), _ptr(out), _stream(ca)))
    return out


def csa_index_topk_workspace(batch: int, n: int, nh_i: int, c_i: int, m: int, k: int) -> int:
    return int(lib().csa_index_topk_workspace(batch, n, nh_i, c_i, m, k))


def csa_index_topk(q_i, w_i, k_i, m: int, k: int, ws: Optional[torch.Tensor] = None,
                   out: Optional[torch.Tensor] = None):
    """Top-k entry indices [B, n, k] int32 (ascending, -1 padded)."""
    B, n, H, ci = q_i.shape
    need = csa_index_topk_workspace(B, n, H, ci, m, k)
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=q_i.device)
    if out is None:
        out = torch.empty((B, n, k), dtype=torch.int32, device=q_i.device)
    _check(lib().csa_index_topk(_ptr(q_i), _ptr(w_i), _ptr(k_i), B, n, H, ci, m, k, _dt(q_i),
                                _ptr(out), _ptr(ws), ws.numel() * ws.element_size(),
                                _stream(q_i)))
    return out


def csa_index_topk_noalloc(q_i, w_i, k_i, m: int, k: int, out: Optional[torch.Tensor] = None):
    """csa_index_topk using the library's built-in score scratch (no workspace).

    For callers that cannot allocate device memory; limited to
    batch * n * (n // m) <= 2**21 scores, and concurrent calls race."""
    B, n, H, ci = q_i.shape
    if out is None:
        out = torch.empty((B, n, k), dtype=torch.int32, device=q_i.device)
    _check(lib().csa_index_topk_noalloc(_ptr(q_i), _ptr(w_i), _ptr(k_i), B, n, H, ci, m, k,
                                        _dt(q_i), _ptr(out), _stream(q_i)))
    return out


def csa_index_topk_lowp(q_i, w_i, k_i, m: int, k: int, fp8_qk: bool = True,
                        bf16_scores: bool = True, ws: Optional[torch.Tensor] = None,
                        out: Optional[torch.Tensor] = None):
    """The indexer + top-k with FP8 query/key scoring and / or bf16-stored
    scores: indices [B, n, k] int32 (ascending, -1 padded)."""
    B, n, H, ci = q_i.shape
    flags = (CSA_INDEX_FP8_QK if fp8_qk else 0) | (CSA_INDEX_BF16_SCORES if bf16_scores else 0)
    need = int(lib().csa_index_topk_lowp_workspace(B, n, H, ci, m, k, flags))
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=q_i.device)
    if out is None:
        out = torch.empty((B, n, k), dtype=torch.int32, device=q_i.device)
    _check(lib().csa_index_topk_lowp(_ptr(q_i), _ptr(w_i), _ptr(k_i), B, n, H, ci, m, k, _dt(q_i),
                                     flags, _ptr(out), _ptr(ws), ws.numel() * ws.element_size(),
                                     _stream(q_i)))
    return out


def csa_sparse_attn(q, kv_comp, idx, kv_win, window: int, sink, scale: float, m: int,
                    out: Optional[torch.Tensor] = None):
    B, n, nh, c = q.shape
    if out is None:
        out = torch.empty_like(q)
    _check(lib().csa_sparse_attn(_ptr(q), _ptr(kv_comp), _ptr(idx), idx.shape[-1], _ptr(kv_win),
                                 window, _ptr(sink), float(scale), B, n, nh, c, m, _dt(q),
                                 _ptr(out), _stream(q)))
    return out


def hca_attn(q, kv_comp, kv_win, window: int, sink, scale: float, m_heavy: int,
             out: Optional[torch.Tensor] = None):
    B, n, nh, c = q.shape
    if out is None:
        out = torch.empty_like(q)
    _check(lib().hca_attn(_ptr(q), _ptr(kv_comp), _ptr(kv_win), window, _ptr(sink), float(scale),
                          B, n, nh, c, m_heavy, _dt(q), _ptr(out), _stream(q)))
    return out


# ------------------------------------------------- RMSNorm and partial RoPE ---

ROPE_BASE = 10000.0
NORM_EPS = 1e-6


def _norm_rope(gamma, eps: float, rope_dims: int, rope_base: float) -> NormRope:
    if gamma is None or gamma.dtype != torch.float32:
        raise ValueError("gamma must be a float32 tensor")
    return NormRope(_ptr(gamma), float(eps), int(rope_dims), float(rope_base))


def csa_norm_rope_rows(x, gamma, pos_mul: int = 1, eps: float = NORM_EPS, rope_dims: int = 64,
                       rope_base: float = ROPE_BASE, out: Optional[torch.Tensor] = None):
    """RMSNorm + rotation of the trailing dims of every row of x [B, n, c] or
    [B, n, heads, c]; row t turns for position t * pos_mul (out may be x)."""
    B, n = x.shape[0], x.shape[1]
    heads = x.shape[2] if x.dim() == 4 else 1
    c = x.shape[-1]
    if out is None:
        out = torch.empty_like(x)
    nr = _norm_rope(gamma, eps, rope_dims, rope_base)
    _check(lib().csa_norm_rope_rows(_ptr(x), B, n, heads, c, int(pos_mul), ctypes.byref(nr),
                                    _dt(x), _ptr(out), _stream(x)))
    return out


def csa_compress_norm_rope(ca, cb, za, zb, ba, bb, m: int, gamma, eps: float = NORM_EPS,
                           rope_dims: int = 64, rope_base: float = ROPE_BASE,
                           out: Optional[torch.Tensor] = None):
    """csa_compress with each entry i RMSNorm-ed and rotated for position m * i."""
    overlap = 1 if cb is not None else 0
    B, n, c = ca.shape
    if out is None:
        out = torch.empty((B, n // m, c), dtype=ca.dtype, device=ca.device)
    nr = _norm_rope(gamma, eps, rope_dims, rope_base)
    _check(lib().csa_compress_norm_rope(_ptr(ca), _ptr(cb), _ptr(za), _ptr(zb), _ptr(ba),
                                        _ptr(bb), B, n, c, m, overlap, _dt(ca), ctypes.byref(nr),
                                        _ptr(out), _stream(ca)))
    return out


def csa_sparse_attn_norm_rope(q, kv_comp, idx, kv_win, window: int, sink, scale: float, m: int,
                              q_gamma, eps: float = NORM_EPS, rope_dims: int = 64,
                              rope_base: float = ROPE_BASE, out: Optional[torch.Tensor] = None):
    """csa_sparse_attn with the query norm + rotation and the output rotation
    by -t; kv_comp and kv_win must already be normed and rotated."""
    B, n, nh, c = q.shape
    if out is None:
        out = torch.empty_like(q)
    nr = _norm_rope(q_gamma, eps, rope_dims, rope_base)
    _check(lib().csa_sparse_attn_norm_rope(_ptr(q), _ptr(kv_comp), _ptr(idx), idx.shape[-1],
                                           _ptr(kv_win), window, _ptr(sink), float(scale), B, n,
                                           nh, c, m, _dt(q), ctypes.byref(nr), _ptr(out),
                                           _stream(q)))
    return out


def hca_attn_norm_rope(q, kv_comp, kv_win, window: int, sink, scale: float, m_heavy: int,
                       q_gamma, eps: float = NORM_EPS, rope_dims: int = 64,
                       rope_base: float = ROPE_BASE, out: Optional[torch.Tensor] = None):
    """hca_attn with the query norm + rotation and the output rotation by -t."""
    B, n, nh, c = q.shape
    if out is None:
        out = torch.empty_like(q)
    nr = _norm_rope(q_gamma, eps, rope_dims, rope_base)
    _check(lib().hca_attn_norm_rope(_ptr(q), _ptr(kv_comp), _ptr(kv_win), window, _ptr(sink),
                                    float(scale), B, n, nh, c, m_heavy, _dt(q), ctypes.byref(nr),
                                    _ptr(out), _stream(q)))
    return out


# ------------------------------------------------------ output projection ---

def csa_grouped_out_proj(o, w1, w2, ws: Optional[torch.Tensor] = None,
                         out: Optional[torch.Tensor] = None):
    """Grouped output projection: o [rows, nh, c] (or [B, n, nh, c]) with
    w1 [G, d_g, nh/G * c] and w2 [d, G * d_g] -> y [rows, d] (bf16)."""
    nh, c = o.shape[-2], o.shape[-1]
    rows = o.numel() // (nh * c)
    G, dg = w1.shape[0], w1.shape[1]
    d = w2.shape[0]
    need = int(lib().csa_grouped_out_proj_workspace(rows, G, dg))
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=o.device)
    if out is None:
        out = torch.empty(o.shape[:-2] + (d,), dtype=o.dtype, device=o.device)
    if o.dtype != torch.bfloat16 or w1.dtype != torch.bfloat16 or w2.dtype != torch.bfloat16:
        raise ValueError("the grouped output projection takes bfloat16 tensors")
    _check(lib().csa_grouped_out_proj(_ptr(o), rows, nh, c, G, dg, d, _ptr(w1), _ptr(w2),
                                      _ptr(ws), ws.numel() * ws.element_size(), _ptr(out),
                                      _stream(o)))
    return out


# ------------------------------------------------------------------- decode ---

class CsaCache:
    """A caller-owned decode cache (one layer, ``batch`` sequences).

    With ``block_table`` (int32 [batch, max_blocks] on the device) the
    compressed entries live in a paged pool of ``num_blocks`` blocks of
    ``block_tokens`` raw tokens each (the classical cache; capacity becomes
    max_blocks * block_tokens // m); the window ring and the compressor tail
    stay per sequence."""

    def __init__(self, batch: int, capacity: int, c: int, rope_dims: int, m: int, window: int,
                 nh: int, is_hca: bool, c_i: int = 0, nh_i: int = 0, k: int = 0,
                 device="cuda", block_table: Optional[torch.Tensor] = None,
                 block_tokens: int = 128, num_blocks: int = 0):
        self.paging = None
        if block_table is not None:
            if block_table.dtype != torch.int32 or block_table.dim() != 2:
                raise ValueError("block_table must be an int32 [batch, max_blocks] tensor")
            self.block_table = block_table
            capacity = block_table.shape[1] * (block_tokens // m)
            self.paging = Paging(int(block_tokens), int(num_blocks), int(block_table.shape[1]),
                                 _ptr(block_table))
        self.desc = CacheDesc(batch, capacity, c, rope_dims, c_i, m, window, nh, nh_i, k,
                              1 if is_hca else 0)
        self.layout = CacheLayout()
        if self.paging is not None:
            _check(lib().csa_paged_cache_layout(ctypes.byref(self.desc), ctypes.byref(self.paging),
                                                ctypes.byref(self.layout)))
        else:
            _check(lib().csa_cache_layout(ctypes.byref(self.desc), ctypes.byref(self.layout)))
        self.buffer = torch.zeros(self.layout.total_bytes, dtype=torch.uint8, device=device)
        ws = int(lib().csa_decode_workspace(ctypes.byref(self.desc)))
        self.workspace = torch.empty(max(ws, 16), dtype=torch.uint8, device=device)

    # views of the regions (for tests and inspection)
    def region(self, name: str, dtype, shape):
        off = getattr(self.layout, name)
        nbytes = int(torch.tensor(shape).prod().item()) * torch.empty((), dtype=dtype).element_size()
        return self.buffer[off:off + nbytes].view(dtype).view(*shape)

    def entries(self):
        """The entry regions as [batch, capacity, ...] (gathered through the
        block table when paged; absent blocks read as zeros)."""
        d = self.desc
        B, cap = d.batch, d.capacity
        rows = B * cap
        if self.paging is not None:
            epb = self.paging.block_tokens // d.m
            rows = self.paging.num_blocks * epb
        out = dict(codes=self.region("entry_fp8", torch.uint8, (rows, d.c - d.rope_dims)),
                   scale=self.region("entry_scale", torch.float32, (rows,)),
                   rope=self.region("entry_rope", torch.bfloat16, (rows, d.rope_dims)))
        if not d.is_hca:
            out["icodes"] = self.region("ikey_fp8", torch.uint8, (rows, d.c_i))
            out["iscale"] = self.region("ikey_scale", torch.float32, (rows,))
        if self.paging is None:
            return {k: v.view(B, cap, *v.shape[1:]) for k, v in out.items()}
        bt = self.block_table.long()
        s = torch.arange(cap, device=bt.device)
        blk = bt[:, s // epb]                                       # [B, cap]
        ok = (blk >= 0) & (blk < self.paging.num_blocks)
        row = torch.where(ok, blk * epb + (s % epb)[None, :], torch.zeros_like(blk))
        res = {}
        for k, v in out.items():
            g = v[row.reshape(-1)].reshape(B, cap, *v.shape[1:]).clone()
            g[~ok] = 0
            res[k] = g
        return res

    def store_entries(self, first: int, kv, ikey=None):
        count = kv.shape[1]
        if self.paging is not None:
            _check(lib().csa_paged_cache_store_entries(
                ctypes.byref(self.desc), ctypes.byref(self.paging), _ptr(self.buffer), first,
                count, _ptr(kv), _ptr(ikey), _dt(kv), _stream(self.buffer)))
            return
        _check(lib().csa_cache_store_entries(ctypes.byref(self.desc), _ptr(self.buffer), first,
                                             count, _ptr(kv), _ptr(ikey), _dt(kv),
                                             _stream(self.buffer)))

    @staticmethod
    def _rows(rows: dict) -> Rows:
        r = Rows()
        for nm in ("ca", "cb", "za", "zb", "ica", "icb", "iza", "izb", "kv_win"):
            t = rows.get(nm)
            if t is not None and t.dtype != torch.bfloat16:
                raise ValueError(f"row stream {nm} must be bfloat16")
            setattr(r, nm, _ptr(t))
        return r

    def write_rows(self, first_pos: int, rows: dict):
        count = rows["kv_win"].shape[1]
        r = self._rows(rows)
        if self.paging is not None:
            _check(lib().csa_paged_cache_write_rows(
                ctypes.byref(self.desc), ctypes.byref(self.paging), _ptr(self.buffer), first_pos,
                count, ctypes.byref(r), _stream(self.buffer)))
            return
        _check(lib().csa_cache_write_rows(ctypes.byref(self.desc), _ptr(self.buffer), first_pos,
                                          count, ctypes.byref(r), _stream(self.buffer)))

    def decode_step(self, pos, rows: dict, biases: dict, sink, scale: float, q, q_i=None,
                    w_i=None, out: Optional[torch.Tensor] = None,
                    sel_out: Optional[torch.Tensor] = None,
                    scores_out: Optional[torch.Tensor] = None):
        """One token per sequence at positions ``pos`` (int64 [B] on device).

        ``rows``: per-stream [B, dim] bf16 tensors; ``biases``: ba, bb, iba, ibb
        fp32; returns out [B, nh, c] bf16.  ``sel_out`` (CSA, optional, int32
        [B, k] on device) receives the selected entry indices; ``scores_out``
        (CSA, optional, fp32 [B, capacity] on device) the indexer scores."""
        if out is None:
            out = torch.empty_like(q)
        r = self._rows({k: v for k, v in rows.items()})
        if sel_out is not None and (sel_out.dtype != torch.int32 or not sel_out.is_contiguous()
                                    or sel_out.numel() != self.desc.batch * self.desc.k):
            raise ValueError("sel_out must be a contiguous int32 [batch, k] tensor")
        if scores_out is not None and (
                scores_out.dtype != torch.float32 or not scores_out.is_contiguous()
                or scores_out.numel() != self.desc.batch * self.desc.capacity):
            raise ValueError("scores_out must be a contiguous float32 [batch, capacity] tensor")
        p = DecodeParams(_ptr(biases.get("ba")), _ptr(biases.get("bb")), _ptr(biases.get("iba")),
                         _ptr(biases.get("ibb")), _ptr(sink), float(scale), _ptr(sel_out),
                         _ptr(scores_out))
        if pos.dtype != torch.int64:
            raise ValueError("pos must be int64")
        if self.paging is not None:
            _check(lib().csa_paged_decode_step(
                ctypes.byref(self.desc), ctypes.byref(self.paging), _ptr(self.buffer), _ptr(pos),
                ctypes.byref(r), ctypes.byref(p), _ptr(q), _ptr(q_i), _ptr(w_i), _ptr(out),
                _ptr(self.workspace), self.workspace.numel(), _stream(q)))
            return out
        _check(lib().csa_decode_step(ctypes.byref(self.desc), _ptr(self.buffer), _ptr(pos),
                                     ctypes.byref(r), ctypes.byref(p), _ptr(q), _ptr(q_i),
                                     _ptr(w_i), _ptr(out), _ptr(self.workspace),
                                     self.workspace.numel(), _stream(q)))
        return out
