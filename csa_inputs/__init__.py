"""Seeded synthetic inputs shared by the oracle, the tests and the benchmark.

This module only draws random tensors and names workload shapes.  It holds
none of the attention layer's arithmetic (no softmax, no visibility rule, no
quantisation), so the CPU oracle and the CUDA library can both consume its
output without sharing any method code.

Every tensor is drawn on the host from ``torch.Generator`` seeded with
``seed * 1_000_003 + tensor_id`` (float32 normal / uniform draws, then scaled
and rounded to the requested dtype with torch's round-to-nearest-even cast),
so the same (seed, tensor_id, shape, dtype) always yields the same bits.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch

_CHUNK = 1 << 25  # elements drawn per generator call (bounds host memory)


def _generator(seed: int, tensor_id: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed((int(seed) * 1_000_003 + int(tensor_id)) & ((1 << 63) - 1))
    return g


def normal(shape, seed: int, tensor_id: int, std: float = 1.0,
           dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    """N(0, std^2) draws of ``shape`` rounded to ``dtype`` (CPU tensor)."""
    g = _generator(seed, tensor_id)
    out = torch.empty(shape, dtype=dtype)
    flat = out.view(-1)
    total = flat.numel()
    for lo in range(0, total, _CHUNK):
        hi = min(total, lo + _CHUNK)
        x = torch.randn(hi - lo, generator=g, dtype=torch.float32)
        if std != 1.0:
            x.mul_(std)
        flat[lo:hi] = x.to(dtype)
    return out


def uniform(shape, seed: int, tensor_id: int, lo: float = 0.0, hi: float = 1.0,
            dtype: torch.dtype = torch.float32) -> torch.Tensor:
    """U(lo, hi) draws of ``shape`` rounded to ``dtype`` (CPU tensor)."""
    g = _generator(seed, tensor_id)
    out = torch.empty(shape, dtype=dtype)
    flat = out.view(-1)
    total = flat.numel()
    for a in range(0, total, _CHUNK):
        b = min(total, a + _CHUNK)
        x = torch.rand(b - a, generator=g, dtype=torch.float32)
        flat[a:b] = (x * (hi - lo) + lo).to(dtype)
    return out


def pinned(t: torch.Tensor) -> torch.Tensor:
    """Copy of ``t`` in page-locked host memory (for timed host->device copies)."""
    return t.pin_memory()


# --------------------------------------------------------------------------
# Workload shapes.  Sizes follow the five benchmark workloads of the layer:
# tiny fp32 CSA prefill, HCA prefill, long CSA prefill, batched CSA decode and
# 1M-context mixed CSA/HCA decode.
# --------------------------------------------------------------------------

BASE_SEED = 20261202


@dataclasses.dataclass(frozen=True)
class Prefill:
    name: str
    kind: str              # "csa" or "hca"
    batch: int
    n: int                 # tokens
    c: int                 # entry / head dim
    m: int                 # compression ratio
    nh: int                # query heads
    window: int
    dtype: torch.dtype
    nh_i: int = 0          # indexer heads (csa)
    c_i: int = 0           # indexer dim (csa)
    k: int = 0             # top-k (csa)
    sink_scalar: Optional[float] = None  # same sink logit for every head
    seed: int = BASE_SEED

    @property
    def scale(self) -> float:
        return 1.0 / float(self.c) ** 0.5


@dataclasses.dataclass(frozen=True)
class Decode:
    name: str
    batch: int
    t: int                 # 0-based position of the decode token
    c: int
    rope_dims: int
    m: int
    nh: int
    window: int
    is_hca: bool
    nh_i: int = 0
    c_i: int = 0
    k: int = 0
    seed: int = BASE_SEED

    @property
    def scale(self) -> float:
        return 1.0 / float(self.c) ** 0.5


TINY_CSA_PREFILL = Prefill("tiny_csa_prefill_fp32_n1024", "csa", 1, 1024, 128, 4, 16, 128,
                           torch.float32, nh_i=4, c_i=64, k=32, sink_scalar=0.0,
                           seed=BASE_SEED + 0)
HCA_PREFILL = Prefill("hca_prefill_bf16_n16384", "hca", 1, 16384, 512, 128, 64, 128,
                      torch.bfloat16, seed=BASE_SEED + 1)
CSA_PREFILL = Prefill("csa_prefill_bf16_n65536", "csa", 1, 65536, 512, 4, 64, 128,
                      torch.bfloat16, nh_i=64, c_i=128, k=512, seed=BASE_SEED + 2)
CSA_DECODE = Decode("csa_decode_b64_ctx131072", 64, 131072, 512, 64, 4, 64, 128, False,
                    nh_i=64, c_i=128, k=512, seed=BASE_SEED + 3)
MIXED_DECODE_CSA = Decode("mixed_decode_b4_ctx1048576_csa", 4, 1048576, 512, 64, 4, 64, 128,
                          False, nh_i=64, c_i=128, k=512, seed=BASE_SEED + 4)
MIXED_DECODE_HCA = Decode("mixed_decode_b4_ctx1048576_hca", 4, 1048576, 512, 64, 128, 64, 128,
                          True, seed=BASE_SEED + 5)

WORKLOADS: Dict[str, object] = {w.name: w for w in (
    TINY_CSA_PREFILL, HCA_PREFILL, CSA_PREFILL, CSA_DECODE, MIXED_DECODE_CSA, MIXED_DECODE_HCA)}


# tensor ids (stable across versions so stored fixtures keep their meaning)
_IDS = dict(ca=1, cb=2, za=3, zb=4, ba=5, bb=6, ica=7, icb=8, iza=9, izb=10, iba=11, ibb=12,
            kv_win=13, q=14, q_i=15, w_i=16, sink=17,
            cache_kv=20, cache_ikey=21)


def prefill_inputs(w: Prefill, n: Optional[int] = None, batch: Optional[int] = None,
                   seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """All host tensors of one prefill layer call.

    CSA: Ca, Cb, Za, Zb [B,n,c]; Ba, Bb [m,c] fp32 ~N(0,0.1); index-key streams
    ica..izb [B,n,c_i] with biases iba, ibb [m,c_i]; q [B,n,nh,c]; q_i
    [B,n,nh_i,c_i]; w_i [B,n,nh_i] fp32 ~U(0,1); kv_win [B,n,c]; sink [nh] fp32.
    HCA: C (ca), Z (za), B (ba) only, plus q, kv_win, sink.
    """
    n = w.n if n is None else n
    B = w.batch if batch is None else batch
    s = w.seed if seed is None else seed
    dt = w.dtype
    out: Dict[str, torch.Tensor] = {}
    out["ca"] = normal((B, n, w.c), s, _IDS["ca"], dtype=dt)
    out["za"] = normal((B, n, w.c), s, _IDS["za"], dtype=dt)
    out["ba"] = normal((w.m, w.c), s, _IDS["ba"], std=0.1, dtype=torch.float32)
    if w.kind == "csa":
        out["cb"] = normal((B, n, w.c), s, _IDS["cb"], dtype=dt)
        out["zb"] = normal((B, n, w.c), s, _IDS["zb"], dtype=dt)
        out["bb"] = normal((w.m, w.c), s, _IDS["bb"], std=0.1, dtype=torch.float32)
        for nm in ("ica", "icb", "iza", "izb"):
            out[nm] = normal((B, n, w.c_i), s, _IDS[nm], dtype=dt)
        for nm in ("iba", "ibb"):
            out[nm] = normal((w.m, w.c_i), s, _IDS[nm], std=0.1, dtype=torch.float32)
        out["q_i"] = normal((B, n, w.nh_i, w.c_i), s, _IDS["q_i"], dtype=dt)
        out["w_i"] = uniform((B, n, w.nh_i), s, _IDS["w_i"])
    out["kv_win"] = normal((B, n, w.c), s, _IDS["kv_win"], dtype=dt)
    out["q"] = normal((B, n, w.nh, w.c), s, _IDS["q"], dtype=dt)
    if w.sink_scalar is not None:
        out["sink"] = torch.full((w.nh,), float(w.sink_scalar), dtype=torch.float32)
    else:
        out["sink"] = normal((w.nh,), s, _IDS["sink"], dtype=torch.float32)
    return out


def decode_inputs(w: Decode, entries: Optional[int] = None, batch: Optional[int] = None,
                  t: Optional[int] = None, steps: int = 1, seed: Optional[int] = None
                  ) -> Dict[str, torch.Tensor]:
    """Host tensors of a decode run.

    ``cache_kv`` [B,E,c] fp32 and ``cache_ikey`` [B,E,c_i] fp32 are the values
    of the E compressed entries already in the cache (each side quantises them
    itself).  ``rows_*`` hold raw per-position rows for positions
    ``t0 - tail .. t0 + steps - 1`` where ``tail = window + 2*m`` (enough to
    rebuild the window ring and the compressor's partial and previous blocks),
    indexed [B, P, dim].  ``q``, ``q_i``, ``w_i`` hold one query per step:
    [steps, B, nh, c] etc.
    """
    B = w.batch if batch is None else batch
    t0 = w.t if t is None else t
    s = w.seed if seed is None else seed
    E = (t0 // w.m) if entries is None else entries
    dt = torch.bfloat16
    tail = w.window + 2 * w.m
    P = tail + steps
    out: Dict[str, torch.Tensor] = {}
    out["cache_kv"] = normal((B, E, w.c), s, _IDS["cache_kv"], dtype=torch.float32)
    for nm in ("ca", "za"):
        out["rows_" + nm] = normal((B, P, w.c), s, _IDS[nm], dtype=dt)
    out["ba"] = normal((w.m, w.c), s, _IDS["ba"], std=0.1, dtype=torch.float32)
    if not w.is_hca:
        out["cache_ikey"] = normal((B, E, w.c_i), s, _IDS["cache_ikey"], dtype=torch.float32)
        for nm in ("cb", "zb"):
            out["rows_" + nm] = normal((B, P, w.c), s, _IDS[nm], dtype=dt)
        out["bb"] = normal((w.m, w.c), s, _IDS["bb"], std=0.1, dtype=torch.float32)
        for nm in ("ica", "icb", "iza", "izb"):
            out["rows_" + nm] = normal((B, P, w.c_i), s, _IDS[nm], dtype=dt)
        for nm in ("iba", "ibb"):
            out[nm] = normal((w.m, w.c_i), s, _IDS[nm], std=0.1, dtype=torch.float32)
        out["q_i"] = normal((steps, B, w.nh_i, w.c_i), s, _IDS["q_i"], dtype=dt)
        out["w_i"] = uniform((steps, B, w.nh_i), s, _IDS["w_i"])
    out["rows_kv_win"] = normal((B, P, w.c), s, _IDS["kv_win"], dtype=dt)
    out["q"] = normal((steps, B, w.nh, w.c), s, _IDS["q"], dtype=dt)
    out["sink"] = normal((w.nh,), s, _IDS["sink"], dtype=torch.float32)
    out["first_pos"] = torch.tensor(t0 - tail, dtype=torch.int64)
    return out
