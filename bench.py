#!/usr/bin/env python
"""Benchmark of the CSA/HCA attention layer on B200 (one JSON line on rank 0).

Headline: CSA prefill of one layer at n = 65536 tokens (c = 512, m = 4,
64 indexer heads x 128, top-k 512, 64 query heads, window 128, bf16), one
step = compress (KV) + compress (index keys) + indexer/top-k + sparse
attention, reported as query-tokens/s.  The same line carries the HCA
prefill layer (n = 16384, m = 128) and the two decode workloads (batch 64 at
context 131072; batch 4 at context 1048576 with one CSA and one HCA layer)
under "workloads", each with its roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

--impl reference times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload.  Several GPUs run independent replicas (the
layer is run on one GPU; no data-path collective), timed as the max over
ranks.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import csa_inputs as G  # noqa: E402

METRIC = "CSA prefill query-tokens/s (n=65536, c=512, top-k 512)"
UNIT = "tokens/s"

# DRAM bytes per call (ncu dram__bytes_read.sum + dram__bytes_write.sum of the
# call's kernels, one capture of the full workload; the summary is under
# profiles/).  A figure is reported only while the kernel sources it was
# measured on are unchanged (sha256 prefix per file), else null.
MEASURED_TRAFFIC = {
    # index_scores_tc_kernel 1126.2 MB read + 2136.1 MB written, topk_rows_staged_kernel
    # 2149.4 MB read + 131.3 MB written (n = 65536; ncu dram__bytes_read/write.sum)
    "index_topk": {"bytes": 5543051520, "sources": {
        'compressed_sparse_attention_11_b200/csrc/indexer_tc.cu': 'e3d3bdb783809238',
        'compressed_sparse_attention_11_b200/csrc/topk.cu': '7d7a94f9ad3e7624',
        'compressed_sparse_attention_11_b200/csrc/sm100.cuh': 'efc54e296506e512',
        'compressed_sparse_attention_11_b200/csrc/common.cuh': '2c8e048cf6f6eadb'}},
    # attn_tc_kernel 4571.7 MB read + 4242.5 MB written (n = 65536)
    "sparse_attn": {"bytes": 8814228992, "sources": {
        'compressed_sparse_attention_11_b200/csrc/attn_tc.cu': '9eaa94c3e12544ce',
        'compressed_sparse_attention_11_b200/csrc/sm100.cuh': 'efc54e296506e512',
        'compressed_sparse_attention_11_b200/csrc/common.cuh': '2c8e048cf6f6eadb',
        'compressed_sparse_attention_11_b200/csrc/rope.cuh': '8af18f1b31f2b303',
        'compressed_sparse_attention_11_b200/csrc/tc_attn_util.cuh': 'fbd5bcb87c834e55'}},
}


# Kernels each timed call launches at the workloads' shapes (the tensor-core
# path).  The roofline line names a kernel: the longest call that is one
# kernel, so that its CUDA-event time is that kernel's launch duration.
CALL_KERNELS = {
    "compress_kv": ("compress_rows_kernel<bf16>",),
    "compress_index_keys": ("compress_rows_kernel<bf16>",),
    "index_topk": ("index_scores_tc_kernel<64,128>", "topk_rows_staged_kernel"),
    "sparse_attn": ("attn_tc_kernel",),
    "compress": ("compress_split_kernel<bf16>",),
    "hca_attn": ("attn_tc_kernel",),
}


def dominant_kernel(calls, per_call_ms):
    """(call, kernel) of the longest single-kernel call."""
    single = [(ms, c) for c, ms in zip(calls, per_call_ms) if len(CALL_KERNELS[c]) == 1]
    ms, call = max(single)
    return call, CALL_KERNELS[call][0]


# ----------------------------------------------------------------- helpers ---

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm_gbs=d["hbm_gbs"], bf16=d["bf16_tflops"],
                    bf16_sustained=d["bf16_tflops_sustained"], source="measured")
    return dict(hbm_gbs=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


def sum_visible(n, m, E=None):
    """sum over t < n of min(floor((t+1)/m), E)."""
    E = n // m if E is None else E
    return sum(min((t + 1) // m, E) for t in range(n))


def sum_entry_sets(n, m, k, window):
    """sum over t of |E_t| = min(k, V(t)) + min(t+1, W) (k=None: dense)."""
    tot = 0
    for t in range(n):
        V = (t + 1) // m
        tot += (V if k is None else min(k, V)) + min(t + 1, window)
    return tot


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during a timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.device = device
        self.proc = None
        self.path = None

    def start(self):
        try:
            uuid = str(torch.cuda.get_device_properties(self.device).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            sel = []
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", *sel, f"--query-gpu={self.FIELDS}", "--format=csv,noheader",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"error": "nvidia-smi unavailable"}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"error": "no samples"}
        sm = [float(r[1].split()[0]) for r in rows if r[1].split()[0].replace(".", "").isdigit()]
        mx = [float(r[2].split()[0]) for r in rows if r[2].split()[0].replace(".", "").isdigit()]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return rank, world, local


def max_over_ranks(x: float, world: int) -> float:
    """The largest of the ranks' values (every rank gets it)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def job_throughput(units_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job units per second: every rank's units over the slowest rank's
    time (replicas: each rank runs the same workload)."""
    return units_per_rank * world / (ms_max * 1e-3)


# ------------------------------------------------------- CSA prefill layer ---

class CsaPrefill:
    """All device buffers of one CSA prefill layer call; step() runs it."""

    def __init__(self, w: G.Prefill, dev):
        import compressed_sparse_attention_11_b200 as csa
        self.csa, self.w, self.dev = csa, w, dev
        self.host = G.prefill_inputs(w)
        self.d = {k: v.to(dev) for k, v in self.host.items()}
        B, n, E = w.batch, w.n, w.n // w.m
        self.kv = torch.empty((B, E, w.c), dtype=w.dtype, device=dev)
        self.ki = torch.empty((B, E, w.c_i), dtype=w.dtype, device=dev)
        self.idx = torch.empty((B, n, w.k), dtype=torch.int32, device=dev)
        self.out = torch.empty_like(self.d["q"])
        nb = csa.csa_index_topk_workspace(B, n, w.nh_i, w.c_i, w.m, w.k)
        self.ws = torch.empty(max(nb, 16), dtype=torch.uint8, device=dev)
        self.calls = ("compress_kv", "compress_index_keys", "index_topk", "sparse_attn")
        self.launches_per_step = sum(len(CALL_KERNELS[c]) for c in self.calls)

    def step(self, ev=None):
        c, d, w = self.csa, self.d, self.w
        if ev: ev[0].record()
        c.csa_compress(d["ca"], d["cb"], d["za"], d["zb"], d["ba"], d["bb"], w.m, out=self.kv)
        if ev: ev[1].record()
        c.csa_compress(d["ica"], d["icb"], d["iza"], d["izb"], d["iba"], d["ibb"], w.m,
                       out=self.ki)
        if ev: ev[2].record()
        c.csa_index_topk(d["q_i"], d["w_i"], self.ki, w.m, w.k, ws=self.ws, out=self.idx)
        if ev: ev[3].record()
        c.csa_sparse_attn(d["q"], self.kv, self.idx, d["kv_win"], w.window, d["sink"], w.scale,
                          w.m, out=self.out)
        if ev: ev[4].record()

    def work(self):
        """Algorithmic work per call: (kind, amount) with kind bytes or flops."""
        w = self.w
        elt = 2 if w.dtype == torch.bfloat16 else 4
        n, E = w.n, w.n // w.m
        sv = sum_visible(n, w.m)
        se = sum_entry_sets(n, w.m, w.k, w.window)
        return {
            "compress_kv": ("bytes", 4 * n * w.c * elt + E * w.c * elt + 2 * w.m * w.c * 4),
            "compress_index_keys": ("bytes", 4 * n * w.c_i * elt + E * w.c_i * elt),
            "index_topk": ("flops", 2 * w.nh_i * w.c_i * sv),
            "sparse_attn": ("flops", 4 * w.nh * w.c * se),
        }

    def h2d_inputs(self, pinned):
        for k, v in pinned.items():
            self.d[k].copy_(v, non_blocking=True)


def time_steps(step_fn, ncalls, K, world, dev):
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(ncalls + 1)] for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    # keep the device busy while the host enqueues the first step, so that the
    # timed region holds device time only (no wait for the first launch)
    torch.cuda._sleep(2_000_000)
    start.record()
    for i in range(K):
        step_fn(evs[i])
    end.record()
    torch.cuda.synchronize()
    total = start.elapsed_time(end)
    per_call = [sum(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(K)) / K
                for j in range(ncalls)]
    return total, per_call


def measured_traffic(call):
    entry = MEASURED_TRAFFIC.get(call)
    if not entry:
        return None
    import hashlib
    for path, digest in entry["sources"].items():
        with open(os.path.join(ROOT, path), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest()[:16] != digest:
                return None
    return entry["bytes"]


def roofline(kind, amount, ms, peaks):
    """Achieved rate of `amount` algorithmic bytes or FLOPs in `ms` against the
    measured peak.  Tensor work is timed in regions of well under a second,
    so it is compared with the burst bf16 figure (the sustained one applies
    to seconds-long loops under the power cap)."""
    if kind == "bytes":
        ach = amount / (ms * 1e-3) / 1e9
        return {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(ach / peaks["hbm_gbs"], 4),
                "algorithmic": amount, "peak_source": peaks["source"] + " hbm_gbs"}
    ach = amount / (ms * 1e-3) / 1e12
    pk = peaks["bf16"]
    return {"bound": "tensor", "achieved": round(ach, 2), "peak": pk, "unit": "TFLOP/s",
            "frac": round(ach / pk, 4), "algorithmic": amount,
            "peak_source": peaks["source"] + " bf16_tflops (burst)"}


def time_region(fn, K, W):
    """Mean ms of fn() over K runs after W warm-up runs (CUDA events)."""
    for _ in range(W):
        fn()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(K):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / K


def bench_prefill_extras(L, dev, K, W, peaks):
    """The 'next' rows on the headline workload's tensors: the layer with the
    query / entry RMSNorm and partial RoPE, the low-precision indexer forms
    (with their recall against the exact selection on sampled rows), and
    the grouped output projection (V4-Flash: 8 groups, d_g 1024, d 4096)."""
    import numpy as np
    csa, d, w = L.csa, L.d, L.w
    out = {}
    # 1. norm + partial RoPE: entries normed as compressed, window rows by the
    #    row kernel, the query in the attention prologue, the output turned back
    g = torch.Generator(device="cpu").manual_seed(7)
    gq = (1.0 + 0.25 * torch.randn(w.c, generator=g)).to(dev)
    gk = (1.0 + 0.25 * torch.randn(w.c, generator=g)).to(dev)
    win_n = torch.empty_like(d["kv_win"])

    def nr_step():
        csa.csa_compress_norm_rope(d["ca"], d["cb"], d["za"], d["zb"], d["ba"], d["bb"], w.m, gk,
                                   out=L.kv)
        csa.csa_compress(d["ica"], d["icb"], d["iza"], d["izb"], d["iba"], d["ibb"], w.m,
                         out=L.ki)
        csa.csa_index_topk(d["q_i"], d["w_i"], L.ki, w.m, w.k, ws=L.ws, out=L.idx)
        csa.csa_norm_rope_rows(d["kv_win"], gk, out=win_n)
        csa.csa_sparse_attn_norm_rope(d["q"], L.kv, L.idx, win_n, w.window, d["sink"], w.scale,
                                      w.m, gq, out=L.out)

    ms_nr = time_region(nr_step, K, W)
    ms_plain = time_region(L.step, K, W)
    ms_rows = time_region(lambda: csa.csa_norm_rope_rows(d["kv_win"], gk, out=win_n), K, W)
    rows_bytes = 2 * d["kv_win"].numel() * 2
    out["norm_rope_layer"] = {
        "metric": "query-tokens/s", "value": round(w.n / (ms_nr * 1e-3), 1),
        "ms_per_step": round(ms_nr, 4), "plain_ms_per_step": round(ms_plain, 4),
        "cost_ms": round(ms_nr - ms_plain, 4),
        "window_rows_kernel": roofline("bytes", rows_bytes, ms_rows, peaks)}
    # 2. low-precision indexer forms, recall against the exact selection
    csa.csa_index_topk(d["q_i"], d["w_i"], L.ki, w.m, w.k, ws=L.ws, out=L.idx)
    ref = L.idx.clone()
    rows = list(range(w.n - 1, w.k * w.m, -(w.n // 512)))
    ref_h = ref[0, rows].cpu().numpy()
    flops = 2 * w.nh_i * w.c_i * sum_visible(w.n, w.m)
    lw = {}
    for name, fp8, bf16s in (("fp8_qk+bf16_scores", True, True), ("fp8_qk", True, False),
                             ("bf16_scores", False, True)):
        nb = csa.lib().csa_index_topk_lowp_workspace(1, w.n, w.nh_i, w.c_i, w.m, w.k,
                                                     (1 if fp8 else 0) | (2 if bf16s else 0))
        ws = torch.empty(nb, dtype=torch.uint8, device=dev)
        idx = torch.empty_like(L.idx)
        fn = lambda: csa.csa_index_topk_lowp(d["q_i"], d["w_i"], L.ki, w.m, w.k,  # noqa: E731
                                             fp8_qk=fp8, bf16_scores=bf16s, ws=ws, out=idx)
        ms = time_region(fn, K, W)
        got = idx[0, rows].cpu().numpy()
        rec = float(np.mean([len(np.intersect1d(a[a >= 0], b[b >= 0])) / max(1, (b >= 0).sum())
                             for a, b in zip(got, ref_h)]))
        lw[name] = {"ms": round(ms, 4), "recall_vs_exact": round(rec, 5),
                    "rows_for_recall": len(rows),
                    "roofline": roofline("flops", flops, ms, peaks)}
        del ws, idx
    lw["exact_ms"] = round(time_region(
        lambda: csa.csa_index_topk(d["q_i"], d["w_i"], L.ki, w.m, w.k, ws=L.ws, out=L.idx), K, W), 4)
    lw["note"] = ("fp8 tensor-core peak taken as 2x the measured bf16 burst figure (the recipe's "
                  "nominal ratio); the roofline lines above are against bf16")
    out["index_topk_lowp"] = lw
    # 3. grouped output projection on the attention output
    G_, dg, dm = 8, 1024, 4096
    kin = w.nh // G_ * w.c
    w1 = (torch.randn(G_, dg, kin, generator=g) * kin ** -0.5).to(torch.bfloat16).to(dev)
    w2 = (torch.randn(dm, G_ * dg, generator=g) * (G_ * dg) ** -0.5).to(torch.bfloat16).to(dev)
    zws = torch.empty(w.n * G_ * dg * 2, dtype=torch.uint8, device=dev)
    y = torch.empty((1, w.n, dm), dtype=torch.bfloat16, device=dev)
    ms_p = time_region(lambda: csa.csa_grouped_out_proj(L.out, w1, w2, ws=zws, out=y), K, W)
    pflops = 2 * w.n * (G_ * dg * kin + dm * G_ * dg)
    out["grouped_out_proj"] = {"shape": f"rows {w.n}, heads {w.nh} x {w.c}, {G_} groups, "
                                        f"d_g {dg}, d {dm}",
                               "ms": round(ms_p, 4), "roofline": roofline("flops", pflops, ms_p,
                                                                          peaks)}
    del w1, w2, zws, y, win_n
    return out


# ------------------------------------------------------------ other layers ---

def bench_hca_prefill(dev, K, W, peaks):
    import compressed_sparse_attention_11_b200 as csa
    w = G.HCA_PREFILL
    h = G.prefill_inputs(w)
    d = {k: v.to(dev) for k, v in h.items()}
    kv = torch.empty((w.batch, w.n // w.m, w.c), dtype=w.dtype, device=dev)
    out = torch.empty_like(d["q"])

    def step(ev):
        ev[0].record()
        csa.csa_compress(d["ca"], None, d["za"], None, d["ba"], None, w.m, out=kv)
        ev[1].record()
        csa.hca_attn(d["q"], kv, d["kv_win"], w.window, d["sink"], w.scale, w.m, out=out)
        ev[2].record()

    for _ in range(W):
        step([torch.cuda.Event(enable_timing=True) for _ in range(3)])
    total, per = time_steps(step, 2, K, 1, dev)
    ms = total / K
    elt = 2
    comp_bytes = 2 * w.n * w.c * elt + (w.n // w.m) * w.c * elt
    attn_flops = 4 * w.nh * w.c * sum_entry_sets(w.n, w.m, None, w.window)
    return {"workload": w.name, "metric": "query-tokens/s", "value": round(w.n / (ms * 1e-3), 1),
            "ms_per_step": round(ms, 4), "calls_ms": {"compress": round(per[0], 4),
                                                      "hca_attn": round(per[1], 4)},
            "roofline": {"compress": roofline("bytes", comp_bytes, per[0], peaks),
                         "hca_attn": roofline("flops", attn_flops, per[1], peaks)}}


def paged_block_table(batch: int, capacity: int, m: int, block_tokens: int = 128,
                      spare: int = 7, seed: int = 17):
    """A block table (int32 [batch, blocks per sequence], on the host) over a
    pool of batch * blocks + spare blocks of block_tokens tokens, enough for
    `capacity` entries per sequence, the physical blocks in a seeded random
    order (no two table slots share a block).  Returns (table, pool size)."""
    epb = block_tokens // m
    nb = (capacity + epb - 1) // epb
    pool = batch * nb + spare
    perm = torch.randperm(pool, generator=torch.Generator().manual_seed(seed))[:batch * nb]
    return perm.view(batch, nb).to(torch.int32), pool


def _decode_layer(w: G.Decode, dev, steps, paged: bool = False):
    """One decode layer's cache and per-step inputs.  ``paged``: the entries in
    a pool of 128-token blocks behind a block table whose physical blocks are
    in a seeded random order (the classical paged cache)."""
    import compressed_sparse_attention_11_b200 as csa
    inp = G.decode_inputs(w, steps=steps)
    E = w.t // w.m
    cap = E + steps // w.m + 2
    if paged:
        bt, pool = paged_block_table(w.batch, cap, w.m)
        bt = bt.to(dev)
        cache = csa.CsaCache(w.batch, cap, w.c, w.rope_dims, w.m, w.window, w.nh, w.is_hca,
                             c_i=w.c_i, nh_i=w.nh_i, k=w.k, device=dev, block_table=bt,
                             block_tokens=128, num_blocks=pool)
    else:
        cache = csa.CsaCache(w.batch, cap, w.c, w.rope_dims, w.m, w.window, w.nh, w.is_hca,
                             c_i=w.c_i, nh_i=w.nh_i, k=w.k, device=dev)
    cache.store_entries(0, inp["cache_kv"].to(dev),
                        None if w.is_hca else inp["cache_ikey"].to(dev))
    names = ("ca", "za", "kv_win") if w.is_hca else \
        ("ca", "cb", "za", "zb", "ica", "icb", "iza", "izb", "kv_win")
    tail = w.window + 2 * w.m
    cache.write_rows(w.t - tail, {nm: inp["rows_" + nm][:, :tail].contiguous().to(dev)
                                  for nm in names})
    bias_keys = ("ba",) if w.is_hca else ("ba", "bb", "iba", "ibb")
    per_step = []
    for s in range(steps):
        per_step.append(dict(
            pos=torch.full((w.batch,), w.t + s, dtype=torch.int64, device=dev),
            rows={nm: inp["rows_" + nm][:, tail + s].contiguous().to(dev) for nm in names},
            q=inp["q"][s].to(dev),
            q_i=None if w.is_hca else inp["q_i"][s].to(dev),
            w_i=None if w.is_hca else inp["w_i"][s].to(dev)))
    biases = {k: inp[k].to(dev) for k in bias_keys}
    sink = inp["sink"].to(dev)
    out = torch.empty((w.batch, w.nh, w.c), dtype=torch.bfloat16, device=dev)
    del inp
    return cache, per_step, biases, sink, out


def decode_bytes(w: G.Decode, t: int):
    """Algorithmic HBM bytes of one decode step at position t (all sequences)."""
    B, c, rope = w.batch, w.c, w.rope_dims
    V = (t + 1) // w.m
    entry = (c - rope) + 4 + 2 * rope
    win = min(t + 1, w.window) * c * 2
    qo = 2 * w.nh * c * 2
    rows = (2 if w.is_hca else 4) * c * 2 + c * 2
    if w.is_hca:
        return B * (V * entry + win + qo + rows)
    ikey = w.c_i + 4
    return B * (V * ikey + min(w.k, V) * entry + win + qo + rows + w.nh_i * (w.c_i * 2 + 4)
                + 4 * w.c_i * 2)


def bench_decode(layers, dev, K, W, peaks, name, paged: bool = False):
    """Times `steps` consecutive decode positions (the last one emits), L2 flushed."""
    steps = 4
    built = [_decode_layer(w, dev, steps, paged) for w in layers]
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    times = []
    for it in range(W + K):
        for s in range(steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for w, (cache, ps, biases, sink, out) in zip(layers, built):
                st = ps[s]
                cache.decode_step(st["pos"], st["rows"], biases, sink, w.scale, st["q"],
                                  st["q_i"], st["w_i"], out=out)
            e1.record()
            torch.cuda.synchronize()
            if it >= W:
                times.append(e0.elapsed_time(e1))
    us = [1000 * t for t in times]
    mean_us = statistics.mean(us)
    nbytes = statistics.mean(sum(decode_bytes(w, w.t + s) for w in layers)
                             for s in range(steps))
    rl = roofline("bytes", nbytes, mean_us / 1000, peaks)
    return {"workload": name, "metric": "decode us/step", "value": round(mean_us, 2),
            "max_us": round(max(us), 2), "steps_timed": len(us), "l2": "flushed before each step",
            "roofline": rl}


# -------------------------------------------------------------- CPU oracle ---

_ORACLE_W = {}


def _oracle_worker_init(tmpdir):
    """Pool worker: one BLAS thread, the sequence's shared arrays mapped from disk."""
    import numpy as np
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass
    for name in ("kv", "ki", "kv_win"):
        _ORACLE_W[name] = np.load(os.path.join(tmpdir, name + ".npy"), mmap_mode="r")


def _oracle_query_row(task):
    """Index scores, top-k and attention of one query row through the oracle."""
    import oracle as O
    t, q_t, qi_t, wi_t, sink, m, k, window, scale = task
    kv, ki, kv_win = _ORACLE_W["kv"], _ORACLE_W["ki"], _ORACLE_W["kv_win"]
    V = O.visible(t, m)
    sc = O.index_scores_row(qi_t, wi_t, ki, V)
    sel = O.topk_row(sc, k)
    Et = O.sparse_entry_set(kv, sel, kv_win, t, m, window)
    O.attend(q_t, Et, sink, scale)
    return t


def oracle_sample(budget_s=12.0, max_procs=32):
    """Times the fp64 oracle on a bounded sample of the CSA prefill workload.

    Compresses the whole sequence (KV and index keys, one process), then runs
    index scores, top-k and attention for strided query rows: first in one
    process with one BLAS thread, then spread over a pool of worker processes
    (one per host core, up to `max_procs`, each with one BLAS thread).  Each
    figure is query tokens per second extrapolated to the workload: the rows
    are sampled uniformly over positions, so their mean cost estimates the
    mean over all n rows."""
    import concurrent.futures as cf
    import multiprocessing as mp
    import shutil

    import numpy as np
    import oracle as O
    w = G.CSA_PREFILL
    inp = G.prefill_inputs(w)
    b = 0
    try:
        from threadpoolctl import threadpool_limits
        limit = threadpool_limits(1)
    except Exception:
        limit = None
    t0 = time.perf_counter()
    kv = O.csa_compress(inp["ca"][b], inp["cb"][b], inp["za"][b], inp["zb"][b], inp["ba"],
                        inp["bb"], w.m)
    ki = O.csa_compress(inp["ica"][b], inp["icb"][b], inp["iza"][b], inp["izb"][b], inp["iba"],
                        inp["ibb"], w.m)
    t_comp = time.perf_counter() - t0
    tmpdir = tempfile.mkdtemp(prefix="csa_oracle_")
    try:
        np.save(os.path.join(tmpdir, "kv.npy"), kv)
        np.save(os.path.join(tmpdir, "ki.npy"), ki)
        np.save(os.path.join(tmpdir, "kv_win.npy"), O.f64(inp["kv_win"][b]))
        sink = O.f64(inp["sink"])
        rows = list(range(w.n - 1, 0, -(w.n // 2048)))   # strided, from the longest row down
        order = [rows[i] for i in np.random.default_rng(0).permutation(len(rows))]

        def task(t):
            return (t, O.f64(inp["q"][b, t]), O.f64(inp["q_i"][b, t]), O.f64(inp["w_i"][b, t]),
                    sink, w.m, w.k, w.window, w.scale)

        # one process, one thread
        _oracle_worker_init(tmpdir)
        done, t1 = 0, time.perf_counter()
        for t in order:
            _oracle_query_row(task(t))
            done += 1
            if time.perf_counter() - t1 > budget_s / 3 and done >= 4:
                break
        per_row_1 = (time.perf_counter() - t1) / done
        if limit is not None:
            limit.restore_original_limits()
        one = {"value": round(1.0 / (t_comp / w.n + per_row_1), 3), "cores": 1,
               "rows": done}

        # a pool of worker processes, one BLAS thread each
        procs = max(1, min(max_procs, os.cpu_count() or 1))
        nrows = max(procs, min(20000, int(procs * (2 * budget_s / 3) / per_row_1)))
        with cf.ProcessPoolExecutor(procs, mp_context=mp.get_context("spawn"),
                                    initializer=_oracle_worker_init,
                                    initargs=(tmpdir,)) as ex:
            list(ex.map(_oracle_query_row, [task(t) for t in order[:procs]]))  # start-up
            tasks = [task(order[i % len(order)]) for i in range(nrows)]
            t2 = time.perf_counter()
            list(ex.map(_oracle_query_row, tasks))
            t_pool = time.perf_counter() - t2
        per_row_p = t_pool / nrows
    finally:
        shutil.rmtree(tmpdir, ignore_errors=True)
    return {"value": round(1.0 / (t_comp / w.n + per_row_p), 3), "unit": UNIT, "cores": procs,
            "kind": "oracle", "one_thread": one,
            "sample": f"full compression of both streams on one core ({t_comp:.1f} s), then "
                      f"index/top-k/attention of strided query rows: {done} rows on one "
                      f"thread, {nrows} rows over {procs} worker processes of one thread "
                      f"({t_pool:.1f} s); extrapolated to n={w.n}"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    t0 = time.perf_counter()
    cb = oracle_sample(budget_s=max(5.0, 20.0 / max(1, args.steps)))
    elapsed = time.perf_counter() - t0
    line = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(G.CSA_PREFILL.n / cb["value"] * 1000, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": G.CSA_PREFILL.name,
                                            "seq_len": G.CSA_PREFILL.n, "batch": 1},
            "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "wall_s": round(elapsed, 1)}
    print(json.dumps(line), flush=True)


# -------------------------------------------------------------------- main ---

def run_profile_case(args):
    """A few steps of one workload, optionally resized, for ncu captures."""
    import dataclasses
    import compressed_sparse_attention_11_b200 as csa
    dev = torch.device("cuda", 0)
    if args.profile in ("prefill", "hca", "next"):
        base = G.HCA_PREFILL if args.profile == "hca" else G.CSA_PREFILL
        w = dataclasses.replace(base, n=args.n) if args.n else base
        if args.profile == "prefill":
            L = CsaPrefill(w, dev)
            for _ in range(args.steps):
                L.step()
        elif args.profile == "next":
            # the 'next' rows once per step: norm + RoPE layer, FP8 / bf16-score
            # indexer, grouped output projection (V4-Flash shapes)
            L = CsaPrefill(w, dev)
            d = L.d
            g = torch.Generator(device="cpu").manual_seed(7)
            gam = (1.0 + 0.25 * torch.randn(w.c, generator=g)).to(dev)
            win_n = torch.empty_like(d["kv_win"])
            idx = torch.empty_like(L.idx)
            kin = w.nh // 8 * w.c
            w1 = (torch.randn(8, 1024, kin, generator=g) * kin ** -0.5).to(torch.bfloat16).to(dev)
            w2 = (torch.randn(4096, 8192, generator=g) * 8192 ** -0.5).to(torch.bfloat16).to(dev)
            y = torch.empty((1, w.n, 4096), dtype=torch.bfloat16, device=dev)
            for _ in range(args.steps):
                csa.csa_compress_norm_rope(d["ca"], d["cb"], d["za"], d["zb"], d["ba"], d["bb"],
                                           w.m, gam, out=L.kv)
                csa.csa_compress(d["ica"], d["icb"], d["iza"], d["izb"], d["iba"], d["ibb"], w.m,
                                 out=L.ki)
                csa.csa_index_topk_lowp(d["q_i"], d["w_i"], L.ki, w.m, w.k, fp8_qk=True,
                                        bf16_scores=True, out=idx)
                csa.csa_norm_rope_rows(d["kv_win"], gam, out=win_n)
                csa.csa_sparse_attn_norm_rope(d["q"], L.kv, idx, win_n, w.window, d["sink"],
                                              w.scale, w.m, gam, out=L.out)
                csa.csa_grouped_out_proj(L.out, w1, w2, out=y)
        else:
            d = {k: v.to(dev) for k, v in G.prefill_inputs(w).items()}
            for _ in range(args.steps):
                kv = csa.csa_compress(d["ca"], None, d["za"], None, d["ba"], None, w.m)
                csa.hca_attn(d["q"], kv, d["kv_win"], w.window, d["sink"], w.scale, w.m)
    else:
        layers = [G.CSA_DECODE] if args.profile == "decode_csa" else \
            [G.MIXED_DECODE_CSA, G.MIXED_DECODE_HCA]
        if args.batch:
            layers = [dataclasses.replace(x, batch=args.batch) for x in layers]
        built = [_decode_layer(x, dev, 4, args.paged) for x in layers]
        for it in range(args.steps):
            for x, (cache, ps, biases, sink, out) in zip(layers, built):
                st = ps[it % 4]
                cache.decode_step(st["pos"], st["rows"], biases, sink, x.scale, st["q"],
                                  st["q_i"], st["w_i"], out=out)
    torch.cuda.synchronize()
    csa.csa_check()
    print(json.dumps({"profile": args.profile, "steps": args.steps, "n": args.n,
                      "batch": args.batch, "paged": args.paged, "ok": True}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=("ours", "reference"))
    ap.add_argument("--skip-extras", action="store_true", help="headline workload only")
    ap.add_argument("--skip-cpu", action="store_true", help="no oracle timing")
    ap.add_argument("--profile", choices=("prefill", "hca", "next", "decode_csa", "decode_mixed"),
                    help="run --steps steps of one workload (for a profiler) and exit")
    ap.add_argument("--n", type=int, default=None, help="--profile prefill/hca/next: tokens")
    ap.add_argument("--batch", type=int, default=None, help="--profile decode_*: sequences")
    ap.add_argument("--paged", action="store_true",
                    help="--profile decode_*: entries in the paged 128-token-block cache")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
        return
    if args.profile:
        run_profile_case(args)
        return
    rank, world, local = dist_setup()
    dev = torch.device("cuda", local)
    import compressed_sparse_attention_11_b200 as csa
    csa.lib()
    peaks = load_peaks()
    w = G.CSA_PREFILL
    L = CsaPrefill(w, dev)
    ncalls = len(L.calls)
    for _ in range(args.warmup):
        L.step()
    torch.cuda.synchronize()
    clk = ClockSampler(dev)
    clk.start()
    total, per_call = time_steps(L.step, ncalls, args.steps, world, dev)
    clocks = clk.stop()
    total = max_over_ranks(total, world)
    ms = total / args.steps
    value = job_throughput(w.n * w.batch, world, ms)
    work = L.work()
    calls = {name: round(t, 4) for name, t in zip(L.calls, per_call)}
    roof = {name: roofline(*work[name], per_call[i], peaks) for i, name in enumerate(L.calls)}
    dom_call, dom_kernel = dominant_kernel(L.calls, per_call)
    dominant = dict(roof[dom_call])
    dominant["kernel"] = dom_kernel
    dominant["call"] = dom_call
    dominant["ms_per_launch"] = calls[dom_call]
    dominant["traffic"] = measured_traffic(dom_call)

    # end to end: every step copies all its inputs from pinned host memory to
    # the device and its whole output back, through the library's public calls.
    # Two steps are in flight: step i's inputs go host -> device on one stream
    # while step i-1 computes on a second and step i-1's output goes
    # device -> host on a third (PCIe carries both directions at once); the
    # device holds two sets of inputs and outputs for it.
    pinned = {k: v.pin_memory() for k, v in L.host.items()}
    out_host = torch.empty(L.out.shape, dtype=L.out.dtype, pin_memory=True)
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = out_host.numel() * out_host.element_size()
    sets = [(L.d, L.out),
            ({k: torch.empty_like(v) for k, v in L.d.items()}, torch.empty_like(L.out))]
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_run(nsteps):
        cur = torch.cuda.current_stream()
        for st in (s_in, s_comp, s_out):
            st.wait_stream(cur)
        comp_done, out_done = [], []
        for i in range(nsteps):
            d, out = sets[i % 2]
            with torch.cuda.stream(s_in):
                if i >= 2:  # step i - 2, the last reader of these inputs, is done
                    s_in.wait_event(comp_done[i - 2])
                for k, v in pinned.items():
                    d[k].copy_(v, non_blocking=True)
                in_ready = torch.cuda.Event()
                in_ready.record(s_in)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(in_ready)
                if i >= 2:  # step i - 2's output has been read back
                    s_comp.wait_event(out_done[i - 2])
                L.d, L.out = d, out
                L.step()
                comp_done.append(torch.cuda.Event())
                comp_done[-1].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[-1])
                out_host.copy_(out, non_blocking=True)
                out_done.append(torch.cuda.Event())
                out_done[-1].record(s_out)
        for st in (s_in, s_comp, s_out):
            cur.wait_stream(st)

    e2e_run(2)
    torch.cuda.synchronize()
    n_e2e = max(3, args.steps)
    barrier(world)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    e2e_run(n_e2e)
    t1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(t0.elapsed_time(t1), world) / n_e2e
    L.d, L.out = sets[0]
    del pinned, out_host, sets

    launches_per_step = L.launches_per_step
    layer_calls = L.calls
    workloads = {}
    if not args.skip_extras:
        workloads["csa_prefill_next_rows"] = bench_prefill_extras(L, dev, max(2, args.steps // 4),
                                                                  2, peaks)
    if not args.skip_extras:
        del L
        torch.cuda.empty_cache()
        workloads["hca_prefill"] = bench_hca_prefill(dev, args.steps, args.warmup, peaks)
        torch.cuda.empty_cache()
        workloads["csa_decode"] = bench_decode([G.CSA_DECODE], dev, max(2, args.steps // 2),
                                               1, peaks, G.CSA_DECODE.name)
        torch.cuda.empty_cache()
        workloads["csa_decode_paged"] = bench_decode([G.CSA_DECODE], dev,
                                                     max(2, args.steps // 2), 1, peaks,
                                                     G.CSA_DECODE.name + "_paged128", paged=True)
        torch.cuda.empty_cache()
        workloads["mixed_decode"] = bench_decode([G.MIXED_DECODE_CSA, G.MIXED_DECODE_HCA], dev,
                                                 max(2, args.steps // 2), 1, peaks,
                                                 "mixed_decode_b4_ctx1048576_csa+hca")
    cpu = None
    if rank == 0 and not args.skip_cpu:
        cpu = oracle_sample()
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": w.name, "seq_len": w.n, "batch": w.batch, "c": w.c,
                       "m": w.m, "top_k": w.k, "heads": w.nh, "index_heads": w.nh_i,
                       "index_dim": w.c_i, "window": w.window,
                       "parallelism": f"replicas x{world}",
                       "l2": "inputs (5.8 GB) larger than L2"},
            "calls_ms": calls,
            "roofline": dominant,
            "roofline_per_call": roof,
            "gpu_launches": launches_per_step * args.steps,
            "kernels_per_call": {c: list(CALL_KERNELS[c]) for c in layer_calls},
            "e2e": {"value": round(w.n * w.batch * world / (e2e_ms * 1e-3), 1), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": round(e2e_ms, 3), "steps": n_e2e,
                    "pipeline": "2 steps in flight: H2D, layer, D2H on three streams"},
            "clocks": clocks,
            "cpu_baseline": cpu,
            "workloads": workloads,
            "peaks": peaks,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
