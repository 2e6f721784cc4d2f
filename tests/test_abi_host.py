"""Host-side checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments before launching anything.

None of these calls reaches a kernel launch: every argument set below fails
validation (or is empty work), so they run on a machine without a GPU.
"""
import ctypes
import os
import re

import pytest
import torch

import compressed_sparse_attention_11_b200 as csa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa.h")
FAKE = 0x10000          # 16-byte aligned, never dereferenced (validation fails first)
MISALIGNED = 0x10004


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([a-z_][a-z0-9_]*)\s*\(",
                       text, flags=re.M)
    return sorted(set(n for n in names if n.startswith(("csa_", "hca_"))))


def test_library_exports_every_declared_function():
    L = csa.lib()
    declared = header_functions()
    assert len(declared) >= 12
    for name in declared:
        assert hasattr(L, name), name
    assert set(declared) == set(csa.EXPORTED)
    assert L.csa_abi_version() == 2


def test_status_strings():
    assert csa.status_string(0) == "CSA_OK"
    assert csa.status_string(-1) == "CSA_ERR_INVALID_ARG"
    assert csa.status_string(-3) == "CSA_ERR_WORKSPACE"
    assert csa.status_string(-5) == "CSA_ERR_TIMEOUT"
    assert csa.status_string(7) == "CSA_ERR_UNKNOWN"


def _compress(**kw):
    a = dict(ca=FAKE, cb=FAKE, za=FAKE, zb=FAKE, ba=FAKE, bb=FAKE, batch=1, n=64, c=128, m=4,
             overlap=1, dt=1, out=FAKE, stream=None)
    a.update(kw)
    L = csa.lib()
    return L.csa_compress(a["ca"], a["cb"], a["za"], a["zb"], a["ba"], a["bb"], a["batch"],
                          a["n"], a["c"], a["m"], a["overlap"], a["dt"], a["out"], a["stream"])


@pytest.mark.parametrize("kw,why", [
    (dict(c=12), "multiple of 8"),
    (dict(c=0), "multiple of 8"),
    (dict(m=0), "m must"),
    (dict(overlap=2), "overlap"),
    (dict(dt=7), "dt must"),
    (dict(batch=-1), "batch"),
    (dict(ca=None), "ca is NULL"),
    (dict(zb=MISALIGNED), "zb is not 16-byte aligned"),
    (dict(out=None), "out is NULL"),
    (dict(overlap=0), "must be NULL"),
])
def test_compress_rejects_bad_arguments(kw, why):
    assert _compress(**kw) == csa.CSA_ERR_INVALID_ARG
    assert why in csa.lib().csa_last_error().decode()


def test_compress_empty_work_is_ok_without_launch():
    assert _compress(batch=0, ca=None, out=None) == csa.CSA_OK
    assert _compress(n=3, ca=None) == csa.CSA_OK      # n < m: no complete entry


def test_index_topk_validation_and_workspace():
    L = csa.lib()
    assert csa.csa_index_topk_workspace(1, 1024, 4, 64, 4, 32) == 1024 * 256 * 4
    assert csa.csa_index_topk_workspace(2, 65536, 64, 128, 4, 512) == 2 * 65536 * 16384 * 4
    call = lambda **kw: L.csa_index_topk(
        kw.get("q", FAKE), kw.get("w", FAKE), kw.get("kk", FAKE), 1, kw.get("n", 64),
        kw.get("nh", 4), kw.get("ci", 64), kw.get("m", 4), kw.get("k", 8), 1,
        kw.get("idx", FAKE), kw.get("ws", FAKE), kw.get("wsb", 1 << 30), None)
    assert call(k=0) == csa.CSA_ERR_INVALID_ARG
    assert call(ci=60) == csa.CSA_ERR_INVALID_ARG
    assert call(nh=0) == csa.CSA_ERR_INVALID_ARG
    assert call(idx=None) == csa.CSA_ERR_INVALID_ARG
    assert call(kk=MISALIGNED) == csa.CSA_ERR_INVALID_ARG
    assert call(wsb=100) == csa.CSA_ERR_WORKSPACE
    assert call(ws=None) == csa.CSA_ERR_WORKSPACE
    assert call(ci=1024, nh=64) == csa.CSA_ERR_UNSUPPORTED


def test_attention_validation():
    L = csa.lib()
    sp = lambda **kw: L.csa_sparse_attn(
        kw.get("q", FAKE), FAKE, kw.get("idx", FAKE), kw.get("k", 8), FAKE, kw.get("win", 128),
        None, kw.get("scale", 0.1), 1, 64, kw.get("nh", 16), kw.get("c", 128), 4, 0,
        kw.get("out", FAKE), None)
    assert sp(k=0) == csa.CSA_ERR_INVALID_ARG
    assert sp(win=0) == csa.CSA_ERR_INVALID_ARG
    assert sp(nh=0) == csa.CSA_ERR_INVALID_ARG
    assert sp(idx=None) == csa.CSA_ERR_INVALID_ARG
    assert sp(scale=float("nan")) == csa.CSA_ERR_INVALID_ARG
    assert sp(c=1024) == csa.CSA_ERR_UNSUPPORTED
    assert sp(c=136) == csa.CSA_ERR_UNSUPPORTED
    hc = lambda **kw: L.hca_attn(FAKE, kw.get("kv", FAKE), FAKE, 128, None, 0.1, 1,
                                 kw.get("n", 256), 16, 128, kw.get("m", 128), 0, FAKE, None)
    assert hc(m=0) == csa.CSA_ERR_INVALID_ARG
    assert hc(kv=None) == csa.CSA_ERR_INVALID_ARG


def _desc(**kw):
    base = dict(batch=64, capacity=32772, c=512, rope_dims=64, c_i=128, m=4, window=128, nh=64,
                nh_i=64, k=512, is_hca=0)
    base.update(kw)
    return csa.CacheDesc(**base)


def test_cache_layout_matches_documented_regions():
    L = csa.lib()
    d = _desc()
    lay = csa.CacheLayout()
    assert L.csa_cache_layout(ctypes.byref(d), ctypes.byref(lay)) == csa.CSA_OK
    B, cap = 64, 32772
    al = lambda x: (x + 255) // 256 * 256
    expect = [("entry_fp8", B * cap * 448), ("entry_scale", B * cap * 4),
              ("entry_rope", B * cap * 64 * 2), ("ikey_fp8", B * cap * 128),
              ("ikey_scale", B * cap * 4), ("window", B * 128 * 512 * 2),
              ("state", B * 2 * 4 * 4 * 512 * 2), ("istate", B * 2 * 4 * 4 * 128 * 2)]
    off = 0
    for name, size in expect:
        assert getattr(lay, name) == off, name
        assert off % 256 == 0
        off = al(off + size)
    assert lay.total_bytes == off
    # per entry: 448 FP8 + 4 scale + 128 bf16 RoPE + 128 FP8 key + 4 key scale
    assert (448 + 4 + 128 + 128 + 4) == 712
    h = _desc(is_hca=1, m=128, capacity=8200, batch=4)
    assert L.csa_cache_layout(ctypes.byref(h), ctypes.byref(lay)) == csa.CSA_OK
    assert lay.ikey_fp8 == lay.ikey_scale == lay.window   # no index keys for HCA


@pytest.mark.parametrize("kw", [dict(c=500), dict(rope_dims=512), dict(rope_dims=4),
                                dict(m=0), dict(window=0), dict(nh=0), dict(c_i=100),
                                dict(k=0), dict(is_hca=3), dict(batch=0), dict(capacity=0)])
def test_cache_desc_rejected(kw):
    L = csa.lib()
    lay = csa.CacheLayout()
    assert L.csa_cache_layout(ctypes.byref(_desc(**kw)), ctypes.byref(lay)) == \
        csa.CSA_ERR_INVALID_ARG
    assert L.csa_decode_workspace(ctypes.byref(_desc(**kw))) == 0


def test_decode_step_validation():
    L = csa.lib()
    d = _desc()
    rows = csa.Rows(*([FAKE] * 9))
    p = csa.DecodeParams(FAKE, FAKE, FAKE, FAKE, None, 0.05)
    ws = L.csa_decode_workspace(ctypes.byref(d))
    assert ws > 0
    call = lambda **kw: L.csa_decode_step(ctypes.byref(d), FAKE, kw.get("pos", FAKE),
                                          ctypes.byref(kw.get("rows", rows)),
                                          ctypes.byref(kw.get("p", p)), FAKE,
                                          kw.get("qi", FAKE), FAKE, FAKE, FAKE,
                                          kw.get("ws", ws), None)
    assert call(pos=None) == csa.CSA_ERR_INVALID_ARG
    assert call(qi=None) == csa.CSA_ERR_INVALID_ARG
    assert call(ws=ws - 1) == csa.CSA_ERR_WORKSPACE
    bad_rows = csa.Rows(*([FAKE] * 8 + [None]))
    assert call(rows=bad_rows) == csa.CSA_ERR_INVALID_ARG
    bad_p = csa.DecodeParams(FAKE, None, FAKE, FAKE, None, 0.05)
    assert call(p=bad_p) == csa.CSA_ERR_INVALID_ARG
    # store / write_rows range checks
    assert L.csa_cache_store_entries(ctypes.byref(d), FAKE, 32770, 5, FAKE, FAKE, 1, None) == \
        csa.CSA_ERR_INVALID_ARG
    assert L.csa_cache_store_entries(ctypes.byref(d), FAKE, 0, 0, None, None, 1, None) == \
        csa.CSA_OK
    assert L.csa_cache_write_rows(ctypes.byref(d), FAKE, -1, 4, ctypes.byref(rows), None) == \
        csa.CSA_ERR_INVALID_ARG


def test_selftest_wait_rejects_limits_out_of_range():
    L = csa.lib()
    assert L.csa_selftest_wait(0, 1, None) == csa.CSA_ERR_INVALID_ARG
    assert L.csa_selftest_wait(2000001, 0, None) == csa.CSA_ERR_INVALID_ARG


def test_binding_rejects_host_tensors_and_bad_layouts():
    """The Python binding only marshals: it refuses what the C ABI cannot take
    (host memory, other dtypes, non-contiguous views) before any call."""
    x = torch.zeros(1, 8, 16)
    with pytest.raises(ValueError, match="CUDA device"):
        csa.csa_compress(x, None, x, None, torch.zeros(4, 16), None, 4)
    with pytest.raises(ValueError, match="dtype"):
        csa._dt(torch.zeros(2, dtype=torch.int32))
    assert csa._dt(torch.zeros(2)) == csa.CSA_F32
    assert csa._dt(torch.zeros(2, dtype=torch.bfloat16)) == csa.CSA_BF16
    assert csa._ptr(None) is None
    with pytest.raises(ValueError, match="CUDA device"):
        csa._ptr(torch.zeros(4, 4).t())


def _noalloc(**kw):
    a = dict(q=FAKE, w=FAKE, k_i=FAKE, batch=1, n=64, nh=4, ci=64, m=4, k=8, dt=1, idx=FAKE)
    a.update(kw)
    return csa.lib().csa_index_topk_noalloc(a["q"], a["w"], a["k_i"], a["batch"], a["n"],
                                            a["nh"], a["ci"], a["m"], a["k"], a["dt"], a["idx"],
                                            None)


@pytest.mark.parametrize("kw,why", [
    (dict(k=0, n=1 << 40), "k must"),          # a bad argument wins over the size check
    (dict(ci=12, n=1 << 40), "multiple of 8"),
    (dict(dt=5, n=1 << 40), "dt must"),
    (dict(m=0), "m must"),
    (dict(n=-1), "must be >= 0"),
])
def test_noalloc_checks_arguments_before_its_size(kw, why):
    assert _noalloc(**kw) == csa.CSA_ERR_INVALID_ARG
    assert why in csa.lib().csa_last_error().decode()


@pytest.mark.parametrize("batch,n,m", [
    (1, 1 << 40, 1),          # batch * n * n/m overflows 64 bits
    (1 << 30, 1 << 20, 4),
    (1, 2050, 2),             # 2050 * 1025 > 2^21
])
def test_noalloc_refuses_sizes_beyond_its_scratch_without_overflow(batch, n, m):
    assert _noalloc(batch=batch, n=n, m=m) == csa.CSA_ERR_UNSUPPORTED
    assert "built-in scratch" in csa.lib().csa_last_error().decode()
