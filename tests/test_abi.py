"""The C ABI library: it loads, exports every declared symbol, and its host
validation rejects bad requests before any CUDA work (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import paged_kv_cache_420_b200 as pkv
from paged_kv_cache_420_b200 import _Pool

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pkv.h")

EINVAL, ERANGE, EALIAS, EUNSUP = 1, 2, 3, 6
FAKE = ctypes.c_void_p(0x10000)  # aligned, never dereferenced by the host checks below
FAKE_ODD = ctypes.c_void_p(0x10008)  # 8-byte but not 16-byte aligned


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*[A-Za-z_][\w \*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)))


def test_library_loads_and_exports_every_declared_symbol():
    lib = pkv.load_library()
    names = declared_functions()
    assert set(names) == set(pkv.EXPORTED), names
    nm = subprocess.run(["nm", "-D", "--defined-only", pkv.LIB_PATH], capture_output=True, text=True).stdout
    for n in names:
        assert hasattr(lib, n)
        assert re.search(rf"\bT {n}$", nm, flags=re.M), n


def test_status_strings_and_version():
    assert pkv.version() == 10100
    for code in range(7):
        assert pkv.status_string(code)
    assert pkv.status_string(99) == "unknown status"


def _pool(nb=8, hkv=2, bs=16, d=128):
    return _Pool(nb, hkv, bs, d)


def test_write_validation():
    lib = pkv.load_library()
    ok = _pool()
    assert lib.pkv_write(FAKE, FAKE, FAKE, 0, FAKE, FAKE, ok, None) == 0  # no tokens: no-op
    assert lib.pkv_write(FAKE, FAKE, FAKE, -1, FAKE, FAKE, ok, None) == EINVAL
    assert lib.pkv_write(None, FAKE, FAKE, 4, FAKE, FAKE, ok, None) == EINVAL
    assert lib.pkv_write(FAKE_ODD, FAKE, FAKE, 4, FAKE, FAKE, ok, None) == EINVAL
    assert lib.pkv_write(FAKE, FAKE, FAKE, 4, FAKE, FAKE, _pool(d=96), None) == EUNSUP
    assert lib.pkv_write(FAKE, FAKE, FAKE, 4, FAKE, FAKE, _pool(bs=24), None) == EUNSUP
    assert lib.pkv_write(FAKE, FAKE, FAKE, 4, FAKE, FAKE, _pool(nb=0), None) == EINVAL


def _pairs(p):
    a = np.ascontiguousarray(np.asarray(p, np.int32).reshape(-1, 2))
    return a, a.ctypes.data_as(ctypes.c_void_p)


def test_copy_pairs_validation():
    lib = pkv.load_library()
    pool = _pool(nb=8)
    for pairs, code in [([[0, 8]], ERANGE), ([[-1, 2]], ERANGE), ([[0, 1], [2, 1]], EALIAS),
                        ([[0, 1], [1, 2]], EALIAS), ([[3, 3]], EALIAS)]:
        arr, ptr = _pairs(pairs)
        assert lib.pkv_copy_blocks(ptr, arr.shape[0], FAKE, FAKE, pool, None) == code, pairs
    arr, ptr = _pairs([[0, 1]])
    assert lib.pkv_copy_blocks(ptr, 0, FAKE, FAKE, pool, None) == 0
    assert lib.pkv_copy_blocks(ptr, 1, FAKE_ODD, FAKE, pool, None) == EINVAL
    assert lib.pkv_copy_blocks(None, 1, FAKE, FAKE, pool, None) == EINVAL


def _decode(lib, **kw):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, tables=FAKE, mbs=4, ctx=FAKE, B=2, Hq=4, scale=0.1, Hkv=2, out=FAKE,
             pool=_pool(hkv=2), max_ctx=64, pt=0, ws=FAKE, ws_bytes=1 << 30)
    a.update(kw)
    return lib.paged_attn_decode(a["q"], a["kc"], a["vc"], a["tables"], a["mbs"], a["ctx"], a["B"], a["Hq"],
                                 a["scale"], a["Hkv"], a["out"], a["pool"], a["max_ctx"], a["pt"], a["ws"],
                                 a["ws_bytes"], None)


def test_decode_validation():
    lib = pkv.load_library()
    assert _decode(lib, B=0) == 0
    assert _decode(lib, Hq=5) == EINVAL  # not a multiple of Hkv
    assert _decode(lib, Hkv=4, Hq=8) == EINVAL  # disagrees with the pool
    assert _decode(lib, Hq=2 * 17, pool=_pool(hkv=2)) == EUNSUP  # g = 17
    assert _decode(lib, pt=24) == EINVAL
    assert _decode(lib, pt=-16) == EINVAL
    assert _decode(lib, q=FAKE_ODD) == EINVAL
    assert _decode(lib, ws=ctypes.c_void_p(0x10010)) == EINVAL  # workspace not 256-B aligned
    assert _decode(lib, ws_bytes=16) == EINVAL
    assert _decode(lib, mbs=0) == EINVAL
    assert _decode(lib, max_ctx=-1) == EINVAL
    assert _decode(lib, out=None) == EINVAL
    assert _decode(lib, pool=_pool(hkv=2, d=256)) == EUNSUP


def _prefill(lib, **kw):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, tables=FAKE, mbs=4, ctx=FAKE, qs=FAKE, B=2, T=32, Hq=4, scale=0.1, Hkv=2,
             out=FAKE, pool=_pool(hkv=2), max_q=16, max_ctx=64, ws=FAKE, ws_bytes=1 << 30)
    a.update(kw)
    f = lib.paged_attn_prefill
    P, I32 = ctypes.c_void_p, ctypes.c_int32
    f.argtypes = [P, P, P, P, I32, P, P, I32, I32, I32, ctypes.c_float, I32, P, _Pool, I32, I32, P,
                  ctypes.c_size_t, P]
    f.restype = ctypes.c_int
    return f(a["q"], a["kc"], a["vc"], a["tables"], a["mbs"], a["ctx"], a["qs"], a["B"], a["T"], a["Hq"],
             a["scale"], a["Hkv"], a["out"], a["pool"], a["max_q"], a["max_ctx"], a["ws"], a["ws_bytes"], None)


def test_prefill_validation():
    lib = pkv.load_library()
    assert _prefill(lib, B=0) == 0
    assert _prefill(lib, T=0) == 0  # no query rows: nothing to launch
    assert _prefill(lib, T=-1) == EINVAL
    assert _prefill(lib, Hq=5) == EINVAL
    assert _prefill(lib, Hq=2 * 17) == EUNSUP
    assert _prefill(lib, scale=0.0) == EINVAL  # the kernel keeps its running max on raw scores
    assert _prefill(lib, scale=-0.1) == EINVAL
    assert _prefill(lib, scale=float("inf")) == EINVAL
    assert _prefill(lib, scale=float("nan")) == EINVAL
    assert _prefill(lib, q=FAKE_ODD) == EINVAL
    assert _prefill(lib, qs=None) == EINVAL
    assert _prefill(lib, ws=ctypes.c_void_p(0x10010)) == EINVAL
    assert _prefill(lib, ws_bytes=16) == EINVAL
    assert _prefill(lib, mbs=0) == EINVAL
    assert _prefill(lib, pool=_pool(hkv=2, bs=8)) == EUNSUP


def test_pool_element_type_validation():
    lib = pkv.load_library()
    ok = _pool()
    fp8 = _Pool(8, 2, 16, 128, 1)
    bad = _Pool(8, 2, 16, 128, 2)
    assert _decode(lib, pool=bad) == EINVAL          # unknown element type
    assert _decode(lib, pool=fp8) == EINVAL          # bf16 decode on an e4m3 pool
    assert lib.pkv_write(FAKE, FAKE, FAKE, 4, FAKE, FAKE, fp8, None) == EINVAL
    f = lib.pkv_write_fp8
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, _Pool, ctypes.c_void_p]
    assert f(FAKE, FAKE, FAKE, 4, FAKE, FAKE, FAKE, FAKE, ok, None) == EINVAL   # e4m3 write on a bf16 pool
    assert _prefill(lib, pool=_Pool(8, 2, 16, 128, 1)) == EINVAL


def test_workspace_size():
    f = pkv.decode_workspace_bytes
    # one partition per sequence: count + entries only
    assert f(4, 4, 4, 64, 64, 512) == 256 + 256
    # 3 partitions: partial (m, l) and accumulators appear
    B, Hq, D, maxP = 8, 64, 128, 3
    expect = 256 + (B * maxP * 8 + 255) // 256 * 256 + (B * Hq * maxP * 8 + 255) // 256 * 256 \
        + (B * Hq * maxP * D * 4 + 255) // 256 * 256
    assert f(B, Hq, 8, D, 1536, 512) == expect
    assert f(B, Hq, 8, D, 1537, 512) > expect
    with pytest.raises(ValueError):
        f(2, 5, 2, 128, 64, 0)
