"""CPU oracle for the paged KV-cache decode step (fp64, plain C + numpy glue).

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only code that may import this package.
The library under ``paged_kv_cache_420_b200`` never imports it, and it shares
no code with that library; the seeded input generators in ``workloads`` are the
only module both sides use.

Functions follow the pages on vLLM's PagedAttention (block table, pos -> block
and offset, attention read through the table, copy-on-write); the C source
``pkv_oracle.c`` cites the passage for each.  Parity pins for every function
are in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pkv_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libpkv_oracle.so")
_lib: Optional[ctypes.CDLL] = None


def build(force: bool = False) -> str:
    """Compiles the C oracle with gcc (-O2 -fopenmp) into oracle/_build/."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        D = ctypes.c_double
        lib.oracle_kv_write.argtypes = [P, P, P, P, P, I, I, I, I, I]
        lib.oracle_copy_blocks.argtypes = [P, P, P, I, I, I, I, I]
        lib.oracle_paged_attention.argtypes = [P, P, P, P, I, P, I, I, I, I, I, I, D, P]
        lib.oracle_attention_partial.argtypes = [P, P, P, P, I, I, I, I, I, I, I, I, D, P, P, P]
        lib.oracle_lse_merge.argtypes = [P, P, P, I, I, P]
        lib.oracle_paged_prefill.argtypes = [P, P, P, P, I, P, P, I, I, I, I, I, I, D, P]
        lib.oracle_swap_out.argtypes = [P, P, P, I, I, I, I, I, P, P]
        lib.oracle_swap_in.argtypes = [P, P, P, I, I, I, I, I, P, P]
        lib.oracle_lru_victims.argtypes = [P, P, I, I, P, P]
        lib.oracle_bm_init.argtypes = [P, P, P, P, P, P, I]
        lib.oracle_bm_alloc.argtypes = [P, P, P, P, P, P, I, P, I, P, P, I, P]
        lib.oracle_bm_free.argtypes = [P, P, P, P, P, P, I, P, I, P]
        lib.oracle_bm_share.argtypes = [P, P, I, P, I, P]
        lib.oracle_bm_append_slots.argtypes = [P, P, P, P, P, P, I, P, I, P, P, I, I, P, P, P, P]
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_decode.restype = D
        lib.oracle_e4m3_encode_array.argtypes = [P, I, P]
        lib.oracle_kv_write_fp8.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I]
        lib.oracle_paged_attention_fp8.argtypes = [P, P, P, P, P, P, I, P, I, I, I, I, I, I, D, P]
        lib.oracle_fnv1a64.argtypes = [P, I]
        lib.oracle_fnv1a64.restype = ctypes.c_uint64
        lib.oracle_prefix_keys.argtypes = [P, I, I, P]
        lib.oracle_prefix_lookup.argtypes = [P, P, P, I, P, P, I, P, P, I, I, P, I, P]
        lib.oracle_prefix_insert.argtypes = [P, I, P, P, I, P, P, I, I, P, I, P]
        lib.oracle_num_threads.argtypes = []
        lib.oracle_set_num_threads.argtypes = [I]
        for f in (lib.oracle_kv_write, lib.oracle_copy_blocks, lib.oracle_paged_attention,
                  lib.oracle_attention_partial, lib.oracle_lse_merge, lib.oracle_num_threads,
                  lib.oracle_set_num_threads,
                  lib.oracle_paged_prefill, lib.oracle_swap_out, lib.oracle_swap_in, lib.oracle_lru_victims,
                  lib.oracle_bm_init, lib.oracle_bm_alloc, lib.oracle_bm_free, lib.oracle_bm_share,
                  lib.oracle_bm_append_slots, lib.oracle_e4m3_encode_array, lib.oracle_kv_write_fp8,
                  lib.oracle_paged_attention_fp8, lib.oracle_prefix_keys,
                  lib.oracle_prefix_lookup, lib.oracle_prefix_insert):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> int:
    """Threads of the oracle's later parallel loops (timing only); returns the
    previous count."""
    return int(_load().oracle_set_num_threads(int(n)))


# ---------------------------------------------------------------------------
# array glue
# ---------------------------------------------------------------------------

def bits(x) -> np.ndarray:
    """bf16 data (torch bf16 tensor, or uint16 bit patterns) -> contiguous uint16."""
    if hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        import torch
        return np.ascontiguousarray(x.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16))
    a = np.ascontiguousarray(x)
    if a.dtype != np.uint16:
        raise TypeError(f"expected bf16 bits (uint16), got {a.dtype}")
    return a


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc == 1:
        raise ValueError(f"oracle {what}: bad argument")
    if rc == 2:
        raise IndexError(f"oracle {what}: index out of range")
    if rc == 3:
        raise ValueError(f"oracle {what}: repeated block id")
    if rc:
        raise RuntimeError(f"oracle {what}: status {rc}")


# ---------------------------------------------------------------------------
# the three operations
# ---------------------------------------------------------------------------

def kv_write(k_cache, v_cache, k, v, slot_mapping):
    """Returns new (k_cache, v_cache) uint16 arrays [NB, Hkv, bs, d] after the
    slot-mapped write of k, v [T, Hkv, d]."""
    kc = bits(k_cache).copy()
    vc = bits(v_cache).copy()
    kb, vb = bits(k), bits(v)
    slots = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    NB, Hkv, bs, d = kc.shape
    T = slots.shape[0]
    assert kb.shape == (T, Hkv, d) and vb.shape == (T, Hkv, d)
    rc = _load().oracle_kv_write(_ptr(kc), _ptr(vc), _ptr(kb), _ptr(vb), _ptr(slots), T, NB, Hkv, bs, d)
    _check(rc, "kv_write")
    return kc, vc


def copy_blocks(k_cache, v_cache, pairs):
    """Returns new (k_cache, v_cache) after copying block src -> dst for every
    (src, dst) in pairs [P, 2] (simultaneous semantics)."""
    kc = bits(k_cache).copy()
    vc = bits(v_cache).copy()
    pr = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32).reshape(-1, 2))
    NB, Hkv, bs, d = kc.shape
    rc = _load().oracle_copy_blocks(_ptr(kc), _ptr(vc), _ptr(pr), pr.shape[0], NB, Hkv, bs, d)
    _check(rc, "copy_blocks")
    return kc, vc


def swap_out(k_cache, v_cache, block_ids):
    """Returns (host_k, host_v) uint16 arrays [n, Hkv, bs, d]: copies of the
    listed blocks of the two caches, in list order."""
    kc, vc = bits(k_cache), bits(v_cache)
    ids = np.ascontiguousarray(block_ids, dtype=np.int32).reshape(-1)
    NB, Hkv, bs, d = kc.shape
    hk = np.zeros((ids.shape[0], Hkv, bs, d), dtype=np.uint16)
    hv = np.zeros_like(hk)
    rc = _load().oracle_swap_out(_ptr(kc), _ptr(vc), _ptr(ids), ids.shape[0], NB, Hkv, bs, d, _ptr(hk), _ptr(hv))
    _check(rc, "swap_out")
    return hk, hv


def swap_in(k_cache, v_cache, host_k, host_v, block_ids):
    """Returns new (k_cache, v_cache) with block ids[i] replaced by host_k[i] /
    host_v[i]; ids must be distinct."""
    kc, vc = bits(k_cache).copy(), bits(v_cache).copy()
    hk, hv = bits(host_k), bits(host_v)
    ids = np.ascontiguousarray(block_ids, dtype=np.int32).reshape(-1)
    NB, Hkv, bs, d = kc.shape
    assert hk.shape == (ids.shape[0], Hkv, bs, d) and hv.shape == hk.shape
    rc = _load().oracle_swap_in(_ptr(hk), _ptr(hv), _ptr(ids), ids.shape[0], NB, Hkv, bs, d, _ptr(kc), _ptr(vc))
    _check(rc, "swap_in")
    return kc, vc


def lru_victims(last_use, evictable, k: int) -> np.ndarray:
    """The k evictable blocks least recently used (oldest last_use first, ties
    by lower block id)."""
    lu = np.ascontiguousarray(last_use, dtype=np.int64).reshape(-1)
    ev = np.ascontiguousarray(evictable, dtype=np.uint8).reshape(-1)
    assert ev.shape == lu.shape
    out = np.zeros(max(k, 1), dtype=np.int32)
    cnt = np.zeros(1, dtype=np.int32)
    rc = _load().oracle_lru_victims(_ptr(lu), _ptr(ev), lu.shape[0], int(k), _ptr(out), _ptr(cnt))
    _check(rc, "lru_victims")
    return out[:int(cnt[0])].copy()


# ---------------------------------------------------------------------------
# block manager (state: free stack, its top, reference counts)
# ---------------------------------------------------------------------------

BM_ERR_NOSPACE, BM_ERR_RANGE, BM_ERR_DOUBLEFREE, BM_ERR_TABLE = 1, 2, 4, 8


class BlockState:
    """free_stack[:top] are the free ids (the next allocation pops
    free_stack[top - 1]); refcount[b] counts the sequences mapping block b;
    block_hash[b] is the prefix key block b holds (0: none); lru_stamp[b] is
    the release clock of a cached block (refcount 0, key kept, evictable),
    -1 for every other block; clock is the next release stamp."""

    def __init__(self, free_stack, top, refcount, block_hash=None, lru_stamp=None, clock=0):
        self.free_stack = np.ascontiguousarray(free_stack, dtype=np.int32)
        self.top = int(top)
        self.refcount = np.ascontiguousarray(refcount, dtype=np.int32)
        n = self.refcount.shape[0]
        self.block_hash = (np.zeros(n, np.uint64) if block_hash is None
                           else np.ascontiguousarray(block_hash, dtype=np.uint64))
        self.lru_stamp = (np.full(n, -1, np.int64) if lru_stamp is None
                          else np.ascontiguousarray(lru_stamp, dtype=np.int64))
        self.clock = int(clock)

    def copy(self):
        return BlockState(self.free_stack.copy(), self.top, self.refcount.copy(), self.block_hash.copy(),
                          self.lru_stamp.copy(), self.clock)

    @property
    def num_blocks(self):
        return self.refcount.shape[0]

    def free_set(self):
        return set(self.free_stack[:self.top].tolist())

    def lru_order(self):
        """Cached blocks, least recently released first (the eviction order)."""
        c = np.flatnonzero(self.lru_stamp >= 0)
        return c[np.argsort(self.lru_stamp[c], kind="stable")].astype(np.int32)


def _bm_call(fn, st: BlockState, *args):
    top = np.array([st.top], dtype=np.int32)
    clock = np.array([st.clock], dtype=np.int64)
    rc = fn(_ptr(st.free_stack), _ptr(top), _ptr(st.refcount), _ptr(st.block_hash), _ptr(st.lru_stamp),
            _ptr(clock), st.num_blocks, *args)
    st.top = int(top[0])
    st.clock = int(clock[0])
    return rc


def bm_init(num_blocks: int) -> BlockState:
    st = BlockState(np.zeros(num_blocks, np.int32), 0, np.zeros(num_blocks, np.int32))
    _check(_bm_call(_load().oracle_bm_init, st), "bm_init")
    return st


def bm_alloc(st: BlockState, counts, capacity: int):
    """Returns (new state, offsets [n+1], ids [capacity], err)."""
    st = st.copy()
    c = np.ascontiguousarray(counts, dtype=np.int32).reshape(-1)
    offsets = np.zeros(c.shape[0] + 1, dtype=np.int32)
    ids = np.full(max(capacity, 1), -1, dtype=np.int32)
    err = np.zeros(1, dtype=np.uint32)
    _check(_bm_call(_load().oracle_bm_alloc, st, _ptr(c), c.shape[0], _ptr(offsets), _ptr(ids), int(capacity),
                    _ptr(err)), "bm_alloc")
    return st, offsets, ids[:capacity], int(err[0])


def bm_free(st: BlockState, ids):
    st = st.copy()
    a = np.ascontiguousarray(ids, dtype=np.int32).reshape(-1)
    err = np.zeros(1, dtype=np.uint32)
    _check(_bm_call(_load().oracle_bm_free, st, _ptr(a), a.shape[0], _ptr(err)), "bm_free")
    return st, int(err[0])


def bm_share(st: BlockState, ids):
    st = st.copy()
    a = np.ascontiguousarray(ids, dtype=np.int32).reshape(-1)
    err = np.zeros(1, dtype=np.uint32)
    _check(_load().oracle_bm_share(_ptr(st.refcount), _ptr(st.lru_stamp), st.num_blocks, _ptr(a), a.shape[0],
                                   _ptr(err)), "bm_share")
    return st, int(err[0])


def bm_append_slots(st: BlockState, block_tables, context_lens, num_new, block_size: int):
    """Returns (new state, tables, context_lens, slot_mapping int64, pairs [P, 2], err)."""
    st = st.copy()
    tables = np.ascontiguousarray(block_tables, dtype=np.int32).copy()
    ctx = np.ascontiguousarray(context_lens, dtype=np.int32).copy()
    nn = np.ascontiguousarray(num_new, dtype=np.int32).reshape(-1)
    B, mbs = tables.shape
    assert ctx.shape == (B,) and nn.shape == (B,)
    slots = np.full(max(int(np.clip(nn, 0, None).sum()), 1), -7, dtype=np.int64)
    pairs = np.zeros((max(B, 1), 2), dtype=np.int32)
    npairs = np.zeros(1, dtype=np.int32)
    err = np.zeros(1, dtype=np.uint32)
    _check(_bm_call(_load().oracle_bm_append_slots, st, _ptr(tables), mbs, _ptr(ctx), _ptr(nn), B, int(block_size),
                    _ptr(slots), _ptr(pairs), _ptr(npairs), _ptr(err)), "bm_append_slots")
    return st, tables, ctx, slots[:int(np.clip(nn, 0, None).sum())], pairs[:int(npairs[0])].copy(), int(err[0])


# ---------------------------------------------------------------------------
# FP8 (e4m3) KV cache
# ---------------------------------------------------------------------------

def e4m3_decode(codes) -> np.ndarray:
    c = np.asarray(codes, dtype=np.uint8)
    f = _load().oracle_e4m3_decode
    return np.array([f(int(v)) for v in c.reshape(-1)], dtype=np.float64).reshape(c.shape)


def e4m3_encode(x) -> np.ndarray:
    a = np.ascontiguousarray(x, dtype=np.float64)
    out = np.zeros(a.shape, dtype=np.uint8)
    _load().oracle_e4m3_encode_array(_ptr(a), a.size, _ptr(out))
    return out


def kv_write_fp8(k_cache8, v_cache8, k, v, slot_mapping, k_scale, v_scale):
    """Returns new uint8 (k_cache, v_cache) [NB, Hkv, bs, d] after the
    quantizing slot-mapped write of bf16 k, v [T, Hkv, d]."""
    kc = np.ascontiguousarray(k_cache8, dtype=np.uint8).copy()
    vc = np.ascontiguousarray(v_cache8, dtype=np.uint8).copy()
    kb, vb = bits(k), bits(v)
    slots = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    ks = np.ascontiguousarray(k_scale, dtype=np.float32)
    vs = np.ascontiguousarray(v_scale, dtype=np.float32)
    NB, Hkv, bs, d = kc.shape
    T = slots.shape[0]
    assert kb.shape == (T, Hkv, d) and ks.shape == (Hkv,) and vs.shape == (Hkv,)
    rc = _load().oracle_kv_write_fp8(_ptr(kc), _ptr(vc), _ptr(kb), _ptr(vb), _ptr(slots), _ptr(ks), _ptr(vs), T, NB,
                                     Hkv, bs, d)
    _check(rc, "kv_write_fp8")
    return kc, vc


def paged_attention_fp8(q, k_cache8, v_cache8, k_scale, v_scale, block_tables, context_lens,
                        scale: float) -> np.ndarray:
    """fp64 decode attention over an e4m3 pool: K = e4m3(code) * k_scale[h], V likewise."""
    qb = bits(q)
    kc = np.ascontiguousarray(k_cache8, dtype=np.uint8)
    vc = np.ascontiguousarray(v_cache8, dtype=np.uint8)
    ks = np.ascontiguousarray(k_scale, dtype=np.float32)
    vs = np.ascontiguousarray(v_scale, dtype=np.float32)
    tables = np.ascontiguousarray(block_tables, dtype=np.int32)
    ctx = np.ascontiguousarray(context_lens, dtype=np.int32)
    B, Hq, d = qb.shape
    NB, Hkv, bs, d2 = kc.shape
    assert d == d2
    out = np.zeros((B, Hq, d), dtype=np.float64)
    rc = _load().oracle_paged_attention_fp8(_ptr(qb), _ptr(kc), _ptr(vc), _ptr(ks), _ptr(vs), _ptr(tables),
                                            tables.shape[1], _ptr(ctx), B, Hq, Hkv, d, bs, NB,
                                            float(np.float64(np.float32(scale))), _ptr(out))
    _check(rc, "paged_attention_fp8")
    return out


# ---------------------------------------------------------------------------
# prefix caching
# ---------------------------------------------------------------------------

def fnv1a64(data: bytes) -> int:
    buf = np.frombuffer(bytes(data), dtype=np.uint8).copy() if len(data) else np.zeros(1, np.uint8)
    return int(_load().oracle_fnv1a64(_ptr(buf), len(data)))


def prefix_keys(tokens, block_size: int) -> np.ndarray:
    """Chained keys of the full blocks of one prompt."""
    t = np.ascontiguousarray(tokens, dtype=np.int32).reshape(-1)
    keys = np.zeros(max(t.shape[0] // block_size, 1), dtype=np.uint64)
    _load().oracle_prefix_keys(_ptr(t), t.shape[0], int(block_size), _ptr(keys))
    return keys[:t.shape[0] // block_size]


class PrefixCache:
    """cap (key, block) pairs; key 0 = empty."""

    def __init__(self, cap: int):
        self.keys = np.zeros(cap, np.uint64)
        self.vals = np.full(cap, -1, np.int32)

    def copy(self):
        c = PrefixCache(self.keys.shape[0])
        c.keys, c.vals = self.keys.copy(), self.vals.copy()
        return c


def prefix_lookup(st: BlockState, cache: PrefixCache, tokens, query_start, block_size: int, block_tables):
    """Returns (new state, tables, num_cached tokens per sequence)."""
    st = st.copy()
    t = np.ascontiguousarray(tokens, dtype=np.int32).reshape(-1)
    qs = np.ascontiguousarray(query_start, dtype=np.int32)
    tables = np.ascontiguousarray(block_tables, dtype=np.int32).copy()
    B, mbs = tables.shape
    nc = np.zeros(max(B, 1), np.int32)
    _check(_load().oracle_prefix_lookup(_ptr(st.refcount), _ptr(st.lru_stamp), _ptr(st.block_hash), st.num_blocks,
                                        _ptr(cache.keys),
                                        _ptr(cache.vals), cache.keys.shape[0], _ptr(t), _ptr(qs), B,
                                        int(block_size), _ptr(tables), mbs, _ptr(nc)), "prefix_lookup")
    return st, tables, nc[:B]


def prefix_insert(st: BlockState, cache: PrefixCache, tokens, query_start, block_size: int, block_tables):
    """Returns (new state, new cache, err)."""
    st = st.copy()
    cache = cache.copy()
    t = np.ascontiguousarray(tokens, dtype=np.int32).reshape(-1)
    qs = np.ascontiguousarray(query_start, dtype=np.int32)
    tables = np.ascontiguousarray(block_tables, dtype=np.int32)
    B, mbs = tables.shape
    err = np.zeros(1, np.uint32)
    _check(_load().oracle_prefix_insert(_ptr(st.block_hash), st.num_blocks, _ptr(cache.keys),
                                        _ptr(cache.vals), cache.keys.shape[0], _ptr(t), _ptr(qs), B,
                                        int(block_size), _ptr(tables), mbs, _ptr(err)), "prefix_insert")
    return st, cache, int(err[0])


def paged_attention(q, k_cache, v_cache, block_tables, context_lens, scale: float) -> np.ndarray:
    """fp64 decode attention out[B, Hq, d] read through the block tables."""
    qb = bits(q)
    kc, vc = bits(k_cache), bits(v_cache)
    tables = np.ascontiguousarray(block_tables, dtype=np.int32)
    ctx = np.ascontiguousarray(context_lens, dtype=np.int32)
    B, Hq, d = qb.shape
    NB, Hkv, bs, d2 = kc.shape
    assert d == d2 and tables.shape[0] == B and ctx.shape[0] == B
    out = np.zeros((B, Hq, d), dtype=np.float64)
    rc = _load().oracle_paged_attention(_ptr(qb), _ptr(kc), _ptr(vc), _ptr(tables), tables.shape[1],
                                        _ptr(ctx), B, Hq, Hkv, d, bs, NB, float(np.float64(np.float32(scale))),
                                        _ptr(out))
    _check(rc, "paged_attention")
    return out


def paged_prefill(q, k_cache, v_cache, block_tables, context_lens, query_start, scale: float) -> np.ndarray:
    """fp64 chunked-prefill attention out[T, Hq, d]: query row i of sequence
    s's chunk is at position ctx_s - q_len_s + i and sees positions [0, pos]."""
    qb = bits(q)
    kc, vc = bits(k_cache), bits(v_cache)
    tables = np.ascontiguousarray(block_tables, dtype=np.int32)
    ctx = np.ascontiguousarray(context_lens, dtype=np.int32)
    qsl = np.ascontiguousarray(query_start, dtype=np.int32)
    T, Hq, d = qb.shape
    NB, Hkv, bs, d2 = kc.shape
    B = ctx.shape[0]
    assert d == d2 and qsl.shape == (B + 1,) and int(qsl[-1]) == T
    out = np.zeros((T, Hq, d), dtype=np.float64)
    rc = _load().oracle_paged_prefill(_ptr(qb), _ptr(kc), _ptr(vc), _ptr(tables), tables.shape[1], _ptr(ctx),
                                      _ptr(qsl), B, Hq, Hkv, d, bs, NB, float(np.float64(np.float32(scale))),
                                      _ptr(out))
    _check(rc, "paged_prefill")
    return out


def attention_partial(q_row, k_cache, v_cache, table_row, num_q_heads: int, hq: int,
                      t_begin: int, t_end: int, scale: float):
    """(m, l, acc[d]) of one (sequence, query head) over tokens [t_begin, t_end)."""
    qb = bits(q_row).reshape(-1)
    kc, vc = bits(k_cache), bits(v_cache)
    tr = np.ascontiguousarray(table_row, dtype=np.int32).reshape(-1)
    NB, Hkv, bs, d = kc.shape
    m = np.zeros(1)
    l = np.zeros(1)
    acc = np.zeros(d)
    rc = _load().oracle_attention_partial(_ptr(qb), _ptr(kc), _ptr(vc), _ptr(tr), NB, num_q_heads, Hkv,
                                          d, bs, hq, t_begin, t_end,
                                          float(np.float64(np.float32(scale))), _ptr(m), _ptr(l), _ptr(acc))
    _check(rc, "attention_partial")
    return float(m[0]), float(l[0]), acc


def lse_merge(m, l, acc) -> np.ndarray:
    """Merges P partial results: m [P], l [P], acc [P, d] -> out [d]."""
    m = np.ascontiguousarray(m, dtype=np.float64)
    l = np.ascontiguousarray(l, dtype=np.float64)
    acc = np.ascontiguousarray(acc, dtype=np.float64)
    P, d = acc.shape
    out = np.zeros(d)
    rc = _load().oracle_lse_merge(_ptr(m), _ptr(l), _ptr(acc), P, d, _ptr(out))
    _check(rc, "lse_merge")
    return out


def decode_step(w, attention: bool = True):
    """Applies one whole step of a ``workloads.Workload`` on the CPU:
    copy-on-write pairs, then the slot-mapped write, then attention.
    Returns (k_cache_bits, v_cache_bits, out_f64 or None)."""
    kc, vc = bits(w.k_cache), bits(w.v_cache)
    if len(w.copy_pairs):
        kc, vc = copy_blocks(kc, vc, w.copy_pairs)
    kc, vc = kv_write(kc, vc, w.k_new, w.v_new, w.slot_mapping)
    out = paged_attention(w.q, kc, vc, w.block_tables, w.context_lens, w.scale) if attention else None
    return kc, vc, out
