"""Python binding of libpkv.so: paged KV-cache write, copy-on-write block copy
and paged decode attention on B200 (sm_100a).

Argument marshalling only.  Every step of the path runs in the library's CUDA
kernels; torch supplies device memory and streams.  There is no CPU fallback:
if libpkv.so is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpkv.so")

PKV_OK = 0
STATUS_NAMES = {0: "PKV_OK", 1: "PKV_EINVAL", 2: "PKV_ERANGE", 3: "PKV_EALIAS", 4: "PKV_ECUDA",
                5: "PKV_EDEVICE", 6: "PKV_EUNSUPPORTED"}
DEVERR_SLOT, DEVERR_BLOCK, DEVERR_CONTEXT, DEVERR_TIMEOUT, DEVERR_LAYOUT = 0x1, 0x2, 0x4, 0x8, 0x10

# Every symbol include/pkv.h declares.
EXPORTED = ("pkv_write", "pkv_copy_blocks", "pkv_decode_workspace_bytes", "paged_attn_decode",
            "paged_attn_decode_static_ws", "pkv_prefill_workspace_bytes", "paged_attn_prefill",
            "pkv_get_device_error", "pkv_selftest_bounded_wait", "pkv_status_string", "pkv_version",
            "pkv_swap_out", "pkv_swap_in", "pkv_lru_victims", "pkv_bm_state_bytes", "pkv_bm_init", "pkv_bm_alloc",
            "pkv_bm_free", "pkv_bm_share", "pkv_bm_append_slots", "pkv_copy_blocks_dev", "pkv_write_fp8",
            "paged_attn_decode_fp8", "pkv_prefix_cache_bytes", "pkv_prefix_cache_init", "pkv_prefix_lookup",
            "pkv_prefix_insert")
STATIC_WS_BYTES = 32 << 20  # PKV_STATIC_WS_BYTES


class PkvError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)} ({status_string(status)})")


KV_BF16, KV_E4M3 = 0, 1  # pkv_pool.kv_dtype


class _Pool(ctypes.Structure):
    _fields_ = [("num_blocks", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("kv_dtype", ctypes.c_int32)]


_lib: Optional[ctypes.CDLL] = None


def load_library() -> ctypes.CDLL:
    """Loads libpkv.so from this package directory (raises if it is absent)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m paged_kv_cache_420_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        P, I32, I64, F, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
        lib.pkv_write.argtypes = [P, P, P, I32, P, P, _Pool, P]
        lib.pkv_copy_blocks.argtypes = [P, I32, P, P, _Pool, P]
        lib.pkv_decode_workspace_bytes.argtypes = [I32, I32, I32, I32, I32, I32]
        lib.pkv_decode_workspace_bytes.restype = SZ
        lib.paged_attn_decode.argtypes = [P, P, P, P, I32, P, I32, I32, F, I32, P, _Pool, I32, I32, P, SZ, P]
        lib.pkv_get_device_error.argtypes = [ctypes.POINTER(I32), P]
        lib.pkv_swap_out.argtypes = [P, P, _Pool, P, I32, P, P, P]
        lib.pkv_swap_in.argtypes = [P, P, P, I32, P, P, _Pool, P]
        lib.pkv_lru_victims.argtypes = [P, P, I32, I32, P, P]
        lib.pkv_bm_state_bytes.argtypes = [I32]
        lib.pkv_bm_state_bytes.restype = SZ
        lib.pkv_bm_init.argtypes = [P, I32, P]
        lib.pkv_bm_alloc.argtypes = [P, I32, P, I32, P, P, I32, P]
        lib.pkv_bm_free.argtypes = [P, I32, P, I32, P]
        lib.pkv_bm_share.argtypes = [P, I32, P, I32, P]
        lib.pkv_bm_append_slots.argtypes = [P, I32, P, I32, P, P, I32, I32, P, I64, P, P, P]
        lib.pkv_copy_blocks_dev.argtypes = [P, P, I32, P, P, _Pool, P]
        lib.pkv_write_fp8.argtypes = [P, P, P, I32, P, P, P, P, _Pool, P]
        lib.pkv_prefix_cache_bytes.argtypes = [I32]
        lib.pkv_prefix_cache_bytes.restype = SZ
        lib.pkv_prefix_cache_init.argtypes = [P, I32, P]
        lib.pkv_prefix_lookup.argtypes = [P, I32, P, I32, P, P, I32, I32, P, I32, P, P]
        lib.pkv_prefix_insert.argtypes = [P, I32, P, I32, P, P, I32, I32, P, I32, P]
        lib.paged_attn_decode_fp8.argtypes = [P, P, P, P, P, P, I32, P, I32, I32, F, I32, P, _Pool, I32, I32, P, SZ,
                                              P]
        lib.pkv_status_string.argtypes = [ctypes.c_int]
        lib.pkv_status_string.restype = ctypes.c_char_p
        lib.pkv_version.restype = I32
        for f in ("pkv_write", "pkv_copy_blocks", "paged_attn_decode", "pkv_get_device_error", "pkv_swap_out",
                  "pkv_swap_in", "pkv_lru_victims", "pkv_bm_init", "pkv_bm_alloc", "pkv_bm_free", "pkv_bm_share",
                  "pkv_bm_append_slots", "pkv_copy_blocks_dev", "pkv_write_fp8", "paged_attn_decode_fp8",
                  "pkv_prefix_cache_init", "pkv_prefix_lookup", "pkv_prefix_insert"):
            getattr(lib, f).restype = ctypes.c_int
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load_library().pkv_status_string(int(status)).decode()


def version() -> int:
    return int(load_library().pkv_version())


def _check(status: int, what: str):
    if status != PKV_OK:
        raise PkvError(status, what)


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _pool(k_cache: torch.Tensor) -> _Pool:
    if k_cache.dim() != 4:
        raise ValueError("cache must be [num_blocks, num_kv_heads, block_size, head_dim]")
    nb, hkv, bs, d = k_cache.shape
    return _Pool(nb, hkv, bs, d, KV_E4M3 if k_cache.dtype == torch.uint8 else KV_BF16)


def _need_cache(t: torch.Tensor, name: str):
    """A pool tensor: bf16, or uint8 e4m3 codes."""
    _need(t, name, torch.uint8 if t.dtype == torch.uint8 else torch.bfloat16)


def _need(t: torch.Tensor, name: str, dtype, cuda=True):
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if cuda and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")


def pkv_write(k: torch.Tensor, v: torch.Tensor, slot_mapping: torch.Tensor, k_cache: torch.Tensor,
              v_cache: torch.Tensor, stream=None) -> None:
    """cache[slot // bs][h][slot % bs] = k[t][h] (and v) for every token t with slot >= 0."""
    for t, n in ((k, "k"), (v, "v"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _need(t, n, torch.bfloat16)
    _need(slot_mapping, "slot_mapping", torch.int64)
    if v_cache.shape != k_cache.shape or k.shape != v.shape:
        raise ValueError("k/v and k_cache/v_cache shapes must match")
    T = slot_mapping.shape[0]
    if k.shape != (T, k_cache.shape[1], k_cache.shape[3]):
        raise ValueError(f"k must be [num_tokens, num_kv_heads, head_dim], got {tuple(k.shape)}")
    st = load_library().pkv_write(_ptr(k), _ptr(v), _ptr(slot_mapping), T, _ptr(k_cache), _ptr(v_cache),
                                  _pool(k_cache), _stream(stream))
    _check(st, "pkv_write")


def pkv_copy_blocks(src_dst_pairs, k_cache: torch.Tensor, v_cache: torch.Tensor, stream=None) -> None:
    """Copies block src -> dst of both caches for every (src, dst) host pair (bf16 or e4m3 pools)."""
    for t, n in ((k_cache, "k_cache"), (v_cache, "v_cache")):
        _need_cache(t, n)
    if v_cache.dtype != k_cache.dtype:
        raise TypeError("k_cache and v_cache must have the same element type")
    pairs = np.ascontiguousarray(np.asarray(src_dst_pairs, dtype=np.int32).reshape(-1, 2))
    st = load_library().pkv_copy_blocks(pairs.ctypes.data_as(ctypes.c_void_p), pairs.shape[0], _ptr(k_cache),
                                        _ptr(v_cache), _pool(k_cache), _stream(stream))
    _check(st, "pkv_copy_blocks")


def _host_blocks(t: torch.Tensor, name: str, k_cache: torch.Tensor, n: int):
    if t.dtype != k_cache.dtype or not t.is_contiguous() or t.is_cuda:
        raise ValueError(f"{name} must be a contiguous host tensor of the pool's element type")
    if not t.is_pinned():
        raise ValueError(f"{name} must be pinned host memory")
    if t.numel() < n * k_cache[0].numel():
        raise ValueError(f"{name} holds fewer than {n} blocks")


def _block_ids(block_ids) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(block_ids, dtype=np.int32).reshape(-1))


def pkv_swap_out(k_cache: torch.Tensor, v_cache: torch.Tensor, block_ids, host_k: torch.Tensor,
                 host_v: torch.Tensor, stream=None) -> None:
    """host_k[i] / host_v[i] := block block_ids[i] of k_cache / v_cache (pinned
    host tensors of at least len(block_ids) blocks); asynchronous on the stream."""
    for t, n in ((k_cache, "k_cache"), (v_cache, "v_cache")):
        _need_cache(t, n)
    ids = _block_ids(block_ids)
    _host_blocks(host_k, "host_k", k_cache, ids.shape[0])
    _host_blocks(host_v, "host_v", k_cache, ids.shape[0])
    st = load_library().pkv_swap_out(_ptr(k_cache), _ptr(v_cache), _pool(k_cache), ids.ctypes.data_as(ctypes.c_void_p),
                                     ids.shape[0], _ptr(host_k), _ptr(host_v), _stream(stream))
    _check(st, "pkv_swap_out")


def pkv_swap_in(host_k: torch.Tensor, host_v: torch.Tensor, block_ids, k_cache: torch.Tensor,
                v_cache: torch.Tensor, stream=None) -> None:
    """Block block_ids[i] of k_cache / v_cache := host_k[i] / host_v[i] (ids distinct)."""
    for t, n in ((k_cache, "k_cache"), (v_cache, "v_cache")):
        _need_cache(t, n)
    ids = _block_ids(block_ids)
    _host_blocks(host_k, "host_k", k_cache, ids.shape[0])
    _host_blocks(host_v, "host_v", k_cache, ids.shape[0])
    st = load_library().pkv_swap_in(_ptr(host_k), _ptr(host_v), ids.ctypes.data_as(ctypes.c_void_p), ids.shape[0],
                                    _ptr(k_cache), _ptr(v_cache), _pool(k_cache), _stream(stream))
    _check(st, "pkv_swap_in")


def lru_victims(last_use, evictable, k: int) -> np.ndarray:
    """The k evictable blocks with the oldest last use (ties: lower id), oldest first."""
    lu = np.ascontiguousarray(np.asarray(last_use, dtype=np.int64).reshape(-1))
    ev = np.ascontiguousarray(np.asarray(evictable, dtype=np.uint8).reshape(-1))
    if ev.shape != lu.shape:
        raise ValueError("last_use and evictable must have one entry per block")
    out = np.zeros(max(int(k), 1), dtype=np.int32)
    cnt = ctypes.c_int32(0)
    st = load_library().pkv_lru_victims(lu.ctypes.data_as(ctypes.c_void_p), ev.ctypes.data_as(ctypes.c_void_p),
                                        lu.shape[0], int(k), out.ctypes.data_as(ctypes.c_void_p), ctypes.byref(cnt))
    _check(st, "pkv_lru_victims")
    return out[:cnt.value].copy()


BM_ERR_NOSPACE, BM_ERR_RANGE, BM_ERR_DOUBLEFREE, BM_ERR_TABLE = 1, 2, 4, 8


def bm_state_bytes(num_blocks: int) -> int:
    n = load_library().pkv_bm_state_bytes(int(num_blocks))
    if n == 0:
        raise ValueError("num_blocks must be positive")
    return int(n)


class BlockManager:
    """The block manager's state on the device (free list, reference counts,
    prefix keys, the eviction order of cached blocks) and its per-step calls;
    every array argument is a CUDA int32 tensor."""

    def __init__(self, num_blocks: int, device="cuda", stream=None):
        self.num_blocks = nb = int(num_blocks)
        self.state = torch.empty(bm_state_bytes(num_blocks), dtype=torch.uint8, device=device)
        a = (nb * 4 + 255) // 256 * 256
        h = (nb * 8 + 255) // 256 * 256
        self.header = self.state[:20].view(torch.int32)  # top, error word, cached, ring head, ring tail
        self.free_stack = self.state[256:256 + 4 * nb].view(torch.int32)
        self.refcount = self.state[256 + a:256 + a + 4 * nb].view(torch.int32)
        self.block_hash = self.state[256 + 5 * a:256 + 5 * a + 8 * nb].view(torch.int64)
        self.lru_pos = self.state[256 + 5 * a + h:256 + 5 * a + h + 4 * nb].view(torch.int32)
        self.ring = self.state[256 + 6 * a + h:256 + 6 * a + h + 8 * nb].view(torch.int32)
        _check(load_library().pkv_bm_init(_ptr(self.state), nb, _stream(stream)), "pkv_bm_init")

    def top(self) -> int:
        return int(self.header[0].item())

    def cached(self) -> int:
        """Blocks with no reference that still hold a prefix key."""
        return int(self.header[2].item())

    def lru_order(self):
        """Cached blocks in eviction order (least recently released first), read
        back from the device ring: the entries of head .. tail whose block still
        records that position."""
        import numpy as np
        hdr = self.header.cpu().numpy().view(np.uint32)
        head, tail = int(hdr[3]), int(hdr[4])
        ring = self.ring.cpu().numpy()
        pos_of = self.lru_pos.cpu().numpy().view(np.uint32)
        pos = np.arange(head, tail, dtype=np.int64)
        blocks = ring[pos % (2 * self.num_blocks)]
        live = (blocks >= 0) & (blocks < self.num_blocks)
        live[live] = pos_of[blocks[live]] == pos[live]
        return blocks[live].astype(np.int32)

    def error(self) -> int:
        return int(self.header[1].item()) & 0xFFFFFFFF

    def clear_error(self):
        self.header[1:2].zero_()

    def alloc(self, counts: torch.Tensor, capacity: int, stream=None):
        """Returns (offsets [n+1], ids [capacity]) device tensors."""
        _need(counts, "counts", torch.int32)
        offsets = torch.empty(counts.numel() + 1, dtype=torch.int32, device=self.state.device)
        ids = torch.full((max(int(capacity), 1),), -1, dtype=torch.int32, device=self.state.device)
        _check(load_library().pkv_bm_alloc(_ptr(self.state), self.num_blocks, _ptr(counts), counts.numel(),
                                           _ptr(offsets), _ptr(ids), int(capacity), _stream(stream)), "pkv_bm_alloc")
        return offsets, ids[:int(capacity)]

    def free(self, block_ids: torch.Tensor, stream=None):
        _need(block_ids, "block_ids", torch.int32)
        _check(load_library().pkv_bm_free(_ptr(self.state), self.num_blocks, _ptr(block_ids), block_ids.numel(),
                                          _stream(stream)), "pkv_bm_free")

    def share(self, block_ids: torch.Tensor, stream=None):
        _need(block_ids, "block_ids", torch.int32)
        _check(load_library().pkv_bm_share(_ptr(self.state), self.num_blocks, _ptr(block_ids), block_ids.numel(),
                                           _stream(stream)), "pkv_bm_share")

    def append_slots(self, block_tables: torch.Tensor, context_lens: torch.Tensor, num_new: torch.Tensor,
                     block_size: int, num_tokens: int, stream=None, out=None):
        """Updates block_tables and context_lens in place; returns
        (slot_mapping int64 [num_tokens], cow_pairs [B, 2], num_cow_pairs [1]),
        written into `out` when given (the same three tensors, preallocated)."""
        for t, n in ((block_tables, "block_tables"), (context_lens, "context_lens"), (num_new, "num_new")):
            _need(t, n, torch.int32)
        B, mbs = block_tables.shape
        if context_lens.shape != (B,) or num_new.shape != (B,):
            raise ValueError("context_lens and num_new must be [num_seqs]")
        dev = self.state.device
        if out is None:
            slots = torch.empty(max(int(num_tokens), 1), dtype=torch.int64, device=dev)
            pairs = torch.empty((max(B, 1), 2), dtype=torch.int32, device=dev)
            npairs = torch.empty(1, dtype=torch.int32, device=dev)
        else:
            slots, pairs, npairs = out
            _need(slots, "slot_mapping", torch.int64)
            _need(pairs, "cow_pairs", torch.int32)
            _need(npairs, "num_cow_pairs", torch.int32)
            if slots.numel() < num_tokens or pairs.shape[0] < B:
                raise ValueError("out tensors too small")
        _check(load_library().pkv_bm_append_slots(_ptr(self.state), self.num_blocks, _ptr(block_tables), mbs,
                                                  _ptr(context_lens), _ptr(num_new), B, int(block_size), _ptr(slots),
                                                  int(num_tokens), _ptr(pairs), _ptr(npairs), _stream(stream)),
               "pkv_bm_append_slots")
        return slots[:int(num_tokens)], pairs, npairs


class PrefixCache:
    """Device table of (prefix key, block) pairs for prefix caching."""

    def __init__(self, capacity: int, device="cuda", stream=None):
        n = load_library().pkv_prefix_cache_bytes(int(capacity))
        if n == 0:
            raise ValueError("capacity must be a power of two >= 2")
        self.capacity = int(capacity)
        self.buf = torch.empty(n, dtype=torch.uint8, device=device)
        _check(load_library().pkv_prefix_cache_init(_ptr(self.buf), self.capacity, _stream(stream)),
               "pkv_prefix_cache_init")

    def lookup(self, bm: "BlockManager", tokens: torch.Tensor, query_start: torch.Tensor, block_size: int,
               block_tables: torch.Tensor, stream=None) -> torch.Tensor:
        """Maps cached leading blocks into block_tables; returns num_cached [B] (tokens)."""
        for t, n in ((tokens, "tokens"), (query_start, "query_start"), (block_tables, "block_tables")):
            _need(t, n, torch.int32)
        B, mbs = block_tables.shape
        num_cached = torch.empty(max(B, 1), dtype=torch.int32, device=self.buf.device)
        _check(load_library().pkv_prefix_lookup(_ptr(bm.state), bm.num_blocks, _ptr(self.buf), self.capacity,
                                                _ptr(tokens), _ptr(query_start), B, int(block_size),
                                                _ptr(block_tables), mbs, _ptr(num_cached), _stream(stream)),
               "pkv_prefix_lookup")
        return num_cached[:B]

    def insert(self, bm: "BlockManager", tokens: torch.Tensor, query_start: torch.Tensor, block_size: int,
               block_tables: torch.Tensor, stream=None) -> None:
        for t, n in ((tokens, "tokens"), (query_start, "query_start"), (block_tables, "block_tables")):
            _need(t, n, torch.int32)
        B, mbs = block_tables.shape
        _check(load_library().pkv_prefix_insert(_ptr(bm.state), bm.num_blocks, _ptr(self.buf), self.capacity,
                                                _ptr(tokens), _ptr(query_start), B, int(block_size),
                                                _ptr(block_tables), mbs, _stream(stream)), "pkv_prefix_insert")


def copy_blocks_dev(cow_pairs: torch.Tensor, num_pairs: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                    stream=None) -> None:
    """Copies block src -> dst for the first num_pairs[0] rows of the device
    pair list (as BlockManager.append_slots returns it)."""
    _need(cow_pairs, "cow_pairs", torch.int32)
    _need(num_pairs, "num_pairs", torch.int32)
    for t, n in ((k_cache, "k_cache"), (v_cache, "v_cache")):
        _need_cache(t, n)
    _check(load_library().pkv_copy_blocks_dev(_ptr(cow_pairs), _ptr(num_pairs), cow_pairs.shape[0], _ptr(k_cache),
                                              _ptr(v_cache), _pool(k_cache), _stream(stream)), "pkv_copy_blocks_dev")


def _need_scales(k_scale, v_scale, hkv):
    for t, n in ((k_scale, "k_scale"), (v_scale, "v_scale")):
        _need(t, n, torch.float32)
        if t.numel() != hkv:
            raise ValueError(f"{n} must hold one scale per kv head ({hkv})")


def pkv_write_fp8(k: torch.Tensor, v: torch.Tensor, slot_mapping: torch.Tensor, k_scale: torch.Tensor,
                  v_scale: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, stream=None) -> None:
    """cache[slot // bs][h][slot % bs] = e4m3(fp32(k[t][h]) / scale[h]) (and v) for every token with slot >= 0;
    the caches are uint8 tensors [num_blocks, num_kv_heads, block_size, head_dim]."""
    for t, n in ((k, "k"), (v, "v")):
        _need(t, n, torch.bfloat16)
    for t, n in ((k_cache, "k_cache"), (v_cache, "v_cache")):
        _need(t, n, torch.uint8)
    _need(slot_mapping, "slot_mapping", torch.int64)
    _need_scales(k_scale, v_scale, k_cache.shape[1])
    T = slot_mapping.shape[0]
    if k.shape != (T, k_cache.shape[1], k_cache.shape[3]) or v.shape != k.shape or v_cache.shape != k_cache.shape:
        raise ValueError("k/v must be [num_tokens, num_kv_heads, head_dim] and the caches alike")
    st = load_library().pkv_write_fp8(_ptr(k), _ptr(v), _ptr(slot_mapping), T, _ptr(k_scale), _ptr(v_scale),
                                      _ptr(k_cache), _ptr(v_cache), _pool(k_cache), _stream(stream))
    _check(st, "pkv_write_fp8")


def paged_attn_decode_fp8(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, k_scale: torch.Tensor,
                          v_scale: torch.Tensor, block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float,
                          num_kv_heads: int, out: torch.Tensor, max_context_len: int, partition_tokens: int = 0,
                          workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    """paged_attn_decode over an FP8 (e4m3) pool with per-kv-head K and V scales."""
    for t, n in ((q, "q"), (out, "out")):
        _need(t, n, torch.bfloat16)
    for t, n in ((k_cache, "k_cache"), (v_cache, "v_cache")):
        _need(t, n, torch.uint8)
    _need(block_tables, "block_tables", torch.int32)
    _need(context_lens, "context_lens", torch.int32)
    _need_scales(k_scale, v_scale, num_kv_heads)
    B, Hq, D = q.shape
    if out.shape != q.shape or v_cache.shape != k_cache.shape:
        raise ValueError("out must match q and v_cache must match k_cache")
    if workspace is None:
        workspace = torch.empty(decode_workspace_bytes(B, Hq, num_kv_heads, D, max_context_len, partition_tokens),
                                dtype=torch.uint8, device=q.device)
    st = load_library().paged_attn_decode_fp8(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale), _ptr(v_scale), _ptr(block_tables),
        block_tables.shape[1], _ptr(context_lens), B, Hq, float(scale), int(num_kv_heads), _ptr(out),
        _pool(k_cache), int(max_context_len), int(partition_tokens), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "paged_attn_decode_fp8")


def decode_workspace_bytes(num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                           max_context_len: int, partition_tokens: int = 0) -> int:
    n = load_library().pkv_decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                                  max_context_len, partition_tokens)
    if n == 0:
        raise ValueError("invalid sizes for the decode workspace")
    return int(n)


def paged_attn_decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, block_tables: torch.Tensor,
                      context_lens: torch.Tensor, scale: float, num_kv_heads: int, out: torch.Tensor,
                      max_context_len: int, partition_tokens: int = 0,
                      workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    """out[s][hq] = softmax(scale * q[s][hq] . K^T) V over the context_lens[s]
    tokens of sequence s, read through block_tables[s]."""
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache"), (out, "out")):
        _need(t, n, torch.bfloat16)
    _need(block_tables, "block_tables", torch.int32)
    _need(context_lens, "context_lens", torch.int32)
    B, Hq, D = q.shape
    if out.shape != q.shape or v_cache.shape != k_cache.shape:
        raise ValueError("out must match q, v_cache must match k_cache")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or context_lens.shape != (B,):
        raise ValueError("block_tables must be [B, max_blocks_per_seq], context_lens [B]")
    if workspace is None:
        nbytes = decode_workspace_bytes(B, Hq, num_kv_heads, D, max_context_len, partition_tokens)
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    st = load_library().paged_attn_decode(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), block_tables.shape[1], _ptr(context_lens),
        B, Hq, float(scale), int(num_kv_heads), _ptr(out), _pool(k_cache), int(max_context_len),
        int(partition_tokens), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "paged_attn_decode")


def get_device_error(stream=None) -> int:
    """Reads and clears the device error word (waits for `stream`)."""
    code = ctypes.c_int32(0)
    st = load_library().pkv_get_device_error(ctypes.byref(code), _stream(stream))
    if st not in (PKV_OK, 5):
        raise PkvError(st, "pkv_get_device_error")
    return int(code.value)


def paged_attn_decode_static_ws(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                                block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float,
                                num_kv_heads: int, out: torch.Tensor, max_context_len: int,
                                partition_tokens: int = 0, stream=None) -> None:
    """paged_attn_decode without a workspace argument, for callers that cannot
    allocate device memory (for example a plugin whose host engine owns all
    device memory).  Its scratch is a fixed device array of STATIC_WS_BYTES
    inside libpkv.so, shared by every call on the device: calls that overlap
    on the GPU race.  Requests that need more scratch raise PkvError
    (PKV_EUNSUPPORTED); the first call on a device should come before any
    stream capture."""
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache"), (out, "out")):
        _need(t, n, torch.bfloat16)
    _need(block_tables, "block_tables", torch.int32)
    _need(context_lens, "context_lens", torch.int32)
    B, Hq, D = q.shape
    if out.shape != q.shape or v_cache.shape != k_cache.shape:
        raise ValueError("out must match q, v_cache must match k_cache")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or context_lens.shape != (B,):
        raise ValueError("block_tables must be [B, max_blocks_per_seq], context_lens [B]")
    lib = load_library()
    f = lib.paged_attn_decode_static_ws
    if f.argtypes is None:
        P, I32, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
        f.argtypes = [P, P, P, P, I32, P, I32, I32, F, I32, P, _Pool, I32, I32, P]
        f.restype = ctypes.c_int
    st = f(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), block_tables.shape[1], _ptr(context_lens),
           B, Hq, float(scale), int(num_kv_heads), _ptr(out), _pool(k_cache), int(max_context_len),
           int(partition_tokens), _stream(stream))
    _check(st, "paged_attn_decode_static_ws")


def selftest_bounded_wait(limit_ns: int, stream=None) -> torch.Tensor:
    """Runs the library's bounded on-chip wait against barriers that never
    complete (see pkv_selftest_bounded_wait).  Returns the device int32[3]
    result; the device error word then holds DEVERR_TIMEOUT."""
    lib = load_library()
    f = lib.pkv_selftest_bounded_wait
    if f.argtypes is None:
        f.argtypes = [ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
        f.restype = ctypes.c_int
    res = torch.full((3,), -1, dtype=torch.int32, device="cuda")
    _check(f(int(limit_ns), _ptr(res), _stream(stream)), "pkv_selftest_bounded_wait")
    return res


def prefill_workspace_bytes(num_seqs: int, num_q_heads: int, num_kv_heads: int, max_query_len: int) -> int:
    lib = load_library()
    f = lib.pkv_prefill_workspace_bytes
    f.argtypes = [ctypes.c_int32] * 4
    f.restype = ctypes.c_size_t
    n = f(num_seqs, num_q_heads, num_kv_heads, max_query_len)
    if n == 0:
        raise ValueError("invalid sizes for the prefill workspace")
    return int(n)


def paged_attn_prefill(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, block_tables: torch.Tensor,
                       context_lens: torch.Tensor, query_start: torch.Tensor, scale: float, num_kv_heads: int,
                       out: torch.Tensor, max_query_len: int, max_context_len: int,
                       workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    """Chunked-prefill attention: query row i of sequence s's chunk (rows
    query_start[s]..query_start[s+1]-1) sits at position ctx - q_len + i and
    attends to positions [0, pos] read through block_tables[s]."""
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache"), (out, "out")):
        _need(t, n, torch.bfloat16)
    for t, n in ((block_tables, "block_tables"), (context_lens, "context_lens"), (query_start, "query_start")):
        _need(t, n, torch.int32)
    T, Hq, D = q.shape
    B = context_lens.shape[0]
    if out.shape != q.shape or query_start.shape != (B + 1,) or block_tables.shape[0] != B:
        raise ValueError("shape mismatch among q/out, query_start [B+1], block_tables [B, MBS]")
    if workspace is None:
        workspace = torch.empty(prefill_workspace_bytes(B, Hq, num_kv_heads, max_query_len), dtype=torch.uint8,
                                device=q.device)
    lib = load_library()
    f = lib.paged_attn_prefill
    if f.argtypes is None:
        P, I32, F, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
        f.argtypes = [P, P, P, P, I32, P, P, I32, I32, I32, F, I32, P, _Pool, I32, I32, P, SZ, P]
        f.restype = ctypes.c_int
    st = f(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), block_tables.shape[1], _ptr(context_lens),
           _ptr(query_start), B, T, Hq, float(scale), int(num_kv_heads), _ptr(out), _pool(k_cache),
           int(max_query_len), int(max_context_len), _ptr(workspace), workspace.numel() * workspace.element_size(),
           _stream(stream))
    _check(st, "paged_attn_prefill")
