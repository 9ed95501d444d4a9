"""Seeded synthetic inputs for one paged-KV decode step.

This module only draws numbers: sequence lengths, physical block assignments
(through a simulated free list), copy-on-write pairs and the Q/K/V values.  It
holds none of the write, copy or attention arithmetic.  The CUDA library's
tests and benchmark and the CPU oracle both consume what it returns, and
nothing else is shared between those two sides.

Physical pool layout (the library's ABI): ``k_cache[num_blocks][num_kv_heads]
[block_size][head_dim]`` bf16, the same for ``v_cache``.  A slot number names
one token row of the pool as ``physical_block * block_size + offset``.

Every workload describes the state *before* one decode step and the inputs of
that step:

1. ``copy_pairs`` (host int32 ``[P, 2]``, ``(src, dst)``): copy-on-write copies
   of shared blocks, applied first;
2. ``k_new``/``v_new``/``slot_mapping``: one new token per sequence, written at
   position ``context_lens[s] - 1``;
3. ``q``/``block_tables``/``context_lens``: the decode query of each sequence.
   ``context_lens`` counts the token written in step 2, and ``block_tables``
   already points at the copy-on-write destinations of step 1.

Integer structure (lengths, tables, free lists) is drawn on the host with
``numpy.random.default_rng(seed)``.  Bulk values (pool, q, k, v ~ N(0,1),
rounded to bf16) are drawn with a ``torch.Generator`` seeded with the same seed
on ``values_device``; CPU and CUDA generators give different streams, so a test
that compares against the oracle draws its values on one device and moves them.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np
import torch

BF16_NAN_BITS = 0x7FC0  # quiet NaN bit pattern used to poison unused pool rows

WORKLOADS = (
    "tiny",
    "llama2-7b",
    "llama2-13b",
    "llama3-8b-gqa-prefix",
    "llama2-70b-long",
)


@dataclasses.dataclass
class Workload:
    name: str
    seed: int
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    max_blocks_per_seq: int
    scale: float
    context_lens: np.ndarray  # int32 [B]
    block_tables: np.ndarray  # int32 [B, MBS]; -1 beyond each sequence's blocks
    slot_mapping: np.ndarray  # int64 [B]
    copy_pairs: np.ndarray  # int32 [P, 2]
    partition_tokens: int  # 0 = let the library choose
    q: torch.Tensor  # bf16 [B, Hq, D]
    k_new: torch.Tensor  # bf16 [B, Hkv, D]
    v_new: torch.Tensor  # bf16 [B, Hkv, D]
    k_cache: torch.Tensor  # bf16 [NB, Hkv, bs, D]
    v_cache: torch.Tensor  # bf16 [NB, Hkv, bs, D]
    description: str = ""

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.num_seqs else 0

    def tensors(self):
        return dict(q=self.q, k_new=self.k_new, v_new=self.v_new,
                    k_cache=self.k_cache, v_cache=self.v_cache)


# --------------------------------------------------------------------------
# helpers
# --------------------------------------------------------------------------

def _nblocks(n_tokens: int, block_size: int) -> int:
    return (int(n_tokens) + block_size - 1) // block_size


def _normal_bf16(shape, gen: torch.Generator, device) -> torch.Tensor:
    """N(0,1) fp32 draws rounded to bf16 (round-to-nearest-even), drawn in
    chunks along dim 0 so that a multi-GB pool needs no full fp32 copy."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    if out.numel() == 0 or gen is None:  # "meta": shapes only, no values
        return out
    per_row = max(1, out[0].numel())
    rows = max(1, (1 << 26) // per_row)
    for r0 in range(0, shape[0], rows):
        r1 = min(shape[0], r0 + rows)
        chunk = torch.randn((r1 - r0,) + tuple(shape[1:]), generator=gen,
                            device=device, dtype=torch.float32)
        out[r0:r1].copy_(chunk)
    return out


def _slots_for_new_tokens(tables: np.ndarray, ctx: np.ndarray, bs: int) -> np.ndarray:
    """Slot of the token at position ctx-1 of every sequence (input encoding:
    physical block id * block_size + offset)."""
    B = len(ctx)
    slots = np.empty(B, dtype=np.int64)
    for s in range(B):
        pos = int(ctx[s]) - 1
        slots[s] = int(tables[s, pos // bs]) * bs + pos % bs
    return slots


def _tables_array(per_seq_blocks: Sequence[Sequence[int]], mbs: int) -> np.ndarray:
    t = np.full((len(per_seq_blocks), max(mbs, 1)), -1, dtype=np.int32)
    for s, blks in enumerate(per_seq_blocks):
        t[s, :len(blks)] = np.asarray(blks, dtype=np.int32)
    return t


def _finish(name, seed, ctx, per_seq_blocks, pre_cow_blocks, copy_pairs, NB,
            Hq, Hkv, D, bs, values_device, poison, partition_tokens, description):
    ctx = np.asarray(ctx, dtype=np.int32)
    B = len(ctx)
    mbs = max([len(b) for b in per_seq_blocks] + [1])
    tables = _tables_array(per_seq_blocks, mbs)
    slots = _slots_for_new_tokens(tables, ctx, bs) if B else np.zeros(0, np.int64)
    pairs = np.asarray(copy_pairs, dtype=np.int32).reshape(-1, 2)

    gen = None
    if str(values_device) != "meta":
        gen = torch.Generator(device=values_device)
        gen.manual_seed(int(seed))
    q = _normal_bf16((B, Hq, D), gen, values_device)
    k_new = _normal_bf16((B, Hkv, D), gen, values_device)
    v_new = _normal_bf16((B, Hkv, D), gen, values_device)
    k_cache = _normal_bf16((NB, Hkv, bs, D), gen, values_device)
    v_cache = _normal_bf16((NB, Hkv, bs, D), gen, values_device)

    if poison and gen is not None:
        # Rows that hold no token of any sequence before the step get NaN bits:
        # a kernel that reads past a context length, or a copy/write that goes
        # missing, then shows up as NaN instead of as a small numeric drift.
        live = np.zeros((NB, bs), dtype=bool)
        for s in range(B):
            blks = pre_cow_blocks[s]
            for pos in range(int(ctx[s]) - 1):
                live[blks[pos // bs], pos % bs] = True
        dead = torch.from_numpy(~live).to(values_device)
        nan = torch.tensor(BF16_NAN_BITS, dtype=torch.int16).view(torch.bfloat16)
        nan = nan.to(values_device)
        mask = dead[:, None, :, None].expand(NB, Hkv, bs, D)
        k_cache = torch.where(mask, nan, k_cache)
        v_cache = torch.where(mask, nan, v_cache)

    scale = float(np.float32(1.0 / math.sqrt(D)))
    return Workload(name=name, seed=seed, num_seqs=B, num_q_heads=Hq,
                    num_kv_heads=Hkv, head_dim=D, block_size=bs, num_blocks=NB,
                    max_blocks_per_seq=mbs, scale=scale, context_lens=ctx,
                    block_tables=tables, slot_mapping=slots, copy_pairs=pairs,
                    partition_tokens=partition_tokens, q=q, k_new=k_new,
                    v_new=v_new, k_cache=k_cache, v_cache=v_cache,
                    description=description)


E4M3_NAN_CODE = 0x7F  # an FP8 (e4m3) NaN code, used to poison unused FP8 pool rows


def fp8_pools(w: Workload, seed: Optional[int] = None):
    """An FP8 (e4m3) pool of the workload's shape: (k_cache8, v_cache8,
    k_scale, v_scale).  Codes are drawn directly: a random sign, an exponent
    field uniform in [1, 9] and a random mantissa (magnitudes 2^-6 .. 7.5), so
    that code * scale spans a few binades; rows that are NaN in the workload's
    bf16 pool (poison) get the NaN code.  Scales: one per kv head, uniform in
    [0.05, 0.5], for K and for V.  Nothing here quantizes."""
    seed = w.seed if seed is None else seed
    dev = w.k_cache.device
    gen = torch.Generator(device=dev)
    gen.manual_seed(int(seed) + 7919)
    shape = tuple(w.k_cache.shape)

    def codes():
        sign = torch.randint(0, 2, shape, generator=gen, device=dev, dtype=torch.int32) << 7
        expo = torch.randint(1, 10, shape, generator=gen, device=dev, dtype=torch.int32) << 3
        mant = torch.randint(0, 8, shape, generator=gen, device=dev, dtype=torch.int32)
        return (sign | expo | mant).to(torch.uint8)

    k8, v8 = codes(), codes()
    for src, dst in ((w.k_cache, k8), (w.v_cache, v8)):
        dead = src.view(torch.int16) == torch.tensor(BF16_NAN_BITS, dtype=torch.int16, device=dev)
        dst.masked_fill_(dead, E4M3_NAN_CODE)
    rng = np.random.default_rng(int(seed) + 104729)
    k_scale = torch.from_numpy(rng.uniform(0.05, 0.5, w.num_kv_heads).astype(np.float32)).to(dev)
    v_scale = torch.from_numpy(rng.uniform(0.05, 0.5, w.num_kv_heads).astype(np.float32)).to(dev)
    return k8, v8, k_scale, v_scale


def _pop_tables(ctx, bs, free: list) -> list:
    """Pops each sequence's blocks (logical order) from the end of ``free``."""
    out = []
    for n in ctx:
        out.append([free.pop() for _ in range(_nblocks(n, bs))])
    return out


# --------------------------------------------------------------------------
# generic generator (tests use it for small ragged cases)
# --------------------------------------------------------------------------

def make_custom(context_lens: Sequence[int], num_q_heads: int, num_kv_heads: int,
                head_dim: int, block_size: int, seed: int = 0,
                pool_factor: float = 1.5, values_device="cpu", poison=False,
                share_prefix_tokens: int = 0, group_size: int = 1,
                partition_tokens: int = 0, name: str = "custom") -> Workload:
    """Sequences of the given lengths on a shuffled free list.

    With ``share_prefix_tokens > 0`` consecutive groups of ``group_size``
    sequences map the blocks that cover their first
    ``min(share_prefix_tokens, ctx-1)`` tokens to the same physical ids
    (``share_prefix_tokens`` must be a multiple of the block size)."""
    rng = np.random.default_rng(seed)
    ctx = [int(c) for c in context_lens]
    bs = block_size
    need = sum(_nblocks(c, bs) for c in ctx) + 1
    NB = max(int(math.ceil(pool_factor * need)), 1)
    free = [int(x) for x in rng.permutation(NB)]
    if share_prefix_tokens:
        assert share_prefix_tokens % bs == 0
        nshared = share_prefix_tokens // bs
        per_seq = []
        group_prefix = None
        for s, c in enumerate(ctx):
            if s % group_size == 0:
                group_prefix = [free.pop() for _ in range(nshared)]
            nb = _nblocks(c, bs)
            # blocks fully before the new token's position may be shared
            nshare = min(nshared, (c - 1) // bs)
            blks = group_prefix[:nshare] + [free.pop() for _ in range(nb - nshare)]
            per_seq.append(blks)
    else:
        per_seq = _pop_tables(ctx, bs, free)
    return _finish(name, seed, ctx, per_seq, per_seq, [], NB, num_q_heads,
                   num_kv_heads, head_dim, bs, values_device, poison,
                   partition_tokens, f"custom lens={ctx}")


# --------------------------------------------------------------------------
# the five decode-step workloads
# --------------------------------------------------------------------------

def _tiny(seed, values_device, poison, block_size=None):
    # 4 sequences, ctx {1,17,33,64}, 4 q = 4 kv heads, d 64, bs 16, pool of 32
    # blocks handed out by a seeded permutation in logical order.
    rng = np.random.default_rng(seed)
    bs = 16 if block_size is None else block_size
    ctx = [1, 17, 33, 64]
    NB = 32
    perm = [int(x) for x in rng.permutation(NB)]
    per_seq, k = [], 0
    for c in ctx:
        n = _nblocks(c, bs)
        per_seq.append(perm[k:k + n])
        k += n
    return _finish("tiny", seed, ctx, per_seq, per_seq, [], NB, 4, 4, 64, bs,
                   values_device, poison, 0,
                   "4 seqs ctx {1,17,33,64}, MHA 4 heads, d64, bs16, pool 32")


def _llama2_7b(seed, values_device, poison, block_size=None):
    rng = np.random.default_rng(seed)
    bs = 16 if block_size is None else block_size
    B, H, D = 64, 32, 128
    ctx = [int(x) for x in rng.integers(128, 2048, size=B, endpoint=True)]
    need = sum(_nblocks(c, bs) for c in ctx)
    NB = int(math.ceil(1.2 * need))
    free = [int(x) for x in rng.permutation(NB)]
    per_seq = _pop_tables(ctx, bs, free)
    return _finish("llama2-7b", seed, ctx, per_seq, per_seq, [], NB, H, H, D, bs,
                   values_device, poison, 0,
                   "B64, MHA 32 heads, d128, bs16, ctx U[128,2048], pool 1.2x, shuffled free list")


def _lognormal_len(rng) -> int:
    prompt = int(np.clip(round(float(rng.lognormal(math.log(300.0), 1.0))), 16, 3072))
    return prompt + int(rng.integers(0, 512, endpoint=True))


def _llama2_13b(seed, values_device, poison, block_size=None):
    rng = np.random.default_rng(seed)
    bs = 16 if block_size is None else block_size
    B, H, D = 128, 40, 128
    ctx = [_lognormal_len(rng) for _ in range(B)]
    need = sum(_nblocks(c, bs) for c in ctx)
    NB = int(math.ceil(1.2 * need))
    # Fragment the free list: 1000 seeded steps, each allocating a sequence of
    # a length from the same distribution (p = 0.5) or freeing a random live
    # one.  An allocation that does not fit is skipped.  Afterwards the live
    # sequences are released in random order, and the measured batch pops its
    # blocks from the resulting (scrambled) LIFO free list.
    free = list(range(NB - 1, -1, -1))
    live, next_id = {}, 0
    for _ in range(1000):
        if not live or rng.random() < 0.5:
            n = _nblocks(_lognormal_len(rng), bs)
            if n <= len(free):
                live[next_id] = [free.pop() for _ in range(n)]
                next_id += 1
        else:
            keys = sorted(live)
            victim = keys[int(rng.integers(len(keys)))]
            free.extend(reversed(live.pop(victim)))
    for key in [sorted(live)[i] for i in rng.permutation(len(live))]:
        free.extend(reversed(live.pop(key)))
    per_seq = _pop_tables(ctx, bs, free)
    return _finish("llama2-13b", seed, ctx, per_seq, per_seq, [], NB, H, H, D, bs,
                   values_device, poison, 0,
                   f"B128, MHA 40 heads, d128, bs{bs}, ctx lognormal(ln300,1) clip[16,3072] "
                   "+ U[0,512], pool 1.2x fragmented by 1000 alloc/free steps")


def _llama3_8b_gqa_prefix(seed, values_device, poison, block_size=None):
    rng = np.random.default_rng(seed)
    bs = 16 if block_size is None else block_size
    B, Hq, Hkv, D = 256, 32, 8, 128
    groups, per_group, prefix = 32, 8, 1024
    assert prefix % bs == 0
    nshared = prefix // bs
    # 8 sequences (distinct groups) are copy-on-write forks: their newest token
    # falls inside the group's shared prefix at a non-zero in-block offset, so
    # the shared block that holds it is copied to a private block first.
    fork_groups = rng.choice(groups, size=8, replace=False)
    fork_members = rng.integers(0, per_group, size=8)
    forked = {int(g) * per_group + int(m) for g, m in zip(fork_groups, fork_members)}
    ctx = []
    for s in range(B):
        if s in forked:
            j = int(rng.integers(512 // bs, nshared))  # shared block of the new token
            o = int(rng.integers(1, bs))  # non-zero offset inside it
            ctx.append(j * bs + o + 1)
        else:
            ctx.append(int(rng.integers(prefix + 1, 8192, endpoint=True)))
    need = groups * nshared
    for s in range(B):
        need += 1 if s in forked else _nblocks(ctx[s], bs) - nshared
    NB = int(math.ceil(1.2 * need))
    free = [int(x) for x in rng.permutation(NB)]
    shared = [[free.pop() for _ in range(nshared)] for _ in range(groups)]
    per_seq, pre_cow, pairs = [], [], []
    for s in range(B):
        g = s // per_group
        if s in forked:
            j = (ctx[s] - 1) // bs
            dst = free.pop()
            pre_cow.append(shared[g][:j + 1])
            per_seq.append(shared[g][:j] + [dst])
            pairs.append((shared[g][j], dst))
        else:
            own = [free.pop() for _ in range(_nblocks(ctx[s], bs) - nshared)]
            per_seq.append(shared[g] + own)
            pre_cow.append(per_seq[-1])
    return _finish("llama3-8b-gqa-prefix", seed, ctx, per_seq, pre_cow, pairs, NB,
                   Hq, Hkv, D, bs, values_device, poison, 0,
                   "B256 in 32 groups of 8 sharing a 1024-token prefix, GQA 32q/8kv, d128, "
                   "bs16, ctx U[1025,8192]; 8 forked seqs (ctx<=1024) copy-on-write their "
                   "shared partial block")


def _llama2_70b_long(seed, values_device, poison, block_size=None):
    rng = np.random.default_rng(seed)
    bs = 16 if block_size is None else block_size
    B, Hq, Hkv, D = 8, 64, 8, 128
    ctx = [int(x) for x in rng.permutation([32768, 65536, 98304, 131072] * 2)]
    need = sum(_nblocks(c, bs) for c in ctx)
    NB = int(math.ceil(1.2 * need))
    free = [int(x) for x in rng.permutation(NB)]
    per_seq = _pop_tables(ctx, bs, free)
    return _finish("llama2-70b-long", seed, ctx, per_seq, per_seq, [], NB, Hq, Hkv,
                   D, bs, values_device, poison, 512,
                   f"B8, GQA 64q/8kv, d128, bs{bs}, ctx {{32K,64K,96K,128K}}x2, "
                   "split-K partitions of 512 tokens")


_BUILDERS = {
    "tiny": _tiny,
    "llama2-7b": _llama2_7b,
    "llama2-13b": _llama2_13b,
    "llama3-8b-gqa-prefix": _llama3_8b_gqa_prefix,
    "llama2-70b-long": _llama2_70b_long,
}


def make(name: str, seed: int = 0, values_device="cpu", poison: bool = False,
         block_size: Optional[int] = None) -> Workload:
    """Builds one of the named decode-step workloads."""
    if name not in _BUILDERS:
        raise KeyError(f"unknown workload {name!r}; choose from {WORKLOADS}")
    return _BUILDERS[name](seed, values_device, poison, block_size)


def subset(w: Workload, num_seqs: int) -> Workload:
    """The first ``num_seqs`` sequences of a workload, on a pool compacted to
    the blocks they reference (and their copy-on-write sources), with tables,
    slots and pairs renumbered.  For smaller profiling and test cases."""
    n = min(int(num_seqs), w.num_seqs)
    tables = w.block_tables[:n]
    refd = set(int(b) for b in tables[tables >= 0].ravel())
    pairs = [(int(s), int(d)) for s, d in w.copy_pairs if int(d) in refd]
    used = sorted(refd | {s for s, _ in pairs})
    new_id = {b: i for i, b in enumerate(used)}
    remap = np.vectorize(lambda b: new_id[int(b)] if b >= 0 else -1, otypes=[np.int32])
    new_tables = remap(tables) if tables.size else tables.copy()
    bs = w.block_size
    slots = np.array([new_id[int(s) // bs] * bs + int(s) % bs for s in w.slot_mapping[:n]], dtype=np.int64)
    sel = torch.tensor(used, dtype=torch.long, device=w.k_cache.device)
    return dataclasses.replace(
        w, num_seqs=n, num_blocks=len(used), context_lens=w.context_lens[:n].copy(),
        block_tables=new_tables.astype(np.int32), slot_mapping=slots,
        copy_pairs=np.array([(new_id[s], new_id[d]) for s, d in pairs], dtype=np.int32).reshape(-1, 2),
        q=w.q[:n].contiguous(), k_new=w.k_new[:n].contiguous(), v_new=w.v_new[:n].contiguous(),
        k_cache=w.k_cache.index_select(0, sel).contiguous(), v_cache=w.v_cache.index_select(0, sel).contiguous(),
        description=w.description + f" (first {n} sequences)")


# --------------------------------------------------------------------------
# chunked prefill: several new tokens per sequence
# --------------------------------------------------------------------------

@dataclasses.dataclass
class PrefillWorkload:
    """State before one prefill chunk and its inputs: sequence s already holds
    prefix_lens[s] tokens; its chunk of q_len_s = query_start[s+1] -
    query_start[s] new tokens is written at positions prefix..ctx-1 (slot
    mapping) and then attends causally.  context_lens counts the chunk."""
    name: str
    seed: int
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    max_blocks_per_seq: int
    scale: float
    context_lens: np.ndarray  # int32 [B]
    query_start: np.ndarray  # int32 [B + 1]
    block_tables: np.ndarray  # int32 [B, MBS]
    slot_mapping: np.ndarray  # int64 [T]
    q: torch.Tensor  # bf16 [T, Hq, D]
    k_new: torch.Tensor  # bf16 [T, Hkv, D]
    v_new: torch.Tensor  # bf16 [T, Hkv, D]
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    description: str = ""

    @property
    def num_tokens(self) -> int:
        return int(self.query_start[-1])

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.num_seqs else 0

    @property
    def max_query_len(self) -> int:
        return int(np.diff(self.query_start).max()) if self.num_seqs else 0


def make_prefill_custom(prefix_lens: Sequence[int], chunk_lens: Sequence[int], num_q_heads: int,
                        num_kv_heads: int, head_dim: int, block_size: int, seed: int = 0,
                        pool_factor: float = 1.2, values_device="cpu", poison=False,
                        name: str = "prefill-custom", description: str = "") -> PrefillWorkload:
    rng = np.random.default_rng(seed)
    bs = block_size
    prefix = [int(x) for x in prefix_lens]
    chunk = [int(x) for x in chunk_lens]
    ctx = [p + c for p, c in zip(prefix, chunk)]
    need = sum(_nblocks(c, bs) for c in ctx) + 1
    NB = max(int(math.ceil(pool_factor * need)), 1)
    free = [int(x) for x in rng.permutation(NB)]
    per_seq = _pop_tables(ctx, bs, free)
    mbs = max([len(b) for b in per_seq] + [1])
    tables = _tables_array(per_seq, mbs)
    qsl = np.zeros(len(ctx) + 1, dtype=np.int32)
    qsl[1:] = np.cumsum(chunk)
    T = int(qsl[-1])
    slots = np.empty(T, dtype=np.int64)
    for s, (p0, c) in enumerate(zip(prefix, chunk)):
        for i in range(c):
            pos = p0 + i
            slots[qsl[s] + i] = int(tables[s, pos // bs]) * bs + pos % bs
    gen = None
    if str(values_device) != "meta":
        gen = torch.Generator(device=values_device)
        gen.manual_seed(int(seed))
    Hq, Hkv, D = num_q_heads, num_kv_heads, head_dim
    q = _normal_bf16((T, Hq, D), gen, values_device)
    k_new = _normal_bf16((T, Hkv, D), gen, values_device)
    v_new = _normal_bf16((T, Hkv, D), gen, values_device)
    k_cache = _normal_bf16((NB, Hkv, bs, D), gen, values_device)
    v_cache = _normal_bf16((NB, Hkv, bs, D), gen, values_device)
    if poison and gen is not None:
        live = np.zeros((NB, bs), dtype=bool)
        for s in range(len(ctx)):
            for pos in range(prefix[s]):
                live[per_seq[s][pos // bs], pos % bs] = True
        dead = torch.from_numpy(~live).to(values_device)
        nan = torch.tensor(BF16_NAN_BITS, dtype=torch.int16).view(torch.bfloat16).to(values_device)
        mask = dead[:, None, :, None].expand(NB, Hkv, bs, D)
        k_cache = torch.where(mask, nan, k_cache)
        v_cache = torch.where(mask, nan, v_cache)
    return PrefillWorkload(name=name, seed=seed, num_seqs=len(ctx), num_q_heads=Hq, num_kv_heads=Hkv,
                           head_dim=D, block_size=bs, num_blocks=NB, max_blocks_per_seq=mbs,
                           scale=float(np.float32(1.0 / math.sqrt(D))),
                           context_lens=np.asarray(ctx, dtype=np.int32), query_start=qsl, block_tables=tables,
                           slot_mapping=slots, q=q, k_new=k_new, v_new=v_new, k_cache=k_cache,
                           v_cache=v_cache, description=description or f"prefix={prefix} chunk={chunk}")


PREFILL_WORKLOADS = ("llama2-13b-prefill", "llama3-8b-prefill")


def make_prefill(name: str, seed: int = 0, values_device="cpu", poison: bool = False,
                 block_size: Optional[int] = None) -> PrefillWorkload:
    """Chunked-prefill workloads: 8 sequences, each with an already cached
    prefix of U[0, L] tokens and a new 512-token chunk (Llama-2-13B: 40 MHA
    heads, L = 3072; Llama-3-8B: 32 q / 8 kv heads, L = 7680)."""
    rng = np.random.default_rng(seed)
    bs = 16 if block_size is None else block_size
    if name == "llama2-13b-prefill":
        Hq, Hkv, L = 40, 40, 3072
    elif name == "llama3-8b-prefill":
        Hq, Hkv, L = 32, 8, 7680
    else:
        raise KeyError(f"unknown prefill workload {name!r}; choose from {PREFILL_WORKLOADS}")
    prefix = [int(x) for x in rng.integers(0, L, size=8, endpoint=True)]
    return make_prefill_custom(prefix, [512] * 8, Hq, Hkv, 128, bs, seed=seed, values_device=values_device,
                               poison=poison, name=name,
                               description=f"B8, {Hq}q/{Hkv}kv heads, d128, bs{bs}, cached prefix U[0,{L}], "
                                           "512-token chunk each")
