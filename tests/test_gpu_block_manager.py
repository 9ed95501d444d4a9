"""GPU parity of the device block manager against the oracle's sequential
block manager: every call's outputs and the whole state (free list, top,
reference counts, prefix keys, the eviction order of cached blocks, error
word) are compared bit for bit after each step.
Cases: random operation mixes, forks whose sharers append together (more
sharers than a warp, across the 1024-sequence chunk boundary), the worked
example, errors, and a whole decode step driven from the device state."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_420_b200 as pkv
import workloads
from tests._gpu_util import assert_attention_close, bits_equal

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _same_state(bm: pkv.BlockManager, st: oracle.BlockState, err_expected: int):
    torch.cuda.synchronize()
    assert bm.top() == st.top
    assert np.array_equal(bm.free_stack.cpu().numpy()[:st.top], st.free_stack[:st.top])
    assert np.array_equal(bm.refcount.cpu().numpy(), st.refcount)
    assert np.array_equal(bm.block_hash.cpu().numpy().view(np.uint64), st.block_hash)
    assert np.array_equal(bm.lru_order(), st.lru_order()) and bm.cached() == len(st.lru_order())
    assert bm.error() == err_expected


def _dev(a, dtype=torch.int32):
    return torch.as_tensor(np.ascontiguousarray(a)).to(dtype).cuda()


class Mirror:
    """Applies each operation to the device manager and to the oracle."""

    def __init__(self, nb, B, mbs, bs):
        self.bm = pkv.BlockManager(nb)
        self.st = oracle.bm_init(nb)
        self.err = 0
        self.bs = bs
        self.tables = np.full((B, mbs), -1, np.int32)
        self.ctx = np.zeros(B, np.int32)
        self.t_dev = _dev(self.tables)
        self.c_dev = _dev(self.ctx)
        _same_state(self.bm, self.st, 0)

    def append(self, num_new):
        nn = np.asarray(num_new, np.int32)
        T = int(np.clip(nn, 0, None).sum())
        slots, pairs, npairs = self.bm.append_slots(self.t_dev, self.c_dev, _dev(nn), self.bs, T)
        self.st, tables, ctx, oslots, opairs, e = oracle.bm_append_slots(self.st, self.tables, self.ctx, nn, self.bs)
        self.err |= e
        torch.cuda.synchronize()
        assert np.array_equal(self.t_dev.cpu().numpy(), tables)
        assert np.array_equal(self.c_dev.cpu().numpy(), ctx)
        assert np.array_equal(slots.cpu().numpy(), oslots)
        k = int(npairs.item())
        assert k == len(opairs) and np.array_equal(pairs.cpu().numpy()[:k], opairs)
        self.tables, self.ctx = tables, ctx
        _same_state(self.bm, self.st, self.err)
        return slots, pairs, npairs, opairs

    def fork(self, a, b):
        """Sequence b (after releasing its blocks) becomes a parallel sample of a."""
        self.release(b)
        nblk = (int(self.ctx[a]) + self.bs - 1) // self.bs
        self.tables[b, :nblk] = self.tables[a, :nblk]
        self.ctx[b] = self.ctx[a]
        self.t_dev.copy_(_dev(self.tables))
        self.c_dev.copy_(_dev(self.ctx))
        if nblk:
            self.bm.share(_dev(self.tables[a, :nblk]))
            self.st, e = oracle.bm_share(self.st, self.tables[a, :nblk])
            self.err |= e
        _same_state(self.bm, self.st, self.err)

    def release(self, b):
        nblk = (int(self.ctx[b]) + self.bs - 1) // self.bs
        if nblk:
            self.bm.free(_dev(self.tables[b, :nblk]))
            self.st, e = oracle.bm_free(self.st, self.tables[b, :nblk])
            self.err |= e
        self.tables[b] = -1
        self.ctx[b] = 0
        self.t_dev.copy_(_dev(self.tables))
        self.c_dev.copy_(_dev(self.ctx))
        _same_state(self.bm, self.st, self.err)


@pytest.mark.parametrize("seed", range(4))
def test_random_operation_mix(seed):
    rng = np.random.default_rng(seed)
    m = Mirror(nb=300, B=40, mbs=24, bs=int(rng.choice([4, 16])))
    for _ in range(30):
        r = rng.random()
        if r < 0.55:
            m.append(rng.integers(0, 9, 40) * (rng.random(40) < 0.8))
        elif r < 0.8:
            a, b = rng.choice(40, 2, replace=False)
            m.fork(int(a), int(b))
        else:
            m.release(int(rng.integers(40)))


def test_fork_storm_across_warps_and_chunks():
    """1500 sequences: 60 parents, each with 24 forks spread over the batch, all
    appending one token into the shared partly filled block in one step."""
    rng = np.random.default_rng(1)
    B = 1500
    m = Mirror(nb=6000, B=B, mbs=8, bs=16)
    parents = np.arange(60)
    m.append(np.where(np.isin(np.arange(B), parents), rng.integers(17, 31, B), 0))  # partly filled 2nd block
    forks = rng.permutation(np.arange(60, B))[:60 * 24].reshape(60, 24)
    for p_, kids in zip(parents, forks):
        for kid in kids:
            nblk = (int(m.ctx[p_]) + 15) // 16
            m.tables[kid, :nblk] = m.tables[p_, :nblk]
            m.ctx[kid] = m.ctx[p_]
    shared = np.concatenate([np.repeat(m.tables[p_, :(m.ctx[p_] + 15) // 16][None], 24, 0).reshape(-1)
                             for p_ in parents])
    m.t_dev.copy_(_dev(m.tables))
    m.c_dev.copy_(_dev(m.ctx))
    m.bm.share(_dev(shared))
    m.st, _ = oracle.bm_share(m.st, shared)
    _same_state(m.bm, m.st, 0)
    active = np.zeros(B, np.int32)
    active[np.concatenate([parents, forks.reshape(-1)])] = 1
    slots, pairs, npairs, opairs = m.append(active)
    assert len(opairs) == 60 * 24  # every sharer but the last in order copies


def test_worked_example_on_device():
    g = json.load(open(os.path.join(GOLDEN, "block_manager_example.json")))
    bm = pkv.BlockManager(g["num_blocks"])
    for step in g["steps"]:
        if step["op"] == "append":
            t = _dev(step["tables"])
            c = _dev(step["context_lens"])
            slots, pairs, npairs = bm.append_slots(t, c, _dev(step["num_new"]), g["block_size"],
                                                   int(sum(step["num_new"])))
            torch.cuda.synchronize()
            assert t.cpu().tolist() == step["expect_tables"]
            assert c.cpu().tolist() == step["expect_context_lens"]
            assert slots.cpu().tolist() == step["expect_slots"]
            assert pairs.cpu().numpy()[:int(npairs.item())].tolist() == step["expect_pairs"]
            assert bm.top() == step["expect_top"]
        elif step["op"] == "fork":
            bm.share(_dev(step["share"]))
        elif step["op"] == "free":
            bm.free(_dev(step["ids"]))
            assert bm.top() == step["expect_top"]
        elif step["op"] == "alloc":
            off, ids = bm.alloc(_dev(step["counts"]), 16)
            torch.cuda.synchronize()
            assert ids.cpu().numpy()[:int(off[-1].item())].tolist() == step["expect_ids"]
        if "expect_refcount" in step:
            torch.cuda.synchronize()
            assert bm.refcount.cpu().tolist() == step["expect_refcount"]
        assert bm.error() == 0


def test_alloc_free_parity_and_errors():
    rng = np.random.default_rng(3)
    bm = pkv.BlockManager(700)
    st = oracle.bm_init(700)
    err = 0
    for _ in range(6):
        counts = rng.integers(0, 40, 2100).astype(np.int32) * (rng.random(2100) < 0.02)
        off, ids = bm.alloc(_dev(counts), 500)
        st, ooff, oids, e = oracle.bm_alloc(st, counts, 500)
        err |= e
        torch.cuda.synchronize()
        assert np.array_equal(off.cpu().numpy(), ooff)
        assert np.array_equal(ids.cpu().numpy()[:ooff[-1]], oids[:ooff[-1]])
        _same_state(bm, st, err)
        held = np.flatnonzero(st.refcount > 0)
        batch = rng.choice(held, min(len(held), 300)).astype(np.int32) if len(held) else np.zeros(0, np.int32)
        # no double frees: at most refcount occurrences of each block
        keep = []
        seen = {}
        for b_ in batch:
            seen[b_] = seen.get(b_, 0) + 1
            if seen[b_] <= st.refcount[b_]:
                keep.append(b_)
        batch = np.array(keep, np.int32)
        if len(batch):
            bm.free(_dev(batch))
            st, e = oracle.bm_free(st, batch)
            err |= e
            _same_state(bm, st, err)
    assert err & oracle.BM_ERR_NOSPACE
    # error paths: out of range, double free (the set of free blocks still matches)
    bm.clear_error()
    bm.free(_dev([700, -1]))
    torch.cuda.synchronize()
    assert bm.error() == oracle.BM_ERR_RANGE
    bm.clear_error()
    held = int(np.flatnonzero(st.refcount == 1)[0])
    bm.free(_dev([held, held]))
    st, e = oracle.bm_free(st, [held, held])
    torch.cuda.synchronize()
    assert bm.error() & oracle.BM_ERR_DOUBLEFREE and e & oracle.BM_ERR_DOUBLEFREE
    assert set(bm.free_stack.cpu().numpy()[:bm.top()].tolist()) == st.free_set()


def test_append_errors_match():
    m = Mirror(nb=10, B=4, mbs=4, bs=4)
    m.append([5, 3, 0, 0])          # 3 blocks
    m.append([12, 1, 1, 0])         # seq0 outgrows its row (TABLE): it and every later one unchanged
    m.release(0)
    m.append([0, 1, 30, 2])         # seq2 asks for more than its row
    m.append([8, 8, 8, 8])          # 8 blocks: fits
    m.append([4, 4, 4, 4])          # one block left: seq0 gets it, seq1 on find none (NOSPACE)
    assert m.err & oracle.BM_ERR_TABLE and m.err & oracle.BM_ERR_NOSPACE


def test_decode_step_driven_by_the_device_block_manager():
    """Forks share a prefix; one decode step appends a token to every sequence
    from the device state, copies the copy-on-write pairs on the device, writes
    the new K/V at the produced slots and runs decode attention: the result
    equals the oracle's step on the oracle's own tables."""
    rng = np.random.default_rng(11)
    B, Hq, Hkv, D, bs, nb, mbs = 24, 8, 2, 128, 16, 400, 40
    m = Mirror(nb=nb, B=B, mbs=mbs, bs=bs)
    m.append(np.where(np.arange(B) < 8, rng.integers(20, 300, B), 0))
    for kid in range(8, B):
        m.fork(kid % 8, kid)
    g = torch.Generator().manual_seed(5)
    kc = torch.randn((nb, Hkv, bs, D), generator=g).to(torch.bfloat16)
    vc = torch.randn((nb, Hkv, bs, D), generator=g).to(torch.bfloat16)
    k_new = torch.randn((B, Hkv, D), generator=g).to(torch.bfloat16)
    v_new = torch.randn((B, Hkv, D), generator=g).to(torch.bfloat16)
    q = torch.randn((B, Hq, D), generator=g).to(torch.bfloat16)
    kd, vd = kc.cuda(), vc.cuda()
    slots, pairs, npairs, opairs = m.append(np.ones(B, np.int32))
    assert len(opairs) > 0
    pkv.copy_blocks_dev(pairs, npairs, kd, vd)
    pkv.pkv_write(k_new.cuda(), v_new.cuda(), slots, kd, vd)
    out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device="cuda")
    pkv.paged_attn_decode(q.cuda(), kd, vd, m.t_dev, m.c_dev, 1 / np.sqrt(D), Hkv, out, int(m.ctx.max()))
    torch.cuda.synchronize()
    okc, ovc = oracle.copy_blocks(kc, vc, opairs)
    okc, ovc = oracle.kv_write(okc, ovc, k_new, v_new, slots.cpu().numpy())
    assert bits_equal(kd, okc) and bits_equal(vd, ovc)
    ref = oracle.paged_attention(q, okc, ovc, m.tables, m.ctx, float(np.float32(1 / np.sqrt(D))))
    assert_attention_close(out, ref, "device block manager step")


def _systems(rng, bs, n_sys=4, vocab=100):
    return [rng.integers(0, vocab, bs * int(rng.integers(1, 4))) for _ in range(n_sys)]


def _prompts(rng, n, bs, systems, vocab=100):
    """Prompts: one of the system prompts (1-3 blocks) plus a private tail."""
    n_sys = len(systems)
    out = []
    for _ in range(n):
        tail = rng.integers(0, vocab, int(rng.integers(0, 3 * bs)))
        out.append(np.concatenate([systems[int(rng.integers(n_sys))], tail]).astype(np.int32))
    return out


def _serve_both(bm, pc, st, ocache, prompts, bs, mbs):
    tokens = np.concatenate(prompts).astype(np.int32)
    qs = np.concatenate([[0], np.cumsum([len(p) for p in prompts])]).astype(np.int32)
    B = len(prompts)
    tables = np.full((B, mbs), -1, np.int32)
    t_dev = _dev(tables)
    cached = pc.lookup(bm, _dev(tokens), _dev(qs), bs, t_dev)
    st, otab, ocached = oracle.prefix_lookup(st, ocache, tokens, qs, bs, tables)
    torch.cuda.synchronize()
    assert np.array_equal(cached.cpu().numpy(), ocached)
    assert np.array_equal(t_dev.cpu().numpy(), otab)
    need = np.array([len(p) for p in prompts], np.int32) - ocached
    c_dev = _dev(ocached)
    slots, pairs, npairs = bm.append_slots(t_dev, c_dev, _dev(need), bs, int(need.sum()))
    st, otab, octx, oslots, opairs, err = oracle.bm_append_slots(st, otab, ocached, need, bs)
    torch.cuda.synchronize()
    assert np.array_equal(t_dev.cpu().numpy(), otab) and np.array_equal(slots.cpu().numpy(), oslots)
    pc.insert(bm, _dev(tokens), _dev(qs), bs, t_dev)
    st, ocache, e2 = oracle.prefix_insert(st, ocache, tokens, qs, bs, otab)
    torch.cuda.synchronize()
    assert np.array_equal(bm.block_hash.cpu().numpy().view(np.uint64), st.block_hash)
    _same_state(bm, st, err | e2)
    return st, ocache, otab, octx, ocached


@pytest.mark.parametrize("seed,B,bs", [(0, 40, 4), (1, 1300, 4), (2, 64, 16)])
def test_prefix_cache_rounds_match_oracle(seed, B, bs):
    """Rounds of requests sharing system prompts: lookup, the remaining blocks
    through append_slots, insert; some sequences end between rounds."""
    rng = np.random.default_rng(seed)
    mbs = 8
    nb = B * mbs * 2
    bm = pkv.BlockManager(nb)
    pc = pkv.PrefixCache(1 << int(np.ceil(np.log2(4 * B * mbs))))
    st = oracle.bm_init(nb)
    ocache = oracle.PrefixCache(4 * B * mbs)
    live = []
    total_hits = 0
    systems = _systems(rng, bs)
    for rnd in range(3):
        prompts = _prompts(rng, B, bs, systems)
        if rnd == 1:
            prompts[B // 2] = prompts[B // 2 - 1].copy()  # the same prompt twice in one batch
        st, ocache, tables, ctx, cached = _serve_both(bm, pc, st, ocache, prompts, bs, mbs)
        total_hits += int((cached > 0).sum())
        live.append((tables, ctx))
        # half of the oldest round's sequences end
        old_tables, old_ctx = live[0]
        ends = np.flatnonzero(rng.random(len(old_ctx)) < 0.5)
        ids = np.concatenate([old_tables[b, :(old_ctx[b] + bs - 1) // bs] for b in ends]) if len(ends) else []
        ids = np.asarray(ids, np.int32)
        if len(ids):
            bm.free(_dev(ids))
            st, _ = oracle.bm_free(st, ids)
            _same_state(bm, st, 0)
            assert np.array_equal(bm.block_hash.cpu().numpy().view(np.uint64), st.block_hash)
        old_ctx[ends] = 0
    assert total_hits > 0 and st.block_hash.any()


def test_cached_blocks_worked_example_on_device():
    """The cached-block worked example (a system prompt served again after its
    first request finished; free blocks before cached ones; least recently
    released evicted first, its key dropped) replayed on the device."""
    from tests.test_oracle_prefix import run_eviction_example
    g = json.load(open(os.path.join(GOLDEN, "prefix_eviction_example.json")))
    bs = g["block_size"]
    bm = pkv.BlockManager(g["num_blocks"])
    pc = pkv.PrefixCache(g["cache_capacity"])

    def serve(prompt):
        tokens = _dev(prompt)
        qs = _dev([0, len(prompt)])
        t = _dev(np.full((1, 8), -1, np.int32))
        cached = pc.lookup(bm, tokens, qs, bs, t)
        need = _dev([len(prompt)]) - cached
        bm.append_slots(t, cached.clone(), need.to(torch.int32), bs, len(prompt))
        pc.insert(bm, tokens, qs, bs, t)
        torch.cuda.synchronize()
        err = bm.error()
        bm.clear_error()
        return int(cached[0].item()), t[0].cpu().numpy(), err

    def finish(row, n):
        bm.free(_dev(row[:-(-n // bs)]))

    def state():
        torch.cuda.synchronize()
        return (bm.refcount.cpu().numpy(), bm.free_stack.cpu().numpy()[:bm.top()], bm.lru_order(),
                bm.block_hash.cpu().numpy().view(np.uint64))

    run_eviction_example(serve, finish, state)


@pytest.mark.parametrize("seed,B,nb,rounds", [(0, 6, 40, 40), (1, 24, 90, 12), (2, 1100, 3000, 3)])
def test_cached_blocks_under_pressure_match_oracle(seed, B, nb, rounds):
    """Rounds of requests sharing system prompts on a pool too small to keep
    every prefix: lookups revive cached blocks, allocation evicts the least
    recently released, all requests finish between rounds.  The whole state,
    the eviction order included, is compared after every call."""
    rng = np.random.default_rng(seed)
    bs, mbs = 4, 8
    bm = pkv.BlockManager(nb)
    pc = pkv.PrefixCache(1 << 12)
    st = oracle.bm_init(nb)
    ocache = oracle.PrefixCache(1 << 12)
    systems = _systems(rng, bs, n_sys=6)
    hits = evictions_seen = 0
    for rnd in range(rounds):
        prompts = _prompts(rng, B, bs, systems)
        cached_before = len(st.lru_order())
        st, ocache, tables, ctx, cached = _serve_both(bm, pc, st, ocache, prompts, bs, mbs)
        bm.clear_error()
        hits += int((cached > 0).sum())
        evictions_seen += int(cached_before > len(st.lru_order()))
        ids = np.concatenate([tables[b, :(ctx[b] + bs - 1) // bs] for b in range(B) if ctx[b] > 0]).astype(np.int32)
        if len(ids):
            bm.free(_dev(ids))
            st, e = oracle.bm_free(st, ids)
            _same_state(bm, st, e)
            bm.clear_error()
    assert hits > 0 and evictions_seen > 0 and len(st.lru_order()) > 0


def test_alloc_takes_cached_blocks_after_the_free_stack():
    rng = np.random.default_rng(5)
    bs, B, mbs, nb = 4, 8, 6, 60
    bm = pkv.BlockManager(nb)
    pc = pkv.PrefixCache(256)
    st = oracle.bm_init(nb)
    ocache = oracle.PrefixCache(256)
    systems = _systems(rng, bs, n_sys=3)
    st, ocache, tables, ctx, _ = _serve_both(bm, pc, st, ocache, _prompts(rng, B, bs, systems), bs, mbs)
    ids = np.concatenate([tables[b, :(ctx[b] + bs - 1) // bs] for b in range(B)]).astype(np.int32)
    bm.free(_dev(ids))
    st, _ = oracle.bm_free(st, ids)
    _same_state(bm, st, 0)
    assert len(st.lru_order()) > 0
    counts = np.array([st.top, 2, 1, 3, 50], np.int32)  # the free stack, then cached blocks, then too many
    off, out_ids = bm.alloc(_dev(counts), 100)
    st, ooff, oids, e = oracle.bm_alloc(st, counts, 100)
    torch.cuda.synchronize()
    assert np.array_equal(off.cpu().numpy(), ooff)
    assert np.array_equal(out_ids.cpu().numpy()[:ooff[-1]], oids[:ooff[-1]])
    _same_state(bm, st, e)
    assert e == oracle.BM_ERR_NOSPACE


def test_eviction_ring_compacts_in_order():
    """The same prompts served and finished round after round on a pool large
    enough to evict nothing: every hit leaves a dead entry in the eviction
    ring and every release appends one, so the ring fills up and is compacted
    (its tail moves back); the order of the cached blocks stays the oracle's."""
    rng = np.random.default_rng(9)
    bs, mbs, nb = 4, 8, 40
    bm = pkv.BlockManager(nb)
    pc = pkv.PrefixCache(256)
    st = oracle.bm_init(nb)
    ocache = oracle.PrefixCache(256)
    prompts = _prompts(rng, 3, bs, _systems(rng, bs, n_sys=2))
    compactions = 0
    for rnd in range(60):
        st, ocache, tables, ctx, cached = _serve_both(bm, pc, st, ocache, prompts, bs, mbs)
        ids = np.concatenate([tables[b, :(ctx[b] + bs - 1) // bs] for b in range(len(prompts))]).astype(np.int32)
        tail_before = int(bm.header[4].item())
        bm.free(_dev(ids))
        st, e = oracle.bm_free(st, ids)
        _same_state(bm, st, e)
        compactions += int(int(bm.header[4].item()) < tail_before)
    assert compactions > 0
