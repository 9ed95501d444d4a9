"""Pins for the oracle's prefix cache (intelliparadigm.com section 3.1,
--enable-prefix-caching; section 2.1's allocation sketch shares a block whose
prefix matches).  The hash is pinned by FNV-1a's published test vectors; the
cache by a worked example, by the chaining (equal block contents under
different prefixes do not match), by the cached state of released keyed
blocks and their least-recently-released eviction (a second worked example),
and by a composition pin: a prompt served partly from the cache attends to
exactly its own tokens."""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
BS = 4


def test_fnv1a64_published_vectors():
    g = json.load(open(os.path.join(GOLDEN, "fnv1a64_vectors.json")))
    for v in g["vectors"]:
        assert oracle.fnv1a64(v["ascii"].encode()) == int(v["fnv1a64"], 16)


def test_keys_chain_over_the_prefix():
    a = np.arange(12, dtype=np.int32)
    b = a.copy()
    b[1] = 99  # differs only in block 0
    ka, kb = oracle.prefix_keys(a, BS), oracle.prefix_keys(b, BS)
    assert len(ka) == 3 and np.all(ka != kb)  # block 1 and 2 contents equal, keys differ through the chain
    assert np.array_equal(oracle.prefix_keys(a[:8], BS), ka[:2])  # a key depends only on its prefix
    # the block digest covers every byte of every token
    c = a.copy()
    c[5] += 1 << 24
    assert oracle.prefix_keys(c, BS)[0] == ka[0] and oracle.prefix_keys(c, BS)[1] != ka[1]


def _serve(st, cache, prompts, mbs=8):
    """Lookup, then blocks for the rest through append_slots, then insert."""
    tokens = np.concatenate(prompts).astype(np.int32)
    qs = np.concatenate([[0], np.cumsum([len(p) for p in prompts])]).astype(np.int32)
    B = len(prompts)
    tables = np.full((B, mbs), -1, np.int32)
    st, tables, cached = oracle.prefix_lookup(st, cache, tokens, qs, BS, tables)
    need = np.array([len(p) for p in prompts], np.int32) - cached
    st, tables, ctx, slots, pairs, err = oracle.bm_append_slots(st, tables, cached, need, BS)
    assert err == 0 and len(pairs) == 0
    st, cache, err = oracle.prefix_insert(st, cache, tokens, qs, BS, tables)
    assert err == 0
    return st, cache, tables, ctx, cached, slots


def test_worked_example():
    st = oracle.bm_init(32)
    cache = oracle.PrefixCache(64)
    sys_prompt = [7, 7, 8, 9, 1, 2, 3, 4]  # two blocks
    p0 = np.array(sys_prompt + [10, 11, 12], np.int32)
    st, cache, t0, _, c0, _ = _serve(st, cache, [p0])
    assert c0.tolist() == [0] and t0[0, :3].tolist() == [0, 1, 2]
    # a second request with the same two-block system prompt maps blocks 0 and 1
    p1 = np.array(sys_prompt + [20, 21, 22, 23, 24], np.int32)
    st, cache, t1, _, c1, _ = _serve(st, cache, [p1])
    assert c1.tolist() == [8] and t1[0, :2].tolist() == [0, 1] and t1[0, 2:4].tolist() == [3, 4]
    assert st.refcount[:5].tolist() == [2, 2, 1, 1, 1]
    # a request that differs in the second block shares only the first
    p2 = np.array([7, 7, 8, 9, 1, 2, 3, 5, 6], np.int32)
    st, cache, t2, _, c2, _ = _serve(st, cache, [p2])
    assert c2.tolist() == [4] and t2[0, 0] == 0 and t2[0, 1] not in (1,)
    # a prompt that is exactly the two cached blocks keeps its last block to compute
    st, cache, t3, _, c3, _ = _serve(st, cache, [np.array(sys_prompt, np.int32)])
    assert c3.tolist() == [4]


def _key_names(prompts, bs):
    """Key value -> name <prompt><block index> for every full block of the prompts."""
    names = {}
    for name, p in prompts.items():
        for i, k in enumerate(oracle.prefix_keys(np.asarray(p, np.int32), bs)):
            names.setdefault(int(k), f"{name}{i}")
    return names


def run_eviction_example(serve, finish, state):
    """Replays the cached-block worked example through serve(prompt) ->
    (num_cached, table row, err) and finish(table row, n_tokens); state() ->
    (refcount, free stack [:top], lru order, block_hash)."""
    g = json.load(open(os.path.join(GOLDEN, "prefix_eviction_example.json")))
    names = _key_names(g["prompts"], g["block_size"])
    rows = {}
    for step in g["steps"]:
        prompt = np.asarray(g["prompts"][step["prompt"]], np.int32)
        if step["op"] == "serve":
            cached, row, err = serve(prompt)
            n_blk = -(-len(prompt) // g["block_size"])
            assert cached == step["expect_cached"], step
            assert list(row[:n_blk]) == step["expect_table"], step
            assert err == step["expect_err"], step
            rows[step["prompt"]] = row
        else:
            finish(rows[step["prompt"]], len(prompt))
        refcount, free, lru, block_hash = state()
        assert list(refcount) == step["expect_refcount"], step
        assert list(free) == step["expect_free"], step
        assert list(lru) == step["expect_lru"], step
        keys = {str(b): names[int(h)] for b, h in enumerate(block_hash) if h}
        assert keys == step["expect_keys"], step
    return g


def test_cached_blocks_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "prefix_eviction_example.json")))
    bs = g["block_size"]
    box = {"st": oracle.bm_init(g["num_blocks"]), "cache": oracle.PrefixCache(g["cache_capacity"])}

    def serve(prompt):
        tokens = prompt.astype(np.int32)
        qs = np.array([0, len(prompt)], np.int32)
        tables = np.full((1, 8), -1, np.int32)
        st, tables, cached = oracle.prefix_lookup(box["st"], box["cache"], tokens, qs, bs, tables)
        need = np.array([len(prompt)], np.int32) - cached
        st, tables, ctx, slots, pairs, err = oracle.bm_append_slots(st, tables, cached, need, bs)
        st, box["cache"], e2 = oracle.prefix_insert(st, box["cache"], tokens, qs, bs, tables)
        box["st"] = st
        return int(cached[0]), tables[0], err | e2

    def finish(row, n):
        box["st"], err = oracle.bm_free(box["st"], row[:-(-n // bs)])
        assert err == 0

    def state():
        st = box["st"]
        return st.refcount, st.free_stack[:st.top], st.lru_order(), st.block_hash

    run_eviction_example(serve, finish, state)


def test_release_keeps_the_key_and_share_revives():
    """A keyed block whose count reaches zero keeps its key and joins the
    eviction order; mapping it again (a fork) takes it off; an unkeyed block
    returns to the free stack."""
    st = oracle.bm_init(16)
    cache = oracle.PrefixCache(32)
    p = np.arange(9, dtype=np.int32)
    st, cache, t, ctx, _, _ = _serve(st, cache, [p])
    keys = oracle.prefix_keys(p, BS)
    st, _ = oracle.bm_free(st, t[0, :3])
    assert np.array_equal(st.block_hash[t[0, :2]], keys)
    assert st.lru_order().tolist() == t[0, :2].tolist()
    assert int(t[0, 2]) in st.free_set() and st.block_hash[t[0, 2]] == 0
    st, err = oracle.bm_share(st, t[0, 1:2])
    assert err == 0 and st.lru_order().tolist() == [int(t[0, 0])] and st.refcount[t[0, 1]] == 1
    st2, cache2, t2, _, cached, _ = _serve(st, cache, [p])
    assert cached.tolist() == [8] and t2[0, :2].tolist() == t[0, :2].tolist()
    assert st2.lru_order().tolist() == [] and st2.refcount[t[0, 0]] == 1 and st2.refcount[t[0, 1]] == 2


def test_allocation_evicts_least_recently_released_first():
    """With the free stack empty, bm_alloc hands out cached blocks in release
    order and drops their keys; a lookup of an evicted prefix then misses."""
    st = oracle.bm_init(4)
    cache = oracle.PrefixCache(16)
    prompts = [np.arange(5, dtype=np.int32) + 100 * i for i in range(2)]  # one full block each, 2 blocks
    st, cache, t, ctx, _, _ = _serve(st, cache, prompts)
    assert st.top == 0
    st, _ = oracle.bm_free(st, [t[1, 0], t[1, 1], t[0, 0], t[0, 1]])  # prompt 1's keyed block is released first
    assert st.lru_order().tolist() == [int(t[1, 0]), int(t[0, 0])]
    assert sorted(st.free_set()) == sorted([int(t[1, 1]), int(t[0, 1])])
    st, off, ids, err = oracle.bm_alloc(st, [3], 8)
    assert err == 0 and ids[:3].tolist() == [int(t[0, 1]), int(t[1, 1]), int(t[1, 0])]
    assert st.block_hash[t[1, 0]] == 0 and st.block_hash[t[0, 0]] != 0 and st.lru_order().tolist() == [int(t[0, 0])]
    tables = np.full((2, 8), -1, np.int32)
    tokens = np.concatenate(prompts)
    qs = np.array([0, 5, 10], np.int32)
    _, _, cached = oracle.prefix_lookup(st, cache, tokens, qs, BS, tables)
    assert cached.tolist() == [4, 0]  # prompt 0's block is still cached, prompt 1's was evicted
    st, off, ids, err = oracle.bm_alloc(st, [2], 8)  # one cached block left: the request does not fit
    assert err == oracle.BM_ERR_NOSPACE and off.tolist() == [0, 0]


def test_first_sequence_in_order_becomes_holder():
    st = oracle.bm_init(32)
    cache = oracle.PrefixCache(64)
    p = np.arange(10, dtype=np.int32)
    st, cache, t, _, cached, _ = _serve(st, cache, [p, p.copy()])  # same prompt twice in one batch: both miss
    assert cached.tolist() == [0, 0]
    first = t[0, :2]
    assert np.array_equal(st.block_hash[first], oracle.prefix_keys(p, BS)[:2])
    assert np.all(st.block_hash[t[1, :2]] == 0)
    st, cache, t2, _, cached, _ = _serve(st, cache, [p])
    assert cached.tolist() == [8] and np.array_equal(t2[0, :2], first)


def test_cached_prompt_attends_to_its_own_tokens():
    """Composition pin: prompts served partly from the cache (K/V written only
    for the uncached tokens) give the same attention as dense attention over
    each prompt's own K/V."""
    rng = np.random.default_rng(3)
    import torch
    NB, Hkv, D = 40, 2, 32
    kc = np.zeros((NB, Hkv, BS, D), np.uint16)
    vc = np.zeros_like(kc)
    st = oracle.bm_init(NB)
    cache = oracle.PrefixCache(128)
    vocab_k = rng.standard_normal((50, Hkv, D)).astype(np.float32)  # K/V of a token is a function of the token
    vocab_v = rng.standard_normal((50, Hkv, D)).astype(np.float32)

    def bf(x):
        return torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)

    shared = rng.integers(0, 50, 8)
    prompts = [np.concatenate([shared, rng.integers(0, 50, n)]).astype(np.int32) for n in (3, 6, 1)]
    for batch in ([prompts[0]], [prompts[1], prompts[2]]):
        st, cache, tables, ctx, cached, slots = _serve(st, cache, batch)
        new_tok = np.concatenate([p[c:] for p, c in zip(batch, cached)])
        kc, vc = oracle.kv_write(kc, vc, bf(vocab_k[new_tok]), bf(vocab_v[new_tok]), slots)
        q = bf(rng.standard_normal((len(batch), 4, D)).astype(np.float32))
        out = oracle.paged_attention(q, kc, vc, tables, ctx, 0.25)
        for b, p in enumerate(batch):
            K = oracle.bf16_bits_to_f64(bf(vocab_k[p]))
            V = oracle.bf16_bits_to_f64(bf(vocab_v[p]))
            Q = oracle.bf16_bits_to_f64(q[b])
            for h in range(4):
                z = 0.25 * K[:, h // 2] @ Q[h]
                w = np.exp(z - z.max())
                assert np.allclose(out[b, h], (w[:, None] * V[:, h // 2]).sum(0) / w.sum(), atol=1e-12)
    assert cached.tolist() == [8, 8]
