"""Pins for the oracle's block manager (wkbse.com section 3.1; intelliparadigm.com
section 2.1, items 1-2 and the block-allocation sketch).

A hand-worked example fixes the allocation order and the copy-on-write rule;
a composition pin ties append_slots to the independently pinned kv_write,
copy_blocks and paged_attention (tokens written at the produced slots must be
exactly what each sequence's table walk attends over); invariants and a pure
Python restatement of the free rule cover the rest.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_block_manager_worked_example_golden():
    g = json.load(open(os.path.join(GOLDEN, "block_manager_example.json")))
    st = oracle.bm_init(g["num_blocks"])
    for step in g["steps"]:
        if step["op"] == "append":
            st, tables, ctx, slots, pairs, err = oracle.bm_append_slots(st, step["tables"], step["context_lens"],
                                                                         step["num_new"], g["block_size"])
            assert err == 0
            assert tables.tolist() == step["expect_tables"]
            assert ctx.tolist() == step["expect_context_lens"]
            assert slots.tolist() == step["expect_slots"]
            assert pairs.tolist() == step["expect_pairs"]
            assert st.top == step["expect_top"]
        elif step["op"] == "fork":
            st, err = oracle.bm_share(st, step["share"])
            assert err == 0
        elif step["op"] == "free":
            st, err = oracle.bm_free(st, step["ids"])
            assert err == 0 and st.top == step["expect_top"]
        elif step["op"] == "alloc":
            st, off, ids, err = oracle.bm_alloc(st, step["counts"], 16)
            assert err == 0 and ids[:off[-1]].tolist() == step["expect_ids"]
        if "expect_refcount" in step:
            assert st.refcount.tolist() == step["expect_refcount"]


def _random_run(seed, nb=64, bs=4, B=6, mbs=12, steps=12):
    """Random appends, forks and frees; yields the state after every step."""
    rng = np.random.default_rng(seed)
    st = oracle.bm_init(nb)
    tables = np.full((B, mbs), -1, np.int32)
    ctx = np.zeros(B, np.int32)
    for _ in range(steps):
        r = rng.random()
        if r < 0.6:
            nn = rng.integers(0, 7, B).astype(np.int32)
            st, tables, ctx, slots, pairs, err = oracle.bm_append_slots(st, tables, ctx, nn, bs)
        elif r < 0.8:
            a, b = rng.choice(B, 2, replace=False)
            held = (ctx[b] + bs - 1) // bs
            if held:
                st, _ = oracle.bm_free(st, tables[b, :held])
            nblk = (ctx[a] + bs - 1) // bs
            tables[b] = -1
            tables[b, :nblk] = tables[a, :nblk]
            ctx[b] = ctx[a]
            st, _ = oracle.bm_share(st, tables[a, :nblk])
        else:
            b = int(rng.integers(B))
            held = (ctx[b] + bs - 1) // bs
            st, _ = oracle.bm_free(st, tables[b, :held])
            tables[b] = -1
            ctx[b] = 0
        yield st, tables, ctx, bs


@pytest.mark.parametrize("seed", range(8))
def test_conservation_invariants(seed):
    for st, tables, ctx, bs in _random_run(seed):
        held = [tables[b, :(ctx[b] + bs - 1) // bs] for b in range(len(ctx))]
        mapped = np.concatenate(held) if held else np.zeros(0, np.int32)
        counts = np.bincount(mapped, minlength=st.num_blocks)
        assert np.array_equal(counts, st.refcount)                      # references = table entries
        free = st.free_stack[:st.top]
        assert len(set(free.tolist())) == st.top                          # no block listed twice
        assert set(free.tolist()) == set(np.flatnonzero(st.refcount == 0).tolist())


@pytest.mark.parametrize("seed", range(6))
def test_append_block_counts_closed_form(seed):
    rng = np.random.default_rng(100 + seed)
    bs, B, mbs, nb = 16, 8, 40, 400
    st = oracle.bm_init(nb)
    tables = np.full((B, mbs), -1, np.int32)
    ctx = np.zeros(B, np.int32)
    for _ in range(4):
        nn = rng.integers(0, 90, B).astype(np.int32)
        top0 = st.top
        st, t2, c2, slots, pairs, err = oracle.bm_append_slots(st, tables, ctx, nn, bs)
        assert err == 0 and len(pairs) == 0  # nothing shared
        need = sum(math.ceil((ctx[b] + nn[b]) / bs) - math.ceil(ctx[b] / bs) for b in range(B))
        assert top0 - st.top == need
        assert np.array_equal(c2, ctx + nn)
        tables, ctx = t2, c2


def test_slots_feed_the_table_walk():
    """Composition pin: after append_slots, applying the copy pairs and writing
    each new token at its slot, paged attention over every sequence equals
    dense attention over that sequence's own tokens."""
    rng = np.random.default_rng(7)
    import torch
    bs, Hkv, D, nb, mbs = 16, 2, 64, 40, 8
    st = oracle.bm_init(nb)
    B = 3
    tables = np.full((B, mbs), -1, np.int32)
    ctx = np.zeros(B, np.int32)
    kc = np.zeros((nb, Hkv, bs, D), np.uint16)
    vc = np.zeros_like(kc)
    toks_k = [[] for _ in range(B)]
    toks_v = [[] for _ in range(B)]

    def bf(x):
        return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)

    for step, nn in enumerate(([20, 5, 0], [1, 1, 0], "fork", [1, 1, 1], [3, 0, 17])):
        if nn == "fork":  # sequence 2 becomes a parallel sample of sequence 0
            nblk = (ctx[0] + bs - 1) // bs
            tables[2, :nblk] = tables[0, :nblk]
            ctx[2] = ctx[0]
            toks_k[2], toks_v[2] = list(toks_k[0]), list(toks_v[0])
            st, _ = oracle.bm_share(st, tables[0, :nblk])
            continue
        nn = np.array(nn, np.int32)
        st, tables, ctx2, slots, pairs, err = oracle.bm_append_slots(st, tables, ctx, nn, bs)
        assert err == 0
        if len(pairs):
            kc, vc = oracle.copy_blocks(kc, vc, pairs)
        T = int(nn.sum())
        k_new = bf(rng.standard_normal((T, Hkv, D)))
        v_new = bf(rng.standard_normal((T, Hkv, D)))
        kc, vc = oracle.kv_write(kc, vc, k_new, v_new, slots)
        o = 0
        for b in range(B):
            for t in range(nn[b]):
                toks_k[b].append(k_new[o])
                toks_v[b].append(v_new[o])
                o += 1
        ctx = ctx2
    q = bf(rng.standard_normal((B, 4, D)))
    scale = 1 / 8
    out = oracle.paged_attention(q, kc, vc, tables, ctx, scale)
    for b in range(B):
        K = oracle.bf16_bits_to_f64(np.stack(toks_k[b]))  # [n, Hkv, D]
        V = oracle.bf16_bits_to_f64(np.stack(toks_v[b]))
        Q = oracle.bf16_bits_to_f64(q[b])
        for h in range(4):
            z = float(np.float32(scale)) * K[:, h // 2] @ Q[h]
            w = np.exp(z - z.max())
            ref = (w[:, None] * V[:, h // 2]).sum(0) / w.sum()
            assert np.allclose(out[b, h], ref, atol=1e-12)


def _free_python(stack, top, ref, ids):
    stack, ref = list(stack[:top]), ref.copy()
    for b in ids:
        if ref[b] > 0:
            ref[b] -= 1
            if ref[b] == 0:
                stack.append(b)
    return stack, ref


@pytest.mark.parametrize("seed", range(6))
def test_free_matches_python_restatement(seed):
    rng = np.random.default_rng(seed)
    st = oracle.bm_init(30)
    st, off, ids, _ = oracle.bm_alloc(st, [20], 20)
    st, _ = oracle.bm_share(st, rng.choice(ids, 8))
    batch = rng.choice(ids, 25)  # repeats
    want_stack, want_ref = _free_python(st.free_stack, st.top, st.refcount, batch)
    st2, err = oracle.bm_free(st, batch)
    assert st2.free_stack[:st2.top].tolist() == want_stack
    assert np.array_equal(st2.refcount, want_ref)


def test_errors():
    st = oracle.bm_init(6)
    st, off, ids, err = oracle.bm_alloc(st, [4, 3, 1], 10)
    assert err & oracle.BM_ERR_NOSPACE and off.tolist() == [0, 4, 4, 4]  # in order: the later 1 is not served
    st, err = oracle.bm_free(st, [0, 0])
    assert err & oracle.BM_ERR_DOUBLEFREE and st.refcount[0] == 0 and st.free_set() >= {0}
    st, err = oracle.bm_free(st, [6])
    assert err & oracle.BM_ERR_RANGE
    tables = np.full((1, 2), -1, np.int32)
    st2, t2, c2, slots, pairs, err = oracle.bm_append_slots(st, tables, [0], [9], 4)
    assert err & oracle.BM_ERR_TABLE and slots.tolist() == [-1] * 9 and c2.tolist() == [0]
