"""Pins of the CPU oracle to things other than itself (no GPU needed).

Each test ties one oracle function to a fact fixed by the pages or by the
mathematics: a count the pages print, a closed form, an invariant the paged
layout must satisfy (placement freedom, sharing, copy-on-write), a library
routine for the dense special case, or brute force on tiny inputs.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(x) -> np.ndarray:
    """float array -> bf16 bit patterns (round to nearest even, via torch)."""
    t = torch.from_numpy(np.array(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _f64(b) -> np.ndarray:
    return oracle.bf16_bits_to_f64(b)


def _rand_bits(rng, shape):
    return _bf16(rng.standard_normal(shape))


def _paged_from_dense(rng, dense_k, dense_v, bs, extra_blocks=3):
    """Scatters per-sequence dense K/V ([n_s, Hkv, d] bf16 bits each) into a
    paged pool with shuffled physical ids, using the oracle's write.
    Returns (k_cache, v_cache, tables)."""
    Hkv, d = dense_k[0].shape[1], dense_k[0].shape[2]
    nblk = [(k.shape[0] + bs - 1) // bs for k in dense_k]
    NB = sum(nblk) + extra_blocks
    perm = rng.permutation(NB)
    mbs = max(nblk + [1])
    tables = np.full((len(dense_k), mbs), -1, dtype=np.int32)
    k_cache = _bf16(np.full((NB, Hkv, bs, d), np.nan))
    v_cache = k_cache.copy()
    j = 0
    for s, k in enumerate(dense_k):
        tables[s, :nblk[s]] = perm[j:j + nblk[s]]
        j += nblk[s]
        n = k.shape[0]
        pos = np.arange(n)
        slots = tables[s, pos // bs].astype(np.int64) * bs + pos % bs
        k_cache, v_cache = oracle.kv_write(k_cache, v_cache, k, dense_v[s], slots)
    return k_cache, v_cache, tables


# --------------------------------------------------------------------------
# block count and addressing
# --------------------------------------------------------------------------

def test_block_count_golden():
    g = json.load(open(os.path.join(GOLDEN, "block_count.json")))
    for case in g["cases"]:
        n, bs, nb = case["tokens"], case["block_size"], case["blocks"]
        w = workloads.make_custom([n], 1, 1, 64, bs, seed=1)
        assert int((w.block_tables[0] >= 0).sum()) == nb
        # the oracle reads exactly `nb` table entries: poisoning the ones after
        # them changes nothing, poisoning the last one makes the read fail
        tables = np.full((1, nb + 2), -7, dtype=np.int32)
        tables[0, :nb] = w.block_tables[0, :nb]
        ctx = np.array([n], np.int32)
        out = oracle.paged_attention(w.q, w.k_cache, w.v_cache, tables, ctx, w.scale)
        assert np.isfinite(out).all()
        tables[0, nb - 1] = -7
        with pytest.raises(IndexError):
            oracle.paged_attention(w.q, w.k_cache, w.v_cache, tables, ctx, w.scale)


def test_write_roundtrip_and_untouched_rows():
    rng = np.random.default_rng(3)
    NB, Hkv, bs, d, T = 9, 3, 16, 64, 40
    kc, vc = _rand_bits(rng, (NB, Hkv, bs, d)), _rand_bits(rng, (NB, Hkv, bs, d))
    k, v = _rand_bits(rng, (T, Hkv, d)), _rand_bits(rng, (T, Hkv, d))
    slots = rng.choice(NB * bs, size=T, replace=False).astype(np.int64)
    slots[[3, 17]] = -1  # padding tokens
    kc2, vc2 = oracle.kv_write(kc, vc, k, v, slots)
    written = np.zeros((NB, bs), bool)
    for t, s in enumerate(slots):
        if s < 0:
            continue
        # numpy's own 4-D indexing of the [NB][Hkv][bs][d] layout
        assert np.array_equal(kc2[s // bs, :, s % bs, :], k[t])
        assert np.array_equal(vc2[s // bs, :, s % bs, :], v[t])
        written[s // bs, s % bs] = True
    keep = ~written
    assert np.array_equal(kc2.transpose(0, 2, 1, 3)[keep], kc.transpose(0, 2, 1, 3)[keep])
    assert np.array_equal(vc2.transpose(0, 2, 1, 3)[keep], vc.transpose(0, 2, 1, 3)[keep])
    # padding tokens left no trace anywhere
    for t in (3, 17):
        assert not (kc2 == k[t][None, :, None, :]).all(axis=(1, 3)).any()


def test_write_rejects_out_of_range_slot():
    rng = np.random.default_rng(4)
    kc = _rand_bits(rng, (2, 1, 16, 64))
    k = _rand_bits(rng, (1, 1, 64))
    with pytest.raises(IndexError):
        oracle.kv_write(kc, kc, k, k, np.array([2 * 16], np.int64))


# --------------------------------------------------------------------------
# copy-on-write
# --------------------------------------------------------------------------

def test_copy_blocks_simultaneous_semantics():
    rng = np.random.default_rng(5)
    NB, Hkv, bs, d = 8, 2, 16, 64
    kc, vc = _rand_bits(rng, (NB, Hkv, bs, d)), _rand_bits(rng, (NB, Hkv, bs, d))
    pairs = np.array([[0, 1], [1, 2], [5, 4], [5, 7]], np.int32)  # chain and fan-out
    kc2, vc2 = oracle.copy_blocks(kc, vc, pairs)
    ek, ev = kc.copy(), vc.copy()
    ek[pairs[:, 1]] = kc[pairs[:, 0]]  # numpy fancy assignment reads all sources first
    ev[pairs[:, 1]] = vc[pairs[:, 0]]
    assert np.array_equal(kc2, ek) and np.array_equal(vc2, ev)
    assert np.array_equal(kc2[2], kc[1])  # old contents of block 1, not the new ones


def test_copy_on_write_isolates_sharers():
    """After copying shared block b -> b' and writing a token into b', the
    sequences that still map b see unchanged outputs (intelliparadigm.com,
    section 2.1 item 2: COW for shared prefixes)."""
    rng = np.random.default_rng(6)
    Hkv, Hq, bs, d = 2, 4, 16, 64
    NB = 6
    kc, vc = _rand_bits(rng, (NB, Hkv, bs, d)), _rand_bits(rng, (NB, Hkv, bs, d))
    q = _rand_bits(rng, (2, Hq, d))
    tables = np.array([[0, 1], [0, 1]], np.int32)  # both share blocks 0 and 1
    ctx = np.array([25, 25], np.int32)
    before = oracle.paged_attention(q, kc, vc, tables, ctx, 0.125)
    kc2, vc2 = oracle.copy_blocks(kc, vc, np.array([[1, 4]], np.int32))
    tables2 = np.array([[0, 1], [0, 4]], np.int32)
    kn, vn = _rand_bits(rng, (1, Hkv, d)), _rand_bits(rng, (1, Hkv, d))
    # position 24 = logical block 1 (now physical 4), offset 8
    kc2, vc2 = oracle.kv_write(kc2, vc2, kn, vn, np.array([4 * bs + 8], np.int64))
    after = oracle.paged_attention(q, kc2, vc2, tables2, ctx, 0.125)
    assert np.array_equal(after[0], before[0])
    assert not np.allclose(after[1], before[1])
    # the forked sequence equals a fresh dense computation with the new token
    k1 = np.concatenate([kc[0], kc[1]], axis=1)[:, :25].copy()
    v1 = np.concatenate([vc[0], vc[1]], axis=1)[:, :25].copy()
    k1[:, 24] = kn[0]
    v1[:, 24] = vn[0]
    for hq in range(Hq):
        h = hq // (Hq // Hkv)
        z = 0.125 * _f64(k1[h]) @ _f64(q[1, hq])
        expect = scipy.special.softmax(z) @ _f64(v1[h])
        np.testing.assert_allclose(after[1, hq], expect, rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------

@pytest.mark.parametrize("lens,Hq,Hkv,d,bs", [
    ([1, 17, 33, 64], 4, 4, 64, 16),
    ([5, 16, 31, 48, 100], 8, 2, 64, 16),
    ([40, 129, 7], 8, 1, 128, 32),
    ([300, 45], 6, 3, 128, 128),
])
def test_attention_equals_dense_library_softmax(lens, Hq, Hkv, d, bs):
    """The paged result equals textbook dense attention on the same tokens laid
    out contiguously (wkbse.com section 3.1: the kernel reads the same K/V
    through the block table)."""
    rng = np.random.default_rng(sum(lens) + Hq)
    dense_k = [_rand_bits(rng, (n, Hkv, d)) for n in lens]
    dense_v = [_rand_bits(rng, (n, Hkv, d)) for n in lens]
    q = _rand_bits(rng, (len(lens), Hq, d))
    kc, vc, tables = _paged_from_dense(rng, dense_k, dense_v, bs)
    scale = float(np.float32(1 / math.sqrt(d)))
    out = oracle.paged_attention(q, kc, vc, tables, np.array(lens, np.int32), scale)
    g = Hq // Hkv
    for s, n in enumerate(lens):
        for hq in range(Hq):
            K = _f64(dense_k[s][:, hq // g, :])
            V = _f64(dense_v[s][:, hq // g, :])
            w = scipy.special.softmax(scale * (K @ _f64(q[s, hq])))
            np.testing.assert_allclose(out[s, hq], w @ V, rtol=1e-11, atol=1e-12)


def test_attention_equals_torch_sdpa_gqa():
    """Second library routine: torch's scaled_dot_product_attention in fp64
    with grouped KV heads."""
    rng = np.random.default_rng(11)
    lens, Hq, Hkv, d, bs = [70, 3, 48], 8, 2, 64, 16
    dense_k = [_rand_bits(rng, (n, Hkv, d)) for n in lens]
    dense_v = [_rand_bits(rng, (n, Hkv, d)) for n in lens]
    q = _rand_bits(rng, (len(lens), Hq, d))
    kc, vc, tables = _paged_from_dense(rng, dense_k, dense_v, bs)
    out = oracle.paged_attention(q, kc, vc, tables, np.array(lens, np.int32), 0.125)
    for s, n in enumerate(lens):
        Q = torch.from_numpy(_f64(q[s]))[None, :, None, :]  # [1, Hq, 1, d]
        K = torch.from_numpy(_f64(dense_k[s])).permute(1, 0, 2)[None]  # [1, Hkv, n, d]
        V = torch.from_numpy(_f64(dense_v[s])).permute(1, 0, 2)[None]
        ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, scale=0.125, enable_gqa=True)
        np.testing.assert_allclose(out[s], ref[0, :, 0, :].numpy(), rtol=1e-11, atol=1e-12)


def test_permutation_of_physical_blocks_changes_nothing():
    """Blocks may sit anywhere in the pool (wkbse.com section 3.1): moving
    every block to another physical id and renaming the table entries
    leaves the output bit-identical."""
    w = workloads.make("tiny", seed=2)
    kc, vc, out = oracle.decode_step(w)
    rng = np.random.default_rng(9)
    pi = rng.permutation(w.num_blocks)
    kp, vp = np.empty_like(kc), np.empty_like(vc)
    kp[pi] = kc
    vp[pi] = vc
    tp = np.where(w.block_tables >= 0, pi[np.maximum(w.block_tables, 0)], -1).astype(np.int32)
    out2 = oracle.paged_attention(w.q, kp, vp, tp, w.context_lens, w.scale)
    assert np.array_equal(out, out2)


def test_shared_prefix_blocks_equal_duplicated_blocks():
    """Tables that point at the same physical prefix blocks give exactly the
    result of private copies of those blocks (block sharing, wkbse.com 3.1;
    intelliparadigm.com 2.1)."""
    w = workloads.make_custom([70, 70, 90, 40], 4, 2, 64, 16, seed=5,
                              share_prefix_tokens=64, group_size=4)
    t = w.block_tables
    assert (t[0, :4] == t[1, :4]).all() and (t[0, :2] == t[3, :2]).all()
    kc, vc = oracle.bits(w.k_cache), oracle.bits(w.v_cache)
    out = oracle.paged_attention(w.q, kc, vc, t, w.context_lens, w.scale)
    # duplicate every shared block into fresh ids
    NB = w.num_blocks
    t2 = t.copy()
    extra_k, extra_v = [], []
    seen = set()
    for s in range(1, w.num_seqs):
        for j in range(t.shape[1]):
            b = int(t[s, j])
            if b >= 0 and (b in set(t[:s].ravel().tolist()) or b in seen):
                t2[s, j] = NB + len(extra_k)
                extra_k.append(kc[b])
                extra_v.append(vc[b])
    kc2 = np.concatenate([kc, np.stack(extra_k)])
    vc2 = np.concatenate([vc, np.stack(extra_v)])
    out2 = oracle.paged_attention(w.q, kc2, vc2, t2, w.context_lens, w.scale)
    assert np.array_equal(out, out2)
    # same suffix data and same q through shared blocks -> same output
    q_same = oracle.bits(w.q).copy()
    q_same[1] = q_same[0]
    out3 = oracle.paged_attention(q_same, kc, vc, t, np.array([64, 64, 90, 40], np.int32), w.scale)
    assert np.array_equal(out3[0], out3[1])


def test_uniform_attention_gives_mean_of_v():
    rng = np.random.default_rng(12)
    NB, Hkv, bs, d, Hq = 6, 2, 16, 64, 4
    kc = np.broadcast_to(_rand_bits(rng, (1, Hkv, 1, d)), (NB, Hkv, bs, d)).copy()
    vc = _rand_bits(rng, (NB, Hkv, bs, d))
    q = _rand_bits(rng, (2, Hq, d))
    tables = np.array([[3, 1, 4], [0, 5, 2]], np.int32)
    ctx = np.array([37, 20], np.int32)
    out = oracle.paged_attention(q, kc, vc, tables, ctx, 0.3)
    g = Hq // Hkv
    for s in range(2):
        rows = [vc[tables[s, i // bs], :, i % bs, :] for i in range(ctx[s])]
        mean = _f64(np.stack(rows)).mean(axis=0)  # [Hkv, d]
        for hq in range(Hq):
            np.testing.assert_allclose(out[s, hq], mean[hq // g], rtol=1e-13, atol=1e-14)
    # q = 0 and scale = 0 give the same closed form with arbitrary keys
    kc_r = _rand_bits(rng, (NB, Hkv, bs, d))
    out_q0 = oracle.paged_attention(np.zeros_like(q), kc_r, vc, tables, ctx, 0.3)
    out_s0 = oracle.paged_attention(q, kc_r, vc, tables, ctx, 0.0)
    np.testing.assert_allclose(out_q0, out, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(out_s0, out, rtol=1e-13, atol=1e-14)


def test_single_token_gives_its_value_row_exactly():
    w = workloads.make("tiny", seed=0)
    kc, vc, out = oracle.decode_step(w)
    assert w.context_lens[0] == 1
    b = w.block_tables[0, 0]
    for hq in range(w.num_q_heads):
        assert np.array_equal(out[0, hq], _f64(vc[b, hq, 0]))
        assert np.array_equal(out[0, hq], _f64(oracle.bits(w.v_new)[0, hq]))


def test_one_hot_attention_selects_one_value_row():
    rng = np.random.default_rng(13)
    Hkv, bs, d = 1, 16, 64
    kc = _bf16(0.01 * rng.standard_normal((3, Hkv, bs, d)))
    vc = _rand_bits(rng, (3, Hkv, bs, d))
    q = _bf16(np.ones((1, 1, d)))
    kc[2, 0, 5] = _bf16(np.full(d, 4.0))  # score 256*scale vs ~0 elsewhere
    out = oracle.paged_attention(q, kc, vc, np.array([[1, 2, 0]], np.int32), np.array([40], np.int32), 1.0)
    np.testing.assert_allclose(out[0, 0], _f64(vc[2, 0, 5]), rtol=0, atol=1e-12)


def test_gqa_head_mapping_is_contiguous_groups():
    """hkv = hq // (Hq/Hkv): kv head h holds the constant value h+1 in V, so the
    output of query head hq is exactly hq // g + 1."""
    rng = np.random.default_rng(14)
    NB, Hkv, bs, d, Hq = 4, 2, 16, 64, 8
    kc = _rand_bits(rng, (NB, Hkv, bs, d))
    vc = _bf16(np.broadcast_to(np.arange(1, Hkv + 1, dtype=np.float32)[None, :, None, None], (NB, Hkv, bs, d)))
    q = _rand_bits(rng, (1, Hq, d))
    out = oracle.paged_attention(q, kc, vc, np.array([[2, 0, 3]], np.int32), np.array([45], np.int32), 0.125)
    for hq in range(Hq):
        np.testing.assert_allclose(out[0, hq], hq // (Hq // Hkv) + 1, rtol=1e-14)


def test_two_token_closed_form_golden():
    g = json.load(open(os.path.join(GOLDEN, "attention_two_tokens.json")))
    d, bs = g["head_dim"], g["block_size"]
    kc = _bf16(np.zeros((1, 1, bs, d)))
    vc = kc.copy()
    kc[0, 0, :2] = _bf16(g["k"])
    vc[0, 0, :2] = _bf16(g["v"])
    q = _bf16(np.array(g["q"]).reshape(1, 1, d))
    out = oracle.paged_attention(q, kc, vc, np.array([[0]], np.int32), np.array([2], np.int32), g["scale"])
    np.testing.assert_allclose(out[0, 0], g["out"], rtol=1e-15)


def test_context_len_zero_gives_zero_output():
    w = workloads.make_custom([20, 5], 2, 2, 64, 16, seed=1)
    out = oracle.paged_attention(w.q, w.k_cache, w.v_cache, w.block_tables,
                                 np.array([0, 5], np.int32), w.scale)
    assert (out[0] == 0).all() and np.abs(out[1]).sum() > 0


def test_brute_force_pure_python_tiny():
    """Independent pure-Python brute force (math.exp, Python floats, token
    lookup through the table by hand) on the tiny workload."""
    w = workloads.make("tiny", seed=4)
    kc, vc, out = oracle.decode_step(w)
    qf = _f64(oracle.bits(w.q))
    kf, vf = _f64(kc), _f64(vc)
    bs = w.block_size
    for s in range(w.num_seqs):
        n = int(w.context_lens[s])
        for hq in range(w.num_q_heads):
            h = hq * w.num_kv_heads // w.num_q_heads
            scores = []
            for i in range(n):
                blk = int(w.block_tables[s][i // bs])
                row = kf[blk][h][i % bs]
                scores.append(w.scale * sum(float(a) * float(b) for a, b in zip(qf[s][hq], row)))
            top = max(scores)
            ws = [math.exp(z - top) for z in scores]
            tot = sum(ws)
            for c in range(0, w.head_dim, 7):
                val = sum(ws[i] * float(vf[int(w.block_tables[s][i // bs])][h][i % bs][c]) for i in range(n)) / tot
                assert abs(val - out[s, hq, c]) <= 1e-12 * (1 + abs(val))


# --------------------------------------------------------------------------
# split-K log-sum-exp merge
# --------------------------------------------------------------------------

@pytest.mark.parametrize("psize", [16, 512, None, "ragged"])
def test_split_merge_equals_unsplit(psize):
    w = workloads.make_custom([1000, 16, 513], 4, 2, 64, 16, seed=8)
    kc, vc = oracle.bits(w.k_cache), oracle.bits(w.v_cache)
    full = oracle.paged_attention(w.q, kc, vc, w.block_tables, w.context_lens, w.scale)
    rng = np.random.default_rng(1)
    for s in range(w.num_seqs):
        n = int(w.context_lens[s])
        if psize is None:
            cuts = [0, n]
        elif psize == "ragged":
            cuts = sorted(set([0, n] + rng.integers(0, n + 1, size=5).tolist()))
        else:
            cuts = list(range(0, n, psize)) + [n]
        for hq in range(w.num_q_heads):
            parts = [oracle.attention_partial(oracle.bits(w.q)[s, hq], kc, vc, w.block_tables[s],
                                              w.num_q_heads, hq, a, b, w.scale)
                     for a, b in zip(cuts[:-1], cuts[1:])]
            parts.append(oracle.attention_partial(oracle.bits(w.q)[s, hq], kc, vc, w.block_tables[s],
                                                  w.num_q_heads, hq, n, n, w.scale))  # empty piece
            m = [p[0] for p in parts]
            l = [p[1] for p in parts]
            acc = np.stack([p[2] for p in parts])
            merged = oracle.lse_merge(m, l, acc)
            np.testing.assert_allclose(merged, full[s, hq], rtol=1e-12, atol=1e-13)


def test_lse_merge_closed_form():
    """Two single-token pieces with scores 0 and ln 3 weigh their rows 1:3."""
    m = [0.0, math.log(3.0)]
    l = [1.0, 1.0]
    acc = np.array([[1.0, 0.0], [0.0, 1.0]])
    np.testing.assert_allclose(oracle.lse_merge(m, l, acc), [0.25, 0.75], rtol=1e-15)
