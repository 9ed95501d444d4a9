"""Pins of the oracle's chunked-prefill attention (no GPU).

A chunk of q_len new tokens at the end of a sequence of ctx tokens: query row
i is at position ctx - q_len + i and sees positions [0, pos] (a token sees
itself and its past).  Pinned against torch's scaled_dot_product_attention in
fp64 with an explicit bottom-right causal mask on the same tokens laid out
densely, and against pure-Python brute force.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads


def _dense(w, kc, vc, s):
    """Dense K/V [Hkv, ctx, d] of sequence s, gathered with numpy's own 4-D
    indexing of the pool."""
    n = int(w.context_lens[s])
    pos = np.arange(n)
    blk = w.block_tables[s, pos // w.block_size]
    k = oracle.bf16_bits_to_f64(kc[blk, :, pos % w.block_size, :])  # [n, Hkv, d]
    v = oracle.bf16_bits_to_f64(vc[blk, :, pos % w.block_size, :])
    return k.transpose(1, 0, 2), v.transpose(1, 0, 2)


@pytest.mark.parametrize("prefix,chunk,Hq,Hkv,d,bs", [
    ([0, 5, 40], [7, 16, 33], 4, 4, 64, 16),
    ([100, 0], [64, 1], 8, 2, 128, 32),
    ([31, 17, 0, 64], [1, 20, 48, 3], 6, 3, 64, 16),
])
def test_prefill_equals_sdpa_with_bottom_right_causal_mask(prefix, chunk, Hq, Hkv, d, bs):
    w = workloads.make_prefill_custom(prefix, chunk, Hq, Hkv, d, bs, seed=sum(prefix) + Hq)
    kc, vc = oracle.kv_write(w.k_cache, w.v_cache, w.k_new, w.v_new, w.slot_mapping)
    out = oracle.paged_prefill(w.q, kc, vc, w.block_tables, w.context_lens, w.query_start, w.scale)
    q = oracle.bf16_bits_to_f64(oracle.bits(w.q))
    for s in range(w.num_seqs):
        a, b = int(w.query_start[s]), int(w.query_start[s + 1])
        L, S = b - a, int(w.context_lens[s])
        if L == 0:
            continue
        K, V = _dense(w, kc, vc, s)
        # query i may see key j iff j <= S - L + i (bottom-right aligned)
        mask = torch.from_numpy(np.arange(S)[None, :] <= (S - L + np.arange(L))[:, None])
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[a:b]).permute(1, 0, 2)[None], torch.from_numpy(K)[None], torch.from_numpy(V)[None],
            attn_mask=mask, scale=float(np.float32(w.scale)), enable_gqa=True)
        np.testing.assert_allclose(out[a:b], ref[0].permute(1, 0, 2).numpy(), rtol=1e-11, atol=1e-12)


def test_prefill_single_token_chunks_equal_decode():
    w = workloads.make_prefill_custom([10, 33, 0], [1, 1, 1], 8, 4, 64, 16, seed=3)
    kc, vc = oracle.kv_write(w.k_cache, w.v_cache, w.k_new, w.v_new, w.slot_mapping)
    a = oracle.paged_prefill(w.q, kc, vc, w.block_tables, w.context_lens, w.query_start, w.scale)
    b = oracle.paged_attention(w.q, kc, vc, w.block_tables, w.context_lens, w.scale)
    assert np.array_equal(a, b)


def test_prefill_brute_force_python():
    w = workloads.make_prefill_custom([3, 0], [5, 4], 2, 1, 64, 16, seed=5)
    kc, vc = oracle.kv_write(w.k_cache, w.v_cache, w.k_new, w.v_new, w.slot_mapping)
    out = oracle.paged_prefill(w.q, kc, vc, w.block_tables, w.context_lens, w.query_start, w.scale)
    qf = oracle.bf16_bits_to_f64(oracle.bits(w.q))
    kf, vf = oracle.bf16_bits_to_f64(kc), oracle.bf16_bits_to_f64(vc)
    for s in range(w.num_seqs):
        a, b = int(w.query_start[s]), int(w.query_start[s + 1])
        n = int(w.context_lens[s])
        for t in range(a, b):
            pos = n - (b - a) + (t - a)
            for hq in range(2):
                z = []
                for j in range(pos + 1):
                    blk = int(w.block_tables[s][j // 16])
                    z.append(w.scale * sum(float(x) * float(y) for x, y in zip(qf[t][hq], kf[blk][0][j % 16])))
                top = max(z)
                e = [math.exp(x - top) for x in z]
                for c in (0, 13, 63):
                    val = sum(e[j] * float(vf[int(w.block_tables[s][j // 16])][0][j % 16][c])
                              for j in range(pos + 1)) / sum(e)
                    assert abs(val - out[t, hq, c]) <= 1e-12 * (1 + abs(val))


def test_prefill_rejects_chunk_longer_than_context():
    w = workloads.make_prefill_custom([0], [4], 2, 2, 64, 16, seed=1)
    with pytest.raises(ValueError):
        oracle.paged_prefill(w.q, w.k_cache, w.v_cache, w.block_tables, np.array([3], np.int32),
                             w.query_start, w.scale)


def test_named_prefill_workloads():
    for name in workloads.PREFILL_WORKLOADS:
        w = workloads.make_prefill(name, seed=0, values_device="meta")
        assert w.num_seqs == 8 and w.num_tokens == 8 * 512
        assert (np.diff(w.query_start) == 512).all()
        assert len(set(w.slot_mapping.tolist())) == w.num_tokens
