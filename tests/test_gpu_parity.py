"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Writes and copies must be bit-exact; decode attention must stay within
max-abs 2e-2 and relative L2 5e-3 of the fp64 oracle.  Cases span several
pipeline stages and partitions, ragged tails, every GQA kernel variant,
both head dims, several block sizes, poisoned (NaN) unused pool rows and the
degenerate lengths 0 and 1.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_420_b200 as pkv
import workloads
from tests._gpu_util import (assert_attention_close, bits_equal, device_inputs, no_device_error, run_step,
                             to_cuda)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clear_device_error():
    if torch.cuda.is_available():
        pkv.get_device_error()
    yield


# ------------------------------------------------------------------ write ---

@pytest.mark.parametrize("poison", [False, True])
def test_tiny_step_write_and_attention(poison):
    w = to_cuda(workloads.make("tiny", seed=0, poison=poison))
    kc, vc, out = run_step(w)
    okc, ovc, ref = oracle.decode_step(w)
    assert bits_equal(kc, okc) and bits_equal(vc, ovc)
    assert_attention_close(out, ref, "tiny")
    # context length 1 attends to the new token only: out = v_new rounded to bf16
    assert torch.equal(out[0], w.v_new[0])
    no_device_error()


def test_write_padding_and_out_of_range_slot():
    rng = np.random.default_rng(1)
    NB, Hkv, bs, D, T = 12, 4, 32, 128, 50
    kc = torch.randn(NB, Hkv, bs, D, device="cuda").to(torch.bfloat16)
    vc = torch.randn(NB, Hkv, bs, D, device="cuda").to(torch.bfloat16)
    k = torch.randn(T, Hkv, D, device="cuda").to(torch.bfloat16)
    v = torch.randn(T, Hkv, D, device="cuda").to(torch.bfloat16)
    slots = rng.choice(NB * bs, size=T, replace=False).astype(np.int64)
    slots[[0, 9, 33]] = -1
    ref_k, ref_v = oracle.kv_write(kc, vc, k, v, slots)
    bad = slots.copy()
    bad[5] = NB * bs + 7  # outside the pool: skipped and reported
    ref_bad_k, ref_bad_v = oracle.kv_write(kc, vc, np.delete(oracle.bits(k), 5, 0), np.delete(oracle.bits(v), 5, 0),
                                           np.delete(slots, 5))
    kc2, vc2 = kc.clone(), vc.clone()
    pkv.pkv_write(k, v, torch.from_numpy(slots).cuda(), kc2, vc2)
    torch.cuda.synchronize()
    assert bits_equal(kc2, ref_k) and bits_equal(vc2, ref_v)
    no_device_error()
    kc3, vc3 = kc.clone(), vc.clone()
    pkv.pkv_write(k, v, torch.from_numpy(bad).cuda(), kc3, vc3)
    assert pkv.get_device_error() == pkv.DEVERR_SLOT
    assert bits_equal(kc3, ref_bad_k) and bits_equal(vc3, ref_bad_v)


@pytest.mark.parametrize("D,bs,Hkv", [(64, 16, 1), (128, 16, 8), (128, 128, 2), (64, 1024, 3)])
def test_write_shapes_bit_exact(D, bs, Hkv):
    rng = np.random.default_rng(D + bs + Hkv)
    NB, T = 7, 33
    kc = torch.randn(NB, Hkv, bs, D, device="cuda").to(torch.bfloat16)
    vc = torch.randn(NB, Hkv, bs, D, device="cuda").to(torch.bfloat16)
    k = torch.randn(T, Hkv, D, device="cuda").to(torch.bfloat16)
    v = torch.randn(T, Hkv, D, device="cuda").to(torch.bfloat16)
    slots = rng.choice(NB * bs, size=T, replace=False).astype(np.int64)
    ref_k, ref_v = oracle.kv_write(kc, vc, k, v, slots)
    pkv.pkv_write(k, v, torch.from_numpy(slots).cuda(), kc, vc)
    torch.cuda.synchronize()
    assert bits_equal(kc, ref_k) and bits_equal(vc, ref_v)
    no_device_error()


# ------------------------------------------------------------------- copy ---

@pytest.mark.parametrize("npairs,D,bs,Hkv", [(1, 128, 16, 8), (37, 64, 32, 2), (1500, 128, 16, 4)])
def test_copy_blocks_bit_exact(npairs, D, bs, Hkv):
    rng = np.random.default_rng(npairs)
    NB = 2 * npairs + 5
    ids = rng.permutation(NB)
    pairs = np.stack([ids[:npairs], ids[npairs:2 * npairs]], axis=1).astype(np.int32)
    kc = torch.randn(NB, Hkv, bs, D, device="cuda").to(torch.bfloat16)
    vc = torch.randn(NB, Hkv, bs, D, device="cuda").to(torch.bfloat16)
    ref_k, ref_v = oracle.copy_blocks(kc, vc, pairs)
    pkv.pkv_copy_blocks(pairs, kc, vc)
    torch.cuda.synchronize()
    assert bits_equal(kc, ref_k) and bits_equal(vc, ref_v)


def test_copy_blocks_fan_out_from_one_source():
    kc = torch.randn(10, 2, 16, 64, device="cuda").to(torch.bfloat16)
    vc = torch.randn(10, 2, 16, 64, device="cuda").to(torch.bfloat16)
    pairs = np.array([[3, 0], [3, 1], [3, 7]], np.int32)
    ref_k, ref_v = oracle.copy_blocks(kc, vc, pairs)
    pkv.pkv_copy_blocks(pairs, kc, vc)
    torch.cuda.synchronize()
    assert bits_equal(kc, ref_k) and bits_equal(vc, ref_v)


def test_copy_then_write_leaves_sharers_unchanged():
    """Copy-on-write: after copying a shared block and writing into the copy,
    the sequence that still maps the original sees the old output exactly."""
    w = to_cuda(workloads.make_custom([70, 70], 4, 2, 128, 16, seed=3, share_prefix_tokens=64, group_size=2))
    d = device_inputs(w)
    out0 = torch.empty_like(w.q)
    pkv.paged_attn_decode(w.q, w.k_cache, w.v_cache, d["tables"], d["ctx"], w.scale, 2, out0, max_context_len=70)
    t = w.block_tables.copy()
    shared = int(t[1, 3])
    fresh = int(np.setdiff1d(np.arange(w.num_blocks), t.ravel())[0])
    kc, vc = w.k_cache.clone(), w.v_cache.clone()
    pkv.pkv_copy_blocks([[shared, fresh]], kc, vc)
    t[1, 3] = fresh
    pos = 3 * 16 + 5
    knew = torch.randn(1, 2, 128, device="cuda").to(torch.bfloat16)
    pkv.pkv_write(knew, knew, torch.tensor([fresh * 16 + 5], device="cuda"), kc, vc)
    out1 = torch.empty_like(w.q)
    pkv.paged_attn_decode(w.q, kc, vc, torch.from_numpy(t).cuda(), d["ctx"], w.scale, 2, out1, max_context_len=70)
    torch.cuda.synchronize()
    assert torch.equal(out1[0], out0[0])
    assert not torch.equal(out1[1], out0[1])
    okc, ovc = oracle.copy_blocks(w.k_cache, w.v_cache, [[shared, fresh]])
    okc, ovc = oracle.kv_write(okc, ovc, knew, knew, np.array([fresh * 16 + 5]))
    assert bits_equal(kc, okc) and bits_equal(vc, ovc)
    ref = oracle.paged_attention(w.q, okc, ovc, t, w.context_lens, w.scale)
    assert_attention_close(out1, ref, f"cow pos {pos}")


# ---------------------------------------------------------------- decode ----

DECODE_CASES = [
    # lens, Hq, Hkv, D, bs, partition_tokens
    ([1, 17, 33, 64], 4, 4, 64, 16, 0),                 # the tiny shape
    ([1000, 5, 16, 31, 257, 640], 8, 8, 128, 16, 0),    # MHA, several stages, ragged tails
    ([1000, 5, 16, 31, 257, 640], 8, 8, 128, 16, 64),   # MHA, forced split-K
    ([700, 3, 129, 1500], 8, 4, 128, 32, 0),            # g = 2 (tensor-core path, padded to 4 heads)
    ([700, 3, 129, 1500], 8, 4, 64, 32, 128),           # g = 2, d 64, split
    ([900, 2, 48, 333], 12, 4, 128, 16, 0),             # g = 3 (tensor-core path, padded tile)
    ([900, 2, 48, 333, 4097], 32, 8, 128, 16, 0),       # g = 4
    ([900, 2, 48, 333, 4097], 32, 8, 128, 16, 16),      # g = 4, one-stage partitions
    ([2049, 17, 512, 513], 64, 8, 128, 128, 512),       # g = 8, bs 128
    ([2049, 17, 512, 513], 64, 8, 64, 16, 0),           # g = 8, d 64
    ([1111, 7, 300], 32, 2, 128, 16, 256),              # g = 16 (two n-tiles)
    ([1111, 7, 300], 16, 1, 64, 64, 0),                 # g = 16, d 64, bs 64
    ([15, 16, 17, 31, 32, 33, 47, 48, 49], 2, 1, 128, 16, 32),  # boundaries around stages/partitions
    # partition groups (4 partitions, one per consumer warp): whole groups, a
    # ragged last partition inside a group, groups followed by single partitions
    ([2048, 2047, 2049, 1537, 1535, 2576], 8, 8, 128, 16, 512),    # MHA (CUDA-core path)
    ([2048, 2047, 2049, 1537, 1535, 2576], 32, 8, 128, 16, 256),   # g = 4 (tensor-core path)
    ([2048, 2047, 2049, 1537, 1535, 2576], 16, 1, 64, 32, 128),    # g = 16, d 64
    ([3000, 1024, 1025, 9], 64, 8, 128, 1024, 256),               # bs 1024: partitions and groups inside one block
    ([1000, 47, 48, 49, 2000], 8, 2, 128, 48, 0),                 # bs 48 (not a power of two), g = 4
    ([1000, 47, 48, 49, 2000], 2, 2, 128, 48, 96),                # bs 48, MHA, split
]


@pytest.mark.parametrize("lens,Hq,Hkv,D,bs,pt", DECODE_CASES)
@pytest.mark.parametrize("poison", [False, True])
def test_decode_parity(lens, Hq, Hkv, D, bs, pt, poison):
    w = to_cuda(workloads.make_custom(lens, Hq, Hkv, D, bs, seed=len(lens) * 31 + Hq, poison=poison,
                                      partition_tokens=pt))
    kc, vc, out = run_step(w)
    okc, ovc, ref = oracle.decode_step(w)
    assert bits_equal(kc, okc) and bits_equal(vc, ovc)
    assert_attention_close(out, ref, f"lens={lens} g={Hq // Hkv} D={D} bs={bs} pt={pt}")
    no_device_error()


def test_decode_context_zero_rows_are_zero():
    w = to_cuda(workloads.make_custom([40, 1, 90], 4, 2, 128, 16, seed=2))
    d = device_inputs(w)
    ctx = torch.tensor([0, 1, 90], dtype=torch.int32, device="cuda")
    out = torch.full_like(w.q, 7.0)
    pkv.paged_attn_decode(w.q, w.k_cache, w.v_cache, d["tables"], ctx, w.scale, 2, out, max_context_len=90)
    ref = oracle.paged_attention(w.q, w.k_cache, w.v_cache, w.block_tables, np.array([0, 1, 90], np.int32), w.scale)
    assert (out[0] == 0).all()
    assert_attention_close(out, ref, "ctx 0")
    no_device_error()


def test_decode_permuted_pool_is_bit_identical():
    w = to_cuda(workloads.make_custom([300, 45, 1000], 32, 8, 128, 16, seed=4))
    d = device_inputs(w)
    out = torch.empty_like(w.q)
    pkv.paged_attn_decode(w.q, w.k_cache, w.v_cache, d["tables"], d["ctx"], w.scale, 8, out, max_context_len=1000)
    pi = torch.from_numpy(np.random.default_rng(5).permutation(w.num_blocks)).cuda()
    kp, vp = torch.empty_like(w.k_cache), torch.empty_like(w.v_cache)
    kp[pi] = w.k_cache
    vp[pi] = w.v_cache
    t = torch.from_numpy(w.block_tables).cuda().long()
    tp = torch.where(t >= 0, pi[t.clamp(min=0)], t).to(torch.int32)
    out2 = torch.empty_like(w.q)
    pkv.paged_attn_decode(w.q, kp, vp, tp, d["ctx"], w.scale, 8, out2, max_context_len=1000)
    torch.cuda.synchronize()
    assert torch.equal(out, out2)


def test_decode_shared_blocks_equal_private_copies():
    w = to_cuda(workloads.make_custom([200, 200, 150, 90], 8, 8, 128, 16, seed=6, share_prefix_tokens=128,
                                      group_size=4))
    d = device_inputs(w)
    out = torch.empty_like(w.q)
    pkv.paged_attn_decode(w.q, w.k_cache, w.v_cache, d["tables"], d["ctx"], w.scale, 8, out, max_context_len=200)
    # duplicate the shared blocks of sequences 1..3 into fresh ids
    t = w.block_tables.copy()
    NB = w.num_blocks
    kc = torch.cat([w.k_cache, w.k_cache[torch.from_numpy(t[1:, :8].ravel().astype(np.int64)).cuda()]])
    vc = torch.cat([w.v_cache, w.v_cache[torch.from_numpy(t[1:, :8].ravel().astype(np.int64)).cuda()]])
    t[1:, :8] = (NB + np.arange(3 * 8)).reshape(3, 8)
    out2 = torch.empty_like(w.q)
    pkv.paged_attn_decode(w.q, kc, vc, torch.from_numpy(t).cuda(), d["ctx"], w.scale, 8, out2, max_context_len=200)
    torch.cuda.synchronize()
    assert torch.equal(out, out2)


def test_split_and_unsplit_agree():
    w = to_cuda(workloads.make_custom([3000, 1234, 77], 32, 8, 128, 16, seed=7))
    outs = []
    for pt in (16, 512, 4096):
        _, _, out = run_step(w, partition_tokens=pt)
        outs.append(out)
    _, _, ref = oracle.decode_step(w)
    for o in outs:
        assert_attention_close(o, ref, "split")
    diff = (outs[0].float() - outs[2].float()).abs().max().item()
    assert diff <= 2e-2


def test_uniform_keys_give_mean_of_values():
    w = to_cuda(workloads.make_custom([100, 37], 8, 2, 128, 16, seed=8))
    w.k_cache = w.k_cache[:1, :, :1].expand_as(w.k_cache).contiguous()
    d = device_inputs(w)
    out = torch.empty_like(w.q)
    pkv.paged_attn_decode(w.q, w.k_cache, w.v_cache, d["tables"], d["ctx"], w.scale, 2, out, max_context_len=100)
    torch.cuda.synchronize()
    vf = w.v_cache.double().cpu().numpy()
    for s, n in enumerate([100, 37]):
        rows = [vf[w.block_tables[s][i // 16], :, i % 16] for i in range(n)]
        mean = np.mean(rows, axis=0)
        for hq in range(8):
            np.testing.assert_allclose(out[s, hq].double().cpu().numpy(), mean[hq // 4], atol=2e-2, rtol=0)


def test_bad_block_id_and_context_are_reported():
    w = to_cuda(workloads.make_custom([64, 64], 4, 4, 128, 16, seed=9))
    d = device_inputs(w)
    out = torch.empty_like(w.q)
    t = d["tables"].clone()
    t[0, 2] = w.num_blocks + 5
    pkv.paged_attn_decode(w.q, w.k_cache, w.v_cache, t, d["ctx"], w.scale, 4, out, max_context_len=64)
    assert pkv.get_device_error() & pkv.DEVERR_BLOCK
    assert torch.isfinite(out.float()).all()
    ctx = d["ctx"].clone()
    ctx[1] = 10_000  # beyond the table (4 blocks = 64 tokens): clamped and reported
    pkv.paged_attn_decode(w.q, w.k_cache, w.v_cache, d["tables"], ctx, w.scale, 4, out, max_context_len=64)
    assert pkv.get_device_error() & pkv.DEVERR_CONTEXT
    ref = oracle.paged_attention(w.q, w.k_cache, w.v_cache, w.block_tables, np.array([64, 64], np.int32), w.scale)
    assert_attention_close(out, ref, "clamped ctx")
    # the same bad id inside a partition group (16-token partitions: one group of 4)
    ws = torch.empty(pkv.decode_workspace_bytes(2, 4, 4, 128, 64, 16), dtype=torch.uint8, device="cuda")
    pkv.paged_attn_decode(w.q, w.k_cache, w.v_cache, t, d["ctx"], w.scale, 4, out, max_context_len=64,
                          partition_tokens=16, workspace=ws)
    assert pkv.get_device_error() & pkv.DEVERR_BLOCK
    assert torch.isfinite(out.float()).all()
    good = torch.empty_like(out)
    pkv.paged_attn_decode(w.q, w.k_cache, w.v_cache, d["tables"], d["ctx"], w.scale, 4, good, max_context_len=64,
                          partition_tokens=16, workspace=ws)
    torch.cuda.synchronize()
    assert pkv.get_device_error() == 0
    assert torch.equal(out[1], good[1])  # the other sequence is untouched by the bad entry


def test_many_sequences_over_planner_chunk():
    """More than 1024 sequences (several planner chunks), short ragged lengths."""
    lens = list(np.random.default_rng(10).integers(1, 80, size=1300))
    w = to_cuda(workloads.make_custom(lens, 8, 1, 64, 16, seed=10, partition_tokens=32))
    kc, vc, out = run_step(w)
    okc, ovc, ref = oracle.decode_step(w)
    assert bits_equal(kc, okc)
    assert_attention_close(out, ref, "1300 seqs")
    no_device_error()


def test_many_sequences_with_partition_groups():
    """More than 1024 sequences with partition groups: the planner lists the
    groups of every chunk before all single partitions."""
    lens = list(np.random.default_rng(12).integers(1, 200, size=1500))
    w = to_cuda(workloads.make_custom(lens, 8, 2, 64, 16, seed=12, partition_tokens=32))
    kc, vc, out = run_step(w)
    okc, ovc, ref = oracle.decode_step(w)
    assert bits_equal(kc, okc)
    assert_attention_close(out, ref, "1500 seqs, groups")
    no_device_error()
