"""GPU parity of chunked-prefill paged attention against the fp64 oracle.

Cases span query tiles (128 rows = tokens x GQA group), chunks shorter and
longer than a tile, prefixes that are empty or end mid-block, key counts that
end inside a 16-key stage, GQA group sizes 1..16 (including ones that do not
divide a tile, leaving padding rows), both head dims, several block sizes and
poisoned unused pool rows.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_420_b200 as pkv
import workloads
from tests._gpu_util import assert_attention_close, bits_equal, no_device_error

pytestmark = pytest.mark.gpu


def run_prefill(w):
    for name in ("q", "k_new", "v_new", "k_cache", "v_cache"):
        setattr(w, name, getattr(w, name).to("cuda").contiguous())
    kc, vc = w.k_cache.clone(), w.v_cache.clone()
    pkv.pkv_write(w.k_new, w.v_new, torch.from_numpy(w.slot_mapping).cuda(), kc, vc)
    out = torch.full_like(w.q, float("nan"))
    pkv.paged_attn_prefill(w.q, kc, vc, torch.from_numpy(w.block_tables).cuda(),
                           torch.from_numpy(w.context_lens).cuda(), torch.from_numpy(w.query_start).cuda(),
                           w.scale, w.num_kv_heads, out, w.max_query_len, w.max_context_len)
    torch.cuda.synchronize()
    return kc, vc, out


CASES = [
    # prefix lens, chunk lens, Hq, Hkv, D, bs
    ([0, 5, 40], [7, 16, 33], 4, 4, 64, 16),
    ([0, 100, 17], [64, 65, 130], 8, 8, 128, 16),        # MHA, 128-token tiles
    ([300, 0, 33], [200, 129, 1], 32, 8, 128, 16),       # g = 4: 32-token tiles
    ([1000, 7], [100, 63], 64, 8, 128, 128),             # g = 8, bs 128
    ([50, 0], [31, 17], 12, 4, 64, 32),                  # g = 3: 42-token tiles (two padding rows)
    ([17, 260], [40, 9], 32, 2, 128, 16),                # g = 16
    ([0], [256], 2, 1, 128, 16),                         # g = 2, whole-sequence prefill
    ([2000, 15, 16], [1, 1, 1], 8, 4, 128, 16),          # single-token chunks (= decode)
    ([0, 513], [384, 300], 8, 8, 64, 16),                # MHA head dim 64, several 128-token tiles
    ([70], [200], 20, 4, 128, 32),                       # g = 5: 25-token tiles, 3 padding rows
    ([129, 1], [777, 64], 14, 2, 128, 16),               # g = 7: 18-token tiles, long chunk
    ([100, 2000, 0], [300, 130, 513], 8, 2, 128, 48),    # bs 48 (not a power of two), g = 4, many items
]


@pytest.mark.parametrize("prefix,chunk,Hq,Hkv,D,bs", CASES)
@pytest.mark.parametrize("poison", [False, True])
def test_prefill_parity(prefix, chunk, Hq, Hkv, D, bs, poison):
    w = workloads.make_prefill_custom(prefix, chunk, Hq, Hkv, D, bs, seed=sum(prefix) + Hq + D, poison=poison)
    kc, vc, out = run_prefill(w)
    okc, ovc = oracle.kv_write(w.k_cache, w.v_cache, w.k_new, w.v_new, w.slot_mapping)
    assert bits_equal(kc, okc)
    ref = oracle.paged_prefill(w.q, okc, ovc, w.block_tables, w.context_lens, w.query_start, w.scale)
    assert_attention_close(out, ref, f"prefix={prefix} chunk={chunk} g={Hq // Hkv} D={D} bs={bs}")
    no_device_error()


@pytest.mark.parametrize("case", [1, 2, 4, 0])
def test_prefill_out_only_16_byte_aligned(case):
    """`out` 16 bytes past a 32-byte boundary takes the 16-byte store path of
    the epilogue; it must write the same bits as the paired 32-byte stores."""
    w = workloads.make_prefill_custom(*CASES[case], seed=5)
    kc, vc, out = run_prefill(w)
    base = torch.full((out.numel() + 8,), float("nan"), dtype=out.dtype, device="cuda")
    out16 = base[8:].view(out.shape)
    assert out16.data_ptr() % 32 == 16 and out.data_ptr() % 32 == 0
    pkv.paged_attn_prefill(w.q, kc, vc, torch.from_numpy(w.block_tables).cuda(),
                           torch.from_numpy(w.context_lens).cuda(), torch.from_numpy(w.query_start).cuda(),
                           w.scale, w.num_kv_heads, out16, w.max_query_len, w.max_context_len)
    torch.cuda.synchronize()
    no_device_error()
    assert torch.equal(out16, out)  # also false if any element stayed NaN


def test_prefill_single_token_equals_decode_kernel():
    w = workloads.make_prefill_custom([300, 1000, 0], [1, 1, 1], 32, 8, 128, 16, seed=9)
    kc, vc, out = run_prefill(w)
    dec = torch.empty_like(out)
    pkv.paged_attn_decode(w.q, kc, vc, torch.from_numpy(w.block_tables).cuda(),
                          torch.from_numpy(w.context_lens).cuda(), w.scale, w.num_kv_heads, dec, w.max_context_len)
    torch.cuda.synchronize()
    assert (out.float() - dec.float()).abs().max().item() <= 2e-2


@pytest.mark.parametrize("name", workloads.PREFILL_WORKLOADS)
def test_named_prefill_workload_full_size(name):
    w = workloads.make_prefill(name, seed=0, values_device="cuda")
    kc0, vc0 = w.k_cache.cpu(), w.v_cache.cpu()
    kc, vc, out = run_prefill(w)
    no_device_error()
    assert torch.isfinite(out.float()).all()
    okc, ovc = oracle.kv_write(kc0, vc0, w.k_new, w.v_new, w.slot_mapping)
    assert bits_equal(kc, okc) and bits_equal(vc, ovc)
    # sampled rows: the first and last 128 query rows of every sequence's chunk
    rows = np.unique(np.concatenate(
        [np.r_[a:min(b, a + 128), max(a, b - 128):b]
         for a, b in zip(w.query_start[:-1].astype(int), w.query_start[1:].astype(int))]))
    sub_q = w.q[torch.from_numpy(rows).cuda()]
    # oracle on single-row chunks with the rows' own context lengths
    seq_of = np.searchsorted(w.query_start, rows, side="right") - 1
    ctx = (w.context_lens[seq_of] - (w.query_start[seq_of + 1] - rows) + 1).astype(np.int32)
    qs = np.arange(len(rows) + 1, dtype=np.int32)
    ref = oracle.paged_prefill(sub_q, okc, ovc, w.block_tables[seq_of], ctx, qs, w.scale)
    assert_attention_close(out[torch.from_numpy(rows).cuda()], ref, name)
