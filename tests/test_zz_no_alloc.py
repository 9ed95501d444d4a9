"""paged_attn_decode_static_ws: decode attention without a workspace argument.

It serves callers that cannot allocate device memory, such as a plugin whose
host engine has reserved all device memory for its own pools and hands out no
allocator, or a latency-critical path that must not call cudaMalloc.  Its
scratch is a fixed device array inside libpkv.so shared by every call.

This file sorts last so that a run stopping at the first failure has already
run every other test.  The test calls the new entry point through the C ABI
several times in a row, on different inputs (each call reuses scratch the one
before left behind).  Each output must equal paged_attn_decode's with a
caller-provided workspace bit for bit (same kernels, same plan, deterministic),
and stay within the attention tolerance of the fp64 oracle.
"""
import ctypes

import pytest
import torch

import oracle
import paged_kv_cache_420_b200 as pkv
import workloads
from tests._gpu_util import assert_attention_close, to_cuda

pytestmark = pytest.mark.gpu


def _inputs(w):
    return (torch.from_numpy(w.block_tables).cuda(), torch.from_numpy(w.context_lens).cuda())


def _abi_static(lib, w, tables, ctx, out, pt, max_ctx=None):
    f = lib.paged_attn_decode_static_ws
    P, I32, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
    f.argtypes = [P, P, P, P, I32, P, I32, I32, F, I32, P, pkv._Pool, I32, I32, P]
    f.restype = ctypes.c_int
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    max_ctx = w.max_context_len if max_ctx is None else max_ctx
    return f(P(w.q.data_ptr()), P(w.k_cache.data_ptr()), P(w.v_cache.data_ptr()), P(tables.data_ptr()),
             tables.shape[1], P(ctx.data_ptr()), w.num_seqs, w.num_q_heads, w.scale, w.num_kv_heads,
             P(out.data_ptr()), pkv._pool(w.k_cache), max_ctx, pt, stream)


def test_static_scratch_decode_matches_workspace_decode_twice():
    lib = pkv.load_library()
    cases = [
        # split-K with several partitions per sequence, GQA tensor-core path
        (workloads.make_custom([3000, 17, 1025, 513], 32, 8, 128, 16, seed=21, poison=True), 256),
        # MHA CUDA-core path, head dim 64; the 700-token sequence takes two of
        # the default 512-token partitions, so this call splits too
        (workloads.make_custom([700, 1, 64, 129, 31], 8, 8, 64, 32, seed=22, poison=True), 0),
        # every context within one partition: no partial results and no reduce
        # kernel, the attention kernel writes out directly
        (workloads.make_custom([300, 1, 64, 129, 31], 16, 4, 128, 16, seed=24, poison=True), 0),
    ]
    for w, pt in cases:
        to_cuda(w)
        tables, ctx = _inputs(w)
        # the step's write comes first: the poisoned pool holds NaN at each
        # sequence's newest position until then
        pkv.pkv_write(w.k_new, w.v_new, torch.from_numpy(w.slot_mapping).cuda(), w.k_cache, w.v_cache)
        ref = torch.empty_like(w.q)
        pkv.paged_attn_decode(w.q, w.k_cache, w.v_cache, tables, ctx, w.scale, w.num_kv_heads, ref,
                              w.max_context_len, pt)
        out = torch.full_like(w.q, float("nan"))
        assert _abi_static(lib, w, tables, ctx, out, pt) == 0
        torch.cuda.synchronize()
        assert pkv.get_device_error() == 0
        assert torch.equal(out, ref)
        exact = oracle.paged_attention(w.q, oracle.bits(w.k_cache), oracle.bits(w.v_cache), w.block_tables,
                                       w.context_lens, w.scale)
        assert_attention_close(out, exact, f"static scratch, lens={list(w.context_lens)}")


def test_static_scratch_rejects_requests_beyond_its_size():
    lib = pkv.load_library()
    w = to_cuda(workloads.make_custom([64], 64, 8, 128, 16, seed=23))
    tables, ctx = _inputs(w)
    out = torch.zeros_like(w.q)
    big_ctx = 1 << 22  # 8192 partitions x 64 heads x 520 B of partials: far above the scratch size
    need = pkv.decode_workspace_bytes(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, big_ctx, 512)
    assert need > pkv.STATIC_WS_BYTES
    assert _abi_static(lib, w, tables, ctx, out, 512, max_ctx=big_ctx) == 6  # PKV_EUNSUPPORTED
    torch.cuda.synchronize()
    assert (out == 0).all()  # nothing was enqueued
