"""GPU parity of the FP8 (e4m3) KV cache against the oracle: the quantizing
write bit for bit (saturation, padding slots, several scales), and decode
attention over e4m3 pools within the attention tolerance (GQA groups 1 to 16
on both the CUDA-core and the tensor-core paths, ragged contexts, split-K
partitions, poisoned unused rows)."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_420_b200 as pkv
import workloads
from tests._gpu_util import assert_attention_close, no_device_error

pytestmark = pytest.mark.gpu


def _codes(t):
    return t.cpu().numpy()


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("scale_kind", ["unit", "small", "mixed"])
def test_write_fp8_bit_exact(D, scale_kind):
    rng = np.random.default_rng(D)
    NB, Hkv, bs, T = 20, 4, 16, 37
    g = torch.Generator().manual_seed(D)
    k = (torch.randn((T, Hkv, D), generator=g) * 4).to(torch.bfloat16)
    v = torch.randn((T, Hkv, D), generator=g).to(torch.bfloat16)
    slots = rng.choice(NB * bs, T, replace=False).astype(np.int64)
    slots[[3, 11]] = -1
    ks = {"unit": [1, 1, 1, 1], "small": [0.004, 0.003, 0.002, 0.001], "mixed": [0.3, 1.7, 0.011, 9.0]}[scale_kind]
    ks = np.array(ks, np.float32)
    vs = ks[::-1].copy()
    kc8 = torch.from_numpy(rng.integers(0, 256, (NB, Hkv, bs, D)).astype(np.uint8))
    vc8 = torch.from_numpy(rng.integers(0, 256, (NB, Hkv, bs, D)).astype(np.uint8))
    kd, vd = kc8.cuda(), vc8.cuda()
    pkv.pkv_write_fp8(k.cuda(), v.cuda(), torch.from_numpy(slots).cuda(), torch.from_numpy(ks).cuda(),
                      torch.from_numpy(vs).cuda(), kd, vd)
    torch.cuda.synchronize()
    ok, ov = oracle.kv_write_fp8(kc8.numpy(), vc8.numpy(), k, v, slots, ks, vs)
    assert np.array_equal(_codes(kd), ok) and np.array_equal(_codes(vd), ov)
    if scale_kind == "small":
        assert (ok == 0x7E).any() and (ok == 0xFE).any()  # saturation exercised
    no_device_error()


def _run_decode(w, k8, v8, ks, vs, pt=0):
    out = torch.full_like(w.q, float("nan"))
    pkv.paged_attn_decode_fp8(w.q, k8, v8, ks, vs, torch.from_numpy(w.block_tables).cuda(),
                              torch.from_numpy(w.context_lens).cuda(), w.scale, w.num_kv_heads, out,
                              int(w.context_lens.max()), partition_tokens=pt)
    torch.cuda.synchronize()
    return out


CASES = [
    # context lens, Hq, Hkv, partition tokens
    ([1, 15, 16, 17, 31, 100], 8, 8, 0),
    ([5, 200, 511, 513], 16, 8, 0),          # g = 2: tensor-core path (padded to 4 heads)
    ([1000, 3000, 77], 4, 4, 256),           # split-K partitions
    ([4096, 2049, 16], 8, 4, 512),           # g = 2, split-K
    ([1, 15, 16, 17, 31, 100], 32, 8, 0),    # g = 4
    ([200, 511, 1000], 64, 8, 256),          # g = 8, split-K
    ([50, 129], 12, 4, 0),                   # g = 3 (padded to 4)
    ([33, 700], 16, 1, 0),                   # g = 16
    ([2048, 2047, 2049, 1537, 2576], 8, 8, 512),   # partition groups, MHA
    ([2048, 2047, 2049, 1537, 2576], 32, 8, 256),  # partition groups, g = 4
]


@pytest.mark.parametrize("ctx,Hq,Hkv,pt", CASES)
@pytest.mark.parametrize("poison", [False, True])
def test_decode_fp8_parity(ctx, Hq, Hkv, pt, poison):
    """A decode step: the new token quantized into its slot, then attention."""
    w = workloads.make_custom(ctx, Hq, Hkv, 128, 16, seed=sum(ctx) + Hq, poison=poison)
    k8, v8, ks, vs = workloads.fp8_pools(w)
    kd, vd = k8.cuda(), v8.cuda()
    pkv.pkv_write_fp8(w.k_new.cuda(), w.v_new.cuda(), torch.from_numpy(w.slot_mapping).cuda(), ks.cuda(), vs.cuda(),
                      kd, vd)
    w.q = w.q.cuda()
    out = _run_decode(w, kd, vd, ks.cuda(), vs.cuda(), pt)
    ok, ov = oracle.kv_write_fp8(k8.numpy(), v8.numpy(), w.k_new, w.v_new, w.slot_mapping, ks.numpy(), vs.numpy())
    assert np.array_equal(_codes(kd), ok) and np.array_equal(_codes(vd), ov)
    ref = oracle.paged_attention_fp8(w.q, ok, ov, ks.numpy(), vs.numpy(), w.block_tables, w.context_lens, w.scale)
    assert_attention_close(out, ref, f"fp8 ctx={ctx} g={Hq // Hkv} pt={pt} poison={poison}")
    no_device_error()


def test_write_then_decode_fp8():
    """A decode step on an FP8 pool: the new token's K/V quantized by the write,
    then attention -- against the oracle's write and attention."""
    w = workloads.make("llama2-7b", seed=3, values_device="cpu")
    w = workloads.subset(w, 24)
    k8, v8, ks, vs = workloads.fp8_pools(w)
    kd, vd = k8.cuda(), v8.cuda()
    pkv.pkv_write_fp8(w.k_new.cuda(), w.v_new.cuda(), torch.from_numpy(w.slot_mapping).cuda(), ks.cuda(), vs.cuda(),
                      kd, vd)
    w.q = w.q.cuda()
    out = _run_decode(w, kd, vd, ks.cuda(), vs.cuda())
    ok, ov = oracle.kv_write_fp8(k8.numpy(), v8.numpy(), w.k_new, w.v_new, w.slot_mapping, ks.numpy(), vs.numpy())
    assert np.array_equal(_codes(kd), ok) and np.array_equal(_codes(vd), ov)
    ref = oracle.paged_attention_fp8(w.q, ok, ov, ks.numpy(), vs.numpy(), w.block_tables, w.context_lens, w.scale)
    assert_attention_close(out, ref, "fp8 llama2-7b step")


def test_fp8_decode_matches_bf16_decode_on_exact_values():
    """With power-of-two scales the dequantized pool is exact in bf16: the FP8
    kernel and the bf16 kernel on that pool agree to the attention tolerance."""
    w = workloads.make_custom([37, 500, 1025], 8, 8, 128, 16, seed=5)
    k8, v8, _, _ = workloads.fp8_pools(w)
    ks = torch.full((8,), 0.25)
    vs = torch.full((8,), 0.125)
    w.q = w.q.cuda()
    out8 = _run_decode(w, k8.cuda(), v8.cuda(), ks.cuda(), vs.cuda())
    kb = torch.from_numpy(oracle.e4m3_decode(k8.numpy()) * 0.25).to(torch.bfloat16).cuda()
    vb = torch.from_numpy(oracle.e4m3_decode(v8.numpy()) * 0.125).to(torch.bfloat16).cuda()
    out = torch.empty_like(w.q)
    pkv.paged_attn_decode(w.q, kb, vb, torch.from_numpy(w.block_tables).cuda(), torch.from_numpy(w.context_lens).cuda(),
                          w.scale, 8, out, 1025)
    torch.cuda.synchronize()
    assert (out8.float() - out.float()).abs().max().item() <= 2e-2


def test_fp8_refuses_unsupported_shapes():
    w = workloads.make_custom([20], 4, 4, 64, 16, seed=1)  # head dim 64
    k8, v8, ks, vs = workloads.fp8_pools(w)
    w.q = w.q.cuda()
    with pytest.raises(pkv.PkvError):
        _run_decode(w, k8.cuda(), v8.cuda(), ks.cuda(), vs.cuda())


def test_named_workload_fp8_full_size_sampled():
    """The Llama-2-13B batch with an FP8 pool: every output finite, sampled
    sequences against the oracle."""
    w = workloads.make("llama2-13b", seed=0, values_device="cuda")
    k8, v8, ks, vs = workloads.fp8_pools(w)
    out = _run_decode(w, k8, v8, ks, vs)
    assert torch.isfinite(out.float()).all()
    no_device_error()
    pick = [0, 17, 63, 127]
    ref = oracle.paged_attention_fp8(w.q[pick].cpu(), k8.cpu().numpy(), v8.cpu().numpy(), ks.cpu().numpy(),
                                     vs.cpu().numpy(), w.block_tables[pick], w.context_lens[pick], w.scale)
    assert_attention_close(out[pick], ref, "fp8 llama2-13b sampled")


def _as_u16(a):
    """An e4m3 pool [NB, Hkv, bs, D] viewed as 2-byte units [NB, Hkv, bs, D/2]:
    whole-block copies move the same bytes either way."""
    a = np.ascontiguousarray(a)
    return a.view(np.uint16).reshape(a.shape[:-1] + (a.shape[-1] // 2,))


def test_fp8_pool_copy_and_swap_match_oracle():
    rng = np.random.default_rng(4)
    NB, Hkv, bs, D = 64, 8, 16, 128
    k8 = rng.integers(0, 256, (NB, Hkv, bs, D)).astype(np.uint8)
    v8 = rng.integers(0, 256, (NB, Hkv, bs, D)).astype(np.uint8)
    kd, vd = torch.from_numpy(k8).cuda(), torch.from_numpy(v8).cuda()
    pairs = np.array([[3, 40], [7, 41], [63, 0], [12, 13]], np.int32)
    pkv.pkv_copy_blocks(pairs, kd, vd)
    torch.cuda.synchronize()
    ok, ov = oracle.copy_blocks(_as_u16(k8), _as_u16(v8), pairs)
    assert np.array_equal(_as_u16(kd.cpu().numpy()), ok) and np.array_equal(_as_u16(vd.cpu().numpy()), ov)
    # the device-sourced copy, with a count on the device
    pd = torch.from_numpy(np.array([[40, 50], [41, 51], [5, 52]], np.int32)).cuda()
    pkv.copy_blocks_dev(pd, torch.tensor([2], dtype=torch.int32, device="cuda"), kd, vd)
    torch.cuda.synchronize()
    ok, ov = oracle.copy_blocks(ok, ov, np.array([[40, 50], [41, 51]], np.int32))
    assert np.array_equal(_as_u16(kd.cpu().numpy()), ok) and np.array_equal(_as_u16(vd.cpu().numpy()), ov)
    # swap out and back into other blocks
    ids = np.array([50, 3, 63], np.int32)
    hk = torch.empty((3, Hkv, bs, D), dtype=torch.uint8).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    pkv.pkv_swap_out(kd, vd, ids, hk, hv)
    torch.cuda.synchronize()
    ohk, ohv = oracle.swap_out(ok, ov, ids)
    assert np.array_equal(_as_u16(hk.numpy()), ohk) and np.array_equal(_as_u16(hv.numpy()), ohv)
    dst = np.array([20, 21, 22], np.int32)
    pkv.pkv_swap_in(hk, hv, dst, kd, vd)
    torch.cuda.synchronize()
    ok, ov = oracle.swap_in(ok, ov, ohk, ohv, dst)
    assert np.array_equal(_as_u16(kd.cpu().numpy()), ok) and np.array_equal(_as_u16(vd.cpu().numpy()), ov)
