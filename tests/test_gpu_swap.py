"""GPU parity of block swap-out / swap-in against the oracle: bit-exact, for
arbitrary bf16 bit patterns (NaN payloads included), repeated ids on the way
out, more ids than one launch carries, both head dims and several block
sizes; pageable host memory is refused."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_420_b200 as pkv

pytestmark = pytest.mark.gpu


def _pool(nb, hkv, bs, d, seed):
    g = torch.Generator().manual_seed(seed)
    kc = torch.randint(-32768, 32767, (nb, hkv, bs, d), generator=g, dtype=torch.int16)
    vc = torch.randint(-32768, 32767, (nb, hkv, bs, d), generator=g, dtype=torch.int16)
    return kc.view(torch.bfloat16), vc.view(torch.bfloat16)


def _bits(t):
    return oracle.bits(t)


def _pinned(n, hkv, bs, d):
    return torch.empty((n, hkv, bs, d), dtype=torch.bfloat16).pin_memory()


CASES = [
    # num_blocks, Hkv, bs, D, n
    (64, 8, 16, 128, 20),
    (40, 1, 32, 64, 40),
    (300, 40, 16, 128, 7),
    (16, 2, 128, 128, 16),
    (3000, 1, 16, 64, 2500),  # two launches
]


@pytest.mark.parametrize("nb,hkv,bs,d,n", CASES)
def test_swap_out_parity(nb, hkv, bs, d, n):
    kc, vc = _pool(nb, hkv, bs, d, seed=nb + n)
    rng = np.random.default_rng(nb)
    ids = rng.integers(0, nb, n).astype(np.int32)  # repeats allowed
    kd, vd = kc.cuda(), vc.cuda()
    hk, hv = _pinned(n, hkv, bs, d), _pinned(n, hkv, bs, d)
    pkv.pkv_swap_out(kd, vd, ids, hk, hv)
    torch.cuda.synchronize()
    ok_k, ok_v = oracle.swap_out(kc, vc, ids)
    assert np.array_equal(_bits(hk), ok_k) and np.array_equal(_bits(hv), ok_v)
    # the pool was only read
    assert np.array_equal(_bits(kd), _bits(kc)) and np.array_equal(_bits(vd), _bits(vc))


@pytest.mark.parametrize("nb,hkv,bs,d,n", CASES)
def test_swap_in_parity_and_round_trip(nb, hkv, bs, d, n):
    kc, vc = _pool(nb, hkv, bs, d, seed=3 * nb + n)
    rng = np.random.default_rng(nb + 1)
    ids = rng.permutation(nb)[:n].astype(np.int32)  # distinct
    hk_src, hv_src = _pool(n, hkv, bs, d, seed=7 * n)
    hk, hv = _pinned(n, hkv, bs, d), _pinned(n, hkv, bs, d)
    hk.copy_(hk_src)
    hv.copy_(hv_src)
    kd, vd = kc.cuda(), vc.cuda()
    pkv.pkv_swap_in(hk, hv, ids, kd, vd)
    torch.cuda.synchronize()
    ok_k, ok_v = oracle.swap_in(kc, vc, hk_src, hv_src, ids)
    assert np.array_equal(_bits(kd), ok_k) and np.array_equal(_bits(vd), ok_v)
    # round trip: out again, back into a zeroed pool
    hk2, hv2 = _pinned(n, hkv, bs, d), _pinned(n, hkv, bs, d)
    pkv.pkv_swap_out(kd, vd, ids, hk2, hv2)
    z_k, z_v = torch.zeros_like(kd), torch.zeros_like(vd)
    pkv.pkv_swap_in(hk2, hv2, ids, z_k, z_v)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(hk2), _bits(hk_src)) and np.array_equal(_bits(hv2), _bits(hv_src))
    assert np.array_equal(_bits(z_k)[ids], ok_k[ids]) and np.array_equal(_bits(z_v)[ids], ok_v[ids])


def test_swap_then_lru_preemption_cycle():
    """A preemption cycle: LRU victims of a pool go out, their blocks are reused
    (overwritten), and they come back into other free blocks -- equal to the
    copy-on-write copy of (victim, new block) pairs on the original pool."""
    nb, hkv, bs, d = 96, 8, 16, 128
    kc, vc = _pool(nb, hkv, bs, d, seed=5)
    rng = np.random.default_rng(5)
    last_use = rng.integers(0, 30, nb)
    evictable = rng.random(nb) < 0.5
    victims = pkv.lru_victims(last_use, evictable, 12)
    assert np.array_equal(victims, oracle.lru_victims(last_use, evictable, 12))
    free = np.setdiff1d(np.arange(nb), victims)[:len(victims)].astype(np.int32)
    kd, vd = kc.cuda(), vc.cuda()
    hk, hv = _pinned(len(victims), hkv, bs, d), _pinned(len(victims), hkv, bs, d)
    pkv.pkv_swap_out(kd, vd, victims, hk, hv)
    kd[torch.from_numpy(victims).long().cuda()] = 0  # reused by another request
    pkv.pkv_swap_in(hk, hv, free, kd, vd)
    torch.cuda.synchronize()
    ok_k, ok_v = oracle.copy_blocks(kc, vc, np.stack([victims, free], 1))
    keep = np.setdiff1d(np.arange(nb), victims)
    assert np.array_equal(_bits(kd)[keep], ok_k[keep]) and np.array_equal(_bits(vd), ok_v)


def test_swap_refuses_pageable_and_device_buffers():
    lib = pkv.load_library()
    kd, vd = (t.cuda() for t in _pool(8, 2, 16, 64, seed=1))
    ids = np.array([1, 2], dtype=np.int32)
    pageable = torch.empty((2, 2, 16, 64), dtype=torch.bfloat16)
    dev = torch.empty((2, 2, 16, 64), dtype=torch.bfloat16, device="cuda")
    for buf in (pageable, dev):
        st = lib.pkv_swap_out(ctypes.c_void_p(kd.data_ptr()), ctypes.c_void_p(vd.data_ptr()), pkv._pool(kd),
                              ids.ctypes.data_as(ctypes.c_void_p), 2, ctypes.c_void_p(buf.data_ptr()),
                              ctypes.c_void_p(buf.data_ptr()), None)
        assert st == 1
    with pytest.raises(ValueError):
        pkv.pkv_swap_out(kd, vd, ids, pageable, pageable)
