"""Pins for the oracle's swap-out / swap-in and LRU victim choice
(intelliparadigm.com article 2012396, section 2.1, item 3; ai-stack.site
"Nano-vLLM 原理", practice 5).

Swap is pinned against copy_blocks (an independently pinned function): moving
blocks out to host memory and back into other blocks must equal the
copy-on-write copy of those pairs.  The LRU choice is pinned by a worked
example written out by hand and by the characterisation of the answer.
"""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _pool(nb=12, hkv=3, bs=16, d=8, seed=0):
    rng = np.random.default_rng(seed)
    kc = rng.integers(0, 1 << 16, size=(nb, hkv, bs, d), dtype=np.uint16)
    vc = rng.integers(0, 1 << 16, size=(nb, hkv, bs, d), dtype=np.uint16)
    return kc, vc


def test_swap_out_then_in_equals_copy_blocks():
    kc, vc = _pool()
    src = [3, 7, 0, 11]
    dst = [5, 1, 9, 2]
    hk, hv = oracle.swap_out(kc, vc, src)
    k2, v2 = oracle.swap_in(kc, vc, hk, hv, dst)
    k3, v3 = oracle.copy_blocks(kc, vc, np.stack([src, dst], 1))
    assert np.array_equal(k2, k3) and np.array_equal(v2, v3)


def test_swap_round_trip_restores_and_swap_out_reads_only():
    kc, vc = _pool(seed=1)
    k0, v0 = kc.copy(), vc.copy()
    ids = [4, 0, 10]
    hk, hv = oracle.swap_out(kc, vc, ids)
    assert np.array_equal(kc, k0) and np.array_equal(vc, v0)
    # the blocks are overwritten (as when reused by another request), then restored
    trash_k, trash_v = oracle.swap_in(kc, vc, np.zeros_like(hk), np.ones_like(hv), ids)
    assert not np.array_equal(trash_k, k0)
    k2, v2 = oracle.swap_in(trash_k, trash_v, hk, hv, ids)
    assert np.array_equal(k2, k0) and np.array_equal(v2, v0)


def test_swap_of_a_permutation_is_a_gather():
    kc, vc = _pool(nb=9, seed=2)
    perm = np.random.default_rng(3).permutation(9).astype(np.int32)
    hk, hv = oracle.swap_out(kc, vc, perm)
    k2, v2 = oracle.swap_in(np.zeros_like(kc), np.zeros_like(vc), hk, hv, np.arange(9))
    assert np.array_equal(k2, np.take(kc, perm, axis=0)) and np.array_equal(v2, np.take(vc, perm, axis=0))
    # the key and value regions stay separate (a block holds both)
    assert not np.array_equal(k2, v2)


def test_swap_rejects_bad_ids():
    kc, vc = _pool()
    with pytest.raises(IndexError):
        oracle.swap_out(kc, vc, [0, 12])
    hk, hv = oracle.swap_out(kc, vc, [1, 2])
    with pytest.raises(ValueError):
        oracle.swap_in(kc, vc, hk, hv, [4, 4])
    assert oracle.swap_out(kc, vc, [])[0].shape == (0, 3, 16, 8)


def test_lru_worked_example_golden():
    g = json.load(open(os.path.join(GOLDEN, "lru_victims_example.json")))
    got = oracle.lru_victims(g["last_use"], g["evictable"], g["k"])
    assert got.tolist() == g["victims"]


@pytest.mark.parametrize("seed", range(6))
def test_lru_characterisation(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 60))
    last = rng.integers(0, 12, size=n)  # many ties
    ev = rng.random(n) < 0.7
    k = int(rng.integers(0, n + 3))
    v = oracle.lru_victims(last, ev, k)
    cand = np.flatnonzero(ev)
    assert len(v) == min(k, len(cand)) and len(set(v.tolist())) == len(v)
    assert ev[v].all()
    # ordered oldest first, ties by id, and nothing left behind is older
    keys = list(zip(last[v].tolist(), v.tolist()))
    assert keys == sorted(keys)
    rest = np.setdiff1d(cand, v)
    if len(v) and len(rest):
        assert max(keys) < min(zip(last[rest].tolist(), rest.tolist()))
    # equal to a stable library sort of the candidates
    order = cand[np.lexsort((cand, last[cand]))]
    assert np.array_equal(v, order[:len(v)])
