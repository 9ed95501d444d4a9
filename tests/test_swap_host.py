"""Host side of swap: the library's LRU victim choice against the oracle, and
the swap entry points' validation before any CUDA work (no GPU needed)."""
import ctypes

import numpy as np
import pytest

import oracle
import paged_kv_cache_420_b200 as pkv
from paged_kv_cache_420_b200 import _Pool

EINVAL, ERANGE, EALIAS = 1, 2, 3
FAKE = ctypes.c_void_p(0x10000)


@pytest.mark.parametrize("seed", range(8))
def test_lru_victims_match_oracle(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(0, 2000))
    last = rng.integers(0, int(rng.integers(1, 50)), n)  # heavy ties
    ev = rng.random(n) < rng.random()
    for k in (0, 1, int(rng.integers(0, n + 1)), n + 7):
        assert np.array_equal(pkv.lru_victims(last, ev, k), oracle.lru_victims(last, ev, k))


def test_lru_validation():
    lib = pkv.load_library()
    cnt = ctypes.c_int32(-1)
    assert lib.pkv_lru_victims(None, None, 0, 3, None, ctypes.byref(cnt)) == EINVAL  # k > 0 needs victims
    out = (ctypes.c_int32 * 4)()
    assert lib.pkv_lru_victims(None, None, 0, 3, out, ctypes.byref(cnt)) == 0 and cnt.value == 0
    assert lib.pkv_lru_victims(None, None, -1, 0, None, ctypes.byref(cnt)) == EINVAL
    assert lib.pkv_lru_victims(None, None, 5, 0, None, ctypes.byref(cnt)) == EINVAL


def _ids(*v):
    a = np.asarray(v, dtype=np.int32)
    return a, a.ctypes.data_as(ctypes.c_void_p)


def test_swap_validation():
    lib = pkv.load_library()
    pool = _Pool(8, 2, 16, 128)
    a, ids = _ids(0, 3, 7)
    assert lib.pkv_swap_out(FAKE, FAKE, pool, ids, 0, FAKE, FAKE, None) == 0
    assert lib.pkv_swap_out(FAKE, FAKE, pool, ids, -1, FAKE, FAKE, None) == EINVAL
    assert lib.pkv_swap_out(FAKE, FAKE, pool, None, 3, FAKE, FAKE, None) == EINVAL
    assert lib.pkv_swap_out(FAKE, FAKE, pool, ids, 3, None, FAKE, None) == EINVAL
    b, bad = _ids(0, 8)
    assert lib.pkv_swap_out(FAKE, FAKE, pool, bad, 2, FAKE, FAKE, None) == ERANGE
    c, dup = _ids(4, 1, 4)
    assert lib.pkv_swap_in(FAKE, FAKE, dup, 3, FAKE, FAKE, pool, None) == EALIAS
    assert lib.pkv_swap_in(FAKE, FAKE, bad, 2, FAKE, FAKE, pool, None) == ERANGE
    assert lib.pkv_swap_out(FAKE, FAKE, _Pool(8, 2, 8, 128), ids, 3, FAKE, FAKE, None) != 0  # bs not a multiple of 16
    # host memory the device cannot address (here: any pointer, or pageable memory) is refused
    host = np.zeros(3 * 2 * 16 * 128, dtype=np.uint16)
    hp = host.ctypes.data_as(ctypes.c_void_p)
    assert lib.pkv_swap_out(FAKE, FAKE, pool, ids, 3, hp, hp, None) == EINVAL


def test_block_manager_host_validation():
    """Host checks of the device block manager's entry points (no GPU work)."""
    lib = pkv.load_library()
    assert lib.pkv_bm_state_bytes(0) == 0
    assert lib.pkv_bm_state_bytes(10) == 256 + 7 * 256 + 2 * 256  # 7 int32 arrays, keys and ring
    assert lib.pkv_bm_state_bytes(100) == 256 + 7 * 512 + 2 * 1024
    assert lib.pkv_bm_state_bytes((1 << 29) + 1) == 0  # above the supported pool size
    assert lib.pkv_prefix_cache_bytes(0) == 0 and lib.pkv_prefix_cache_bytes(48) == 0  # power of two
    assert lib.pkv_prefix_cache_bytes(64) == 512 + 2 * 256
    assert lib.pkv_prefix_cache_init(FAKE, 48, None) == EINVAL
    assert lib.pkv_bm_init(None, 8, None) == EINVAL
    assert lib.pkv_bm_init(ctypes.c_void_p(0x10080), 8, None) == EINVAL  # state not 256-B aligned
    assert lib.pkv_bm_init(FAKE, 0, None) == EINVAL
    assert lib.pkv_bm_alloc(FAKE, 8, FAKE, -1, FAKE, FAKE, 4, None) == EINVAL
    assert lib.pkv_bm_alloc(FAKE, 8, FAKE, 2, None, FAKE, 4, None) == EINVAL
    assert lib.pkv_bm_free(FAKE, 8, None, 0, None) == 0
    assert lib.pkv_bm_free(FAKE, 8, None, 3, None) == EINVAL
    assert lib.pkv_bm_share(FAKE, 8, ctypes.c_void_p(0x10002), 3, None) == EINVAL  # ids not 4-B aligned
    args = [FAKE, 8, FAKE, 4, FAKE, FAKE, 2, 16, FAKE, 32, FAKE, FAKE, None]
    bad = list(args); bad[8] = None  # no slot mapping
    assert lib.pkv_bm_append_slots(*bad) == EINVAL
    bad = list(args); bad[9] = -1  # negative capacity
    assert lib.pkv_bm_append_slots(*bad) == EINVAL
    bad = list(args); bad[7] = 0  # block size
    assert lib.pkv_bm_append_slots(*bad) == EINVAL
    pool = _Pool(8, 2, 16, 128)
    assert lib.pkv_copy_blocks_dev(FAKE, FAKE, 0, FAKE, FAKE, pool, None) == 0
    assert lib.pkv_copy_blocks_dev(None, FAKE, 4, FAKE, FAKE, pool, None) == EINVAL
