"""Parity at the full sizes of the five decode-step workloads, in the launch
configuration the benchmark times.

Pools after the copy-on-write copies and the write are compared bit-exactly
with the oracle's; attention is compared on a seeded sample of sequences that
the fp64 oracle computes one by one (all of them when the batch is small), and
every output row must be finite.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._gpu_util import assert_attention_close, bits_equal, no_device_error, run_step

pytestmark = pytest.mark.gpu

CASES = [
    ("tiny", 16, None),
    ("llama2-7b", 16, 16),
    ("llama2-13b", 16, None),
    ("llama2-13b", 32, 32),
    ("llama3-8b-gqa-prefix", 16, 24),
    ("llama2-70b-long", 16, 2),
    ("llama2-70b-long", 128, 2),
]


@pytest.mark.parametrize("name,bs,sample", CASES)
def test_full_size_step(name, bs, sample):
    w = workloads.make(name, seed=0, values_device="cuda", block_size=bs)
    kc0, vc0 = w.k_cache.cpu(), w.v_cache.cpu()
    kc, vc, out = run_step(w)
    no_device_error()
    assert torch.isfinite(out.float()).all()
    okc, ovc = oracle.bits(kc0), oracle.bits(vc0)
    if len(w.copy_pairs):
        okc, ovc = oracle.copy_blocks(okc, ovc, w.copy_pairs)
    okc, ovc = oracle.kv_write(okc, ovc, w.k_new, w.v_new, w.slot_mapping)
    assert bits_equal(kc, okc) and bits_equal(vc, ovc)
    B = w.num_seqs
    if sample is None or sample >= B:
        idx = np.arange(B)
    else:
        rng = np.random.default_rng(123)
        idx = np.sort(rng.choice(B, size=sample, replace=False))
        if len(w.copy_pairs):  # always include the copy-on-write forks
            forks = [int(np.nonzero((w.block_tables == d).any(axis=1))[0][0]) for d in w.copy_pairs[:, 1]]
            idx = np.union1d(idx, forks)
    q = w.q[torch.from_numpy(idx).cuda()]
    ref = oracle.paged_attention(q, okc, ovc, w.block_tables[idx], w.context_lens[idx], w.scale)
    assert_attention_close(out[torch.from_numpy(idx).cuda()], ref, f"{name} bs{bs}")
