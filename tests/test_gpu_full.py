"""Parity at the full sizes of the five decode-step workloads, in the launch
configuration the benchmark times.

Pools after the copy-on-write copies and the write are compared bit-exactly
with the oracle's.  Attention is compared with the fp64 oracle on every
sequence of the 7B, 13B and long-context batches (the long-context batch
includes both 131,072-token sequences, 256 partitions each), and on 64 of the
256 shared-prefix sequences: a seeded sample, every copy-on-write fork, and one
whole group of 8 sharers.  Every output row must be finite.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._gpu_util import assert_attention_close, bits_equal, no_device_error, run_step

pytestmark = pytest.mark.gpu

# (workload, block size, sampled sequences; None = all)
CASES = [
    ("tiny", 16, None),
    ("llama2-7b", 16, None),
    ("llama2-13b", 16, None),
    ("llama2-13b", 32, None),
    ("llama3-8b-gqa-prefix", 16, 64),
    ("llama2-70b-long", 16, None),
    ("llama2-70b-long", 128, None),
]
SHARERS_PER_GROUP = 8  # the shared-prefix batch: groups of 8 consecutive sequences


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
        must = set()
        if len(w.copy_pairs):  # every copy-on-write fork, and the whole group of the first one
            forks = [int(np.nonzero((w.block_tables == d).any(axis=1))[0][0]) for d in w.copy_pairs[:, 1]]
            g0 = forks[0] // SHARERS_PER_GROUP * SHARERS_PER_GROUP
            must = set(forks) | set(range(g0, g0 + SHARERS_PER_GROUP))
        rest = np.array(sorted(set(range(B)) - must))
        rng = np.random.default_rng(123)
        extra = rng.choice(rest, size=max(0, sample - len(must)), replace=False)
        idx = np.array(sorted(must | set(int(x) for x in extra)))
        assert len(idx) == sample
    q = w.q[torch.from_numpy(idx).cuda()]
    ref = oracle.paged_attention(q, okc, ovc, w.block_tables[idx], w.context_lens[idx], w.scale)
    assert_attention_close(out[torch.from_numpy(idx).cuda()], ref, f"{name} bs{bs}")
