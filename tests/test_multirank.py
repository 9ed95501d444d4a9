"""Host logic of the multi-GPU benchmark on CPU: two gloo ranks.

The decode path shards by sequence with no data exchange, so `bench.py --gpus
N` runs one independent seeded batch per rank.  These tests check the parts
that do not need a GPU: each rank gets its own batch, the timing is the
slowest rank's, bytes are summed over ranks, and the reference arm runs on
rank 0 only.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        class A:
            workload, block_size, seed, max_seqs = "llama2-13b", None, 0, 0
        w = bench.make_workload(A, rank, "meta")
        ms = [10.0, 14.0][rank]
        nbytes = bench.step_bytes(w)
        ms_max, bytes_all, seqs_all = bench.combine_ranks(dist, ms, nbytes, w.num_seqs, "cpu")
        gathered = [None] * world
        dist.all_gather_object(gathered, (int(w.context_lens.sum()), nbytes))
        results[rank] = dict(ms_max=ms_max, bytes_all=bytes_all, seqs_all=seqs_all, mine=nbytes, all=gathered,
                             ref=bench.run_reference(type("R", (), dict(steps=1, warmup=0, workload="tiny",
                                                                         block_size=None, seed=0))(), rank, world))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling_reduction():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        results = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, results)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=300)
            assert p.exitcode == 0
        r0, r1 = results[0], results[1]
    # the slowest rank's time, summed bytes and sequences
    assert r0["ms_max"] == r1["ms_max"] == 14.0
    assert r0["bytes_all"] == r1["bytes_all"] == r0["mine"] + r1["mine"]
    assert r0["seqs_all"] == 256
    # each rank drew its own batch (seed + rank)
    (tok0, b0), (tok1, b1) = r0["all"]
    assert tok0 != tok1 and b0 != b1
    # whole-job throughput uses every rank's bytes over the slowest time
    assert bench.whole_job_gbs(r0["bytes_all"], 10, r0["ms_max"]) == pytest.approx(
        (r0["mine"] + r1["mine"]) * 10 / 0.014 / 1e9)
    # the CPU reference arm runs on rank 0 only
    assert r0["ref"]["impl"] == "reference" and r1["ref"] is None
