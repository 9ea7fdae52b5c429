"""Replica mode of the benchmark on CPU: two gloo ranks, no GPU.

Each rank runs an independent problem (its own seed), the step time is the
max over ranks, and the whole-job value counts every rank's work.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from block_sparse_attention_threshold_b200 import synthetic as syn
        w = bench.rank_workload(syn.workload("tiny_n1024"), rank, world)
        q, _, _ = syn.generate_bf16(w)
        local_ms = 10.0 + 5.0 * rank
        ms = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        val = bench.whole_job_tflops(w.dense_flops(), world, ms)
        out.put((rank, w.seed, int(q.astype("int64").sum()), ms, val))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_replicas():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, s0, h0, ms0, v0), (r1, s1, h1, ms1, v1) = res
    assert s0 != s1 and h0 != h1          # independent problems
    assert ms0 == ms1 == 15.0             # max over ranks
    from block_sparse_attention_threshold_b200 import synthetic as syn
    flops = syn.workload("tiny_n1024").dense_flops()
    assert v0 == pytest.approx(2 * flops / 15e-3 / 1e12)


def test_single_rank_is_identity():
    from block_sparse_attention_threshold_b200 import synthetic as syn
    w = syn.workload("tiny_n1024")
    assert bench.rank_workload(w, 0, 1) is w
    assert bench.max_over_ranks(3.0, 1, None) == 3.0
