"""Replica plumbing of bench.py on CPU: world_size 2 over gloo. Each rank reports its own
time; the whole-job throughput uses the slowest rank and counts every rank's units."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        secs = [0.010, 0.025][rank]
        value, t = bench.combine(1e9, secs, world)
        bench.barrier()
        q.put((rank, value, t))
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_use_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, value, t in res:
        assert t == pytest.approx(0.025)
        assert value == pytest.approx(2e9 / 0.025)


def test_reference_arm_other_ranks_print_nothing():
    import bench
    import argparse
    args = argparse.Namespace(workload="decode8b", steps=1, warmup=0)
    assert bench.run_reference(args, world=2, rank=1) is None


def test_work_model_closed_forms():
    import bench
    arch = bench.LLAMA8B
    # weight bytes of one layer: qkv + o + gate_up + down, int8
    wbytes = 6144 * 4096 + 4096 * 4096 + 28672 * 4096 + 4096 * 14336
    assert bench.gemm_bytes(1, 6144, 4096) == 6144 * 4096 + 4096 + 4 + 4 * 6144 + 2 * 6144
    ops, nbytes, gops, gbytes = bench.layer_work(arch, 1)
    assert ops == 2 * wbytes and gbytes > wbytes and nbytes > gbytes
    # the pages' size arithmetic: 8e9 weights are 14.9 GiB in bf16 and 7.45 GiB in int8
    assert round(8e9 * 2 / 1024 ** 3, 1) == 14.9 and round(8e9 / 1024 ** 3, 2) == 7.45
