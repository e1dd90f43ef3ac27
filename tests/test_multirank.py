"""The multi-process plumbing of bench.py on CPU with the gloo backend
(world size 2, 127.0.0.1): the timing reduction takes the slowest rank on
every rank, the job throughput counts every rank's work, and the oracle
reference arm runs and prints on rank 0 only."""
import contextlib
import io
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(1.5 + rank, "cpu")       # rank 1 is the slow one
        zero = bench.max_over_ranks(0.0, "cpu")
        buf = io.StringIO()

        class Args:
            gpus, steps, warmup, cpu_sample_groups, qjl_rows = world, 1, 0, 1, 0
            value_scale, rnorm_f16 = "norm", False

        cfg = bench.synth.KV_CONFIGS["llama3.1-8b_32k_b3"].scaled(layers=1, batch=1, kv_heads=1, seq=256)
        with contextlib.redirect_stdout(buf):
            if rank != 0:  # the reference arm returns at once on the other ranks
                bench.run_reference(Args, cfg)
        dist.barrier()
        q.put((rank, ms, zero, buf.getvalue()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [2.5, 2.5]
    assert [r[2] for r in res] == [0.0, 0.0]
    assert res[1][3] == ""  # rank 1 printed nothing
    # weak scaling: both ranks' bytes over the slowest rank's time
    assert bench.job_throughput(10 ** 9, world, 2.5) == pytest.approx(800.0)


def test_single_process_reduction_is_identity():
    assert bench.max_over_ranks(3.25, "cpu") == 3.25
