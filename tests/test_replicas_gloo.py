"""The N > 1 path of bench.py ("replicas only": independent replicas, no data
collective) on CPU with two gloo ranks: the timed region's result is the
slowest rank's time on every rank, the job throughput counts every replica,
and the reference arm runs on rank 0 only."""
import contextlib
import io
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        got = bench.max_over_ranks(ms, "cpu")
        dist.barrier()
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            if rank != 0:  # the reference arm's non-zero ranks leave without work
                bench.run_reference(type("A", (), {"steps": 1, "warmup": 0, "gpus": world})(), rank)
        out[rank] = (got, buf.getvalue())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    assert res[1][1] == ""


def test_job_throughput_counts_every_replica():
    tok = 32768
    one = bench.job_throughput(1, tok, 13.0)
    assert bench.job_throughput(4, tok, 13.0) == pytest.approx(4 * one)
    assert one == pytest.approx(tok / 0.013)
