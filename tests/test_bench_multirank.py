"""The benchmark's N > 1 path on CPU ranks (gloo, world size 2): every rank
scans its own independent workload (weak scaling, no data-path collective)
and the job's time is the slowest rank's, reduced with one all-reduce MAX."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank-local timings: rank 1 is the slower one on the device, rank 0 end to end
        total_ms = [100.0, 130.0][rank]
        e2e_s = [0.9, 0.5][rank]
        got = bench.max_over_ranks(dist, [total_ms, e2e_s], "cpu")
        sigma, _ = synth.channel_sigma(rank, 8)      # each rank's own workload
        out[rank] = (got, sigma.sum())
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_rank_and_shard_by_seed():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(2, port, out), nprocs=2, join=True,
                           start_method="spawn")
        res = dict(out)
    assert res[0][0] == res[1][0] == [130.0, 0.9]
    assert res[0][1] != res[1][1]            # independent (rank-seeded) sessions


def test_throughput_counts_every_rank():
    v, e = bench.job_throughput(keys_per_step=8 * 131072 * 3, steps=30, world=2,
                                total_ms=2000.0, e2e_seconds=4.0)
    keys = 8 * 131072 * 3 * 30 * 2
    assert v == pytest.approx(keys / 2.0 / 1e9)
    assert e == pytest.approx(keys / 4.0 / 1e9)
    assert bench.max_over_ranks(None, [1.5, 2], "cpu") == [1.5, 2.0]


def test_reference_arm_runs_on_rank_zero_only(capsys, monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = type("A", (), dict(gpus=2, steps=1, warmup=0))()
    bench.run_reference(args, "qwen3_8b_layer_128k", bench.WORKLOADS["qwen3_8b_layer_128k"])
    assert capsys.readouterr().out == ""
