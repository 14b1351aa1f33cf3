"""Host logic of the multi-GPU benchmark path, run as two gloo ranks on CPU.

The decode path shards by sequence with no data-path collective: each rank runs its own
sequences, and only a MAX all-reduce of device times (plus barriers) crosses ranks.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import bench
    from mla_latent_kv_42_b200 import synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = bench.rank_workload(synth.workload("production_b128_ragged_paged_bf16"), rank)
        lens = synth.cached_lengths(w)
        mine = [10.0 + rank, 3.0 * (1 - rank), 7.0]
        got = bench.max_over_ranks(mine, torch.device("cpu"), world)
        dist.barrier()
        q.put((rank, w.seed, lens.tolist()[:8], got))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_own_distinct_sequences():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = dict()
    for _ in range(2):
        rank, seed, lens, got = q.get(timeout=120)
        out[rank] = (seed, lens, got)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out[0][2] == out[1][2] == [11.0, 3.0, 7.0]          # element-wise max over ranks
    assert out[0][0] != out[1][0] and out[0][1] != out[1][1]    # each rank has its own sequences


def test_job_metric_aggregates_ranks_and_layers():
    import bench
    # 20 steps of 12 layers took 240 ms on the slowest of 4 ranks: each rank advanced 240 layer-steps
    assert bench.job_us_per_layer_step(240.0, 20, 12, 4) == pytest.approx(250.0)
    assert bench.job_us_per_layer_step(10.0, 10, 1, 1) == pytest.approx(1000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import argparse
    import bench
    monkeypatch.setenv("RANK", "1")
    args = argparse.Namespace(workload="running_b1_n256_fp16", steps=1, warmup=3, gpus=2)
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""
