"""Multi-process host logic of bench.py on CPU (gloo, world size 2): the step
time is the max over ranks, every rank takes the same collective steps, and
the reference arm runs on rank 0 only."""

import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        bench.barrier(dist)
        t = bench.max_over_ranks(10.0 + rank, dist)
        bench.barrier(dist)
        out[rank] = t
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    port = _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    assert out[0] == 11.0 and out[1] == 11.0


def test_single_process_is_identity():
    assert bench.max_over_ranks(3.5, None) == 3.5
    assert bench.max_over_ranks(3.5, dist) == 3.5     # no process group initialised


def test_reference_arm_only_on_rank0(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = bench.argparse.Namespace(steps=1, warmup=3, target_sparsity=0.95, gpus=2)
    assert bench.run_reference(args, bench.WORKLOADS["pr1"], "pr1") == 0
