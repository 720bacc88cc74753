"""The multi-rank plumbing of bench.py on CPU: two gloo ranks, each running
its own replica, time = max over ranks, whole-job value = all ranks' units
over that time (weak scaling).  No GPU and no data-path collective."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, w, local = bench.dist_env()
    assert (r, w, local) == (rank, world, rank)
    d = bench.init_dist(w, "gloo")
    assert d is not None and d.get_world_size() == world
    dev = torch.device("cpu")
    # each rank "measured" a different time; every rank must agree on the max
    ms = 10.0 + 5.0 * rank
    bench.barrier(d, dev)
    m = bench.max_over_ranks(ms, d, dev)
    value = bench.weak_scaling_value(256 * 48 * 48, 4, w, m)
    out[rank] = (m, value)
    bench.barrier(d, dev)
    d.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_and_value():
    world = 2
    port = _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0] == out[1]
    m, value = out[0]
    assert m == 15.0
    assert value == pytest.approx(2 * 256 * 48 * 48 * 4 / 0.015)


def test_single_rank_needs_no_process_group():
    assert bench.init_dist(1, "gloo") is None
    assert bench.max_over_ranks(3.5, None, torch.device("cpu")) == 3.5


def test_reference_arm_prints_only_on_rank_zero(capsys):
    args = bench.parse_args(["--impl", "reference", "--steps", "1", "--warmup", "0",
                             "--cpu-seconds", "0.05"])
    bench.run_reference(args, rank=1, world=2)
    assert capsys.readouterr().out == ""
