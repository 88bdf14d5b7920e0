"""Host logic of the multi-GPU bench (replicas, no data-path collective) on
CPU ranks over gloo, world size 2: the timing is the max over ranks and
every replica draws its own tokens while sharing the model."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from expert_routing_grouped_layer_b200 import workloads as W


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        timed = bench.max_over_ranks(1.5 + rank, "cpu")
        cfg = W.CONFIGS["tiny_bf16"]
        x = W.make_inputs(cfg.replace(seed=bench.replica_seed(cfg.seed, rank)))["x"]
        wg = W.make_inputs(cfg)["gate_w"]
        xf = x.float().contiguous()  # gloo gathers float32, not 16-bit tensors
        xs = [torch.zeros_like(xf) for _ in range(world)]
        dist.all_gather(xs, xf)
        ws = [torch.zeros_like(wg) for _ in range(world)]
        dist.all_gather(ws, wg)
        out[rank] = (timed, not torch.equal(xs[0], xs[1]), torch.equal(ws[0], ws[1]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_timing_and_replica_inputs():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world,
                       start_method="spawn")
    assert out[0][0] == out[1][0] == 2.5  # max over ranks
    assert out[0][1] and out[0][2]  # different tokens, same router weights


def test_single_process_timing_is_identity():
    assert bench.max_over_ranks(3.25, "cpu") == 3.25
    assert bench.replica_seed(11, 0) == 11 and bench.replica_seed(11, 1) != 11
