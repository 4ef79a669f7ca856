"""Multi-process data parallelism on CPU (gloo, world size 2).

Each rank takes its shard of a global batch, computes the gradient of its
shard's mean loss with the CPU oracle, and the ranks average the gradients with
adjoint_gradients_b200.dp.  The result must equal the single-process gradient of
the global batch's mean loss.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from adjoint_gradients_b200 import dp
from adjoint_gradients_b200.inputs import random_case


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, B, n, L, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x, theta, y = random_case(42, B, n, L)
        sl = dp.shard(B, world, rank)
        E = oracle.forward(x[sl], theta)
        g, _ = oracle.adjoint(x[sl], theta, oracle.loss_seed(E, y[sl]))
        t = torch.from_numpy(g.copy())
        dp.average_gradients(t)
        if rank == 0:
            np.save(out, t.numpy())
    finally:
        dist.destroy_process_group()


def test_shards_cover_the_batch():
    for B in (1, 7, 64, 85):
        for world in (1, 2, 3, 8):
            idx = np.concatenate([np.arange(B)[dp.shard(B, world, r)] for r in range(world)])
            np.testing.assert_array_equal(idx, np.arange(B))


def test_two_rank_gradient_average_matches_global_batch(tmp_path):
    B, n, L = 8, 5, 3
    out = str(tmp_path / "g.npy")
    mp.start_processes(_worker, args=(2, _free_port(), B, n, L, out), nprocs=2, start_method="spawn")
    got = np.load(out)
    x, theta, y = random_case(42, B, n, L)
    E = oracle.forward(x, theta)
    want, _ = oracle.adjoint(x, theta, oracle.loss_seed(E, y))
    np.testing.assert_allclose(got, want, atol=1e-12)
