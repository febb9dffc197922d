"""Head-parallel multi-GPU forward: the host logic on CPU, world size 2 over gloo.

The forward pass shards into independent heads.  Each rank computes its
contiguous slice of the flattened B*H heads; the optional gather brings the
slices back in order.  Here each rank's forward is the float64 oracle on the
CPU, so the test checks the partition and the gather against one
single-process oracle call on all heads.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import monarch_attention
from structured_sub_quadratic_b200.inputs import iid_qkv
from structured_sub_quadratic_b200.parallel import head_parallel_forward, head_shard


def oracle_forward(q, k, v, b1, b2, T, c1, c2):
    o = monarch_attention(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                          b1, b2, T, c1, c2)
    return torch.from_numpy(o).to(q.dtype)


@pytest.mark.parametrize("n,world", [(12, 1), (12, 2), (12, 5), (3, 8), (0, 3), (384, 8)])
def test_head_shard_covers_every_head_once(n, world):
    shards = [head_shard(n, r, world) for r in range(world)]
    owned = [h for lo, hi in shards for h in range(lo, hi)]
    assert owned == list(range(n))
    sizes = [hi - lo for lo, hi in shards]
    assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)


def test_head_shard_rejects_bad_requests():
    for args in [(4, 2, 2), (4, -1, 2), (4, 0, 0), (-1, 0, 1)]:
        with pytest.raises(ValueError):
            head_shard(*args)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v = iid_qkv(2, 3, 6 * 5, 16, torch.float32, seed=21)
        mine = head_parallel_forward(q, k, v, 6, 5, 2, 2, 1, forward=oracle_forward)
        full = head_parallel_forward(q, k, v, 6, 5, 2, 2, 1, gather=True, forward=oracle_forward)
        lo, hi = head_shard(6, rank, world)
        local = head_parallel_forward(q.reshape(6, 30, 16)[lo:hi], k.reshape(6, 30, 16)[lo:hi],
                                      v.reshape(6, 30, 16)[lo:hi], 6, 5, 2, 2, 1, local=True,
                                      forward=oracle_forward)
        out[rank] = (mine.numpy(), full.numpy(), local.numpy(), (lo, hi))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_head_parallel_forward_over_gloo_matches_one_process(world):
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    q, k, v = iid_qkv(2, 3, 6 * 5, 16, torch.float32, seed=21)
    ref = oracle_forward(q, k, v, 6, 5, 2, 2, 1).numpy()
    flat = ref.reshape(6, 30, 16)
    for rank in range(world):
        mine, full, local, (lo, hi) = out[rank]
        np.testing.assert_array_equal(mine, flat[lo:hi])
        np.testing.assert_array_equal(local, flat[lo:hi])
        np.testing.assert_array_equal(full, ref)


def test_single_process_forward_is_the_whole_batch():
    q, k, v = iid_qkv(1, 2, 4 * 4, 8, torch.float32, seed=3)
    o = head_parallel_forward(q, k, v, 4, 4, 1, forward=oracle_forward, gather=True)
    np.testing.assert_array_equal(o.numpy(), oracle_forward(q, k, v, 4, 4, 1, 1, 1).numpy())
