"""Head-parallel MonarchAttention over several GPUs, one process per GPU.

The B*H heads of a forward pass are independent problems (every step of the
method works inside one head), so the multi-GPU form shards the heads: each
rank runs the forward pass of a contiguous slice of the flattened (B*H) head
index on its own GPU, with its own stream and the library's per-device
workspace.  Nothing crosses GPUs on the data path: no peer loads and no
collective.  The one optional collective is the gather of the output slices
when the caller wants every rank to hold the whole output
(``gather=True``, an all-gather over the process group).

Use with ``torch.distributed`` initialised (NCCL on GPUs), one rank per GPU:

    from structured_sub_quadratic_b200 import parallel
    lo, hi = parallel.head_shard(B * H, rank, world)
    out = parallel.head_parallel_forward(q, k, v, b1, b2, T, c1, c2)

``q``, ``k``, ``v`` may hold every head (the rank takes its slice) or just the
rank's slice (``local=True``).
"""
from __future__ import annotations

import torch


def head_shard(n_heads: int, rank: int, world: int):
    """[lo, hi) of the flattened heads owned by `rank`: contiguous slices
    whose sizes differ by at most one, the larger ones first (so every head is
    owned by exactly one rank, and a rank may own none when world > n_heads)."""
    if world < 1 or not (0 <= rank < world) or n_heads < 0:
        raise ValueError(f"bad shard request: n_heads={n_heads} rank={rank} world={world}")
    base, extra = divmod(n_heads, world)
    lo = rank * base + min(rank, extra)
    hi = lo + base + (1 if rank < extra else 0)
    return lo, hi


def _dist():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        return dist, dist.get_rank(), dist.get_world_size()
    return None, 0, 1


def head_parallel_forward(q, k, v, b1, b2, T, c1=1, c2=1, *, local=False, gather=False,
                          forward=None):
    """MonarchAttention forward of this rank's heads.

    q, k, v: (B, H, N, d) with every head (``local=False``; the rank's
    contiguous slice of the flattened heads is taken), or (n_local, N, d) /
    (1, n_local, N, d) holding just this rank's heads (``local=True``).
    Returns this rank's output heads as (n_local, N, d), or with
    ``gather=True`` the whole (B, H, N, d) output on every rank (requires
    ``local=False``).  ``forward`` is the per-rank forward of a (1, n, N, d)
    batch; the default is the library's C-ABI forward on the current device.
    """
    if forward is None:
        from . import api
        forward = api.monarch_attn_fwd
    dist, rank, world = _dist()
    if local:
        if gather:
            raise ValueError("gather=True needs every head in q, k, v (local=False)")
        heads = q.reshape(-1, q.shape[-2], q.shape[-1])
        lo, hi = 0, heads.shape[0]
        qs, ks, vs = (x.reshape(-1, x.shape[-2], x.shape[-1]) for x in (q, k, v))
    else:
        if q.dim() != 4:
            raise ValueError("expected (B, H, N, d) tensors")
        B, H, N, d = q.shape
        lo, hi = head_shard(B * H, rank, world)
        qs, ks, vs = (x.reshape(B * H, N, d)[lo:hi] for x in (q, k, v))
    n_local = hi - lo
    N, d = qs.shape[-2], qs.shape[-1]
    if n_local > 0:
        o = forward(qs.contiguous().view(1, n_local, N, d), ks.contiguous().view(1, n_local, N, d),
                    vs.contiguous().view(1, n_local, N, d), b1, b2, T, c1, c2)
        o = o.reshape(n_local, N, d)
    else:
        o = qs.new_empty((0, N, d))
    if not gather:
        return o
    B, H = q.shape[0], q.shape[1]
    full = q.new_empty((B * H, N, d))
    if dist is None or world == 1:
        full.copy_(o)
        return full.view(B, H, N, d)
    # shards differ in size by at most one head: every rank sends a buffer of
    # the largest shard's size (one all-gather of equal parts), then each
    # rank's valid heads are copied into their place
    width = head_shard(B * H, 0, world)[1]
    send = q.new_zeros((width, N, d))
    send[:n_local].copy_(o)
    recv = q.new_empty((world * width, N, d))
    dist.all_gather_into_tensor(recv, send)
    for r in range(world):
        rlo, rhi = head_shard(B * H, r, world)
        full[rlo:rhi].copy_(recv[r * width:r * width + (rhi - rlo)])
    return full.view(B, H, N, d)
