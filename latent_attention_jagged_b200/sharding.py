"""Multi-GPU data parallelism for the forward: users are independent (each
user's layers touch only that user's rows) and the weights are small, so a
batch is split by user across ranks, each rank runs its share on its own GPU
with replicated weights, and no collective touches the data path.  The only
exchange is the optional gather of the outputs back into batch order.

Split rule: longest-processing-time first on the per-user algorithmic FLOPs
of the pyramid schedule (the same count as `cost.py`), so that ranks finish
together even for skewed length mixes.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Sequence

import heapq
import numpy as np


def user_flops(lengths: Sequence[int], dims) -> np.ndarray:
    """Algorithmic FLOPs of each user's whole forward (absorbed form)."""
    T = np.asarray(lengths, dtype=np.int64)
    d, h, r, dc, m = dims.d, dims.heads, dims.rank, dims.d_ctx, dims.ffn_mult
    tot = np.zeros(T.shape[0], dtype=np.float64)
    for k in dims.keep:
        n = np.minimum(T, k)
        q = n + dims.n_q
        P = dims.n_q * T + n * T - n * (n - 1) // 2
        tot += (2.0 * T * d * r + 2.0 * q * d * h * r + 2.0 * dc * h * r + 4.0 * h * r * P
                + 2.0 * q * h * r * d + 4.0 * m * q * d * d)
        T = n
    if dims.d_out:
        tot += 2.0 * d * dims.d_out
    return tot


def lpt_partition(costs: Sequence[float], world: int) -> List[np.ndarray]:
    """Assign items to `world` bins, largest first, each to the least-loaded
    bin; every bin keeps its items in ascending original order."""
    if world < 1:
        raise ValueError("world must be >= 1")
    costs = np.asarray(costs, dtype=np.float64)
    order = sorted(range(costs.shape[0]), key=lambda i: (-costs[i], i))
    heap = [(0.0, r) for r in range(world)]
    bins: List[List[int]] = [[] for _ in range(world)]
    for i in order:
        load, r = heapq.heappop(heap)
        bins[r].append(i)
        heapq.heappush(heap, (load + float(costs[i]), r))
    return [np.array(sorted(b), dtype=np.int64) for b in bins]


@dataclass
class Shard:
    users: np.ndarray       # global user indices of this rank, ascending
    offsets: np.ndarray     # int64 [len(users)+1], rows of the sub-batch
    rows: np.ndarray        # int64 [sum T]: global row index of each sub-batch row


def make_shard(offsets: np.ndarray, users: np.ndarray) -> Shard:
    offsets = np.asarray(offsets, dtype=np.int64)
    lens = offsets[users + 1] - offsets[users]
    sub = np.zeros(users.shape[0] + 1, dtype=np.int64)
    np.cumsum(lens, out=sub[1:])
    rows = np.concatenate([np.arange(offsets[u], offsets[u + 1], dtype=np.int64) for u in users]) \
        if users.size else np.zeros(0, dtype=np.int64)
    return Shard(users=users, offsets=sub, rows=rows)


def shard_batch(offsets: np.ndarray, dims, world: int) -> List[Shard]:
    """Split one jagged batch into `world` per-rank sub-batches (LPT on FLOPs)."""
    offsets = np.asarray(offsets, dtype=np.int64)
    lengths = offsets[1:] - offsets[:-1]
    parts = lpt_partition(user_flops(lengths, dims), world)
    return [make_shard(offsets, p) for p in parts]


def gather_outputs(local_out, shard: Shard, batch: int, group=None):
    """All-gather every rank's per-user outputs and put them back in batch
    order (torch.distributed; the only collective of the multi-GPU path)."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    tail = tuple(local_out.shape[1:])
    n_local = torch.tensor([local_out.shape[0]], dtype=torch.int64, device=local_out.device)
    counts = [torch.zeros_like(n_local) for _ in range(world)]
    dist.all_gather(counts, n_local, group=group)
    cmax = int(max(int(c.item()) for c in counts))
    pad = torch.zeros((cmax,) + tail, dtype=local_out.dtype, device=local_out.device)
    pad[: local_out.shape[0]] = local_out
    idx = torch.full((cmax,), -1, dtype=torch.int64, device=local_out.device)
    idx[: shard.users.shape[0]] = torch.as_tensor(shard.users, device=local_out.device)
    outs = [torch.empty_like(pad) for _ in range(world)]
    idxs = [torch.empty_like(idx) for _ in range(world)]
    dist.all_gather(outs, pad, group=group)
    dist.all_gather(idxs, idx, group=group)
    full = torch.zeros((batch,) + tail, dtype=local_out.dtype, device=local_out.device)
    for o, i, c in zip(outs, idxs, counts):
        k = int(c.item())
        full[i[:k]] = o[:k]
    return full
