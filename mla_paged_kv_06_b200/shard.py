"""Host-side data parallelism for paged MLA decode: one process per GPU.

Sequences of a decode batch are independent (each row of the output reads only its
own sequence's pages), so a batch splits across ranks with no exchange on the data
path. This module holds the host logic of that split:

- `shard_batch` assigns sequences to ranks so that every rank gets about the same
  number of KV pages (longest-first greedy onto the least-loaded rank; each sequence
  also costs a fixed overhead, the same per-(sequence, row tile) term the split-KV
  scheduler uses).
- `make_shard` cuts a rank's inputs out of a global batch: its q rows, its lengths,
  and a compact page pool holding only the pages its sequences own, with the block
  table renumbered into that pool. Each rank then runs `mla_get_metadata` and
  `mla_decode_fwd` on its own shard, on its own GPU.
- `rank_seed` gives each rank its own batch when every rank decodes a batch of the same
  shape (weak scaling, as the benchmark runs).
- `max_over_ranks` reduces a per-rank time to the job's time (the slowest rank).

Nothing here touches a GPU. The results of the shards, placed back at their indices,
equal the results of the whole batch.
"""

from __future__ import annotations

import torch

from .workloads import BLOCK_SIZE, DecodeInputs

# Fixed cost of one sequence in pages: the same per-item overhead the split-KV
# scheduler charges, so a rank of many short sequences is not under-counted.
SEQUENCE_OVERHEAD_PAGES = 3


def sequence_cost(length: int, tiles: int = 1) -> int:
    """Work of one sequence in page units: its pages plus a fixed overhead, per row tile."""
    pages = (int(length) + BLOCK_SIZE - 1) // BLOCK_SIZE
    return tiles * (pages + SEQUENCE_OVERHEAD_PAGES)


def shard_batch(seqlens, world: int, tiles: int = 1) -> list[list[int]]:
    """Sequence indices of each rank, balanced by `sequence_cost`.

    Longest sequence first, each onto the rank with the least cost so far (ties go to
    the lower rank; equal lengths keep batch order). Every index appears in exactly
    one shard; each shard lists its indices in increasing order. A rank may get an
    empty shard when there are fewer sequences than ranks.
    """
    if world < 1:
        raise ValueError("world must be >= 1")
    lens = [int(x) for x in torch.as_tensor(seqlens).tolist()]
    order = sorted(range(len(lens)), key=lambda b: (-lens[b], b))
    load = [0] * world
    shards: list[list[int]] = [[] for _ in range(world)]
    for b in order:
        r = min(range(world), key=lambda k: (load[k], k))
        shards[r].append(b)
        load[r] += sequence_cost(lens[b], tiles)
    return [sorted(s) for s in shards]


def make_shard(x: DecodeInputs, indices) -> DecodeInputs:
    """The inputs of the sequences `indices` of `x`, with a compact page pool.

    The pool keeps the shard's pages in first-use order. Block-table entries past a
    sequence's last page point at page 0 of the shard pool (the decode never reads
    them). An empty shard, or one whose sequences are all empty, gets a one-page pool
    of zeros so that every pointer stays valid.
    """
    idx = [int(i) for i in indices]
    seqlens = x.seqlens[idx].clone() if idx else torch.zeros(0, dtype=torch.int32)
    q = x.q[idx].clone() if idx else x.q[:0].clone()
    nblk = [(int(L) + BLOCK_SIZE - 1) // BLOCK_SIZE for L in seqlens.tolist()]
    max_blocks = max(nblk + [1])
    remap: dict[int, int] = {}
    table = torch.zeros((len(idx), max_blocks), dtype=torch.int32)
    for row, (b, n) in enumerate(zip(idx, nblk)):
        for j in range(n):
            phys = int(x.block_table[b, j])
            if phys not in remap:
                remap[phys] = len(remap)
            table[row, j] = remap[phys]
    if remap:
        kcache = x.kcache[list(remap.keys())].clone()
    else:
        kcache = torch.zeros((1,) + tuple(x.kcache.shape[1:]), dtype=x.kcache.dtype)
    return DecodeInputs(q, kcache, table, seqlens, x.scale, x.causal, x.workload, x.seed)


def rank_seed(seed: int, rank: int) -> int:
    """Seed of rank `rank`'s batch when every rank decodes its own batch of the same
    shape (weak scaling): distinct per rank, equal to `seed` on rank 0."""
    return int(seed) + int(rank)


def max_over_ranks(value: float, dist=None, device: str | torch.device = "cpu") -> float:
    """The largest `value` over all ranks of the default process group (or `value`
    itself without one). NCCL groups need `device` to be this rank's GPU."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
