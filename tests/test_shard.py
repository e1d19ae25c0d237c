"""Data-parallel host logic on CPU: batch sharding, per-shard page pools and the
max-over-ranks reduction, in one process and as two gloo ranks.

The decode's sequences are independent, so the oracle's result for a shard must equal,
bit for bit, the rows of the whole batch's result at the shard's indices (the oracle
computes every sequence on its own, in the same order, from the same values).
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from mla_paged_kv_06_b200 import shard as sh
from mla_paged_kv_06_b200 import workloads as wl


def _oracle(x):
    return oracle.decode(x.q, x.kcache, x.block_table, x.seqlens, x.scale, x.causal)


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_shard_batch_partitions_and_balances(world):
    lens = wl.draw_seqlens("uniform:1,8192", 128, seed=3)
    shards = sh.shard_batch(lens, world)
    assert len(shards) == world
    flat = sorted(i for s in shards for i in s)
    assert flat == list(range(128))
    assert all(s == sorted(s) for s in shards)
    loads = [sum(sh.sequence_cost(int(lens[i])) for i in s) for s in shards]
    # longest-first greedy: the spread is at most the largest single cost
    assert max(loads) - min(loads) <= max(sh.sequence_cost(int(L)) for L in lens.tolist())


def test_shard_batch_more_ranks_than_sequences():
    shards = sh.shard_batch([5, 700, 64], 5)
    assert sorted(i for s in shards for i in s) == [0, 1, 2]
    assert sum(1 for s in shards if not s) == 2
    assert shards[0] == [1]                     # the longest goes to rank 0


def test_shard_batch_is_deterministic_and_rejects_bad_world():
    lens = [100, 100, 100, 5000, 1]
    assert sh.shard_batch(lens, 2) == sh.shard_batch(torch.tensor(lens), 2)
    with pytest.raises(ValueError):
        sh.shard_batch(lens, 0)


def test_make_shard_pool_holds_only_owned_pages():
    x = wl.make_paged_inputs([130, 1, 64, 65, 0], 1, 16, seed=2, spare_blocks=3, poison=True)
    y = sh.make_shard(x, [0, 3, 4])
    assert y.batch == 3 and y.seqlens.tolist() == [130, 65, 0]
    assert y.num_blocks == 3 + 2                # ceil(130/64) + ceil(65/64) pages
    assert int(y.block_table.max()) < y.num_blocks
    # page contents follow the renumbering
    for row, b in enumerate([0, 3]):
        for j in range(int(wl.blocks_needed(y.seqlens[row:row + 1])[0])):
            a = x.kcache[int(x.block_table[b, j])]
            c = y.kcache[int(y.block_table[row, j])]
            assert torch.equal(a.view(torch.int16), c.view(torch.int16))


def test_make_shard_empty():
    x = wl.make_paged_inputs([10, 20], 2, 8, seed=1)
    y = sh.make_shard(x, [])
    assert y.batch == 0 and y.num_blocks == 1 and y.block_table.shape == (0, 1)


@pytest.mark.parametrize("world", [2, 3])
def test_shard_results_reassemble_the_batch(world):
    x = wl.make_paged_inputs([300, 1, 64, 129, 5, 700, 0, 65], 2, 8, seed=4, causal=True,
                             spare_blocks=2, poison=True)
    ref_out, ref_lse = _oracle(x)
    out = np.full_like(ref_out, np.nan)
    lse = np.full_like(ref_lse, np.nan)
    for idx in sh.shard_batch(x.seqlens, world):
        if not idx:
            continue
        o, l = _oracle(sh.make_shard(x, idx))
        out[idx], lse[idx] = o, l
    assert np.array_equal(out, ref_out)
    assert np.array_equal(lse, ref_lse, equal_nan=True)


def test_rank_seed_and_single_process_reduction():
    assert sh.rank_seed(0, 0) == 0 and sh.rank_seed(5, 3) == 8
    assert len({sh.rank_seed(7, r) for r in range(8)}) == 8
    assert sh.max_over_ranks(2.5) == 2.5


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, result_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # every rank builds the same global batch, decodes its shard, gathers the pieces
        x = wl.make_paged_inputs([300, 1, 64, 129, 5, 700, 0, 65, 2000], 1, 16, seed=6,
                                 spare_blocks=2, poison=True)
        idx = sh.shard_batch(x.seqlens, world)[rank]
        piece = _oracle(sh.make_shard(x, idx)) if idx else None
        gathered = [None] * world
        dist.all_gather_object(gathered, (idx, piece))
        # the job's time is the slowest rank's
        slowest = sh.max_over_ranks(1.0 + rank, dist)
        # weak scaling: every rank's own batch differs
        own = wl.make_paged_inputs([37], 1, 16, seed=sh.rank_seed(0, rank))
        seeds = [None] * world
        dist.all_gather_object(seeds, own.q.float().sum().item())
        if rank == 0:
            ref_out, ref_lse = _oracle(x)
            out = np.full_like(ref_out, np.nan)
            lse = np.full_like(ref_lse, np.nan)
            seen = []
            for i, p in gathered:
                seen += i
                if p is not None:
                    out[i], lse[i] = p
            ok = (sorted(seen) == list(range(x.batch)) and np.array_equal(out, ref_out)
                  and np.array_equal(lse, ref_lse, equal_nan=True)
                  and slowest == float(world) and len(set(seeds)) == world)
            with open(os.path.join(result_dir, "ok"), "w") as f:
                f.write("1" if ok else "0")
        else:
            assert slowest == float(world)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_decode_and_reduce(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    assert (tmp_path / "ok").read_text() == "1"
