"""Split-KV across ranks, host side (no GPU): the page plan, the per-rank slices and
the exchange, checked by decoding every rank's slice with the oracle and merging the
parts with the oracle's combine; the result must equal the oracle on the whole batch.
Also run as two and three gloo ranks that exchange their partials for real.
"""

import datetime
import os
import random
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from mla_paged_kv_06_b200 import splitkv as skv
from mla_paged_kv_06_b200 import workloads as wl


def _oracle(x):
    return oracle.decode(x.q, x.kcache, x.block_table, x.seqlens, x.scale, x.causal)


def _merge(parts):
    """oracle.combine over rank partials given as (out [b,s_q,h_q,512], lse [b,h_q,s_q])."""
    b, s_q, h_q, _ = parts[0][0].shape
    po = np.stack([o.reshape(-1, 512) for o, _ in parts])
    pl = np.stack([np.transpose(l, (0, 2, 1)).reshape(-1) for _, l in parts])
    out, lse = oracle.combine(po, pl)
    return out.reshape(b, s_q, h_q, 512), np.transpose(lse.reshape(b, s_q, h_q), (0, 2, 1))


def _close(a, b, tol=1e-12):
    (oa, la), (ob, lb) = a, b
    assert np.array_equal(np.isfinite(la), np.isfinite(lb))
    fin = np.isfinite(lb)
    assert np.abs(oa - ob).max() <= tol
    if fin.any():
        assert np.abs(la[fin] - lb[fin]).max() <= tol


LENGTHS = [0, 1, 2, 63, 64, 65, 127, 129, 300, 1000]


@pytest.mark.parametrize("world", [1, 2, 3, 4, 7])
@pytest.mark.parametrize("s_q, causal", [(1, False), (2, True), (4, True), (16, True), (3, False)])
def test_plan_partitions_pages_and_respects_the_causal_rule(world, s_q, causal):
    plan = skv.plan_kv_split(LENGTHS, world, s_q, causal)
    for b, L in enumerate(LENGTHS):
        P = (L + 63) // 64
        # contiguous, in rank order, covering [0, P) once
        assert plan.page_begin[0][b] == 0 and plan.page_end[world - 1][b] == P
        for g in range(world):
            assert plan.page_begin[g][b] <= plan.page_end[g][b]
            if g:
                assert plan.page_begin[g][b] == plan.page_end[g - 1][b]
        assert sum(plan.tokens[g][b] for g in range(world)) == L
        for g in range(world - 1):
            if plan.tokens[g][b]:
                assert plan.tokens[g][b] == 64 * (plan.page_end[g][b] - plan.page_begin[g][b])
                if causal:       # every token of a non-last rank is seen by every query
                    assert 64 * plan.page_end[g][b] <= L - s_q + 1
        if not causal:           # balanced to within one page
            counts = [plan.page_end[g][b] - plan.page_begin[g][b] for g in range(world)]
            assert max(counts) - min(counts) <= 1
        assert plan.rank_causal(world - 1) == causal
        assert not any(plan.rank_causal(g) for g in range(world - 1))


def test_plan_rejects_bad_arguments():
    with pytest.raises(ValueError):
        skv.plan_kv_split([5], 0)
    with pytest.raises(ValueError):
        skv.plan_kv_split([5], 2, s_q=0)
    with pytest.raises(ValueError):
        skv.plan_kv_split([-1], 2)


@pytest.mark.parametrize("world", [2, 3, 4])
@pytest.mark.parametrize("s_q, h_q, causal", [(1, 16, False), (2, 8, True), (4, 4, True),
                                               (3, 5, False)])
def test_rank_slices_merge_to_the_whole_decode(world, s_q, h_q, causal):
    x = wl.make_paged_inputs([0, 1, 3, 64, 65, 130, 200, 70], s_q, h_q, seed=40 + world,
                             causal=causal, spare_blocks=3, poison=True)
    plan = skv.plan_kv_split(x.seqlens, world, s_q, causal)
    parts = []
    for g in range(world):
        xr = skv.make_kv_slice(x, plan, g)
        assert xr.causal == (causal and g == world - 1)
        # the compact pool holds exactly the rank's pages
        assert xr.kcache.shape[0] == max(1, sum(plan.page_end[g][b] - plan.page_begin[g][b]
                                                for b in range(x.batch)))
        parts.append(_oracle(xr))
    _close(_merge(parts), _oracle(x))


def test_more_ranks_than_pages_and_all_empty():
    x = wl.make_paged_inputs([5, 0], 2, 4, seed=47, causal=True, spare_blocks=1, poison=True)
    plan = skv.plan_kv_split(x.seqlens, 4, 2, True)
    parts = [_oracle(skv.make_kv_slice(x, plan, g)) for g in range(4)]
    merged = _merge(parts)
    _close(merged, _oracle(x))
    assert np.all(merged[0][1] == 0) and np.all(np.isneginf(merged[1][1]))


def test_a_non_last_rank_decoded_causally_is_caught():
    # planted mistake: every rank applies the causal mask to its own slice
    x = wl.make_paged_inputs([200, 130], 2, 4, seed=48, causal=True, spare_blocks=1)
    plan = skv.plan_kv_split(x.seqlens, 2, 2, True)
    parts = []
    for g in range(2):
        xr = skv.make_kv_slice(x, plan, g)
        xr.causal = True
        parts.append(_oracle(xr))
    with pytest.raises(AssertionError):
        _close(_merge(parts), _oracle(x), tol=1e-6)


def test_a_plan_that_ignores_the_causal_rule_is_caught():
    # planted mistake: the last rank holds fewer than s_q - 1 tokens (plain even split),
    # so rank 1 decodes tokens that query 0 must not see
    L, s_q, world = 129, 4, 3
    x = wl.make_paged_inputs([L], s_q, 4, seed=49, causal=True)
    plan = skv.plan_kv_split([L], world, s_q, causal=False)  # no causal adjustment
    assert plan.tokens[2][0] < s_q - 1 and 64 * plan.page_end[1][0] > L - s_q + 1
    plan.causal = True
    parts = [_oracle(skv.make_kv_slice(x, plan, g)) for g in range(world)]
    with pytest.raises(AssertionError):
        _close(_merge(parts), _oracle(x), tol=1e-6)
    good = skv.plan_kv_split([L], world, s_q, causal=True)
    assert good.tokens[2][0] >= s_q - 1
    parts = [_oracle(skv.make_kv_slice(x, good, g)) for g in range(world)]
    _close(_merge(parts), _oracle(x))


def test_random_plans_merge_exactly():
    rng = random.Random(50)
    for case in range(12):
        world = rng.randint(2, 5)
        s_q = rng.choice([1, 2, 3, 5])
        causal = rng.random() < 0.6
        lens = [rng.choice([0, 1, rng.randint(1, 400)]) for _ in range(rng.randint(1, 4))]
        x = wl.make_paged_inputs(lens, s_q, 3, seed=100 + case, causal=causal,
                                 spare_blocks=1, poison=True)
        plan = skv.plan_kv_split(x.seqlens, world, s_q, causal)
        parts = [_oracle(skv.make_kv_slice(x, plan, g)) for g in range(world)]
        _close(_merge(parts), _oracle(x))


def test_exchange_without_a_process_group_returns_the_own_part():
    o = torch.randn(2, 1, 4, 512)
    l = torch.randn(2, 4, 1)
    po, pl = skv.exchange_partials(o, l)
    assert po.shape == (1, 2, 1, 4, 512) and torch.equal(po[0], o) and torch.equal(pl[0], l)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, result_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # every rank builds the same global inputs, decodes only its slice, then the
        # partials are exchanged in the layout the device combine reads
        x = wl.make_paged_inputs([700, 1, 0, 130, 64], 2, 4, seed=51, causal=True,
                                 spare_blocks=2, poison=True)
        plan = skv.plan_kv_split(x.seqlens, world, 2, True)
        out, lse = _oracle(skv.make_kv_slice(x, plan, rank))
        o_parts, lse_parts = skv.exchange_partials(torch.from_numpy(out), torch.from_numpy(lse))
        ok = tuple(o_parts.shape) == (world,) + out.shape
        ok = ok and torch.equal(o_parts[rank], torch.from_numpy(out))
        parts = [(o_parts[g].numpy(), lse_parts[g].numpy()) for g in range(world)]
        merged = _merge(parts)
        ref = _oracle(x)
        try:
            _close(merged, ref)
        except AssertionError:
            ok = False
        flags = [None] * world
        dist.all_gather_object(flags, bool(ok))
        if rank == 0:
            with open(os.path.join(result_dir, "ok"), "w") as f:
                f.write("1" if all(flags) else "0")
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_exchange_partials_and_merge(tmp_path, world):
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    assert (tmp_path / "ok").read_text() == "1"
