"""Pins of the cache-append oracle (CPU only).

The append is checked against things other than itself: the decode oracle's own gather
(which defines where token t of a sequence lives), a round trip through a cache the
input generator built with the longer lengths, and the untouched rest of the pool.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import kv_append as ka
from mla_paged_kv_06_b200 import workloads as wl


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _cut(full, lens_old, s_new):
    """kv_new = the rows at positions [L, L + s_new) of a cache built with the longer
    lengths, read with the decode oracle's gather; the cache with those slots wiped."""
    bt = full.block_table
    kv_new = np.zeros((full.batch, s_new, 576), dtype=np.uint16)
    wiped = _bits(full.kcache).copy()
    bits = _bits(full.kcache)
    for b, L in enumerate(lens_old):
        rows = oracle.gather_tokens(bits, bt[b], L + s_new)      # exact: 0..65535 as fp64
        kv_new[b] = np.asarray(rows[L:L + s_new], dtype=np.uint16)
        for j in range(s_new):
            t = L + j
            wiped[int(bt[b, t // 64]), t % 64, 0, :] = 0x7FC0          # bf16 NaN
    return kv_new, wiped


@pytest.mark.parametrize("lens_old, s_new", [
    ([0, 63, 64, 127, 1000], 1),
    ([63, 1, 62], 2),             # crosses a page boundary
    ([5, 200], 4),
])
def test_round_trip_restores_the_longer_cache(lens_old, s_new):
    full = wl.make_paged_inputs([L + s_new for L in lens_old], 1, 16, seed=31,
                                spare_blocks=2, poison=True)
    kv_new, wiped = _cut(full, lens_old, s_new)
    got = ka.append(wiped, full.block_table, lens_old, kv_new)
    assert np.array_equal(got, _bits(full.kcache))


def test_only_the_new_positions_change():
    x = wl.make_paged_inputs([70, 3, 128], 1, 16, seed=32, spare_blocks=3, poison=True)
    lens_old = [70, 3, 120]
    g = np.random.default_rng(5)
    kv_new = g.integers(0, 1 << 15, size=(3, 2, 576), dtype=np.uint16)
    before = _bits(x.kcache)
    after = ka.append(x.kcache, x.block_table, lens_old, kv_new)
    changed = np.argwhere((after != before).any(axis=-1).reshape(x.num_blocks, 64))
    expect = set()
    for b, L in enumerate(lens_old):
        for j in range(2):
            t = L + j
            expect.add((int(x.block_table[b, t // 64]), t % 64))
            assert np.array_equal(after[int(x.block_table[b, t // 64]), t % 64, 0], kv_new[b, j])
    assert {tuple(map(int, c)) for c in changed} <= expect


def test_decode_after_append_equals_decode_of_the_longer_cache():
    lens_old, s_new = [100, 64, 1], 1
    full = wl.make_paged_inputs([L + s_new for L in lens_old], 1, 8, seed=33, spare_blocks=1)
    kv_new, wiped = _cut(full, lens_old, s_new)
    cache = torch.from_numpy(ka.append(wiped, full.block_table, lens_old, kv_new).view(np.int16))
    cache = cache.view(torch.bfloat16)
    a = oracle.decode(full.q, cache, full.block_table, full.seqlens, full.scale, False)
    b = oracle.decode(full.q, full.kcache, full.block_table, full.seqlens, full.scale, False)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_out_of_range_positions_and_blocks_raise():
    x = wl.make_paged_inputs([64], 1, 8, seed=34)
    kv_new = np.zeros((1, 1, 576), dtype=np.uint16)
    with pytest.raises(IndexError):
        ka.append(x.kcache, x.block_table, [64], kv_new)          # table holds one page
    bt = x.block_table.clone()
    bt[0, 0] = x.num_blocks
    with pytest.raises(IndexError):
        ka.append(x.kcache, bt, [3], kv_new)


def test_a_planted_off_by_one_is_caught():
    def shifted(kcache, block_table, seqlens, kv_new):
        return ka.append(kcache, block_table, [int(L) - 1 for L in seqlens], kv_new)
    lens_old, s_new = [63, 10], 2
    full = wl.make_paged_inputs([L + s_new for L in lens_old], 1, 8, seed=35, spare_blocks=1)
    kv_new, wiped = _cut(full, lens_old, s_new)
    assert not np.array_equal(shifted(wiped, full.block_table, lens_old, kv_new),
                              _bits(full.kcache))
