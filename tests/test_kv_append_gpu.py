"""GPU parity of the cache append (mla_kv_append) against the CPU oracle, through the
C ABI: a byte copy, so the whole pool must match bit for bit."""

import numpy as np
import pytest
import torch

import oracle
from oracle import kv_append as ka
from mla_paged_kv_06_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _mla():
    from mla_paged_kv_06_b200 import mla
    return mla


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _run(kcache, block_table, lens, kv_new):
    mla = _mla()
    kc = kcache.cuda()
    mla.mla_kv_append(kv_new.cuda(), block_table.cuda(), torch.tensor(lens, dtype=torch.int32).cuda(), kc)
    torch.cuda.synchronize()
    st, word = mla.mla_get_last_device_error()
    return kc, st, word


@pytest.mark.parametrize("lens_old, s_new", [
    ([0, 63, 64, 127, 1000], 1),
    ([63, 1, 62], 2),
    ([5, 200], 4),
    ([7] * 300, 3),
])
def test_append_matches_oracle_bit_for_bit(lens_old, s_new):
    x = wl.make_paged_inputs([L + s_new for L in lens_old], 1, 8, seed=41, spare_blocks=3,
                             poison=True)
    g = torch.Generator().manual_seed(9)
    kv_new = torch.randn((len(lens_old), s_new, 576), generator=g).to(torch.bfloat16)
    kc, st, word = _run(x.kcache, x.block_table, lens_old, kv_new)
    assert st == 0, hex(word)
    want = ka.append(x.kcache, x.block_table, lens_old, kv_new)
    assert np.array_equal(_bits(kc), want)


def test_decode_after_append_matches_oracle():
    mla = _mla()
    lens_old, s_new = [100, 4000, 63, 1], 1
    full = wl.make_paged_inputs([L + s_new for L in lens_old], 1, 128, seed=42, spare_blocks=2,
                                poison=True)
    # the new rows as they sit in the longer cache, and that cache with their slots wiped
    kv_new = torch.zeros((len(lens_old), s_new, 576), dtype=torch.bfloat16)
    wiped = full.kcache.clone()
    for b, L in enumerate(lens_old):
        for j in range(s_new):
            t = L + j
            blk, slot = int(full.block_table[b, t // 64]), t % 64
            kv_new[b, j] = full.kcache[blk, slot, 0]
            wiped[blk, slot, 0] = float("nan")
    kc, st, _ = _run(wiped, full.block_table, lens_old, kv_new)
    assert st == 0
    d_bt, d_sl = full.block_table.cuda(), full.seqlens.cuda()
    meta, ns = mla.mla_get_metadata(d_sl, full.h_q, full.s_q)
    out, lse = mla.mla_decode_fwd(full.q.cuda(), kc, d_bt, d_sl, full.scale, False, meta, ns)
    torch.cuda.synchronize()
    ref_out, ref_lse = oracle.decode(full.q, full.kcache, full.block_table, full.seqlens,
                                     full.scale, False)
    assert np.abs(out.double().cpu().numpy() - ref_out).max() <= 1e-2
    assert np.abs(lse.double().cpu().numpy() - ref_lse).max() <= 1e-3


def test_bad_positions_and_blocks_are_reported_and_not_written():
    mla = _mla()
    x = wl.make_paged_inputs([64, 10], 1, 8, seed=43, spare_blocks=1)
    kv_new = torch.ones((2, 1, 576), dtype=torch.bfloat16)
    # sequence 0 is full: position 64 is past its one-page table
    kc, st, _ = _run(x.kcache, x.block_table, [64, 10], kv_new)
    assert st == mla.MLA_ERR_DEVICE_BAD_INPUT
    want = ka.append(x.kcache, x.block_table[1:], [10], kv_new[1:])   # only sequence 1
    got = _bits(kc)
    assert np.array_equal(got, want)
    # a block id outside the pool
    bt = x.block_table.clone()
    bt[1, 0] = x.num_blocks + 3
    kc, st, _ = _run(x.kcache, bt, [3, 10], kv_new)
    assert st == mla.MLA_ERR_DEVICE_BAD_INPUT
    assert mla.mla_get_last_device_error()[0] == mla.MLA_OK
