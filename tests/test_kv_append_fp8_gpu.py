"""FP8 cache append on the GPU (mla_kv_append_fp8) against the FP8 oracle's quantizer:
every written row bit for bit, nothing else touched, a whole cache quantized token by
token, and bad positions reported without writing.
"""

import numpy as np
import pytest
import torch

from oracle import fp8_cache as f8
from mla_paged_kv_06_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _mla():
    from mla_paged_kv_06_b200 import mla
    return mla


def _ok():
    mla = _mla()
    torch.cuda.synchronize()
    st, word = mla.mla_get_last_device_error()
    assert st == mla.MLA_OK, (mla.status_string(st), hex(word))


def _rows(n, seed):
    """bf16 rows with every kind of group: wide and narrow ranges, a zero group, exact
    E4M3 values, tiny values in the subnormal range of the codes."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((n, 576), generator=g) * torch.exp(torch.randn((n, 1), generator=g) * 3)
    x[0, 128:256] = 0.0
    x[1 % n, :127] = torch.tensor(f8.e4m3_value(np.arange(0x7F, dtype=np.uint8))).float()
    x[1 % n, 127] = -448.0
    x[2 % n, 256:384] *= 1e-6
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("lens_old, s_new", [([0, 63, 64, 127, 1000], 1), ([63, 1, 62], 2),
                                             ([5, 200, 0], 16)])
def test_written_rows_match_the_oracle_bit_for_bit(lens_old, s_new):
    mla = _mla()
    x = wl.make_paged_inputs([L + s_new for L in lens_old], 1, 8, seed=81, spare_blocks=3)
    nb = x.num_blocks
    g = np.random.default_rng(82)
    before = g.integers(0, 256, size=(nb, 64, 656), dtype=np.uint8)
    cache = torch.from_numpy(before.copy()).cuda()
    kv_new = _rows(len(lens_old) * s_new, 83).reshape(len(lens_old), s_new, 576)
    mla.mla_kv_append_fp8(kv_new.cuda(), x.block_table.cuda(),
                          torch.tensor(lens_old, dtype=torch.int32).cuda(), cache)
    _ok()
    got = cache.cpu().numpy()
    expect = before.copy()
    rows = f8.quantize_rows(kv_new.reshape(-1, 576))
    for b, L in enumerate(lens_old):
        for j in range(s_new):
            t = L + j
            expect[int(x.block_table[b, t // 64]), t % 64] = rows[b * s_new + j]
    assert np.array_equal(got, expect)


def test_a_whole_cache_quantized_token_by_token():
    # every token of a bf16 cache appended into an empty FP8 cache, 16 at a time per
    # sequence, equals the oracle's quantization of the whole cache
    mla = _mla()
    lens = [200, 64, 1, 130]
    x = wl.make_paged_inputs(lens, 1, 8, seed=84)
    cache = torch.zeros((x.num_blocks, 64, 656), dtype=torch.uint8, device="cuda")
    bt = x.block_table.cuda()
    for start in range(0, max(lens), 16):
        for b, L in enumerate(lens):
            n = min(16, L - start)
            if n <= 0:
                continue
            rows = torch.stack([x.kcache[int(x.block_table[b, t // 64]), t % 64, 0]
                                for t in range(start, start + n)])
            mla.mla_kv_append_fp8(rows[None].cuda(), bt[b:b + 1].contiguous(),
                                  torch.tensor([start], dtype=torch.int32).cuda(), cache)
    _ok()
    expect = f8.quantize_cache(x.kcache)
    got = cache.cpu().numpy()
    for b, L in enumerate(lens):
        for t in range(L):
            blk = int(x.block_table[b, t // 64])
            assert np.array_equal(got[blk, t % 64], expect[blk, t % 64]), (b, t)


def test_bad_positions_are_reported_and_not_written():
    mla = _mla()
    x = wl.make_paged_inputs([64], 1, 8, seed=85)
    cache = torch.zeros((x.num_blocks, 64, 656), dtype=torch.uint8, device="cuda")
    kv_new = _rows(1, 86).reshape(1, 1, 576).cuda()
    mla.mla_kv_append_fp8(kv_new, x.block_table.cuda(), torch.tensor([64], dtype=torch.int32).cuda(),
                          cache)                     # past the one-page block table
    torch.cuda.synchronize()
    st, _ = mla.mla_get_last_device_error()
    assert st == mla.MLA_ERR_DEVICE_BAD_INPUT
    assert int(cache.sum()) == 0
