"""Split-KV across devices, on one GPU: the fp32-output decode, the device combine of
partials, and the whole path with the ranks' slices decoded one after another (the
exchange between devices is covered by the gloo tests; on one GPU the gathered parts
are stacked directly). Everything is compared with the oracle.
"""

import numpy as np
import pytest
import torch

import oracle
from mla_paged_kv_06_b200 import splitkv as skv
from mla_paged_kv_06_b200 import workloads as wl

pytestmark = pytest.mark.gpu

ATOL_OUT = 1e-2
ATOL_LSE = 1e-3


def _mla():
    from mla_paged_kv_06_b200 import mla
    return mla


def _dev(x):
    return x.q.cuda(), x.kcache.cuda(), x.block_table.cuda(), x.seqlens.cuda()


def _ok():
    mla = _mla()
    torch.cuda.synchronize()
    st, word = mla.mla_get_last_device_error()
    assert st == mla.MLA_OK, (mla.status_string(st), hex(word))


def _check_oracle(out, lse, x, rows=None):
    ref_out, ref_lse = oracle.decode(x.q, x.kcache, x.block_table, x.seqlens, x.scale,
                                     x.causal)
    o = out.float().cpu().numpy()
    l = lse.cpu().numpy()
    assert np.isfinite(o).all()
    assert np.array_equal(np.isfinite(l), np.isfinite(ref_lse))
    assert np.abs(o - ref_out).max() <= ATOL_OUT
    fin = np.isfinite(ref_lse)
    if fin.any():
        assert np.abs(l[fin] - ref_lse[fin]).max() <= ATOL_LSE


@pytest.mark.parametrize("lens, s_q, h_q, causal", [
    ([37, 130, 0, 1], 1, 16, False),
    ([300, 70, 2000], 2, 64, True),
    ([5000, 64, 3], 1, 128, False),
])
def test_partial_decode_is_the_unrounded_decode(lens, s_q, h_q, causal):
    mla = _mla()
    x = wl.make_paged_inputs(lens, s_q, h_q, seed=60, causal=causal, spare_blocks=2,
                             poison=True)
    q, kc, bt, sl = _dev(x)
    meta, ns = mla.mla_get_metadata(sl, h_q, s_q)
    out_f, lse_f = mla.mla_decode_fwd_partial(q, kc, bt, sl, x.scale, causal, meta, ns)
    out_b, lse_b = mla.mla_decode_fwd(q, kc, bt, sl, x.scale, causal, meta, ns)
    _ok()
    assert out_f.dtype == torch.float32
    # the bf16 call rounds the very same fp32 values (split or not), so they agree bit
    # for bit once the fp32 output is rounded the same way
    assert torch.equal(out_f.to(torch.bfloat16), out_b)
    assert torch.equal(lse_f, lse_b)
    _check_oracle(out_f, lse_f, x)


@pytest.mark.parametrize("parts", [1, 2, 5, 37])
def test_combine_partials_matches_the_oracle_combine(parts):
    mla = _mla()
    g = torch.Generator().manual_seed(61 + parts)
    b, s_q, h_q = 3, 2, 16
    o = torch.randn((parts, b, s_q, h_q, 512), generator=g)
    l = torch.randn((parts, b, h_q, s_q), generator=g) * 4
    # empty parts (-inf, their O is NaN and must not be read), a row no part sees
    if parts > 1:
        l[1, 0] = -float("inf")
        o[1, 0] = float("nan")
    l[:, 2, 3, 1] = -float("inf")
    o[:, 2, 1, 3] = float("nan")
    out, lse = mla.mla_combine_partials(o.cuda().contiguous(), l.cuda().contiguous())
    _ok()
    po = torch.nan_to_num(o, nan=0.0).reshape(parts, -1, 512).double().numpy()
    pl = l.permute(0, 1, 3, 2).reshape(parts, -1).double().numpy()
    ref_o, ref_l = oracle.combine(po, pl)
    ref_o = ref_o.reshape(b, s_q, h_q, 512)
    ref_l = np.transpose(ref_l.reshape(b, s_q, h_q), (0, 2, 1))
    got_o = out.float().cpu().numpy()
    got_l = lse.cpu().numpy()
    assert np.isfinite(got_o).all()
    assert np.array_equal(np.isfinite(got_l), np.isfinite(ref_l))
    # bf16 output: half an ulp of |out| plus fp32 accumulation
    assert np.abs(got_o - ref_o).max() <= 2 ** -7 * max(1.0, np.abs(ref_o).max())
    fin = np.isfinite(ref_l)
    assert np.abs(got_l[fin] - ref_l[fin]).max() <= 1e-5
    assert np.all(got_o[2, 1, 3] == 0) and np.isneginf(got_l[2, 3, 1])


def _split_path(x, world):
    """The ranks' slices decoded one after another on this GPU, stacked in rank order
    as the all-gather would, then merged on the device."""
    mla = _mla()
    plan = skv.plan_kv_split(x.seqlens, world, x.s_q, x.causal)
    o_parts, l_parts = [], []
    for g in range(world):
        xr = skv.make_kv_slice(x, plan, g)
        q, kc, bt, sl = _dev(xr)
        meta, ns = mla.mla_get_metadata(sl, xr.h_q, xr.s_q)
        o, l = mla.mla_decode_fwd_partial(q, kc, bt, sl, xr.scale, xr.causal, meta, ns)
        o_parts.append(o)
        l_parts.append(l)
    out, lse = mla.mla_combine_partials(torch.stack(o_parts), torch.stack(l_parts))
    _ok()
    return out, lse


@pytest.mark.parametrize("world", [2, 3, 4])
@pytest.mark.parametrize("lens, s_q, h_q, causal", [
    ([700, 1, 0, 130, 64], 1, 16, False),
    ([2000, 129, 65], 2, 128, True),
    ([129, 3000], 4, 32, True),
])
def test_split_across_ranks_matches_the_oracle(world, lens, s_q, h_q, causal):
    x = wl.make_paged_inputs(lens, s_q, h_q, seed=62 + world, causal=causal, spare_blocks=2,
                             poison=True)
    out, lse = _split_path(x, world)
    _check_oracle(out, lse, x)


def test_split_of_one_long_sequence_matches_the_single_device_decode():
    # one 64k-token sequence over 4 ranks against the one-device decode of the same
    # inputs (both within tolerance of each other; the oracle on sampled rows)
    mla = _mla()
    x = wl.make_paged_inputs([65536], 1, 128, seed=66)
    out, lse = _split_path(x, 4)
    q, kc, bt, sl = _dev(x)
    meta, ns = mla.mla_get_metadata(sl, 128, 1)
    out1, lse1 = mla.mla_decode_fwd(q, kc, bt, sl, x.scale, False, meta, ns)
    _ok()
    assert (out.float() - out1.float()).abs().max().item() <= ATOL_OUT
    assert (lse - lse1).abs().max().item() <= ATOL_LSE
    K = oracle.gather_tokens(x.kcache, x.block_table[0], 65536)
    for h in (0, 77, 127):
        ro, rl = oracle.decode_partial(x.q[0, 0, h:h + 1], K, x.scale)
        assert np.abs(out[0, 0, h].float().cpu().numpy() - ro[0]).max() <= ATOL_OUT
        assert abs(float(lse[0, h, 0]) - rl[0]) <= ATOL_LSE
