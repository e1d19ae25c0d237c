"""GPU parity of the decode over an FP8 latent cache (mla_decode_fwd_fp8), through the C
ABI, against the FP8 oracle: exact attention over the rows as the format reads them back
(oracle.fp8_cache.decode_fp8). The read-back values are bf16 numbers, so the kernel's
arithmetic after widening a page is the bf16 decode's, and the tolerances are the bf16
decode's: max |out - oracle| <= 1e-2, max |lse - oracle| <= 1e-3, and per row
max |dout| / max |out_oracle| <= 2e-2.
"""

import numpy as np
import pytest
import torch

from oracle import fp8_cache as f8
from mla_paged_kv_06_b200 import workloads as wl

pytestmark = pytest.mark.gpu

ATOL_OUT = 1e-2
ATOL_LSE = 1e-3
REL_OUT = 2e-2


def _mla():
    from mla_paged_kv_06_b200 import mla
    return mla


def run_fp8(x, kc8, num_sms=None):
    mla = _mla()
    q, bt, sl = x.q.cuda(), x.block_table.cuda(), x.seqlens.cuda()
    nsm = num_sms or mla.default_num_sms()
    meta, ns = mla.mla_get_metadata(sl, x.h_q, x.s_q, nsm)
    out, lse = mla.mla_decode_fwd_fp8(q, torch.from_numpy(kc8).cuda(), bt, sl, x.scale, x.causal,
                                      meta, ns, num_sms=nsm)
    torch.cuda.synchronize()
    st, word = mla.mla_get_last_device_error()
    assert st == mla.MLA_OK, (mla.status_string(st), hex(word))
    return out, lse


def compare(out, lse, ref_out, ref_lse, what):
    o = out.double().cpu().numpy()
    l = lse.double().cpu().numpy()
    assert np.isfinite(o).all(), f"{what}: non-finite output"
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isneginf(l), ~fin), f"{what}: empty-row lse mismatch"
    d_o = np.abs(o - ref_out).max()
    d_l = np.abs(l[fin] - ref_lse[fin]).max() if fin.any() else 0.0
    err = np.abs(o - ref_out).reshape(-1, 512).max(axis=1)
    scale = np.abs(ref_out).reshape(-1, 512).max(axis=1)
    rel = float((err[scale > 0] / scale[scale > 0]).max()) if (scale > 0).any() else 0.0
    assert d_o <= ATOL_OUT, f"{what}: max|dout|={d_o:.3e}"
    assert d_l <= ATOL_LSE, f"{what}: max|dlse|={d_l:.3e}"
    assert rel <= REL_OUT, f"{what}: row-relative {rel:.3e}"
    return d_o, d_l, rel


SMALL = [
    # lens, s_q, h_q, causal
    ([37, 130], 1, 16, False),
    ([1, 63, 64, 65, 127, 128, 129, 700], 1, 16, False),
    ([2000, 5, 64], 1, 32, False),
    ([513, 300, 1], 2, 16, True),
    ([258, 3, 1, 0, 64], 3, 7, True),
    ([129, 5], 1, 1, False),
    ([1500, 333], 2, 8, True),
    ([300, 70, 1], 1, 64, False),
    ([900, 129], 2, 32, True),
    ([65, 640], 4, 13, True),
]


@pytest.mark.parametrize("case", SMALL)
@pytest.mark.parametrize("num_sms", [None, 1, 6])
def test_small_parity_against_the_fp8_oracle(case, num_sms):
    lens, s_q, h_q, causal = case
    # a NaN-poisoned pool: the rows no sequence owns quantize to NaN codes and scales
    x = wl.make_paged_inputs(lens, s_q, h_q, seed=sum(lens) + 11, causal=causal,
                             spare_blocks=3, poison=True)
    kc8 = f8.quantize_cache(x.kcache)
    out, lse = run_fp8(x, kc8, num_sms)
    ref_out, ref_lse = f8.decode_fp8(x.q, kc8, x.block_table, x.seqlens, x.scale, causal)
    compare(out, lse, ref_out, ref_lse, f"{case}/{num_sms}")


def test_full_uniform_workload_sampled():
    # The uniform workload's shape (64 x 4096 tokens, 16 heads) in the benchmark's launch
    # configuration. Quantizing the whole 4096-page pool on the CPU takes minutes, so the
    # pages of six sampled sequences are quantized by the oracle and every other page is
    # random bytes (decoded by the kernel like any other, but not compared).
    x = wl.make_workload("uniform", seed=0)
    g = np.random.default_rng(5)
    kc8 = g.integers(0, 256, size=(x.num_blocks, 64, f8.ROW_BYTES), dtype=np.uint8)
    picked = [0, 17, 31, 40, 62, 63]
    for b in picked:
        blocks = x.block_table[b, : (int(x.seqlens[b]) + 63) // 64].long()
        kc8[blocks.numpy()] = f8.quantize_cache(x.kcache[blocks])
    out, lse = run_fp8(x, kc8)
    ref_out, ref_lse = f8.decode_fp8(x.q, kc8, x.block_table, x.seqlens, x.scale, False,
                                     batch_indices=picked)
    d_o, d_l, rel = compare(out[picked], lse[picked], ref_out, ref_lse, "uniform fp8")
    print(f"uniform fp8: max|dout| {d_o:.3e}  max|dlse| {d_l:.3e}  row-relative {rel:.3e}")


def test_block_permutation_is_bit_exact():
    x = wl.make_paged_inputs([130, 2000, 64, 1], 1, 16, seed=5, spare_blocks=2, poison=True)
    kc8 = f8.quantize_cache(x.kcache)
    out, lse = run_fp8(x, kc8)
    g = torch.Generator().manual_seed(4)
    perm = torch.randperm(x.num_blocks, generator=g)
    kc8b = np.empty_like(kc8)
    kc8b[perm.numpy()] = kc8
    bt2 = perm[x.block_table.long()].to(torch.int32)
    y = wl.DecodeInputs(x.q, x.kcache, bt2, x.seqlens, x.scale, x.causal, "perm", 5)
    out2, lse2 = run_fp8(y, kc8b)
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


def test_more_than_64_rows_is_rejected_before_launch():
    mla = _mla()
    x = wl.make_paged_inputs([100], 1, 65, seed=6)
    kc8 = f8.quantize_cache(x.kcache)
    with pytest.raises(mla.MlaError) as e:
        run_fp8(x, kc8)
    assert e.value.status == mla.MLA_ERR_UNSUPPORTED
