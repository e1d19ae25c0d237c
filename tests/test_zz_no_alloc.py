"""The decode entry point that allocates nothing (mla_decode_fwd_noalloc), through the
C ABI: two calls in a row, each compared with mla_decode_fwd on a caller workspace,
and the host-side rejection of sizes beyond its built-in scratch.

Self-contained: it builds its own inputs and passes in a fresh process as well as after
the rest of the suite (the scratch keeps the previous call's partials, which must not
matter).
"""

import ctypes

import pytest
import torch

from mla_paged_kv_06_b200 import workloads as wl

pytestmark = pytest.mark.gpu

ATOL_OUT = 1e-2
ATOL_LSE = 1e-3


def _mla():
    from mla_paged_kv_06_b200 import mla
    return mla


def _dev(x):
    return x.q.cuda(), x.kcache.cuda(), x.block_table.cuda(), x.seqlens.cuda()


def _both(x):
    mla = _mla()
    q, kc, bt, sl = _dev(x)
    meta, ns = mla.mla_get_metadata(sl, x.h_q, x.s_q)
    out_a, lse_a = mla.mla_decode_fwd_noalloc(q, kc, bt, sl, x.scale, x.causal, meta, ns)
    out_b, lse_b = mla.mla_decode_fwd(q, kc, bt, sl, x.scale, x.causal, meta, ns)
    torch.cuda.synchronize()
    st, word = mla.mla_get_last_device_error()
    assert st == mla.MLA_OK, (mla.status_string(st), hex(word))
    return (out_a, lse_a), (out_b, lse_b), meta


def _close(a, b):
    (out_a, lse_a), (out_b, lse_b) = a, b
    assert torch.isfinite(out_a.float()).all()
    assert (out_a.float() - out_b.float()).abs().max().item() <= ATOL_OUT
    fin = torch.isfinite(lse_b)
    assert torch.equal(torch.isfinite(lse_a), fin)
    if fin.any():
        assert (lse_a[fin] - lse_b[fin]).abs().max().item() <= ATOL_LSE


def test_noalloc_matches_workspace_call_twice_in_a_row():
    # first call: long sequences at h_q = 128 split across many units, so partials go
    # through the scratch and the combine reads them back
    x1 = wl.make_paged_inputs([6000, 17, 3000, 900, 8000, 1], 1, 128, seed=21,
                              spare_blocks=2, poison=True)
    a1, b1, meta = _both(x1)
    assert int(meta[0]) > 1                         # more than one work unit
    _close(a1, b1)
    # second call right after, other shapes (causal, two query tokens, two row tiles):
    # the first call's partials still sit in the scratch and must not leak in
    x2 = wl.make_paged_inputs([4000, 65, 2500], 2, 128, seed=22, causal=True,
                              spare_blocks=2, poison=True)
    a2, b2, _ = _both(x2)
    _close(a2, b2)
    # and the first inputs once more give the same result as before
    a3, _, _ = _both(x1)
    assert torch.equal(a3[0], a1[0]) and torch.equal(a3[1], a1[1])


def test_noalloc_rejects_sizes_beyond_its_scratch_before_launch():
    mla = _mla()
    lib = mla.library()
    units = mla.mla_num_work_units(mla.default_num_sms())
    # smallest batch of one-tile work sequences whose worst case exceeds the scratch
    batch = 1
    while mla.mla_workspace_bytes(batch, 128, 1, 2 * units) <= mla.MLA_NOALLOC_SCRATCH_BYTES:
        batch += 1
    # valid pointers of a small problem; the call must refuse on the host before any
    # launch, so the claimed batch is never read through them
    x = wl.make_paged_inputs([70], 1, 128, seed=23)
    q, kc, bt, sl = _dev(x)
    meta, ns = mla.mla_get_metadata(sl, x.h_q, x.s_q)
    out = torch.empty((1, 1, 128, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, 128, 1), dtype=torch.float32, device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = lib.mla_decode_fwd_noalloc(p(q), p(kc), kc.shape[0], p(bt), bt.shape[1], p(sl),
                                    batch, 1, 128, float(x.scale), 0, p(meta), p(ns),
                                    p(out), p(lse), ctypes.c_void_p(0))
    assert st == mla.MLA_ERR_WORKSPACE_TOO_SMALL
    # one below the limit is accepted by the same check (run for real on its own inputs)
    assert mla.mla_workspace_bytes(batch - 1, 128, 1, 2 * units) <= mla.MLA_NOALLOC_SCRATCH_BYTES
    torch.cuda.synchronize()
    assert mla.mla_get_last_device_error()[0] == mla.MLA_OK
