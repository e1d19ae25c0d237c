"""The decode entry point that allocates nothing (mla_decode_fwd_noalloc), through the
C ABI: two calls in a row, each compared with mla_decode_fwd on a caller workspace;
the host-side rejection of sizes beyond its built-in scratch; and the largest size it
accepts, run for real.

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


def _shared_pool_inputs(lens, seed):
    """One-tile (h_q = 128) sequences whose pages all map into one small pool: decode
    only reads the cache, so a large batch needs little memory."""
    batch, pool = len(lens), 64
    nblk = max(1, max((L + 63) // 64 for L in lens))
    g = torch.Generator().manual_seed(seed)
    bt = torch.tensor([[(5 * b + 11 * j) % pool for j in range(nblk)] for b in range(batch)],
                      dtype=torch.int32)
    return wl.DecodeInputs(
        q=torch.randn((batch, 1, 128, 576), generator=g).to(torch.bfloat16),
        kcache=torch.randn((pool, 64, 1, 576), generator=g).to(torch.bfloat16),
        block_table=bt, seqlens=torch.tensor(lens, dtype=torch.int32),
        scale=wl.DEFAULT_SCALE, causal=False, workload="custom", seed=seed)


def test_noalloc_rejects_sizes_beyond_its_scratch_and_runs_the_largest_it_accepts():
    mla = _mla()
    lib = mla.library()
    units = mla.mla_num_work_units(mla.default_num_sms(), 128, 1)
    # smallest batch of one-tile work sequences whose worst case exceeds the scratch
    batch = 1
    while mla.mla_workspace_bytes(batch, 128, 1, 2 * units) <= mla.MLA_NOALLOC_SCRATCH_BYTES:
        batch += 1
    # Every buffer is sized for the claimed batch, so a regression in the size check
    # shows up as a wrong status, never as an access outside these allocations.
    lens = [64 * (20 + (7 * i) % 5) + (13 * i) % 64 for i in range(batch)]
    x = _shared_pool_inputs(lens, seed=23)
    q, kc, bt, sl = _dev(x)
    meta, ns = mla.mla_get_metadata(sl, 128, 1)
    out = torch.empty((batch, 1, 128, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((batch, 128, 1), dtype=torch.float32, device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = lib.mla_decode_fwd_noalloc(p(q), p(kc), kc.shape[0], p(bt), bt.shape[1], p(sl),
                                    batch, 1, 128, float(x.scale), 0, p(meta), p(ns),
                                    p(out), p(lse), ctypes.c_void_p(0))
    assert st == mla.MLA_ERR_WORKSPACE_TOO_SMALL
    torch.cuda.synchronize()
    assert mla.mla_get_last_device_error()[0] == mla.MLA_OK
    # One below the limit is accepted and runs: with lengths of 20-25 pages nearly every
    # unit boundary falls inside a sequence, so nearly every partial slot of the scratch
    # is used (at most work sequences + units chunks). It matches the call on a caller
    # workspace.
    y = _shared_pool_inputs(lens[: batch - 1], seed=24)
    a, b, meta = _both(y)
    _close(a, b)
    ns = mla.mla_get_metadata(y.seqlens.cuda(), 128, 1)[1]
    chunks = int(ns[-1])
    assert chunks >= batch - 1 + (3 * units) // 4, (chunks, batch - 1, units)
