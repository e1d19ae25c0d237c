"""GPU parity of the CUDA decode path against the fp64 CPU oracle, through the C ABI.

Tolerances (the decode's accuracy contract): max |out - oracle| <= 1e-2 on the bf16
output and max |lse - oracle| <= 1e-3 on the fp32 log-sum-exp. Because long sequences
have small outputs (about 1/sqrt(visible tokens)), an absolute bound alone is loose
there, so every comparison also bounds the error of each row relative to that row's
largest output: max_d |out - oracle| / max_d |oracle| <= 2e-2. The derivation: the bf16
rounding of the output contributes at most 2^-9 = 0.002 of the row maximum; the bf16
rounding of the probabilities P before the PV product perturbs each term of the weighted
sum by at most 2^-9 relative, which for an output that sums n comparable terms of
random sign is about 2^-9 / sqrt(3) = 0.0011 of the row's scale per element (times a
few standard deviations over 512 dims and up to 128 rows); 2e-2 leaves a factor of
several over both. Small cases and the full-size workloads (every sequence, in the
benchmark's launch configuration) compare every element with the oracle; a few
properties are checked besides (finite outputs, agreement with the no-split schedule).
"""

import numpy as np
import pytest
import torch

import oracle
from mla_paged_kv_06_b200 import workloads as wl

pytestmark = pytest.mark.gpu

ATOL_OUT = 1e-2
ATOL_LSE = 1e-3
REL_OUT = 2e-2          # per row: max |dout| / max |out_oracle|
# Two GPU results that are each within the tolerance of the oracle can differ by twice
# it (one bf16 ulp is 0.0156 at |o| in [2, 4)), so GPU-vs-GPU comparisons use 2x.
ATOL_PAIR_OUT = 2 * ATOL_OUT
ATOL_PAIR_LSE = 2 * ATOL_LSE


def _mla():
    from mla_paged_kv_06_b200 import mla
    return mla


def to_dev(x):
    return dict(q=x.q.cuda(), kcache=x.kcache.cuda(), block_table=x.block_table.cuda(),
                seqlens=x.seqlens.cuda())


def run(x, d=None, impl="tc", num_sms=None, check_error=True):
    mla = _mla()
    d = d or to_dev(x)
    nsm = num_sms or mla.default_num_sms()
    meta, ns = mla.mla_get_metadata(d["seqlens"], x.h_q, x.s_q, nsm)
    fn = mla.mla_decode_fwd if impl == "tc" else mla.mla_decode_fwd_simt
    out, lse = fn(d["q"], d["kcache"], d["block_table"], d["seqlens"], x.scale, x.causal,
                  meta, ns, num_sms=nsm)
    torch.cuda.synchronize()
    if check_error:
        st, word = mla.mla_get_last_device_error()
        assert st == 0, f"device error {mla.status_string(st)} word={word:#x}"
    return out, lse


def graph_step(x, d):
    """The step as the benchmark times it: mla_get_metadata + mla_decode_fwd captured once
    as a CUDA graph on buffers of their own, then replayed."""
    mla = _mla()
    nsm = mla.default_num_sms()
    meta = torch.empty(mla.mla_metadata_ints(nsm), dtype=torch.int32, device="cuda")
    ns = torch.empty(mla.mla_num_splits_len(x.batch, x.h_q, x.s_q), dtype=torch.int32,
                     device="cuda")
    ws = torch.empty(mla.mla_workspace_bytes(x.batch, x.h_q, x.s_q, nsm), dtype=torch.uint8,
                     device="cuda")
    out = torch.full((x.batch, x.s_q, x.h_q, 512), float("nan"), dtype=torch.bfloat16,
                     device="cuda")
    lse = torch.empty((x.batch, x.h_q, x.s_q), dtype=torch.float32, device="cuda")

    def step():
        mla.mla_get_metadata(d["seqlens"], x.h_q, x.s_q, nsm, meta, ns)
        mla.mla_decode_fwd(d["q"], d["kcache"], d["block_table"], d["seqlens"], x.scale,
                           x.causal, meta, ns, ws, out, lse)

    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    g.replay()
    torch.cuda.synchronize()
    st, word = mla.mla_get_last_device_error()
    assert st == 0, f"device error {mla.status_string(st)} word={word:#x}"
    del g
    return out, lse


def compare(out, lse, ref_out, ref_lse, what=""):
    o = out.double().cpu().numpy()
    l = lse.double().cpu().numpy()
    assert np.isfinite(o).all(), f"{what}: non-finite output"
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isneginf(l), ~fin), f"{what}: empty-row lse mismatch"
    d_o = np.abs(o - ref_out).max() if o.size else 0.0
    d_l = np.abs(l[fin] - ref_lse[fin]).max() if fin.any() else 0.0
    assert d_o <= ATOL_OUT, f"{what}: max|dout|={d_o:.3e}"
    assert d_l <= ATOL_LSE, f"{what}: max|dlse|={d_l:.3e}"
    rel = row_relative_error(o, ref_out)
    assert rel <= REL_OUT, f"{what}: max row-relative error {rel:.3e}"
    return d_o, d_l, rel


def row_relative_error(o, ref_out):
    """Largest over rows of max_d |o - ref| / max_d |ref| (rows whose reference is all
    zero, the empty rows, are compared absolutely above and skipped here)."""
    if o.size == 0:
        return 0.0
    err = np.abs(o - ref_out).reshape(-1, ref_out.shape[-1]).max(axis=1)
    scale = np.abs(ref_out).reshape(-1, ref_out.shape[-1]).max(axis=1)
    nz = scale > 0
    return float((err[nz] / scale[nz]).max()) if nz.any() else 0.0


def oracle_all(x):
    return oracle.decode(x.q, x.kcache, x.block_table, x.seqlens, x.scale, x.causal)


@pytest.mark.parametrize("impl", ["tc", "simt"])
def test_tiny_workload_parity(impl):
    x = wl.make_workload("tiny")
    out, lse = run(x, impl=impl)
    assert tuple(out.shape) == (2, 1, 16, 512) and tuple(lse.shape) == (2, 16, 1)
    compare(out, lse, *oracle_all(x), what=f"tiny/{impl}")


SMALL = [
    # lens, s_q, h_q, causal
    ([1, 63, 64, 65, 127, 128, 129], 1, 16, False),
    ([700, 1, 2000, 64], 1, 128, False),
    ([513, 4096, 1000], 2, 128, True),
    ([300, 65, 2], 2, 64, True),
    ([1500, 333], 1, 64, False),
    ([17, 200, 190], 4, 32, True),
    ([129, 5], 1, 1, False),
    ([258, 3, 1, 0, 64], 3, 7, True),
    ([2500], 1, 100, False),
    ([300, 70], 16, 64, True),        # the largest row count: 1024 rows, 8 tiles
    ([1000], 8, 128, True),
]


@pytest.mark.parametrize("case", SMALL)
@pytest.mark.parametrize("num_sms", [None, 1, 6])
@pytest.mark.parametrize("impl", ["tc", "simt"])
def test_small_parity(case, num_sms, impl):
    lens, s_q, h_q, causal = case
    x = wl.make_paged_inputs(lens, s_q, h_q, seed=sum(lens) + s_q, causal=causal,
                             spare_blocks=3, poison=True)
    out, lse = run(x, impl=impl, num_sms=num_sms)
    compare(out, lse, *oracle_all(x), what=f"{case}/{num_sms}/{impl}")


def test_device_metadata_matches_host_plan():
    mla = _mla()
    # the last two cases are too large for the scheduler's shared-memory table (global
    # path); the last one has two row tiles per sequence, cut tile by tile
    for lens, h_q, s_q in [([37, 130], 16, 1), ([65536, 10, 0, 65536, 3], 64, 1),
                           ([8192] * 128, 128, 2), (list(range(0, 9000, 37)), 128, 1),
                           ([5, 700, 0, 64] * 7500, 16, 1),
                           ([5, 700, 0, 64, 3000] * 4200, 128, 2)]:
        seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
        for nsm in [1, 2, 13, mla.default_num_sms()]:
            meta, ns = mla.mla_get_metadata(seq, h_q, s_q, nsm)
            units = mla.mla_num_work_units(nsm, h_q, s_q)
            hm, hns = mla.mla_plan_host(lens, h_q, s_q, units)
            assert np.array_equal(meta.cpu().numpy()[: hm.size], hm)
            assert np.array_equal(ns.cpu().numpy(), hns)


def test_more_units_than_clusters():
    # A host-planned schedule with more units than the split kernel has clusters: each
    # cluster then runs several units one after another, and the result is unchanged.
    mla = _mla()
    units = 3 * mla.mla_num_work_units(mla.default_num_sms(), 128, 1) + 5
    lens = [3000, 200, 5000, 64, 1, 0, 777, 4100]
    x = wl.make_paged_inputs(lens, 1, 128, seed=71, spare_blocks=2, poison=True)
    hm, hns = mla.mla_plan_host(lens, 128, 1, units)
    assert int(hm[0]) == units
    meta = torch.from_numpy(hm).cuda()
    ns = torch.from_numpy(hns).cuda()
    d = dict(q=x.q.cuda(), kcache=x.kcache.cuda(), block_table=x.block_table.cuda(),
             seqlens=x.seqlens.cuda())
    out, lse = mla.mla_decode_fwd(d["q"], d["kcache"], d["block_table"], d["seqlens"], x.scale,
                                  False, meta, ns, num_sms=2 * units)
    torch.cuda.synchronize()
    st, word = mla.mla_get_last_device_error()
    assert st == mla.MLA_OK, (mla.status_string(st), hex(word))
    compare(out, lse, *oracle_all(x), what="units > clusters")


def test_thirty_thousand_sequences_sharing_a_small_pool():
    # A batch too large for the scheduler's shared-memory table (its global-memory path
    # runs), about 400 work sequences per unit, and a combine grid of 30,000 x 16 CTAs.
    # The sequences map their pages into one 64-page pool (decode only reads the cache),
    # so the inputs stay small. Sampled sequences, empty ones included, match the oracle.
    lens = [(37 * i) % 701 for i in range(30000)]
    batch, nblk_max, pool = len(lens), 11, 64
    g = torch.Generator().manual_seed(74)
    bt = torch.tensor([[(7 * b + 13 * j) % pool for j in range(nblk_max)] for b in range(batch)],
                      dtype=torch.int32)
    x = wl.DecodeInputs(
        q=torch.randn((batch, 1, 1, 576), generator=g).to(torch.bfloat16),
        kcache=torch.randn((pool, 64, 1, 576), generator=g).to(torch.bfloat16),
        block_table=bt, seqlens=torch.tensor(lens, dtype=torch.int32),
        scale=wl.DEFAULT_SCALE, causal=False, workload="custom", seed=74)
    out, lse = run(x)
    o = out.float().cpu().numpy()
    assert np.isfinite(o).all()
    idx = sorted({0, 1, 700, 701, 18947, batch - 1} | set(range(5, batch, 997)))
    ref_out, ref_lse = oracle.decode(x.q, x.kcache, x.block_table, x.seqlens, x.scale, False,
                                     batch_indices=idx)
    compare(out[idx], lse[idx], ref_out, ref_lse, what="30k sequences")
    assert lens[0] == 0 and torch.all(out[0] == 0) and torch.isneginf(lse[0]).all()


FULL = ["uniform", "v3", "spec", "skewed"]


@pytest.mark.parametrize("h_q,s_q,num_sms,chunks", [
    (16, 1, 2, 2), (16, 1, 3, 3), (16, 1, 4, 4), (16, 1, 5, 5), (32, 1, 4, 4),
    (64, 1, 2, 2), (64, 1, 3, 3),
    (16, 1, 8, 8), (16, 1, 9, 9), (16, 1, 17, 17), (16, 1, 33, 33), (16, 1, 148, 129),
    (128, 2, 40, 10), (128, 2, 140, 34),
])
def test_rows_merged_from_many_chunks(h_q, s_q, num_sms, chunks):
    # One long sequence spread over 2 to 148 units, merged by the combine: a row of more
    # than 8 chunks is cut into slices merged by separate CTAs, then the slices are
    # merged (the second run on the same schedule checks that the slice counters start
    # from zero again). Short sequences beside it keep the one-pass merge.
    mla = _mla()
    lens = [40960, 100, 0, 64]
    x = wl.make_paged_inputs(lens, s_q, h_q, seed=chunks + h_q, causal=s_q > 1,
                             spare_blocks=2, poison=True)
    nsm = min(num_sms, mla.default_num_sms())
    _, ns = mla.mla_plan_host(lens, h_q, s_q, mla.mla_num_work_units(nsm, h_q, s_q))
    if nsm == num_sms:
        assert int(ns[1] - ns[0]) == chunks      # the first sequence's chunks (tile 0)
    d = to_dev(x)
    meta, ns = mla.mla_get_metadata(d["seqlens"], x.h_q, x.s_q, nsm)
    res = []
    for _ in range(2):                           # one schedule, two calls
        res.append(mla.mla_decode_fwd(d["q"], d["kcache"], d["block_table"], d["seqlens"],
                                      x.scale, x.causal, meta, ns, num_sms=nsm))
        torch.cuda.synchronize()
        st, word = mla.mla_get_last_device_error()
        assert st == 0, f"device error {mla.status_string(st)} word={word:#x}"
    (out, lse), (out2, lse2) = res
    compare(out, lse, *oracle_all(x), what=f"{h_q}/{s_q}/{nsm}")
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


@pytest.fixture(scope="module")
def full_inputs():
    cache = {}

    def get(name):
        if name not in cache:
            cache.clear()
            x = wl.make_workload(name, seed=0)
            cache[name] = (x, to_dev(x))
        return cache[name]
    return get


@pytest.mark.parametrize("name", FULL)
def test_full_workload_parity(name, full_inputs):
    # every sequence of the full-size workload, element by element, in the benchmark's
    # launch configuration (all SMs, the device scheduler's split schedule)
    x, d = full_inputs(name)
    out, lse = run(x, d)
    ref_out, ref_lse = oracle_all(x)
    d_o, d_l, rel = compare(out, lse, ref_out, ref_lse, what=name)
    print(f"{name}: max|dout| {d_o:.3e}  max|dlse| {d_l:.3e}  max row-relative {rel:.3e}")
    # the benchmark replays the step as a CUDA graph: the replay gives the same bits
    g_out, g_lse = graph_step(x, d)
    assert torch.equal(g_out, out) and torch.equal(g_lse, lse), f"{name}: graph replay differs"


@pytest.mark.parametrize("name", FULL)
def test_full_workload_split_matches_no_split(name, full_inputs):
    x, d = full_inputs(name)
    out_a, lse_a = run(x, d)
    out_b, lse_b = run(x, d, num_sms=1)
    assert (out_a.float() - out_b.float()).abs().max().item() <= ATOL_PAIR_OUT
    assert (lse_a - lse_b).abs().max().item() <= ATOL_PAIR_LSE


def test_full_workload_tc_matches_simt(full_inputs):
    x, d = full_inputs("skewed")
    out_a, lse_a = run(x, d, impl="tc")
    out_b, lse_b = run(x, d, impl="simt")
    assert (out_a.float() - out_b.float()).abs().max().item() <= ATOL_PAIR_OUT
    assert (lse_a - lse_b).abs().max().item() <= ATOL_PAIR_LSE


def test_nan_poison_full_size():
    x = wl.make_workload("v3", seed=3, poison=True)
    assert torch.isnan(x.kcache[:, :, 0, 0].float()).any()
    out, lse = run(x)
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    compare(out, lse, *oracle_all(x), what="v3-poison")


@pytest.mark.parametrize("impl", ["tc", "simt"])
def test_block_permutation_is_bit_exact(impl):
    x = wl.make_paged_inputs([130, 4000, 64, 1], 2, 128, seed=5, causal=True,
                             spare_blocks=2, poison=True)
    out, lse = run(x, impl=impl)
    g = torch.Generator().manual_seed(4)
    perm = torch.randperm(x.num_blocks, generator=g)
    kc2 = torch.empty_like(x.kcache)
    kc2[perm] = x.kcache
    bt2 = perm[x.block_table.long()].to(torch.int32)
    y = wl.DecodeInputs(x.q, kc2, bt2, x.seqlens, x.scale, x.causal, "perm", 5)
    out2, lse2 = run(y, impl=impl)
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


def test_repeat_runs_are_bit_identical():
    x = wl.make_paged_inputs([3000, 17, 900], 1, 128, seed=8)
    d = to_dev(x)
    a = run(x, d)
    b = run(x, d)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_single_token_returns_v_row_exactly():
    x = wl.make_paged_inputs([1, 1, 1], 1, 128, seed=9)
    out, lse = run(x)
    for b in range(3):
        row = x.kcache[int(x.block_table[b, 0]), 0, 0, :512]
        assert torch.equal(out[b, 0].cpu(), row.expand(128, 512))


def test_bad_inputs_report_device_error():
    mla = _mla()
    x = wl.make_paged_inputs([100, 50], 1, 16, seed=10)
    d = to_dev(x)
    # a block id past the pool: recorded, skipped, no fault
    d["block_table"][0, 1] = x.num_blocks + 5
    run(x, d, check_error=False)
    st, word = mla.mla_get_last_device_error()
    assert st == mla.MLA_ERR_DEVICE_BAD_INPUT, (st, hex(word))
    # a length the block table cannot hold: recorded and clamped
    d = to_dev(x)
    d["seqlens"][1] = 64 * x.block_table.shape[1] + 1
    run(x, d, check_error=False)
    st, _ = mla.mla_get_last_device_error()
    assert st == mla.MLA_ERR_DEVICE_BAD_INPUT
    st, _ = mla.mla_get_last_device_error()
    assert st == mla.MLA_OK


@pytest.mark.parametrize("h_q", [16, 128])          # the 1-CTA and the 2-CTA kernel
def test_bounded_wait_gives_up_and_reports_a_timeout(h_q):
    # The test hook makes each CTA's loader wait, before its first copy, on a barrier that
    # nothing completes. Every wait of the kernel then gives up after the (here 2 ms)
    # limit: the launch ends normally with MLA_ERR_DEVICE_TIMEOUT recorded, nothing is in
    # flight, and the device stays usable for the next call.
    mla = _mla()
    x = wl.make_paged_inputs([300, 70, 1], 1, h_q, seed=31)
    d = to_dev(x)
    mla.mla_test_set_stall(True, 2_000_000)
    try:
        run(x, d, check_error=False)
        st, word = mla.mla_get_last_device_error()
    finally:
        mla.mla_test_set_stall(False, 0)
    assert st == mla.MLA_ERR_DEVICE_TIMEOUT, (mla.status_string(st), hex(word))
    assert word & 0xFF == 1                          # the timeout kind
    out, lse = run(x, d)
    compare(out, lse, *oracle_all(x), what="after a timeout")


@pytest.mark.parametrize("h_q", [128, 16])
def test_graph_captured_step_follows_new_lengths(h_q):
    """The step (metadata + decode) captured once as a CUDA graph, as the benchmark and a
    serving loop replay it: after new lengths are written into the same buffer, a replay
    schedules and decodes them (the schedule is computed on the device, so nothing of the
    first lengths is baked into the graph)."""
    mla = _mla()
    lens_a = [3000, 17, 900, 64, 1]
    lens_b = [1500, 9, 899, 1, 1]               # within each row's pages of lens_a
    x = wl.make_paged_inputs(lens_a, 1, h_q, seed=21, spare_blocks=2, poison=True)
    d = to_dev(x)
    nsm = mla.default_num_sms()
    meta = torch.empty(mla.mla_metadata_ints(nsm), dtype=torch.int32, device="cuda")
    ns = torch.empty(mla.mla_num_splits_len(x.batch, h_q, 1), dtype=torch.int32, device="cuda")
    ws = torch.empty(mla.mla_workspace_bytes(x.batch, h_q, 1, nsm), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty((x.batch, 1, h_q, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((x.batch, h_q, 1), dtype=torch.float32, device="cuda")

    def step():
        mla.mla_get_metadata(d["seqlens"], h_q, 1, nsm, meta, ns)
        mla.mla_decode_fwd(d["q"], d["kcache"], d["block_table"], d["seqlens"], x.scale,
                           x.causal, meta, ns, ws, out, lse)

    step()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for lens in (lens_a, lens_b, lens_a):
        sl = torch.tensor(lens, dtype=torch.int32)
        d["seqlens"].copy_(sl)
        out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        st, word = mla.mla_get_last_device_error()
        assert st == 0, f"device error {mla.status_string(st)} word={word:#x}"
        ref = oracle.decode(x.q, x.kcache, x.block_table, sl, x.scale, x.causal)
        compare(out, lse, *ref, what=f"graph replay h_q={h_q} lens={lens}")
    del g


@pytest.mark.parametrize("h_q", [128, 16])
def test_decode_sees_the_writes_of_the_kernel_queued_before_it(h_q):
    """The split kernel is launched with programmatic stream serialization: it may be
    scheduled before the kernel ahead of it ends, and must still read only what that
    kernel wrote. Here a torch kernel rewrites q in place right before the decode, with no
    synchronisation, and the decode must see the new q (it then matches the oracle on it)."""
    mla = _mla()
    x = wl.make_paged_inputs([1500, 64, 700, 1], 1, h_q, seed=31, spare_blocks=2, poison=True)
    d = to_dev(x)
    nsm = mla.default_num_sms()
    meta, ns = mla.mla_get_metadata(d["seqlens"], h_q, 1, nsm)
    mla.mla_decode_fwd(d["q"], d["kcache"], d["block_table"], d["seqlens"], x.scale,
                       x.causal, meta, ns, num_sms=nsm)
    d["q"].mul_(-1.5)                          # queued right before the decode
    out, lse = mla.mla_decode_fwd(d["q"], d["kcache"], d["block_table"], d["seqlens"],
                                  x.scale, x.causal, meta, ns, num_sms=nsm)
    torch.cuda.synchronize()
    st, word = mla.mla_get_last_device_error()
    assert st == 0, f"device error {mla.status_string(st)} word={word:#x}"
    q_new = d["q"].cpu()
    assert torch.equal(q_new, (x.q.cuda() * -1.5).cpu())
    ref = oracle.decode(q_new, x.kcache, x.block_table, x.seqlens, x.scale, x.causal)
    compare(out, lse, *ref, what=f"q rewritten before the decode, h_q={h_q}")
