"""Host-side tests of the C ABI: the library loads without a GPU, exports every function
include/mla.h declares, rejects bad arguments before launching anything, and its host
scheduler (the same arithmetic the device metadata kernel runs) covers every page of
every work sequence exactly once with balanced units."""

import ctypes
import random

import numpy as np
import pytest

from mla_paged_kv_06_b200 import mla


def test_library_exports_every_header_function():
    lib = mla.library()
    names = mla.header_functions()
    assert "mla_get_metadata" in names and "mla_decode_fwd" in names
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings():
    assert mla.status_string(0) == "MLA_OK"
    assert mla.status_string(-4) == "MLA_ERR_WORKSPACE_TOO_SMALL"
    assert mla.status_string(-99) == "MLA_ERR_UNKNOWN"


def test_size_queries():
    assert mla.mla_metadata_ints(148) == 8 * 149
    assert mla.mla_metadata_ints(0) == 0
    assert mla.mla_num_splits_len(128, 128, 1) == 129
    assert mla.mla_num_splits_len(128, 128, 2) == 257
    assert mla.mla_num_splits_len(4, 129, 1) == 0           # h_q beyond 128: rejected
    ws = mla.mla_workspace_bytes(128, 128, 1, 148)
    cap = 128 + 74
    assert ws >= cap * 128 * 512 * 4 + cap * 128 * 4
    assert mla.mla_workspace_bytes(0, 16, 1, 148) == 0


def _decode_args(**over):
    vp = ctypes.c_void_p
    a = dict(q=vp(16), kcache=vp(16), num_blocks=8, block_table=vp(16), max_blocks=4,
             seqlens=vp(16), batch=2, s_q=1, h_q=16, scale=0.07, causal=0, metadata=vp(16),
             num_splits=vp(16), workspace=vp(256), workspace_bytes=1 << 30, out=vp(16),
             lse=vp(16), stream=vp(0))
    a.update(over)
    return list(a.values())


@pytest.mark.parametrize("over,expect", [
    (dict(q=ctypes.c_void_p(0)), mla.MLA_ERR_INVALID_ARG),
    (dict(out=ctypes.c_void_p(0)), mla.MLA_ERR_INVALID_ARG),
    (dict(q=ctypes.c_void_p(18)), mla.MLA_ERR_INVALID_ARG),          # misaligned
    (dict(workspace=ctypes.c_void_p(272)), mla.MLA_ERR_INVALID_ARG),  # not 256-aligned
    (dict(num_blocks=0), mla.MLA_ERR_INVALID_ARG),
    (dict(causal=2), mla.MLA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), mla.MLA_ERR_INVALID_ARG),
    (dict(h_q=129), mla.MLA_ERR_UNSUPPORTED),
    (dict(s_q=17), mla.MLA_ERR_UNSUPPORTED),
    (dict(h_q=128, s_q=9), mla.MLA_ERR_UNSUPPORTED),
    (dict(batch=0), mla.MLA_ERR_UNSUPPORTED),
    (dict(workspace_bytes=1024), mla.MLA_ERR_WORKSPACE_TOO_SMALL),
])
@pytest.mark.parametrize("fn", ["mla_decode_fwd", "mla_decode_fwd_simt"])
def test_decode_rejects_bad_arguments_before_launch(fn, over, expect):
    # Host validation runs before any CUDA call, so this needs no GPU.
    assert getattr(mla.library(), fn)(*_decode_args(**over)) == expect


def test_metadata_rejects_bad_arguments():
    lib = mla.library()
    vp = ctypes.c_void_p
    assert lib.mla_get_metadata(vp(0), 2, 16, 1, 148, vp(16), vp(16), vp(0)) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_get_metadata(vp(16), 2, 16, 1, 0, vp(16), vp(16), vp(0)) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_get_metadata(vp(16), 2, 200, 1, 148, vp(16), vp(16), vp(0)) == mla.MLA_ERR_UNSUPPORTED


# ---------------------------------------------------------------------------------
# Scheduler properties (host planner).

def _walk(meta, ns, lens, h_q, s_q):
    """Expand the schedule into {v: [(unit, chunk, pages...)]} and check its invariants."""
    U = int(meta[0])
    tiles = int(meta[1])
    batch = len(lens)
    assert tiles == -(-(h_q * s_q) // 128) and int(meta[2]) == batch
    V = batch * tiles
    nblk = [-(-max(int(lens[v % batch]), 0) // 64) for v in range(V)]
    seen = {}
    order = []
    for u in range(U):
        vb, kb, ve, ke, cb = (int(x) for x in meta[8 * (u + 1): 8 * (u + 1) + 5])
        v, k, first = vb, kb, True
        while (v, k) < (ve, ke) and v < V:
            if k >= nblk[v]:
                v, k, first = v + 1, 0, False
                continue
            chunk = cb if first else 0
            seen.setdefault(v, []).append((u, chunk, k))
            order.append((v, k))
            k += 1
            if k >= nblk[v] and (v, k) < (ve, ke):
                v, k, first = v + 1, 0, False
    # every page of every work sequence exactly once, in (v, page) order
    expect = [(v, k) for v in range(V) for k in range(nblk[v])]
    assert order == expect
    # chunk counts and indices
    for v in range(V):
        n = int(ns[v + 1] - ns[v])
        units = sorted({u for (u, _, _) in seen.get(v, [])})
        assert n == len(units), (v, n, units)
        for idx, u in enumerate(units):
            chunks = {c for (uu, c, _) in seen[v] if uu == u}
            assert chunks == {idx}, (v, u, chunks, idx)
    return seen, nblk


@pytest.mark.parametrize("case", [
    ([37, 130], 16, 1, 74),
    ([4096] * 64, 16, 1, 74),
    ([1] * 300, 128, 1, 74),
    ([64, 65, 63, 1, 128, 0, 0, 5000, 0], 128, 2, 74),
    ([65536, 10, 10, 65536, 3, 65536, 1, 2], 64, 1, 74),
    ([0, 0, 0], 16, 1, 74),
    ([8192] * 3, 128, 2, 1),
    ([100, 200], 128, 2, 3),
])
def test_schedule_covers_every_page_once(case):
    lens, h_q, s_q, U = case
    meta, ns = mla.mla_plan_host(lens, h_q, s_q, U)
    _walk(meta, ns, lens, h_q, s_q)


def test_schedule_random_and_balanced():
    rng = random.Random(1234)
    for trial in range(60):
        batch = rng.randint(1, 150)
        kind = rng.choice(["uniform", "lognormal", "equal", "giant"])
        if kind == "uniform":
            lens = [rng.randint(0, 9000) for _ in range(batch)]
        elif kind == "lognormal":
            lens = [min(65536, max(1, int(rng.lognormvariate(7, 1.0)))) for _ in range(batch)]
        elif kind == "equal":
            lens = [rng.randint(1, 5000)] * batch
        else:
            lens = [rng.randint(1, 100) for _ in range(batch)]
            lens[rng.randrange(batch)] = 65536
        h_q = rng.choice([16, 32, 64, 128])
        s_q = rng.choice([1, 2])
        U = rng.choice([1, 2, 37, 74])
        meta, ns = mla.mla_plan_host(lens, h_q, s_q, U)
        seen, nblk = _walk(meta, ns, lens, h_q, s_q)
        W = int(meta[5])
        # fixed cost per work sequence, in pages: 1 for the 1-CTA kernel up to 32 query
        # rows per sequence, 2 for it with 33-64 rows, 3 for the 2-CTA kernel; the header
        # records it
        rows = h_q * s_q
        overhead = 1 if rows <= 32 else 2 if rows <= 64 else 3
        assert int(meta[6]) == overhead
        total = sum(overhead + n for n in nblk)
        T = int(meta[1])
        if T > 1 and U >= T:
            # tile-aligned: tile t cuts its own line (the batch's costs) over its units
            assert int(meta[7]) == 1
            line = total // T
            units_t = [(t + 1) * U // T - t * U // T for t in range(T)]
            assert W == max(max(-(-line // n), 4) for n in units_t)
        else:
            assert int(meta[7]) == 0
            assert W == max(-(-total // U), 4)
        # no unit owns more than W pages: the largest unit is within one overhead of ideal
        per_unit = [0] * U
        for v, items in seen.items():
            for (u, _, _) in items:
                per_unit[u] += 1
        assert max(per_unit) <= W


@pytest.mark.parametrize("s_q,U", [(2, 74), (4, 74), (3, 74), (2, 5)])
def test_tile_aligned_units_of_equal_count_stream_the_same_pages(s_q, U):
    # Several row tiles: tile t owns units [t U / T, (t+1) U / T) and cuts the batch's
    # cost line over them alone, so tiles with equal unit counts get the same runs
    rng = random.Random(s_q * 100 + U)
    lens = [rng.randint(0, 9000) for _ in range(57)] + [65536, 1, 0]
    B = len(lens)
    meta, ns = mla.mla_plan_host(lens, 128, s_q, U)
    _walk(meta, ns, lens, 128, s_q)
    T = int(meta[1])
    assert T == s_q and int(meta[7]) == 1
    first = [t * U // T for t in range(T + 1)]
    rec = lambda u: [int(x) for x in meta[8 * (u + 1): 8 * (u + 1) + 5]]
    for t in range(1, T):
        if first[t + 1] - first[t] != first[1] - first[0]:
            continue
        for i in range(first[1] - first[0]):
            a, b = rec(first[0] + i), rec(first[t] + i)
            assert [b[0] - t * B, b[1], b[2] - t * B, b[3], b[4]] == a, (t, i, a, b)
    # every tile's chunk counts are the same
    n = np.diff(ns)
    for t in range(1, T):
        if first[t + 1] - first[t] == first[1] - first[0]:
            assert np.array_equal(n[t * B:(t + 1) * B], n[:B])


def test_schedule_no_split_with_one_unit():
    meta, ns = mla.mla_plan_host([8192, 3, 65536], 128, 2, 1)
    assert np.all(np.diff(ns) == 1)


def test_kv_append_rejects_bad_arguments_before_launch():
    lib = mla.library()
    buf = (ctypes.c_uint16 * 2048)()
    ints = (ctypes.c_int32 * 64)()
    a = ctypes.addressof(buf)
    i = ctypes.addressof(ints)
    # null pointers, bad sizes and misaligned rows fail on the host, before any launch
    assert lib.mla_kv_append(None, 1, i, 4, i, 2, a, 8, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_kv_append(a, 0, i, 4, i, 2, a, 8, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_kv_append(a, 1, i, 0, i, 2, a, 8, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_kv_append(a + 2, 1, i, 4, i, 2, a, 8, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_kv_append(a, 17, i, 4, i, 2, a, 8, None) == mla.MLA_ERR_UNSUPPORTED
    assert lib.mla_kv_append(a, 1, i, 4, i, 0, a, 8, None) == mla.MLA_ERR_UNSUPPORTED


def test_split_kv_entry_points_reject_bad_arguments_before_launch():
    lib = mla.library()
    buf = (ctypes.c_float * 4096)()
    a = ctypes.addressof(buf)
    # mla_combine_partials: null pointers, part counts outside [1, MLA_MAX_PARTS],
    # misaligned buffers and unsupported shapes fail on the host
    assert lib.mla_combine_partials(None, a, 2, 1, 1, 16, a, a, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_combine_partials(a, a, 0, 1, 1, 16, a, a, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_combine_partials(a, a, mla.MLA_MAX_PARTS + 1, 1, 1, 16, a, a,
                                    None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_combine_partials(a + 4, a, 2, 1, 1, 16, a, a, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_combine_partials(a, a + 2, 2, 1, 1, 16, a, a, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_combine_partials(a, a, 2, 1, 1, 129, a, a, None) == mla.MLA_ERR_UNSUPPORTED
    assert lib.mla_combine_partials(a, a, 2, 0, 1, 16, a, a, None) == mla.MLA_ERR_UNSUPPORTED
    # mla_decode_fwd_partial shares mla_decode_fwd's checks: a null or misaligned fp32
    # output is refused
    i = (ctypes.c_int32 * 64)()
    ip = ctypes.addressof(i)
    args = lambda out: (a, a, 8, ip, 4, ip, 1, 1, 16, 0.1, 0, ip, ip, a, 1 << 20, out, a, None)
    assert lib.mla_decode_fwd_partial(*args(None)) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_decode_fwd_partial(*args(a + 4)) == mla.MLA_ERR_INVALID_ARG


def test_kv_append_fp8_rejects_bad_arguments_before_launch():
    lib = mla.library()
    buf = (ctypes.c_uint16 * 2048)()
    ints = (ctypes.c_int32 * 64)()
    a = ctypes.addressof(buf)
    i = ctypes.addressof(ints)
    assert lib.mla_kv_append_fp8(None, 1, i, 4, i, 2, a, 8, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_kv_append_fp8(a, 1, i, 4, i, 2, None, 8, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_kv_append_fp8(a, 0, i, 4, i, 2, a, 8, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_kv_append_fp8(a, 1, i, 4, i, 2, a, 0, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_kv_append_fp8(a, 1, i, 4, i, 2, a + 8, 8, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_kv_append_fp8(a, 17, i, 4, i, 2, a, 8, None) == mla.MLA_ERR_UNSUPPORTED
    assert lib.mla_kv_append_fp8(a, 1, i, 4, i, 0, a, 8, None) == mla.MLA_ERR_UNSUPPORTED
    assert mla.MLA_FP8_ROW_BYTES == 656
