"""Pins for the CPU oracle: each check ties it to something other than itself.

Run without a GPU. Plausible mistakes (a dropped rope term, V taken from the wrong
dims, a wrong causal offset, a transposed page index, a mis-weighted combine) each fail
at least one test here; test_planted_mistakes_are_caught plants them in copies of
the oracle to show it.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import mla_decode as om
from mla_paged_kv_06_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def _ev(x):
    if isinstance(x, str):
        return float(eval(x, {"__builtins__": {}}, {"exp": math.exp, "log": math.log}))
    return float(x)


def _golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


def _build_golden(case):
    B, s_q, h_q = case["batch"], case["s_q"], case["h_q"]
    q = np.zeros((B, s_q, h_q, 576))
    for b, i, h, entries in case["q"]:
        for d, v in entries:
            q[b, i, h, d] = _ev(v)
    kc = np.zeros((case["num_blocks"], 64, 1, 576))
    for blk in case["nan_blocks"]:
        kc[blk] = np.nan
    for blk, slot, entries in case["rows"]:
        for d, v in entries:
            kc[blk, slot, 0, d] = _ev(v)
    bt = np.array(case["block_table"], dtype=np.int64)
    lens = np.array(case["seqlens"], dtype=np.int64)
    return q, kc, bt, lens


def _check_golden(decode_fn):
    for case in _golden_cases():
        q, kc, bt, lens = _build_golden(case)
        out, lse = decode_fn(q, kc, bt, lens, case["scale"], case["causal"])
        expect = np.zeros_like(out)
        for b, i, h, d, e in case["expect_out"]:
            expect[b, i, h, d] = _ev(e)
        np.testing.assert_allclose(out, expect, rtol=0, atol=1e-14, err_msg=case["name"])
        for b, h, i, e in case["expect_lse"]:
            assert abs(lse[b, h, i] - _ev(e)) < 1e-13, case["name"]


def test_golden_worked_examples():
    _check_golden(oracle.decode)


def test_golden_worked_examples_bruteforce():
    _check_golden(oracle.decode_bruteforce)


def _small_case(seed, lens, s_q, h_q, causal, poison=True, spare=3):
    return wl.make_paged_inputs(lens, s_q, h_q, seed=seed, causal=causal,
                                spare_blocks=spare, poison=poison)


def test_bruteforce_matches_on_tiny_workload():
    x = wl.make_workload("tiny")
    a_out, a_lse = oracle.decode(x.q, x.kcache, x.block_table, x.seqlens, x.scale, x.causal)
    b_out, b_lse = oracle.decode_bruteforce(x.q, x.kcache, x.block_table, x.seqlens,
                                            x.scale, x.causal)
    np.testing.assert_allclose(a_out, b_out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(a_lse, b_lse, rtol=0, atol=1e-12)


@pytest.mark.parametrize("seed,lens,s_q,h_q,causal", [
    (1, [1, 64, 65], 1, 3, False),
    (2, [2, 70, 129], 2, 2, True),
    (3, [63, 1, 128], 2, 1, True),
])
def test_bruteforce_matches_random(seed, lens, s_q, h_q, causal):
    x = _small_case(seed, lens, s_q, h_q, causal)
    a = oracle.decode(x.q, x.kcache, x.block_table, x.seqlens, x.scale, causal)
    b = oracle.decode_bruteforce(x.q, x.kcache, x.block_table, x.seqlens, x.scale, causal)
    np.testing.assert_allclose(a[0], b[0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(a[1], b[1], rtol=0, atol=1e-12)


def test_single_token_returns_its_v_row():
    x = _small_case(5, [1, 1], 1, 4, False)
    out, lse = oracle.decode(x.q, x.kcache, x.block_table, x.seqlens, x.scale, False)
    kc = x.kcache.double().numpy()
    q = x.q.double().numpy()
    for b in range(2):
        row = kc[int(x.block_table[b, 0]), 0, 0]
        for h in range(4):
            assert np.array_equal(out[b, 0, h], row[:512])
            s = x.scale * math.fsum(q[b, 0, h, d] * row[d] for d in range(576))
            assert abs(lse[b, h, 0] - s) < 1e-12


def test_equal_scores_give_mean_of_v():
    x = _small_case(6, [37, 200], 1, 2, False)
    q0 = torch.zeros_like(x.q)
    out, lse = oracle.decode(q0, x.kcache, x.block_table, x.seqlens, x.scale, False)
    kc = x.kcache.double().numpy()
    for b, L in enumerate([37, 200]):
        rows = [kc[int(x.block_table[b, t // 64]), t % 64, 0, :512] for t in range(L)]
        mean = np.array([math.fsum(r[d] for r in rows) / L for d in range(512)])
        for h in range(2):
            np.testing.assert_allclose(out[b, 0, h], mean, rtol=0, atol=1e-13)
            assert abs(lse[b, h, 0] - math.log(L)) < 1e-13


def test_block_permutation_invariance():
    x = _small_case(7, [130, 64, 5], 1, 4, False)
    out, lse = oracle.decode(x.q, x.kcache, x.block_table, x.seqlens, x.scale, False)
    g = torch.Generator().manual_seed(99)
    perm = torch.randperm(x.num_blocks, generator=g)          # new id of old block
    kc2 = torch.empty_like(x.kcache)
    kc2[perm] = x.kcache
    bt2 = perm[x.block_table.long()].to(torch.int32)
    out2, lse2 = oracle.decode(x.q, kc2, bt2, x.seqlens, x.scale, False)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


def test_nan_padding_never_reaches_output():
    x = _small_case(8, [2, 63, 65, 127], 2, 3, True)
    assert torch.isnan(x.kcache.float()).any()
    out, lse = oracle.decode(x.q, x.kcache, x.block_table, x.seqlens, x.scale, True)
    assert np.isfinite(out).all() and np.isfinite(lse).all()


def test_causal_reduces_to_single_query():
    x = _small_case(9, [90, 64, 3], 2, 3, True)
    out, lse = oracle.decode(x.q, x.kcache, x.block_table, x.seqlens, x.scale, True)
    # query 1 sees all L tokens: an s_q = 1 call at length L
    o1, l1 = oracle.decode(x.q[:, 1:2], x.kcache, x.block_table, x.seqlens, x.scale, False)
    # query 0 sees L - 1 tokens: an s_q = 1 call at length L - 1
    o0, l0 = oracle.decode(x.q[:, 0:1], x.kcache, x.block_table, x.seqlens - 1, x.scale, False)
    np.testing.assert_allclose(out[:, 1:2], o1, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse[:, :, 1:2], l1, rtol=0, atol=1e-13)
    np.testing.assert_allclose(out[:, 0:1], o0, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse[:, :, 0:1], l0, rtol=0, atol=1e-13)


def test_empty_visible_sets():
    # L = 0, and a causal query that sees nothing (L = 1, s_q = 2, query 0 sees 0 tokens)
    x = _small_case(10, [0, 1], 2, 2, True)
    out, lse = oracle.decode(x.q, x.kcache, x.block_table, x.seqlens, x.scale, True)
    assert np.all(out[0] == 0) and np.all(np.isneginf(lse[0]))
    assert np.all(out[1, 0] == 0) and np.all(np.isneginf(lse[1, :, 0]))
    assert np.isfinite(lse[1, :, 1]).all()


def test_combine_identity_over_splits():
    x = _small_case(11, [300], 1, 8, False, poison=False, spare=0)
    K = om.gather_tokens(x.kcache.double().numpy(), x.block_table[0].numpy(), 300)
    q = x.q[0, 0]
    full_o, full_l = oracle.decode_partial(q, K, x.scale)
    for cuts in ([0, 300], [0, 64, 300], [0, 1, 128, 129, 300], [0, 0, 150, 150, 300]):
        parts = [oracle.decode_partial(q, K[a:b], x.scale) for a, b in zip(cuts, cuts[1:])]
        o, l = oracle.combine(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
        np.testing.assert_allclose(o, full_o, rtol=0, atol=1e-13)
        np.testing.assert_allclose(l, full_l, rtol=0, atol=1e-12)
    # the combined lse is ln of the summed exponentials (natural log, scale inside)
    s = x.scale * (q.double().numpy() @ K.T)
    ref = np.array([math.log(math.fsum(math.exp(v) for v in row)) for row in s])
    np.testing.assert_allclose(full_l, ref, rtol=0, atol=1e-12)


def test_combine_all_empty():
    o, l = oracle.combine(np.ones((3, 2, 512)), np.full((3, 2), -np.inf))
    assert np.all(o == 0) and np.all(np.isneginf(l))


def test_workload_shapes_and_pools():
    for name, w in wl.WORKLOADS.items():
        lens = wl.draw_seqlens(w.seqlen, w.batch, 0)
        assert lens.shape == (w.batch,) and int(lens.min()) >= 1
        if name == "skewed":
            assert int((lens == 65536).sum()) >= 4 and int(lens.max()) <= 65536
        if name == "v3":
            assert 1 <= int(lens.min()) and int(lens.max()) <= 8192
        if name == "spec":
            assert 512 <= int(lens.min()) and int(lens.max()) <= 8192
    t = wl.make_workload("tiny")
    assert t.num_blocks == 8 and t.seqlens.tolist() == [37, 130]
    assert tuple(t.q.shape) == (2, 1, 16, 576) and t.q.dtype == torch.bfloat16
    # every block a sequence owns appears once; the other slots are NaN
    owned = set()
    for b, L in enumerate(t.seqlens.tolist()):
        for j in range((L + 63) // 64):
            owned.add(int(t.block_table[b, j]))
    assert len(owned) == 4
    spare = [i for i in range(8) if i not in owned]
    assert torch.isnan(t.kcache[spare].float()).all()


# ---------------------------------------------------------------------------------
# Planted mistakes: each mutant oracle must fail at least one pin above.

def _mutant_decode(kind):
    def decode(q, kcache, block_table, seqlens, scale, causal, batch_indices=None):
        kc = om._f64(kcache)
        bt = om._i64(block_table)
        lens = om._i64(seqlens)
        qq = om._f64(q)
        B, s_q, h_q, _ = qq.shape
        out = np.zeros((B, s_q, h_q, 512))
        lse = np.full((B, h_q, s_q), -np.inf)
        for b in range(B):
            for i in range(s_q):
                n = om.visible_tokens(int(lens[b]), s_q, i, causal)
                if kind == "causal_off_by_one" and causal:
                    n -= 1
                if n <= 0:
                    continue
                t = np.arange(n)
                if kind == "page_index_swapped":
                    K = kc[bt[b][t % 64 % bt.shape[1]], t // 64 % 64, 0, :]
                else:
                    K = kc[bt[b][t // 64], t % 64, 0, :]
                Kd = K[:, :512] if kind == "drop_rope" else K
                qd = qq[b, i][:, :512] if kind == "drop_rope" else qq[b, i]
                S = scale * (qd @ Kd.T)
                if kind == "scale_outside":
                    S = S / scale
                V = K[:, 64:] if kind == "v_last_dims" else K[:, :512]
                m = S.max(axis=1, keepdims=True)
                E = np.exp(S - m)
                lsum = E.sum(axis=1)
                out[b, i] = (E @ V) / lsum[:, None]
                lse[b, :, i] = m[:, 0] + np.log(lsum) + (1.0 if kind == "lse_shift" else 0.0)
        if kind == "lse_layout":
            lse = lse[:, ::-1, :].copy()
        return out, lse
    return decode


@pytest.mark.parametrize("kind", ["causal_off_by_one", "page_index_swapped", "drop_rope",
                                  "scale_outside", "v_last_dims", "lse_shift", "lse_layout"])
def test_planted_mistakes_are_caught(kind):
    mutant = _mutant_decode(kind)
    with pytest.raises(AssertionError):
        _check_golden(mutant)


# ---------------------------------------------------------------------------------
# decode_partial on its own: its output is the attention over an explicit token set, so
# over the whole visible set of a row it must give what the brute-force loop gives for
# that row. This pins the function independently of combine() (which only relates its
# outputs to each other).

def _partial_vs_bruteforce(partial_fn):
    x = _small_case(12, [70, 130, 1], 2, 3, True)
    bf_out, bf_lse = oracle.decode_bruteforce(x.q, x.kcache, x.block_table, x.seqlens,
                                              x.scale, True)
    kc = x.kcache.double().numpy()
    for b, L in enumerate(x.seqlens.tolist()):
        for i in range(x.s_q):
            n = om.visible_tokens(L, x.s_q, i, True)
            K = om.gather_tokens(kc, x.block_table[b].numpy(), max(n, 0))
            o, l = partial_fn(x.q[b, i], K, x.scale)
            np.testing.assert_allclose(o, bf_out[b, i], rtol=0, atol=1e-12)
            if n > 0:
                np.testing.assert_allclose(l, bf_lse[b, :, i], rtol=0, atol=1e-12)
            else:
                assert np.all(np.isneginf(l)) and np.all(o == 0)


def test_decode_partial_matches_bruteforce_over_a_rows_visible_tokens():
    _partial_vs_bruteforce(oracle.decode_partial)


def test_decode_partial_matches_decode_on_a_workload_sequence():
    x = _small_case(13, [300, 1000], 1, 8, False, poison=False, spare=0)
    out, lse = oracle.decode(x.q, x.kcache, x.block_table, x.seqlens, x.scale, False)
    kc = x.kcache.double().numpy()
    for b, L in enumerate([300, 1000]):
        K = om.gather_tokens(kc, x.block_table[b].numpy(), L)
        o, l = oracle.decode_partial(x.q[b, 0], K, x.scale)
        np.testing.assert_allclose(o, out[b, 0], rtol=0, atol=1e-13)
        np.testing.assert_allclose(l, lse[b, :, 0], rtol=0, atol=1e-12)


def _mutant_partial(kind):
    def partial(q_rows, K_rows, scale):
        qq, K = om._f64(q_rows), om._f64(K_rows)
        if K.shape[0] == 0:
            return np.zeros((qq.shape[0], 512)), np.full(qq.shape[0], -np.inf)
        S = scale * (qq @ K.T)
        m = S.max(axis=1, keepdims=True)
        E = np.exp(S - m)
        lsum = E.sum(axis=1)
        V = K[:, 64:] if kind == "v_last_dims" else K[:, :512]
        o = E @ V
        if kind != "no_normalise":
            o = o / lsum[:, None]
        lse = m[:, 0] + np.log(lsum) if kind != "lse_without_max" else np.log(lsum)
        return o, lse
    return partial


@pytest.mark.parametrize("kind", ["v_last_dims", "no_normalise", "lse_without_max"])
def test_planted_mistakes_in_decode_partial_are_caught(kind):
    with pytest.raises(AssertionError):
        _partial_vs_bruteforce(_mutant_partial(kind))
