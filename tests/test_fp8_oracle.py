"""Pins of the FP8 latent-cache oracle (CPU only): the E4M3 codec against torch's
float8_e4m3fn and against its definition, the quantizer's error bound and byte layout,
and decode over the dequantized cache against the brute-force loop.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import fp8_cache as f8
from mla_paged_kv_06_b200 import workloads as wl


def test_every_code_decodes_like_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().double().numpy()
    assert np.array_equal(f8.e4m3_value(codes), ref, equal_nan=True)
    # the format's landmarks, from the bit fields
    assert f8.e4m3_value(np.uint8(0x7E)) == 448.0
    assert f8.e4m3_value(np.uint8(0x01)) == 2.0 ** -9           # smallest subnormal
    assert f8.e4m3_value(np.uint8(0x08)) == 2.0 ** -6           # smallest normal
    assert np.isnan(f8.e4m3_value(np.uint8(0x7F))) and np.isnan(f8.e4m3_value(np.uint8(0xFF)))


def test_encoder_matches_torch_in_range():
    g = np.random.default_rng(0)
    x = (g.standard_normal(100_000) * np.exp(g.uniform(-14, 6, 100_000))).astype(np.float32)
    # every midpoint between neighbouring values (the ties) and the values themselves
    pos = f8.e4m3_value(np.arange(0x7F, dtype=np.uint8))
    mids = ((pos[1:] + pos[:-1]) / 2).astype(np.float32)
    x = np.concatenate([x, pos.astype(np.float32), mids, -mids, np.float32([0.0, -0.0])])
    x = x[np.abs(x) < 464]                # torch turns |x| >= 464 into NaN, the format saturates
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(f8.e4m3_encode(x), ref)


def test_encoder_saturates_and_keeps_nan():
    x = np.float32([448.0, 449.0, 463.9, 464.0, 480.0, 1e30, -1e30, np.inf, -np.inf, np.nan])
    codes = f8.e4m3_encode(x)
    assert list(codes[:6]) == [0x7E] * 6
    assert codes[6] == 0xFE and codes[7] == 0x7E and codes[8] == 0xFE
    assert codes[9] == f8.E4M3_NAN


def test_ties_go_to_the_even_code():
    # 232 lies halfway between 224 (code 0x76, even) and 240 (0x77): 224; 248 between
    # 240 (0x77) and 256 (0x78): 256; 0.0029296875 between 2^-9 (0x01) and 2^-8 (0x02): 2^-8
    codes = f8.e4m3_encode(np.float32([232.0, 248.0, 0.0029296875]))
    assert list(codes) == [0x76, 0x78, 0x02]


def _row(vals_latent, vals_rope):
    x = torch.tensor(np.concatenate([vals_latent, vals_rope]), dtype=torch.float32)
    return x.to(torch.bfloat16).reshape(1, 576)


def test_byte_layout_of_a_hand_built_row():
    lat = np.zeros(512)
    lat[0] = 448.0              # group 0: amax 448 -> scale 1, code of 448 is 0x7E
    lat[1] = -1.0               # -> 0xB8
    lat[128] = 3.5              # group 1: amax 3.5 -> scale 3.5/448
    lat[256:384] = 0.0          # group 2: all zero -> scale 0, codes 0
    lat[384] = -0.25            # group 3: amax 0.25
    rope = np.arange(64) * 0.5 - 7.0
    q = f8.quantize_rows(_row(lat, rope))[0]
    assert q.shape == (656,)
    assert q[0] == 0x7E and q[1] == 0xB8 and q[2] == 0
    scales = q[512:528].copy().view("<f4")
    assert scales[0] == np.float32(1.0)
    assert scales[1] == np.float32(3.5) / np.float32(448.0)
    assert scales[2] == 0.0 and np.all(q[256:384] == 0)
    assert q[128] == 0x7E and q[384] == 0xFE            # each group's amax maps to +-448
    rope_bits = torch.tensor(rope, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy()
    assert np.array_equal(q[528:656].copy().view("<i2"), rope_bits)
    back = f8.dequantize_rows(q[None])[0]
    assert back[0] == 448.0 and back[1] == -1.0 and back[128] == 3.5     # scales 1 and 2^-7
    # amax 0.25 comes back as 448 times the fp32-rounded scale 0.25 / 448, in fp32, then
    # rounded to bf16: within 2^-24 of 0.25 before the bf16 step, exactly 0.25 after it
    prod = np.float32(448.0) * (np.float32(0.25) / np.float32(448.0))
    assert abs(float(prod) - 0.25) <= 0.25 * 2.0 ** -23
    assert back[384] == -0.25
    assert np.array_equal(back[512:], rope)


def test_a_swapped_scale_order_is_caught():
    # planted mistake: groups 0 and 1 with their scales exchanged must not read back
    lat = np.concatenate([np.full(128, 2.0), np.full(128, 0.5), np.ones(256)])
    q = f8.quantize_rows(_row(lat, np.zeros(64)))[0].copy()
    sc = q[512:528].copy()
    q[512:516], q[516:520] = sc[4:8], sc[0:4]
    assert not np.array_equal(f8.dequantize_rows(q[None])[0][:256], lat[:256])


def test_representable_values_round_trip_exactly():
    g = np.random.default_rng(1)
    pos = f8.e4m3_value(np.arange(0x7F, dtype=np.uint8))
    lat = g.choice(np.concatenate([pos, -pos]), size=512)
    lat[::128] = 448.0                                  # each group's amax 448: scale 1
    x = _row(lat, g.standard_normal(64))
    back = f8.dequantize_rows(f8.quantize_rows(x))[0]
    assert np.array_equal(back[:512], lat)


def test_quantization_error_is_within_the_format_bound():
    # per element: at most half a step of the value's binade (2^-4 relative for normal
    # values), and at most half the subnormal step (2^-10 * scale) below 2^-6 * scale;
    # the read-back then adds the fp32 product's and the bf16 rounding (2^-24 + 2^-9 of the
    # read-back value)
    x = wl.make_paged_inputs([300], 1, 1, seed=2).kcache.reshape(-1, 576)[:300]
    ref = x.float().double().numpy()
    back = f8.dequantize_rows(f8.quantize_rows(x))
    assert np.array_equal(back[:, 512:], ref[:, 512:])          # rope untouched
    q = f8.quantize_rows(x)
    scales = q[:, 512:528].copy().view("<f4").astype(np.float64)
    s = np.repeat(scales, 128, axis=1)
    err = np.abs(back[:, :512] - ref[:, :512])
    bound = (np.maximum(np.abs(ref[:, :512]) * 2.0 ** -4, s * 2.0 ** -10) * (1 + 1e-6)
             + np.abs(back[:, :512]) * (2.0 ** -9 + 2.0 ** -24))
    assert np.all(err <= bound)
    assert err.max() > 0                                # it is a lossy format


def test_read_back_is_the_fp32_product_rounded_to_bf16():
    # an independent route to the same value: torch's E4M3 decode, an fp32 multiply and
    # torch's round-to-nearest-even cast to bf16
    x = wl.make_paged_inputs([200], 1, 1, seed=6).kcache.reshape(-1, 576)[:200]
    q = f8.quantize_rows(x)
    codes = torch.from_numpy(q[:, :512].copy()).view(torch.float8_e4m3fn).float()
    scales = torch.from_numpy(q[:, 512:528].copy().view("<f4")).repeat_interleave(128, dim=1)
    want = (codes * scales).to(torch.bfloat16).double().numpy()
    assert np.array_equal(f8.dequantize_rows(q)[:, :512], want)


def test_bf16_rounding_ties_and_specials():
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: ties go to the even mantissa (1);
    # 1 + 3 * 2^-8 halfway between 1 + 2^-7 and 1 + 2^-6: to 1 + 2^-6; just above a tie
    # rounds up; NaN stays NaN
    x = np.float32([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, 1 + 2.0 ** -8 + 2.0 ** -20, -2.5, np.nan])
    r = f8.round_to_bf16(x)
    assert r[0] == 1.0 and r[1] == 1 + 2.0 ** -6 and r[2] == 1 + 2.0 ** -7 and r[3] == -2.5
    assert np.isnan(r[4])
    g = np.random.default_rng(7)
    y = (g.standard_normal(200_000) * np.exp(g.uniform(-30, 30, 200_000))).astype(np.float32)
    want = torch.from_numpy(y).to(torch.bfloat16).float().numpy()
    assert np.array_equal(f8.round_to_bf16(y), want)


def test_fp8_decode_matches_brute_force_on_the_dequantized_cache():
    x = wl.make_paged_inputs([37, 130, 1], 2, 4, seed=3, causal=True, spare_blocks=2)
    fp8 = f8.quantize_cache(x.kcache)
    deq = f8.dequantize_cache(fp8)
    out, lse = f8.decode_fp8(x.q, fp8, x.block_table, x.seqlens, x.scale, True)
    ref_out, ref_lse = oracle.decode_bruteforce(x.q, deq, x.block_table, x.seqlens, x.scale, True)
    assert np.abs(out - ref_out).max() <= 1e-12
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(lse), fin)
    assert np.abs(lse[fin] - ref_lse[fin]).max() <= 1e-12


def test_fp8_decode_error_against_the_bf16_decode():
    # Not a pin but the format's cost, seen at the output on N(0,1) data: a 2^-4 relative
    # error on every latent dim moves each score by a few hundredths, so outputs move by
    # a few percent of their size. An FP8 kernel is therefore compared with this FP8
    # oracle (the dequantized cache), not with the bf16 decode.
    x = wl.make_paged_inputs([500, 64, 1000], 1, 16, seed=4)
    out8, lse8 = f8.decode_fp8(x.q, f8.quantize_cache(x.kcache), x.block_table, x.seqlens,
                               x.scale, False)
    out, lse = oracle.decode(x.q, x.kcache, x.block_table, x.seqlens, x.scale, False)
    rel = np.sqrt(((out8 - out) ** 2).sum() / (out ** 2).sum())
    assert 1e-3 < rel < 0.1
    assert np.abs(lse8 - lse).max() < 0.1


@pytest.mark.parametrize("n", [1, 7, 64])
def test_cache_shapes(n):
    x = wl.make_paged_inputs([64 * n], 1, 1, seed=5)
    fp8 = f8.quantize_cache(x.kcache)
    assert fp8.shape == (n, 64, 656) and fp8.dtype == np.uint8
    assert f8.dequantize_cache(fp8).shape == (n, 64, 1, 576)
