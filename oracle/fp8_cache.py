"""CPU oracle for an FP8 latent cache: the row format, its quantizer, and decode over it.

TEST INFRASTRUCTURE ONLY, like the rest of this package: only the tests, the package's
`smoke()` check and the benchmark's CPU legs may use it, and it shares no code with the
CUDA path.

Where it comes from
-------------------
The pages use FP8 for training, GEMMs and communication, not for the KV cache: the
DeepSeek-V3 co-design summary (news.chathome.org, paragraph on low-precision-driven
design) for FP8 mixed-precision training; the DeepGEMM page (618zxw.cn, Open Source
Week day 3, paragraphs on the library and on fine-grained scaling) for FP8 GEMMs with
fine-grained scale factors; the DeepEP page (cointeeth.com, feature 3) for FP8
dispatch. They fix no cache format. An FP8 latent cache cuts the bytes a memory-bound
decode streams by 43%, so the format below is this library's own choice, taking from
the GEMM page only the idea of one scale per small group of values:

  one token's row, 656 bytes:
    [0, 512)    the 512 latent dims as FP8 E4M3 codes (OCP E4M3: 1 sign, 4 exponent bits
                with bias 7, 3 mantissa bits, subnormals, no infinities, S.1111.111 = NaN,
                largest finite 448)
    [512, 528)  four fp32 scales, little-endian, one per 128-dim group of the latent dims
    [528, 656)  the 64 rope dims, unchanged bf16, little-endian
  a page is 64 such rows: 41,984 bytes (every row starts on a 16-byte boundary).

Quantizing a bf16 row, group g = dims [128g, 128g + 128):
    amax_g  = max |x_d| over the group                       (exact)
    s_g     = fp32(amax_g / 448)                             (fp32 division, nearest-even)
    code_d  = E4M3(fp32(x_d / s_g)), nearest-even, saturated to +-448    (0 when s_g = 0)
The integer codes are decided in fp32, the precision a kernel would use. Reading back:
    x^_d = bf16(fp32(E4M3 value(code_d) * s_g))     (fp32 product, then bf16, both
                                                     round-to-nearest-even)
and rope dims are read back as they were. The read-back value is a bf16 number: the
operand type a tensor-core decode multiplies, so a decode kernel widens every page into
exactly these values and the CPU side takes the same two roundings in the same order.
Their cost (2^-9 relative at most, with the fp32 step far below it) is small beside the
format's own 2^-4 step. Decode over an FP8 cache is exact attention (the bf16 oracle's
definition) over the read-back rows x^.

Pins (tests/test_fp8_oracle.py, no GPU): every code against torch's float8_e4m3fn, the
encoder against torch's cast on values in range, saturation and rounding ties by the
definition, the read-back against torch's fp32 product and bf16 cast, the bf16 rounding
on its ties, the round trip of representable values, the error bound of the format, the
byte layout on a hand-built row, and decode against the brute-force loop on the
dequantized cache.
"""

from __future__ import annotations

import numpy as np

ROW_BYTES = 656
LATENT = 512
ROPE = 64
GROUP = 128
GROUPS = LATENT // GROUP
SCALE_OFF = LATENT
ROPE_OFF = LATENT + 4 * GROUPS
E4M3_MAX = 448.0
E4M3_NAN = 0x7F


def e4m3_value(codes) -> np.ndarray:
    """fp64 value of each E4M3 code (uint8), from the bit fields."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    val = sign * val
    return np.where((e == 15) & (m == 7), np.nan, val)


# the 127 non-negative finite values in code order (codes 0x00 .. 0x7E), increasing
_POS = e4m3_value(np.arange(0x7F, dtype=np.uint8))


def e4m3_encode(x) -> np.ndarray:
    """E4M3 code of each fp32 value: nearest representable value, ties to the even code,
    magnitudes at or above 448 saturate to 448, NaN gives the NaN code."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    neg = np.signbit(x)
    a = np.abs(x)
    hi = np.searchsorted(_POS, a, side="left").clip(1, len(_POS) - 1)   # _POS[hi-1] < a <= _POS[hi]
    lo = hi - 1
    d_lo = a - _POS[lo]
    d_hi = _POS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(a >= E4M3_MAX, 0x7E, code)
    code = np.where(a == 0.0, 0, code)
    code = code | np.where(neg, 0x80, 0)
    code = np.where(np.isnan(x), E4M3_NAN, code)
    return code.astype(np.uint8)


def _bf16_bits(x) -> np.ndarray:
    if hasattr(x, "view") and hasattr(x, "dtype") and "bfloat16" in str(x.dtype):
        import torch
        return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    return np.asarray(x, dtype=np.uint16)


def _bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def quantize_rows(rows) -> np.ndarray:
    """[n, 576] bf16 rows (torch bf16 or uint16 bit patterns) -> [n, 656] uint8 rows."""
    bits = _bf16_bits(rows).reshape(-1, LATENT + ROPE)
    x = _bits_to_f32(bits)
    n = x.shape[0]
    out = np.zeros((n, ROW_BYTES), dtype=np.uint8)
    scales = np.zeros((n, GROUPS), dtype=np.float32)
    for g in range(GROUPS):
        xg = x[:, GROUP * g: GROUP * (g + 1)]
        amax = np.abs(xg).max(axis=1)
        s = (amax / np.float32(E4M3_MAX)).astype(np.float32)
        scales[:, g] = s
        with np.errstate(divide="ignore", invalid="ignore"):
            ratio = (xg / s[:, None]).astype(np.float32)
        codes = e4m3_encode(ratio)
        codes[s == 0] = 0
        out[:, GROUP * g: GROUP * (g + 1)] = codes
    out[:, SCALE_OFF:ROPE_OFF] = scales.astype("<f4").view(np.uint8).reshape(n, 4 * GROUPS)
    out[:, ROPE_OFF:] = bits[:, LATENT:].astype("<u2").view(np.uint8).reshape(n, 2 * ROPE)
    return out


def round_to_bf16(x32) -> np.ndarray:
    """fp32 values rounded to the nearest bf16 value (ties to even), returned as fp32:
    on the bit pattern, add 0x7FFF plus the lowest kept bit and drop the low 16 bits.
    NaN stays NaN; the format's products never reach the overflow range."""
    x32 = np.asarray(x32, dtype=np.float32)
    bits = x32.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    r = (((bits + 0x7FFF + lsb) >> 16) << 16).astype(np.uint32).view(np.float32)
    return np.where(np.isnan(x32), np.float32(np.nan), r)


def dequantize_rows(q) -> np.ndarray:
    """[n, 656] uint8 rows -> [n, 576] fp64 values: latent dims bf16(fp32(code * scale)),
    rope dims as stored."""
    q = np.asarray(q, dtype=np.uint8).reshape(-1, ROW_BYTES)
    n = q.shape[0]
    scales = q[:, SCALE_OFF:ROPE_OFF].copy().view("<f4")                      # fp32
    vals = e4m3_value(q[:, :LATENT]).astype(np.float32).reshape(n, GROUPS, GROUP)  # exact
    with np.errstate(invalid="ignore", over="ignore"):
        prod = (vals * scales[:, :, None]).astype(np.float32)                   # fp32, nearest-even
    lat = round_to_bf16(prod).astype(np.float64)
    rope = _bits_to_f32(q[:, ROPE_OFF:].copy().view("<u2")).astype(np.float64)
    return np.concatenate([lat.reshape(n, LATENT), rope], axis=1)


def quantize_cache(kcache) -> np.ndarray:
    """bf16 cache [num_blocks, 64, 1, 576] -> FP8 cache [num_blocks, 64, 656] uint8."""
    bits = _bf16_bits(kcache)
    nb = bits.shape[0]
    return quantize_rows(bits.reshape(-1, LATENT + ROPE)).reshape(nb, 64, ROW_BYTES)


def dequantize_cache(fp8_cache) -> np.ndarray:
    """FP8 cache [num_blocks, 64, 656] -> fp64 [num_blocks, 64, 1, 576]."""
    q = np.asarray(fp8_cache, dtype=np.uint8)
    nb = q.shape[0]
    return dequantize_rows(q.reshape(-1, ROW_BYTES)).reshape(nb, 64, 1, LATENT + ROPE)


def decode_fp8(q, fp8_cache, block_table, seqlens, scale: float, causal: bool,
               batch_indices=None):
    """Exact decode attention over the read-back FP8 cache (fp64), for all sequences or
    those in `batch_indices`. Only the pages those sequences own are read back (the
    others are left NaN, and the bf16 oracle never reads a page a sequence does not own)."""
    from .mla_decode import decode
    q8 = np.asarray(fp8_cache, dtype=np.uint8)
    nb = q8.shape[0]
    idx = range(len(seqlens)) if batch_indices is None else list(batch_indices)
    lens = np.asarray(seqlens, dtype=np.int64)
    bt = np.asarray(block_table, dtype=np.int64)
    used = sorted({int(bt[b][j]) for b in idx for j in range((int(lens[b]) + 63) // 64)})
    deq = np.full((nb, 64, 1, LATENT + ROPE), np.nan)
    if used:
        deq[used] = dequantize_rows(q8[used].reshape(-1, ROW_BYTES)).reshape(len(used), 64, 1,
                                                                             LATENT + ROPE)
    return decode(q, deq, block_table, seqlens, scale, causal, batch_indices=batch_indices)
