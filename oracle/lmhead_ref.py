"""fp64 CPU oracle of the online-FP8 LM head (hidden 2560 -> vocabulary 157,184).

TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the
benchmark's CPU-baseline arm may import this module.  The GPU library never
imports it, and it imports nothing from the GPU library.

What the pages say (bpdata article "Harom optimalizacio a Ling-3.0-flash MoE
inferenciajanak", section "Optimalizacio 2: Online FP8 LM head kvantalas"):
the LM head projects the 2,560-wide hidden state onto a 157,184-token
vocabulary; the checkpoint stores it in bf16 and leaves it unquantised, so
every decoded token reads the whole 157,184 x 2,560 matrix.  The optimisation
quantises it dynamically to FP8 when the LM head is built, which roughly
halves the bytes read per token.

Readings this oracle takes where the pages are silent (also listed in the
design notes):
  * FP8 format: e4m3 with no infinities (bias 7, largest finite 448, one NaN
    pattern per sign), rounding to nearest with ties to even, saturating to
    +-448 (an input never exceeds 448 by more than a rounding error here).
  * weights: one fp32 scale per vocabulary row, s_w = max|w_row| / 448
    (fp32 division); codes = e4m3(w / s_w) with the division in fp32.
  * activations: quantised the same way per token at call time ("dynamic").
  * logits[t, v] = s_x[t] * s_w[v] * sum_k e4m3(x)[t, k] * e4m3(w)[v, k]:
    every product of two e4m3 values is exact; the oracle sums in fp64.
  * an all-zero row or token gets scale 1 (its codes are all zero).
Where floating point decides a code, both sides use the same fp32 steps:
fp32 max, fp32 division by 448, fp32 division of each value by the scale.
"""
from __future__ import annotations

import numpy as np

__all__ = ["E4M3_MAX", "e4m3_decode", "e4m3_encode", "quantize_rows", "lm_head_fp8"]

E4M3_MAX = 448.0


def e4m3_decode(codes) -> np.ndarray:
    """e4m3 bytes -> exact float64.

    Bit 7 is the sign, bits 6..3 the exponent field E, bits 2..0 the mantissa
    field M.  E = 0: subnormal M / 8 * 2^-6; E = 1..15: (1 + M / 8) * 2^(E-7),
    except E = 15, M = 7, which is NaN (the format has no infinities).
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def e4m3_encode(values) -> np.ndarray:
    """float32 values -> e4m3 bytes, nearest with ties to even, saturating to +-448.

    Finite inputs only.  The e4m3 grid has spacing 2^(e-3) in the binade
    [2^e, 2^(e+1)) for e = -6..8, and 2^-9 below 2^-6 (subnormals), so a
    magnitude is divided by its spacing (exact: a power of two), rounded to
    an integer n with ties to even, and n is turned into the fields.
    """
    v = np.asarray(values, dtype=np.float32).astype(np.float64)
    sign = np.signbit(v)
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.clip(e, -6, 8)                       # binade exponent (subnormals share -6's spacing)
    spacing = np.exp2(e - 3.0)
    n = np.rint(a / spacing)                    # numpy rint: ties to even
    # n / 8 >= 2 means the value rounded up into the next binade
    up = n >= 16
    e = np.where(up, e + 1, e)
    n = np.where(up, n / 2, n)                  # 16 -> 8 (exact: 16 is even)
    normal = (n >= 8) | (e > -6)
    field_e = np.where(normal & (n >= 8), e + 7, 0)
    field_m = np.where(normal & (n >= 8), n - 8, n)
    code = (field_e.astype(np.int64) << 3) | field_m.astype(np.int64)
    code = np.where(a >= E4M3_MAX, 0x7E, code)  # saturate: 448 = E 15, M 6
    code = np.minimum(code, 0x7E)
    return (code | np.where(sign, 0x80, 0)).astype(np.uint8)


def quantize_rows(rows_f32):
    """Rows (float32 [R, K]) -> (codes uint8 [R, K], scales float32 [R]).

    scale = max|row| / 448 in fp32 (1 for an all-zero row); codes =
    e4m3(row / scale) with the division in fp32.
    """
    w = np.asarray(rows_f32, dtype=np.float32)
    amax = np.max(np.abs(w), axis=1).astype(np.float32)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    q = (w / scale[:, None]).astype(np.float32)
    return e4m3_encode(q), scale


def lm_head_fp8(x_bf16_bits, w_bf16_bits):
    """logits [T, V] (float64) of the online-FP8 LM head.

    x_bf16_bits: bf16 bit patterns [T, H]; w_bf16_bits: bf16 bit patterns
    [V, H].  Returns (logits, x codes, x scales, w codes, w scales).
    """
    def to_f32(bits):
        b = np.asarray(bits, dtype=np.uint16)
        return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)

    xq, xs = quantize_rows(to_f32(np.atleast_2d(x_bf16_bits)))
    wq, ws = quantize_rows(to_f32(np.atleast_2d(w_bf16_bits)))
    xd = e4m3_decode(xq)
    wd = e4m3_decode(wq)
    logits = (xd @ wd.T) * xs.astype(np.float64)[:, None] * ws.astype(np.float64)[None, :]
    return logits, xq, xs, wq, ws
