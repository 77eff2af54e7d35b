"""Pins of the online-FP8 LM-head oracle against what the format and the
mathematics fix (runs without a GPU)."""
import numpy as np
import pytest
import torch

import oracle.lmhead_ref as L


def test_e4m3_decode_literals():
    # bit patterns from the e4m3 definition: sign | 4-bit exponent (bias 7) | 3-bit mantissa
    table = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0, 0x39: 1.125,
             0x3F: 1.875, 0x40: 2.0, 0x7E: 448.0, 0xB8: -1.0, 0xFE: -448.0, 0x81: -(2.0 ** -9)}
    for c, v in table.items():
        assert L.e4m3_decode(np.uint8(c)) == v, hex(c)
    assert np.isnan(L.e4m3_decode(np.uint8(0x7F))) and np.isnan(L.e4m3_decode(np.uint8(0xFF)))


def test_e4m3_positive_codes_are_increasing():
    v = L.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    assert np.all(np.diff(v) > 0)


def test_e4m3_round_trip_of_every_finite_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    back = L.e4m3_encode(L.e4m3_decode(codes).astype(np.float32))
    assert np.array_equal(back, codes)


def test_e4m3_ties_go_to_even_and_large_values_saturate():
    cases = {1.0625: 0x38,            # halfway 1.0 / 1.125 -> even mantissa 0
             1.1875: 0x3A,            # halfway 1.125 / 1.25 -> 1.25 (mantissa 2)
             2.0 ** -10: 0x00,        # halfway 0 / 2^-9 -> 0
             3 * 2.0 ** -10: 0x02,    # halfway 2^-9 / 2^-8 -> 2^-8 (mantissa 2)
             15 * 2.0 ** -10: 0x08,   # halfway 7 * 2^-9 / 2^-6 -> 2^-6 (first normal)
             448.0 * (1 + 2 ** -5): 0x7E, 1000.0: 0x7E, -1000.0: 0xFE, 0.0: 0x00}
    for v, c in cases.items():
        assert L.e4m3_encode(np.float32(v)) == c, v


def test_e4m3_encode_matches_torch_float8_in_range():
    rng = np.random.default_rng(5)
    v = np.concatenate([rng.uniform(-448, 448, 100_000), rng.uniform(-2 ** -5, 2 ** -5, 20_000),
                        rng.standard_normal(20_000) * 3]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(L.e4m3_encode(v), ref)


def test_quantize_rows_scale_and_extremes():
    rng = np.random.default_rng(1)
    w = (rng.standard_normal((6, 256)) * np.array([1, 1e-3, 50, 1, 1, 1])[:, None]).astype(np.float32)
    w[3] = 0.0                                   # all-zero row: scale 1, codes 0
    q, s = L.quantize_rows(w)
    amax = np.abs(w).max(axis=1).astype(np.float32)
    for r in range(6):
        if r == 3:
            assert s[r] == 1.0 and not q[r].any()
            continue
        assert s[r] == np.float32(amax[r] / np.float32(448.0))
        j = int(np.argmax(np.abs(w[r])))
        assert q[r, j] & 0x7F == 0x7E        # the row maximum maps to 448 (up to the sign)
        deq = L.e4m3_decode(q[r]) * s[r]
        # e4m3 keeps 3 mantissa bits: relative error <= 2^-4 above the subnormal range
        big = np.abs(w[r]) >= 2.0 ** -6 * s[r]
        assert np.all(np.abs(deq[big] - w[r][big]) <= 2.0 ** -4 * np.abs(w[r][big]) + 1e-30)


def test_quantize_rows_scale_invariance():
    rng = np.random.default_rng(2)
    w = rng.standard_normal((3, 64)).astype(np.float32)
    q1, s1 = L.quantize_rows(w)
    q2, s2 = L.quantize_rows(w * np.float32(8.0))   # a power of two: every fp32 step scales exactly
    assert np.array_equal(q1, q2) and np.array_equal(s2, s1 * np.float32(8.0))


def _bf16_bits(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_lm_head_matches_python_loops():
    # (a restatement of the sum as loops; the independent pins are the format
    # tests above and the comparison with the unquantised product below)
    rng = np.random.default_rng(3)
    x = _bf16_bits(rng.standard_normal((2, 32)))
    w = _bf16_bits(rng.standard_normal((3, 32)) * 0.02)
    logits, xq, xs, wq, ws = L.lm_head_fp8(x, w)
    xd, wd = L.e4m3_decode(xq), L.e4m3_decode(wq)
    for t in range(2):
        for v in range(3):
            acc = 0.0
            for k in range(32):
                acc += float(xd[t, k]) * float(wd[v, k])
            assert abs(logits[t, v] - acc * float(xs[t]) * float(ws[v])) <= 1e-12 * (1 + abs(acc))


def test_lm_head_close_to_the_unquantised_product():
    rng = np.random.default_rng(4)
    xf = rng.standard_normal((4, 2560)).astype(np.float32)
    wf = (rng.standard_normal((64, 2560)) * 0.02).astype(np.float32)
    x, w = _bf16_bits(xf), _bf16_bits(wf)
    logits = L.lm_head_fp8(x, w)[0]
    xb = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    wb = (w.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ref = xb @ wb.T
    # two e4m3 roundings (relative 2^-4 each, random signs) over 2560 terms; a
    # wrong scale, a transposed operand or a dropped term is far outside this
    assert np.abs(logits - ref).max() <= 0.05 * np.abs(ref).max()
