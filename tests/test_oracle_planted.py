"""Each plausible mistake planted in the LM-head and MXFP4 oracles (on the
CPU, by monkeypatching the oracle) must make at least one of their pins fail:
evidence that the pins constrain what they claim to (runs without a GPU)."""
import numpy as np
import pytest

import oracle.lmhead_ref as L
import oracle.mxfp4_ref as MX
import tests.test_oracle_lmhead as PL
import tests.test_oracle_mxfp4 as PM


def _some_pin_fails(pins):
    for pin in pins:
        try:
            pin()
        except AssertionError:
            return True
    return False


LMHEAD_PINS = [PL.test_e4m3_decode_literals, PL.test_e4m3_positive_codes_are_increasing,
               PL.test_e4m3_round_trip_of_every_finite_code, PL.test_e4m3_ties_go_to_even_and_large_values_saturate,
               PL.test_e4m3_encode_matches_torch_float8_in_range, PL.test_quantize_rows_scale_and_extremes,
               PL.test_quantize_rows_scale_invariance, PL.test_lm_head_close_to_the_unquantised_product]
MXFP4_PINS = [PM.test_e2m1_decode_literals, PM.test_e2m1_decode_matches_ml_dtypes,
              PM.test_ue8m0_decode_matches_torch_and_literals, PM.test_pack_unpack_round_trip_and_nibble_order,
              PM.test_dequantize_hand_worked_row, PM.test_layer_equals_the_w4_oracle_on_shared_weights]


def test_pins_pass_unmodified():
    for pin in LMHEAD_PINS + MXFP4_PINS:
        pin()


@pytest.mark.parametrize("name,mutant", [
    # exponent bias 8 instead of 7
    ("e4m3_decode", lambda orig: (lambda c: orig(c) / 2.0)),
    # round half away from zero instead of ties to even
    ("e4m3_encode", lambda orig: (lambda v: orig(np.nextafter(np.asarray(v, np.float32), np.float32(np.inf))))),
    # scale divides by 447 instead of 448
    ("quantize_rows", lambda orig: (lambda w: (lambda q, s: (q, (s * np.float32(448.0 / 447.0)).astype(np.float32)))(*orig(w)))),
])
def test_lmhead_mutants_are_caught(monkeypatch, name, mutant):
    monkeypatch.setattr(L, name, mutant(getattr(L, name)))
    assert _some_pin_fails(LMHEAD_PINS), name


def test_lmhead_dropped_token_scale_is_caught(monkeypatch):
    orig = L.lm_head_fp8

    def no_x_scale(x, w):
        logits, xq, xs, wq, ws = orig(x, w)
        return logits / xs.astype(np.float64)[:, None], xq, xs, wq, ws
    monkeypatch.setattr(L, "lm_head_fp8", no_x_scale)
    assert _some_pin_fails(LMHEAD_PINS)


@pytest.mark.parametrize("name,mutant", [
    # exponent bias 0 instead of 1
    ("e2m1_decode", lambda orig: (lambda c: orig(c) * 2.0)),
    # high nibble taken as the even index
    ("unpack_e2m1", lambda orig: (lambda p: orig(p).reshape(*np.asarray(p).shape[:-1], -1, 2)[..., ::-1]
                                  .reshape(*np.asarray(p).shape[:-1], -1))),
    # E8M0 bias 128 instead of 127
    ("ue8m0_decode", lambda orig: (lambda e: orig(e) / 2.0)),
    # block scales tiled along K instead of repeated per 32 elements
    ("dequantize_mxfp4", lambda orig: (lambda p, s: MX.e2m1_decode(MX.unpack_e2m1(p))
                                       * np.tile(MX.ue8m0_decode(s), (1,) * (np.asarray(s).ndim - 1) + (32,)))),
])
def test_mxfp4_mutants_are_caught(monkeypatch, name, mutant):
    monkeypatch.setattr(MX, name, mutant(getattr(MX, name)))
    assert _some_pin_fails(MXFP4_PINS), name
