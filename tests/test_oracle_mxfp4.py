"""Pins of the MXFP4 oracle against the format's definition, two library
implementations of its element and scale types, and the pinned W4 oracle on
weights both formats represent exactly (runs without a GPU)."""
import ml_dtypes
import numpy as np
import torch

import oracle.moe_ref as W4
import oracle.mxfp4_ref as MX


def test_e2m1_decode_literals():
    # sign | E (2 bits, bias 1) | M: the 16 codes of the definition
    expect = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    got = MX.e2m1_decode(np.arange(16))
    assert list(got[:8]) == expect
    assert list(got[8:]) == [-v for v in expect]
    assert np.signbit(got[8])  # code 8 is -0


def test_e2m1_decode_matches_ml_dtypes():
    codes = np.arange(16, dtype=np.uint8)
    ref = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(MX.e2m1_decode(codes), ref)


def test_ue8m0_decode_matches_torch_and_literals():
    e = np.arange(255, dtype=np.uint8)
    ref = torch.from_numpy(e).view(torch.float8_e8m0fnu).double().numpy()
    assert np.array_equal(MX.ue8m0_decode(e), ref)
    assert MX.ue8m0_decode(127) == 1.0 and MX.ue8m0_decode(128) == 2.0 and MX.ue8m0_decode(120) == 2.0 ** -7
    assert np.isnan(MX.ue8m0_decode(255))


def test_pack_unpack_round_trip_and_nibble_order():
    rng = np.random.default_rng(0)
    c = rng.integers(0, 16, size=(3, 64), dtype=np.uint8)
    p = MX.pack_e2m1(c)
    assert p.shape == (3, 32) and np.array_equal(MX.unpack_e2m1(p), c)
    assert MX.pack_e2m1(np.array([[0x3, 0xC]], dtype=np.uint8))[0, 0] == 0xC3  # low nibble = even index


def test_dequantize_hand_worked_row():
    # 64 elements, two blocks: block 0 scale 2^-1 (e = 126), block 1 scale 2^3 (e = 130)
    codes = np.zeros((1, 64), dtype=np.uint8)
    codes[0, 0], codes[0, 1], codes[0, 31] = 0x7, 0xB, 0x1     # 6, -1.5, 0.5
    codes[0, 32], codes[0, 63] = 0x5, 0xE                      # 3, -4
    w = MX.dequantize_mxfp4(MX.pack_e2m1(codes), np.array([[126, 130]], dtype=np.uint8))
    expect = np.zeros((1, 64))
    expect[0, 0], expect[0, 1], expect[0, 31] = 3.0, -0.75, 0.25
    expect[0, 32], expect[0, 63] = 24.0, -32.0
    assert np.array_equal(w, expect)


# int4 codes whose halves are E2M1 values, and the E2M1 code of each half
_Q = np.array([0, 1, 2, 3, 4, 6, -1, -2, -3, -4, -6])
_E2M1_OF_HALF = {0: 0x0, 1: 0x1, 2: 0x2, 3: 0x3, 4: 0x4, 6: 0x5, -1: 0x9, -2: 0xA, -3: 0xB, -4: 0xC, -6: 0xD}


def _both_formats(rng, rows, K):
    """The same weights as W4 g32 (q * s, s = 2^(e-128) in bf16) and as
    MXFP4 (e2m1(q / 2) * 2^(e-127))."""
    q = rng.choice(_Q, size=(rows, K))
    e = rng.integers(110, 131, size=(rows, K // 32)).astype(np.uint8)
    s_bits = ((e.astype(np.uint32) - 1) << 23 >> 16).astype(np.uint16)  # bf16 of 2^(e - 128)
    w4 = (W4.pack_int4(q), s_bits)
    codes = np.vectorize(_E2M1_OF_HALF.get)(q).astype(np.uint8)
    mx = (MX.pack_e2m1(codes), e)
    return w4, mx


def test_layer_equals_the_w4_oracle_on_shared_weights():
    rng = np.random.default_rng(1)
    E, H, I, k, T = 16, 128, 64, 4, 5
    layer4, layermx = {}, {}
    for name, (rows, K) in (("gate", (I, H)), ("up", (I, H)), ("down", (H, I))):
        q4, s4, qm, sm = [], [], [], []
        for _ in range(E):
            (a, b), (c, d) = _both_formats(rng, rows, K)
            q4.append(a); s4.append(b); qm.append(c); sm.append(d)
        layer4[f"{name}_q"], layer4[f"{name}_s"] = np.stack(q4), np.stack(s4)
        layermx[f"{name}_q"], layermx[f"{name}_s"] = np.stack(qm), np.stack(sm)
    assert np.array_equal(W4.dequantize(layer4["gate_q"][3], layer4["gate_s"][3]),
                          MX.dequantize_mxfp4(layermx["gate_q"][3], layermx["gate_s"][3]))
    bf = lambda a: W4.f32_to_bf16_bits(np.asarray(a, dtype=np.float32))
    shared = {"router_w": bf(rng.standard_normal((E, H)) * 0.02), "router_bias": None,
              "sh_gate": bf(rng.standard_normal((I, H)) * 0.02), "sh_up": bf(rng.standard_normal((I, H)) * 0.02),
              "sh_down": bf(rng.standard_normal((H, I)) * 0.02)}
    layer4.update(shared)
    layermx.update(shared)
    x = bf(rng.standard_normal((T, H)))
    a = W4.moe_layer(x, layer4, k)
    b = MX.moe_layer_mxfp4(x, layermx, k)
    assert np.array_equal(a["idx"], b["idx"]) and np.array_equal(a["out"], b["out"])
