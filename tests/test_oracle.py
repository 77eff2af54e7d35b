"""Pins for the fp64 oracle: each checks it against something other than itself.

Pins used (none retypes the oracle's own formula):
  * literal bit patterns for the bf16 and int4 formats, and torch's bf16
    rounding as an independent library routine;
  * exhaustive byte round trip of the int4 packing;
  * a special case that reduces to a textbook routine (g = K, unit scales:
    the dequantised GEMV is an integer matrix-vector product);
  * brute force on tiny inputs (pure-Python loops for the grouped dequant
    GEMV and for the shared expert; a full Python sort for the top-k);
  * invariants of the routing weights (positive, non-increasing, sum to 1);
  * a dense evaluation of every expert masked by the routing weights, which
    must equal the sparse per-expert path;
  * a hand-built 4-expert layer whose output is written below as a closed
    form (fixture tests/golden/hand_case_e4_h8_i4.json);
  * the magnitude of the output at the full shape.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads

HERE = os.path.dirname(os.path.abspath(__file__))


def sig(z):
    return 1.0 / (1.0 + math.exp(-z))


def silu_cf(z):
    return z * sig(z)


# ------------------------------------------------------------------ formats

def test_bf16_literals():
    bits = np.array([0x3F80, 0xC000, 0x3F00, 0x0000, 0x8000, 0x4049, 0x7F7F, 0x0001, 0x3C23],
                    dtype=np.uint16)
    want = [1.0, -2.0, 0.5, 0.0, -0.0, 3.140625, 3.3895313892515355e38,
            9.183549615799121e-41, 0.0099487304687500]
    got = oracle.bf16_bits_to_f64(bits)
    for g, w in zip(got, want):
        assert g == w
    assert math.copysign(1.0, got[4]) == -1.0


def test_f32_to_bf16_rounding():
    # literal cases, including both kinds of tie
    vals = np.array([1.0, 3.14159265, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.0, 0.02], dtype=np.float32)
    want = [0x3F80, 0x4049, 0x3F80, 0x3F82, 0xC000, 0x3CA4]
    assert list(oracle.f32_to_bf16_bits(vals)) == want
    # against torch's own round-to-nearest-even conversion
    g = torch.Generator().manual_seed(7)
    v = torch.randn(10000, generator=g) * 3.0
    tb = v.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.f32_to_bf16_bits(v.numpy()), tb)


def test_unpack_literals():
    table = {0x00: (0, 0), 0x01: (1, 0), 0x10: (0, 1), 0x0F: (-1, 0), 0xF0: (0, -1),
             0x87: (7, -8), 0x78: (-8, 7), 0xFF: (-1, -1), 0x88: (-8, -8), 0x77: (7, 7),
             0x9A: (-6, -7), 0x25: (5, 2)}
    b = np.array(list(table.keys()), dtype=np.uint8)
    q = oracle.unpack_int4(b[None, :])[0]
    for j, (lo, hi) in enumerate(table.values()):
        assert (q[2 * j], q[2 * j + 1]) == (lo, hi)


def test_pack_unpack_all_bytes():
    b = np.arange(256, dtype=np.uint8).reshape(4, 64)
    q = oracle.unpack_int4(b)
    assert q.min() == -8 and q.max() == 7
    assert np.array_equal(oracle.pack_int4(q), b)
    pairs = set(zip(q.reshape(-1)[0::2].tolist(), q.reshape(-1)[1::2].tolist()))
    assert len(pairs) == 256
    rng = np.random.default_rng(3)
    qq = rng.integers(-8, 8, size=(7, 96))
    assert np.array_equal(oracle.unpack_int4(oracle.pack_int4(qq)), qq)
    with pytest.raises(ValueError):
        oracle.pack_int4(np.array([[8, 0]]))


def test_dequant_gemv_unit_scales_is_integer_matvec():
    rng = np.random.default_rng(11)
    K = 256
    q = rng.integers(-8, 8, size=(40, K))
    s = np.full((40, 1), 0x3F80, dtype=np.uint16)  # g = K, scale 1.0
    W = oracle.dequantize(oracle.pack_int4(q), s)
    xi = rng.integers(-100, 100, size=K)
    assert np.array_equal(W @ xi.astype(np.float64), np.dot(q, xi).astype(np.float64))


def test_dequant_grouped_bruteforce():
    rng = np.random.default_rng(5)
    rows, K, g = 3, 64, 32
    q = rng.integers(-8, 8, size=(rows, K))
    sv = rng.uniform(0.01, 0.03, size=(rows, K // g)).astype(np.float32)
    sb = oracle.f32_to_bf16_bits(sv)
    x = rng.standard_normal(K)
    W = oracle.dequantize(oracle.pack_int4(q), sb)
    got = W @ x
    for n in range(rows):
        acc = 0.0
        for G in range(K // g):
            s = float(torch.from_numpy(sb.view(np.int16)).view(torch.bfloat16)[n, G].double())
            part = 0.0
            for k in range(G * g, G * g + g):
                part += int(q[n, k]) * float(x[k])
            acc += s * part
        assert abs(acc - got[n]) <= 1e-12 * max(1.0, abs(acc))


# ------------------------------------------------------------------ routing

def test_topk_ties_go_to_lower_index():
    l = np.array([0.5, 2.0, 2.0, 1.0, 2.0, 1.0])
    assert list(oracle.select_topk(l, 2)) == [1, 2]
    assert list(oracle.select_topk(l, 4)) == [1, 2, 4, 3]
    assert list(oracle.select_topk(np.zeros(9), 3)) == [0, 1, 2]


def test_topk_matches_full_python_sort():
    rng = np.random.default_rng(1)
    for trial in range(50):
        E = int(rng.integers(8, 600))
        k = int(rng.integers(1, min(8, E) + 1))
        l = np.round(rng.standard_normal(E), 1)  # many exact ties
        want = sorted(range(E), key=lambda e: (-l[e], e))[:k]
        assert list(oracle.select_topk(l, k)) == want


def test_route_weight_invariants():
    rng = np.random.default_rng(2)
    logits = rng.standard_normal((64, 512)) * 3.0
    idx, w = oracle.route(logits, 8)
    assert np.all(w > 0)
    assert np.all(np.abs(w.sum(1) - 1.0) <= 1e-12)
    assert np.all(np.diff(w, axis=1) <= 1e-15)
    for t in range(64):
        assert len(set(idx[t].tolist())) == 8
        # every kept logit is >= every dropped one
        kept = logits[t, idx[t]]
        dropped = np.delete(logits[t], idx[t])
        assert kept.min() >= dropped.max()


def test_route_k1_weight_is_one():
    idx, w = oracle.route(np.array([[0.1, 3.0, -2.0]]), 1)
    assert idx[0, 0] == 1 and w[0, 0] == 1.0


def test_near_tie_flag():
    l = np.array([[3.0, 2.0, 1.0, 1.0 + 5e-6, 0.0], [3.0, 2.0, 1.0, 0.5, 0.0]])
    assert list(oracle.near_tie(l, 3)) == [True, False]


def test_router_bias_enters_before_selection():
    rng = np.random.default_rng(9)
    H, E = 32, 6
    x = rng.standard_normal((1, H))
    wr = rng.standard_normal((E, H)) * 0.02
    b = np.zeros(E)
    b[5] = 50.0
    l = oracle.router_logits(x, wr, b)
    idx, w = oracle.route(l, 2)
    assert idx[0, 0] == 5
    assert w[0, 0] > 1 - 1e-15


# ------------------------------------------------------------------ FFN

def test_silu_values():
    z = np.array([0.0, 1.0, -1.0, 20.0, -800.0, 800.0])
    s = oracle.silu(z)
    assert s[0] == 0.0
    assert abs(s[1] - 0.7310585786300049) < 1e-16
    assert abs(s[2] + 0.2689414213699951) < 1e-16
    assert abs(s[3] - 20.0 * (1 - 2.0611536181902037e-09)) < 1e-12
    assert s[4] == 0.0 and s[5] == 800.0
    assert np.all(np.isfinite(s))


def _hand_case():
    with open(os.path.join(HERE, "golden", "hand_case_e4_h8_i4.json")) as f:
        c = json.load(f)
    E, H, I = c["num_experts"], c["hidden"], c["inter"]
    b = lambda a: oracle.f32_to_bf16_bits(np.array(a, dtype=np.float32))
    w = {
        "router_w": b(c["router_w"]),
        "router_bias": None,
        "gate_q": oracle.pack_int4(np.array(c["gate_q"])),
        "gate_s": b(c["gate_s"]).reshape(E, I, -1),
        "up_q": oracle.pack_int4(np.array(c["up_q"])),
        "up_s": b(c["up_s"]).reshape(E, I, -1),
        "down_q": oracle.pack_int4(np.array(c["down_q"])),
        "down_s": b(c["down_s"]).reshape(E, H, -1),
        "sh_gate": b(c["sh_gate"]), "sh_up": b(c["sh_up"]), "sh_down": b(c["sh_down"]),
    }
    return c, w, b([c["x"]])


def test_hand_case_closed_form():
    c, w, x = _hand_case()
    r = oracle.moe_layer(x, w, c["top_k"])
    # routing: logits 2, 1, 1, 0 -> experts 0 and 1 (1 beats 2 on the tie)
    assert list(r["logits"][0]) == [2.0, 1.0, 1.0, 0.0]
    assert list(r["idx"][0]) == [0, 1]
    w0, w1 = sig(1.0), sig(-1.0)
    assert abs(r["w"][0, 0] - w0) < 1e-15 and abs(r["w"][0, 1] - w1) < 1e-15
    # expert 0: gate = 0.5*[1, -1, 3, 0], up = [2, 1, 2, -1]
    h = [2 * silu_cf(0.5), 1 * silu_cf(-0.5), 2 * silu_cf(1.5), 0.0]
    y0 = [0.25 * v for v in (h[0], h[1], h[2], h[3], h[0] + h[1], -h[2], 7 * h[0] - 8 * h[3], 0.0)]
    # expert 1: gate = [1, 0, -1, 0], up = 2*[1, 0, 0, 1] -> h = [2 silu(1), 0, 0, 0]
    y1 = [2 * silu_cf(1.0)] * 8
    # shared: gate = [0.5, 0, 0, 0], up = [1, 0, 0, 0], down column 0 = [1, -1, .5, 0, 0, 0, 0, 2]
    hs = silu_cf(0.5)
    S = [hs * v for v in (1, -1, 0.5, 0, 0, 0, 0, 2)]
    want = [w0 * a + w1 * b_ + s for a, b_, s in zip(y0, y1, S)]
    got = r["out"][0]
    for g, wv in zip(got, want):
        assert abs(g - wv) <= 1e-13, (got, want)


def test_hand_case_catches_planted_mistakes(monkeypatch):
    """A plausible mistake planted in the oracle must change the hand-case output."""
    c, w, x = _hand_case()
    base = oracle.moe_layer(x, w, c["top_k"])["out"]
    # 1) nibble order swapped
    orig = oracle.moe_ref.unpack_int4

    def swapped(p):
        q = orig(p)
        q2 = q.copy()
        q2[..., 0::2], q2[..., 1::2] = q[..., 1::2], q[..., 0::2]
        return q2
    monkeypatch.setattr(oracle.moe_ref, "unpack_int4", swapped)
    assert not np.allclose(oracle.moe_layer(x, w, c["top_k"])["out"], base)
    monkeypatch.setattr(oracle.moe_ref, "unpack_int4", orig)
    # 2) tie broken toward the higher index
    orig_sel = oracle.moe_ref.select_topk
    monkeypatch.setattr(oracle.moe_ref, "select_topk",
                        lambda l, k: np.lexsort((-np.arange(len(l)), -np.asarray(l)))[:k])
    assert not np.allclose(oracle.moe_layer(x, w, c["top_k"])["out"], base)
    monkeypatch.setattr(oracle.moe_ref, "select_topk", orig_sel)
    # 3) gate and up exchanged inside the FFN
    orig_ffn = oracle.moe_ref.expert_ffn
    monkeypatch.setattr(oracle.moe_ref, "expert_ffn",
                        lambda xs, g, u, d: orig_ffn(xs, u, g, d))
    assert not np.allclose(oracle.moe_layer(x, w, c["top_k"])["out"], base)


def test_sparse_equals_dense_masked():
    """Evaluate every expert densely, mask with the routing weights, compare."""
    E, H, I, k, T = 16, 64, 32, 4, 6
    lw = workloads.layer_weights(E, H, I, seed=3)
    w = lw.host_arrays()
    x = workloads.tokens(T, H, seed=4).view(torch.int16).numpy().view(np.uint16)
    r = oracle.moe_layer(x, w, k)
    xf = oracle.bf16_bits_to_f64(x)
    # independent dense path: full stacks, einsum over all experts
    Wg = np.stack([oracle.dequantize(w["gate_q"][e], w["gate_s"][e]) for e in range(E)])
    Wu = np.stack([oracle.dequantize(w["up_q"][e], w["up_s"][e]) for e in range(E)])
    Wd = np.stack([oracle.dequantize(w["down_q"][e], w["down_s"][e]) for e in range(E)])
    G = np.einsum("eih,th->tei", Wg, xf)
    U = np.einsum("eih,th->tei", Wu, xf)
    Hh = G / (1 + np.exp(-G)) * U
    Y = np.einsum("ehi,tei->teh", Wd, Hh)
    logits = xf @ oracle.bf16_bits_to_f64(w["router_w"]).T
    mask = np.zeros((T, E))
    for t in range(T):
        keep = sorted(range(E), key=lambda e: (-logits[t, e], e))[:k]
        p = np.exp(logits[t] - logits[t].max())
        p /= p.sum()
        mask[t, keep] = p[keep] / p[keep].sum()
    sg = oracle.bf16_bits_to_f64(w["sh_gate"]) @ xf.T
    su = oracle.bf16_bits_to_f64(w["sh_up"]) @ xf.T
    S = (oracle.bf16_bits_to_f64(w["sh_down"]) @ (sg / (1 + np.exp(-sg)) * su)).T
    dense = np.einsum("te,teh->th", mask, Y) + S
    assert np.allclose(r["out"], dense, rtol=1e-12, atol=1e-12)


def test_shared_expert_bruteforce_when_routed_scales_are_zero():
    E, H, I, k = 4, 16, 8, 2
    lw = workloads.layer_weights(E, H, I, seed=8, group=8)
    w = lw.host_arrays()
    for key in ("gate_s", "up_s", "down_s"):
        w[key] = np.zeros_like(w[key])
    x = workloads.tokens(1, H, seed=9).view(torch.int16).numpy().view(np.uint16)
    got = oracle.moe_layer(x, w, k)["out"][0]
    bf = lambda bits: float(np.array([int(bits) << 16], dtype=np.uint32).view(np.float32)[0])
    xv = [bf(v) for v in x[0]]
    hs = []
    for i in range(I):
        g = sum(bf(w["sh_gate"][i, h]) * xv[h] for h in range(H))
        u = sum(bf(w["sh_up"][i, h]) * xv[h] for h in range(H))
        hs.append(g / (1 + math.exp(-g)) * u)
    for n in range(H):
        want = sum(bf(w["sh_down"][n, i]) * hs[i] for i in range(I))
        assert abs(got[n] - want) <= 1e-13 * max(1.0, abs(want))


def test_tokens_grouped_per_expert_equal_one_by_one():
    E, H, I, k, T = 8, 64, 32, 3, 7
    lw = workloads.layer_weights(E, H, I, seed=12)
    w = lw.host_arrays()
    x = workloads.tokens(T, H, seed=13).view(torch.int16).numpy().view(np.uint16)
    r = oracle.moe_layer(x, w, k)
    for t in range(T):
        rt = oracle.moe_layer(x[t:t + 1], w, k)
        assert np.array_equal(rt["idx"][0], r["idx"][t])
        assert np.allclose(rt["out"][0], r["out"][t], rtol=1e-13, atol=1e-13)


def test_output_magnitude_full_shape():
    """Full-shape layer (32 experts): the output's spread is in the expected range.

    With q uniform on [-8, 7] and s ~ 0.02, a routed weight has rms ~0.093,
    so gate/up values have std ~4.7 and each expert output std ~30; the
    renormalised mix of 8 experts plus a small shared term lands at ~10-40.
    A wrong scale (x32 or /32) or packing error moves it far outside.
    """
    lw = workloads.layer_weights(32, seed=0)
    w = lw.host_arrays()
    x = workloads.tokens(3, seed=0).view(torch.int16).numpy().view(np.uint16)
    out = oracle.moe_layer(x, w, 8)["out"]
    sd = out.std()
    assert 8.0 < sd < 80.0, sd
