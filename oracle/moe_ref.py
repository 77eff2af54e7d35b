"""fp64 CPU oracle of the Ling-3.0-flash routed-expert MoE layer (W4 g32).

TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the
benchmark's CPU-baseline arm may import this module.  The GPU library never
imports it, and it imports nothing from the GPU library.

What the layer is, from the pages:
  * vLLM recipe page "inclusionAI/Ling-3.0-flash", section Overview: 512 routed
    experts with 8 active per token plus one shared expert.
  * same page, section "Single-GPU int4": the int4 variant is a pack-quantized
    checkpoint, symmetric W4 with group_size 32, applied to the routed experts
    only; the shared expert (and attention, lm_head) stay in bf16.
  * bpdata article "Három optimalizáció a Ling-3.0-flash MoE inferenciájának",
    section "Modell és kiinduló konfiguráció": every MoE layer routes each
    token to eight of 512 routed experts and also uses one shared expert; the
    hidden size is 2,560 (same article, baseline paragraph); section
    "Optimalizáció 1": moe_intermediate_size = 768.

Readings this oracle takes where the pages are silent (each one is a
convention the library fixes, listed with the rest in the design notes):
  * gate function: fp32-or-better router logits, softmax over all experts,
    keep the top-k under the order (logit descending, index ascending), then
    renormalise the k kept probabilities to sum to 1.  That equals a softmax
    over the k kept logits alone; both ways are computed and checked.
  * optional per-expert router bias is added to the logits before selection.
  * expert FFN: y = W_down (SiLU(W_gate x) * (W_up x)), SiLU(z) = z / (1 + e^-z).
  * the shared expert is added with weight 1.
  * int4 codes: two's-complement nibbles, two per byte, low nibble = even
    index along K, bytes along K, row-major [rows, K/2]; w = q * s with one
    bf16 scale per `group` consecutive K elements of a row, no zero point.
  * no intermediate rounding: everything stays fp64 from the exactly
    converted bf16 / int inputs to the end.

Everything is plain numpy float64.  A matrix product (numpy @) is the only
library primitive used as a step.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "bf16_bits_to_f64", "f32_to_bf16_bits", "unpack_int4", "pack_int4",
    "dequantize", "router_logits", "select_topk", "renormalized_weights",
    "route", "silu", "expert_ffn", "moe_layer", "near_tie",
]


# ---------------------------------------------------------------- formats

def bf16_bits_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact float64.

    A bf16 value is the top 16 bits of an IEEE binary32, so widening the bits
    by 16 zero bits gives the binary32 with the same value, exactly.
    """
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def f32_to_bf16_bits(values) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest, ties to even (finite inputs)."""
    u = np.asarray(values, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return r.astype(np.uint16)


def unpack_int4(packed) -> np.ndarray:
    """Packed bytes [..., K/2] -> int4 codes as int8 [..., K].

    Byte j holds code 2j in its low nibble and code 2j+1 in its high nibble;
    a nibble v in 0..15 encodes the two's-complement value v (v < 8) or
    v - 16 (v >= 8), so codes lie in [-8, 7] (symmetric W4 with the full
    signed range).
    """
    p = np.asarray(packed, dtype=np.uint8)
    lo = (p & 0x0F).astype(np.int16)
    hi = (p >> 4).astype(np.int16)
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.int8)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def pack_int4(q) -> np.ndarray:
    """int4 codes [..., K] in [-8, 7] -> packed bytes [..., K/2] (inverse of unpack_int4)."""
    q = np.asarray(q)
    if q.shape[-1] % 2:
        raise ValueError("K must be even")
    if q.min(initial=0) < -8 or q.max(initial=0) > 7:
        raise ValueError("int4 codes must lie in [-8, 7]")
    v = (q.astype(np.int16) & 0x0F).astype(np.uint8)
    return (v[..., 0::2] | (v[..., 1::2] << 4)).astype(np.uint8)


def dequantize(packed, scale_bits) -> np.ndarray:
    """W[n, k] = q[n, k] * s[n, k // g] in float64 (exact: q is a small int, s a bf16).

    The group size g is K divided by the number of scales per row.
    """
    q = unpack_int4(packed).astype(np.float64)
    s = bf16_bits_to_f64(scale_bits)
    K = q.shape[-1]
    ng = s.shape[-1]
    if K % ng:
        raise ValueError("K must be a multiple of the number of groups")
    g = K // ng
    return q * np.repeat(s, g, axis=-1)


# ---------------------------------------------------------------- routing

def router_logits(x, router_w, bias=None) -> np.ndarray:
    """l[t, e] = sum_h x[t, h] * Wr[e, h] (+ b[e])."""
    l = np.asarray(x, dtype=np.float64) @ np.asarray(router_w, dtype=np.float64).T
    if bias is not None:
        l = l + np.asarray(bias, dtype=np.float64)[None, :]
    return l


def select_topk(logits_row, k: int) -> np.ndarray:
    """Indices of the k largest logits, ordered by (logit desc, index asc)."""
    l = np.asarray(logits_row, dtype=np.float64)
    order = np.lexsort((np.arange(l.shape[0]), -l))
    return order[:k].astype(np.int64)


def renormalized_weights(logits_row, idx) -> np.ndarray:
    """Softmax over all experts, then renormalise over the selected ones.

    Computed both as (full softmax, renormalise) and as a softmax over the
    selected logits alone; the two are the same quantity and must agree.
    """
    l = np.asarray(logits_row, dtype=np.float64)
    m = l.max()
    p = np.exp(l - m)
    p = p / p.sum()
    w_full = p[idx] / p[idx].sum()
    sel = l[idx]
    ms = sel.max()
    e = np.exp(sel - ms)
    w_sel = e / e.sum()
    if not np.allclose(w_full, w_sel, rtol=1e-12, atol=1e-300):
        raise AssertionError("softmax-then-renormalise disagrees with softmax over the kept logits")
    return w_sel


def route(logits, k: int):
    """Per token: top-k indices and their renormalised weights."""
    logits = np.atleast_2d(np.asarray(logits, dtype=np.float64))
    T = logits.shape[0]
    idx = np.zeros((T, k), dtype=np.int64)
    w = np.zeros((T, k), dtype=np.float64)
    for t in range(T):
        idx[t] = select_topk(logits[t], k)
        w[t] = renormalized_weights(logits[t], idx[t])
    return idx, w


def near_tie(logits, k: int, eps: float = 1e-5) -> np.ndarray:
    """True for tokens whose k-th and (k+1)-th largest logits are within eps."""
    logits = np.atleast_2d(np.asarray(logits, dtype=np.float64))
    if logits.shape[1] <= k:
        return np.zeros(logits.shape[0], dtype=bool)
    s = -np.sort(-logits, axis=1)
    return np.abs(s[:, k - 1] - s[:, k]) < eps


# ---------------------------------------------------------------- FFN

def silu(z) -> np.ndarray:
    """SiLU(z) = z * sigmoid(z) = z / (1 + e^-z)."""
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def expert_ffn(xs, w_gate, w_up, w_down) -> np.ndarray:
    """y = W_down (SiLU(W_gate x) * (W_up x)) for each row x of xs.

    w_gate, w_up: [I, H]; w_down: [H, I]; xs: [m, H] -> y: [m, H].
    """
    g = xs @ w_gate.T
    u = xs @ w_up.T
    h = silu(g) * u
    return h @ w_down.T


# ---------------------------------------------------------------- the layer

def moe_layer(x_bits, weights: dict, top_k: int, dequant=None) -> dict:
    """The routed-expert MoE layer for T tokens, in float64.

    x_bits: bf16 bit patterns [T, H].  weights: the canonical boundary layout
    (bf16 tensors as uint16 bit patterns, packed int4 as uint8, the optional
    router bias as float32) with keys router_w, router_bias, gate_q, gate_s,
    up_q, up_s, down_q, down_s, sh_gate, sh_up, sh_down.  dequant(codes,
    scales) turns one expert matrix's packed codes and scales into float64
    weights (default: the W4 g32 `dequantize`; the MXFP4 oracle passes its own).

    Returns out [T, H] (float64, before the final bf16 rounding), idx [T, k],
    w [T, k] and logits [T, E].
    """
    x = bf16_bits_to_f64(np.atleast_2d(x_bits))
    T, H = x.shape
    wr = bf16_bits_to_f64(weights["router_w"])
    bias = weights.get("router_bias")
    logits = router_logits(x, wr, bias)
    idx, w = route(logits, top_k)

    out = np.zeros((T, H), dtype=np.float64)
    deq = dequantize if dequant is None else dequant
    # routed experts: each selected expert applied to the tokens that chose it
    for e in np.unique(idx):
        toks, slots = np.nonzero(idx == e)
        wg = deq(weights["gate_q"][e], weights["gate_s"][e])
        wu = deq(weights["up_q"][e], weights["up_s"][e])
        wd = deq(weights["down_q"][e], weights["down_s"][e])
        y = expert_ffn(x[toks], wg, wu, wd)
        out[toks] += w[toks, slots][:, None] * y
    # the shared expert, bf16 weights, weight 1
    out += expert_ffn(x, bf16_bits_to_f64(weights["sh_gate"]),
                      bf16_bits_to_f64(weights["sh_up"]),
                      bf16_bits_to_f64(weights["sh_down"]))
    return {"out": out, "idx": idx, "w": w, "logits": logits}
