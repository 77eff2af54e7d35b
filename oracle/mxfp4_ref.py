"""fp64 CPU oracle of the MoE layer with MXFP4 routed-expert weights.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the
benchmark's CPU-baseline arm may import this module.  The GPU library never
imports it, and it imports nothing from the GPU library.

What the pages say: bpdata article "Harom optimalizacio a Ling-3.0-flash MoE
inferenciajanak", sections "Modell es kiindulo konfiguracio" and
"Optimalizacio 1: Humming MXFP4 MoE backend": the profiled checkpoint
(Ling-3.0-flash-fp4) keeps its routed experts in MXFP4 and runs them through
MXFP4 MoE kernels (FlashInfer's, then Humming's).  The pages name the format
but do not define it; this oracle takes the OCP Microscaling (MX) definition
of MXFP4:
  * elements: FP4 E2M1 -- bit 3 sign, bits 2..1 exponent E (bias 1), bit 0
    mantissa M; E = 0 is subnormal, M * 0.5; otherwise (1 + M / 2) * 2^(E-1).
    The 16 codes are +-{0, 0.5, 1, 1.5, 2, 3, 4, 6}; no infinity or NaN.
  * one shared scale per block of 32 consecutive elements: E8M0, an unsigned
    biased exponent, scale = 2^(e - 127), with e = 255 NaN.
  * element value = E2M1 value * block scale.
Readings where the definition leaves the layout open (the same as the W4
layer's boundary): two codes per byte, the low nibble holds the even index
along K, bytes along K, rows row-major [rows, K/2]; one scale byte per 32
elements along K, [rows, K/32].  Everything else in the layer (router,
top-k, renormalisation, SwiGLU, shared expert) is the W4 oracle's.
"""
from __future__ import annotations

import numpy as np

from . import moe_ref

__all__ = ["e2m1_decode", "ue8m0_decode", "unpack_e2m1", "pack_e2m1", "dequantize_mxfp4", "moe_layer_mxfp4"]


def e2m1_decode(codes) -> np.ndarray:
    """4-bit E2M1 codes (0..15) -> exact float64."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64) & 0xF
    sign = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    m = c & 0x1
    mag = np.where(e == 0, m * 0.5, (1.0 + m / 2.0) * np.exp2(e.astype(np.float64) - 1.0))
    return sign * mag


def ue8m0_decode(e) -> np.ndarray:
    """E8M0 scale bytes -> 2^(e - 127) as float64 (255 -> NaN)."""
    b = np.asarray(e, dtype=np.uint8).astype(np.float64)
    return np.where(b == 255, np.nan, np.exp2(b - 127.0))


def unpack_e2m1(packed) -> np.ndarray:
    """[..., K/2] bytes -> [..., K] codes; the low nibble is the even index."""
    b = np.asarray(packed, dtype=np.uint8)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = b & 0xF
    out[..., 1::2] = b >> 4
    return out


def pack_e2m1(codes) -> np.ndarray:
    """[..., K] codes (0..15) -> [..., K/2] bytes (inverse of unpack_e2m1)."""
    c = np.asarray(codes, dtype=np.uint8) & 0xF
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def dequantize_mxfp4(packed, scale_bytes) -> np.ndarray:
    """W[n, k] = e2m1(q[n, k]) * 2^(e[n, k // 32] - 127) in float64 (exact)."""
    v = e2m1_decode(unpack_e2m1(packed))
    s = ue8m0_decode(scale_bytes)
    K, ng = v.shape[-1], s.shape[-1]
    if K % ng:
        raise ValueError("K must be a multiple of the number of blocks")
    return v * np.repeat(s, K // ng, axis=-1)


def moe_layer_mxfp4(x_bits, weights: dict, top_k: int) -> dict:
    """The MoE layer with MXFP4 routed experts: the keys of the W4 layer, with
    gate_q / up_q / down_q holding packed E2M1 codes and gate_s / up_s /
    down_s holding E8M0 scale bytes (uint8)."""
    return moe_ref.moe_layer(x_bits, weights, top_k, dequant=dequantize_mxfp4)
