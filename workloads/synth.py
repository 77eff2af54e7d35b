"""Seeded synthetic inputs for the Ling-shaped W4 g32 MoE layer.

This module only draws random numbers.  It holds none of the layer's
arithmetic: no nibble unpacking, no dequantisation, no routing, no FFN.
Both the fp64 oracle (through the tests) and the GPU library consume what
it produces, in the canonical boundary layout:

  router_w  bf16  [E, H]        ~ N(0, 0.02)   (0.02 is the standard deviation)
  gate_q    uint8 [E, I, H/2]   two int4 codes per byte; every byte uniform
  gate_s    bf16  [E, I, H/32]  0.02 * U(0.5, 1.5)
  up_q      uint8 [E, I, H/2]
  up_s      bf16  [E, I, H/32]
  down_q    uint8 [E, H, I/2]
  down_s    bf16  [E, H, I/32]
  sh_gate   bf16  [I, H]        ~ N(0, 0.02)
  sh_up     bf16  [I, H]
  sh_down   bf16  [H, I]
  x         bf16  [T, H]        ~ N(0, 1)
  lm head   bf16  [V, H]        ~ N(0, 0.02) * exp(U(-1, 1)) per row, V = 157,184
MXFP4 layers (layer_weights_mxfp4) draw the same tensors in the same order,
with E8M0 scale bytes uint8 [E, rows, K/32] uniform in [119, 123] in place of
the bf16 scales (the code bytes are uniform either way).

A uniform byte carries two independent uniform 4-bit codes, so drawing
bytes uniformly is the same as drawing each int4 code uniformly in
[-8, 7]; no packing step is needed here.

Floating values are drawn in fp32 and rounded to bf16 by torch's
round-to-nearest-even conversion.  Values depend on (seed, device type):
torch's CPU and CUDA generators are different streams, so a test that
compares the GPU library with the oracle draws once and hands the same
bytes to both.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

HIDDEN = 2560          # hidden size of the Ling-3.0-flash MoE layer
INTER = 768            # moe_intermediate_size
NUM_EXPERTS = 512      # routed experts
TOP_K = 8              # experts per token
GROUP = 32             # int4 group size along the input dimension


def _gen(seed: int, device) -> torch.Generator:
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(int(seed))
    return g


def _normal_bf16(shape, std, g, device):
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    return (t * std).to(torch.bfloat16)


def _scale_bf16(shape, g, device):
    t = torch.empty(shape, device=device, dtype=torch.float32)
    t.uniform_(0.5, 1.5, generator=g)
    return (t * 0.02).to(torch.bfloat16)


def _bytes(shape, g, device):
    return torch.randint(0, 256, shape, generator=g, device=device, dtype=torch.uint8)


@dataclass
class LayerWeights:
    router_w: torch.Tensor
    gate_q: torch.Tensor
    gate_s: torch.Tensor
    up_q: torch.Tensor
    up_s: torch.Tensor
    down_q: torch.Tensor
    down_s: torch.Tensor
    sh_gate: torch.Tensor
    sh_up: torch.Tensor
    sh_down: torch.Tensor
    router_bias: torch.Tensor | None = None

    @property
    def num_experts(self) -> int:
        return self.router_w.shape[0]

    @property
    def hidden(self) -> int:
        return self.router_w.shape[1]

    @property
    def inter(self) -> int:
        return self.sh_gate.shape[0]

    def tensors(self) -> dict:
        return {k: getattr(self, k) for k in (
            "router_w", "router_bias", "gate_q", "gate_s", "up_q", "up_s",
            "down_q", "down_s", "sh_gate", "sh_up", "sh_down")}

    def to(self, device) -> "LayerWeights":
        kw = {k: (None if v is None else v.to(device)) for k, v in self.tensors().items()}
        return LayerWeights(**kw)

    def host_arrays(self) -> dict:
        """numpy views for the oracle: bf16 as uint16 bit patterns."""
        out = {}
        for k, v in self.tensors().items():
            if v is None:
                out[k] = None
            elif v.dtype == torch.bfloat16:
                out[k] = v.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")
            else:
                out[k] = v.detach().cpu().contiguous().numpy()
        return out


def layer_weights(num_experts: int = NUM_EXPERTS, hidden: int = HIDDEN,
                  inter: int = INTER, seed: int = 0, device="cpu",
                  group: int = GROUP) -> LayerWeights:
    """One MoE layer's weights in the canonical layout, drawn in a fixed order."""
    E, H, I = num_experts, hidden, inter
    if H % 2 or I % 2 or H % group or I % group:
        raise ValueError("hidden and inter must be multiples of the group size")
    g = _gen(seed, device)
    router_w = _normal_bf16((E, H), 0.02, g, device)
    gate_q = _bytes((E, I, H // 2), g, device)
    gate_s = _scale_bf16((E, I, H // group), g, device)
    up_q = _bytes((E, I, H // 2), g, device)
    up_s = _scale_bf16((E, I, H // group), g, device)
    down_q = _bytes((E, H, I // 2), g, device)
    down_s = _scale_bf16((E, H, I // group), g, device)
    sh_gate = _normal_bf16((I, H), 0.02, g, device)
    sh_up = _normal_bf16((I, H), 0.02, g, device)
    sh_down = _normal_bf16((H, I), 0.02, g, device)
    return LayerWeights(router_w, gate_q, gate_s, up_q, up_s, down_q, down_s,
                        sh_gate, sh_up, sh_down)


def _e8m0_bytes(shape, g, device, lo=119, hi=123):
    """E8M0 scale bytes e uniform in [lo, hi]: scales 2^(e - 127) from 2^-8 to 2^-4."""
    return torch.randint(lo, hi + 1, shape, generator=g, device=device, dtype=torch.uint8)


def layer_weights_mxfp4(num_experts: int = NUM_EXPERTS, hidden: int = HIDDEN,
                        inter: int = INTER, seed: int = 0, device="cpu",
                        group: int = GROUP) -> LayerWeights:
    """One MoE layer with MXFP4 routed experts, drawn in the W4 layer's order:
    the codes are uniform bytes (two independent uniform E2M1 codes per byte,
    all 16 codes valid), the scales E8M0 bytes uniform in [119, 123], so that
    the weights' spread is close to the W4 layer's."""
    E, H, I = num_experts, hidden, inter
    if H % 2 or I % 2 or H % group or I % group:
        raise ValueError("hidden and inter must be multiples of the group size")
    g = _gen(seed, device)
    router_w = _normal_bf16((E, H), 0.02, g, device)
    gate_q = _bytes((E, I, H // 2), g, device)
    gate_s = _e8m0_bytes((E, I, H // group), g, device)
    up_q = _bytes((E, I, H // 2), g, device)
    up_s = _e8m0_bytes((E, I, H // group), g, device)
    down_q = _bytes((E, H, I // 2), g, device)
    down_s = _e8m0_bytes((E, H, I // group), g, device)
    sh_gate = _normal_bf16((I, H), 0.02, g, device)
    sh_up = _normal_bf16((I, H), 0.02, g, device)
    sh_down = _normal_bf16((H, I), 0.02, g, device)
    return LayerWeights(router_w, gate_q, gate_s, up_q, up_s, down_q, down_s,
                        sh_gate, sh_up, sh_down)


def tokens(T: int, hidden: int = HIDDEN, seed: int = 0, device="cpu") -> torch.Tensor:
    """x [T, hidden] bf16 ~ N(0, 1) from one seed."""
    g = _gen(seed, device)
    return torch.randn((T, hidden), generator=g, device=device,
                       dtype=torch.float32).to(torch.bfloat16)


BF16_MAX = 3.3895313892515355e38  # largest finite bf16 (0x7F7F)

# Token kinds of extreme magnitude, for the range tests: name -> what it is.
EXTREME_KINDS = {
    "normal": "N(0, 1)",
    "zeros": "all zero",
    "big": "N(0, 1) * 2^20 (|x| far beyond fp16's 65504)",
    "fp16_edge": "N(0, 1) * 2^15 (|x| around and above fp16's 65504)",
    "near_max": "N(0, 1) * 2^125, clipped to bf16's largest finite value",
    "all_max": "every element +-U(0.5, 1) * bf16's largest finite value",
    "subnormal": "every element a random nonzero bf16 subnormal",
    "tiny": "N(0, 1) * 2^-60",
    "mixed": "N(0, 1) with 64 positions bf16 subnormals, 16 at N(0, 1) * 2^-100 "
             "and 4 at +-U(1, 2) * 2^30",
    "tiny_huge": "every element a bf16 subnormal except 3 at +-U(1, 2) * 2^50",
}


def extreme_token(kind: str, hidden: int = HIDDEN, seed: int = 0) -> torch.Tensor:
    """One token x [hidden] bf16 of the given kind (EXTREME_KINDS), on the CPU."""
    g = _gen(seed, "cpu")
    n = torch.randn(hidden, generator=g, dtype=torch.float64)

    def subnormals(m):
        mant = torch.randint(1, 128, (m,), generator=g, dtype=torch.int32)
        sign = torch.randint(0, 2, (m,), generator=g, dtype=torch.int32) << 15
        return (mant | sign).to(torch.int16).view(torch.bfloat16)

    def positions(m):
        return torch.randperm(hidden, generator=g)[:m]

    def signs(m):
        return torch.randint(0, 2, (m,), generator=g, dtype=torch.float64) * 2 - 1

    if kind == "normal":
        x = n.to(torch.bfloat16)
    elif kind == "zeros":
        x = torch.zeros(hidden, dtype=torch.bfloat16)
    elif kind == "big":
        x = (n * 2.0 ** 20).to(torch.bfloat16)
    elif kind == "fp16_edge":
        x = (n * 2.0 ** 15).to(torch.bfloat16)
    elif kind == "near_max":
        x = (n * 2.0 ** 125).clamp(-BF16_MAX, BF16_MAX).to(torch.bfloat16)
    elif kind == "all_max":
        u = torch.empty(hidden, dtype=torch.float64).uniform_(0.5, 1.0, generator=g)
        x = (signs(hidden) * u * BF16_MAX).clamp(-BF16_MAX, BF16_MAX).to(torch.bfloat16)
    elif kind == "subnormal":
        x = subnormals(hidden)
    elif kind == "tiny":
        x = (n * 2.0 ** -60).to(torch.bfloat16)
    elif kind == "mixed":
        x = n.to(torch.bfloat16)
        p = positions(84)
        x[p[:64]] = subnormals(64)
        x[p[64:80]] = (torch.randn(16, generator=g, dtype=torch.float64) * 2.0 ** -100).to(torch.bfloat16)
        u = torch.empty(4, dtype=torch.float64).uniform_(1.0, 2.0, generator=g)
        x[p[80:]] = (signs(4) * u * 2.0 ** 30).to(torch.bfloat16)
    elif kind == "tiny_huge":
        x = subnormals(hidden)
        p = positions(3)
        u = torch.empty(3, dtype=torch.float64).uniform_(1.0, 2.0, generator=g)
        x[p] = (signs(3) * u * 2.0 ** 50).to(torch.bfloat16)
    else:
        raise ValueError(f"unknown token kind {kind!r}")
    return x


def extreme_tokens(kinds, hidden: int = HIDDEN, seed: int = 0, device="cpu") -> torch.Tensor:
    """Tokens of the given kinds, row i of kinds[i] from seed + i."""
    return torch.stack([extreme_token(k, hidden, seed + i) for i, k in enumerate(kinds)]).to(device)


def token_stream(seeds, hidden: int = HIDDEN, device="cpu") -> torch.Tensor:
    """One token per seed, stacked: row i is tokens(1, seed=seeds[i])."""
    rows = [tokens(1, hidden, s, device) for s in seeds]
    return torch.cat(rows, 0) if rows else torch.empty((0, hidden), dtype=torch.bfloat16, device=device)


def zipf_router_bias(num_experts: int = NUM_EXPERTS, s: float = 1.1, seed: int = 0) -> torch.Tensor:
    """Per-expert additive router bias b_e = -s * ln(r_e), fp32 [E].

    r_e is the 1-based rank of expert e under a seeded random permutation, so
    exp(logit + b_e) is proportional to exp(logit) * r_e^-s: a Zipf(s)
    popularity tilt.  Drawn on the CPU so it is the same on every device.
    """
    g = _gen(seed, "cpu")
    perm = torch.randperm(num_experts, generator=g)
    rank = torch.empty(num_experts, dtype=torch.float64)
    rank[perm] = torch.arange(1, num_experts + 1, dtype=torch.float64)
    return (-s * torch.log(rank)).to(torch.float32)


# The five workloads (names describe what they are, with their sizes).
WORKLOADS = {
    "reduced_e32_t1": dict(num_experts=32, T=1, weight_seed=0, token_seeds=[0],
                           note="reduced layer, 32 routed experts, 1 token, seed 0; "
                                "parity also runs tokens from seeds 0..99"),
    "decode_e512_t1": dict(num_experts=512, T=1, weight_seed=0,
                           token_seeds=[1 + t for t in range(1000)],
                           note="full layer, batch-1 decode, 1000 tokens (seed 1+t), each its own call"),
    "verify_e512_t4": dict(num_experts=512, T=4, weight_seed=0,
                           call_seeds=[10000 + i for i in range(250)],
                           note="full layer, 4-token verify batch, 250 calls (seed 10000+i)"),
    "verify_e512_t8": dict(num_experts=512, T=8, weight_seed=0,
                           call_seeds=[30000 + i for i in range(250)],
                           note="full layer, 8-token verify window, 250 calls (seed 30000+i), one launch each"),
    "stack40_e512_t1": dict(num_experts=512, T=1, layers=40,
                            layer_seeds=[100 + l for l in range(40)], tokens=200,
                            note="40 independent full layers back to back, 200 tokens"),
    "prefill_e512_t2048_zipf": dict(num_experts=512, T=2048, weight_seed=0, token_seed=20000,
                                    zipf_s=1.1,
                                    note="full layer, 2048-token prefill chunk, Zipf(1.1) router bias"),
    "decode_e512_t1_mxfp4": dict(num_experts=512, T=1, weight_seed=0, fmt="mxfp4",
                                 token_seeds=[1 + t for t in range(1000)],
                                 note="full layer with MXFP4 routed experts, batch-1 decode, token t from seed 1+t"),
    "prefill_e512_t2048_zipf_mxfp4": dict(num_experts=512, T=2048, weight_seed=0, token_seed=20000,
                                          zipf_s=1.1, fmt="mxfp4",
                                          note="full layer with MXFP4 routed experts, 2048-token prefill chunk, "
                                               "Zipf(1.1) router bias"),
}


VOCAB = 157_184        # LM-head vocabulary of Ling-3.0-flash


def lm_head_weights(vocab: int = VOCAB, hidden: int = HIDDEN, seed: int = 0, device="cpu") -> torch.Tensor:
    """LM head W [vocab, hidden] bf16: N(0, 0.02) times a per-row factor
    exp(U(-1, 1)), so that the rows' ranges (and their FP8 scales) differ."""
    g = _gen(seed, device)
    w = torch.randn((vocab, hidden), generator=g, device=device, dtype=torch.float32)
    f = torch.empty((vocab, 1), device=device, dtype=torch.float32)
    f.uniform_(-1.0, 1.0, generator=g)
    return (w * (0.02 * torch.exp(f))).to(torch.bfloat16)


LMHEAD_WORKLOADS = {
    "lmhead_fp8_v157184_t1": dict(vocab=VOCAB, T=1, weight_seed=7, token_seed=30000,
                                  note="online-FP8 LM head, 157,184 x 2,560, one token per call"),
    "lmhead_fp8_v157184_t8": dict(vocab=VOCAB, T=8, weight_seed=7, token_seed=40000,
                                  note="online-FP8 LM head, 157,184 x 2,560, 8 tokens per call"),
}


def stack_token_seed(t: int, layer: int) -> int:
    """Seed of the input of token t at layer `layer` in the 40-layer stack."""
    return 1_000_000 + 1000 * t + layer

