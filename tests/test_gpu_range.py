"""Tokens of extreme magnitude against the fp64 oracle (needs a B200).

The token kinds (workloads.EXTREME_KINDS) cover the input format's range:
|x| far beyond fp16's 65504, |x| up to bf16's largest finite value (outputs
and, for "all_max", router logits beyond fp32's range), tokens made of bf16
subnormals, tiny tokens whose outputs sit near bf16's smallest values, and
tokens mixing subnormal, ordinary and huge values.  They run through the
decode kernel (T = 1, 4 and 8), the token-grouped path (T = 37 on the
32-expert layer, which splits its experts between the GEMV kernels and the
tensor-core tiles; T = 20 on the full layer) and both MXFP4 paths,
with and without a router bias, and are compared with the bar of
tests.parity.compare_range.
"""
import numpy as np
import pytest
import torch

import oracle
import oracle.mxfp4_ref as MX
import workloads
import weight_only_int4_fp32_b200 as lm
from tests.parity import bits, compare_range

pytestmark = pytest.mark.gpu

DEV = "cuda"
KINDS = list(workloads.EXTREME_KINDS)
T4_GROUPS = [("normal", "big", "tiny", "mixed"),
             ("near_max", "subnormal", "fp16_edge", "all_max"),
             ("tiny_huge", "zeros", "big", "normal")]


def _cuda(tensors: dict) -> dict:
    return {k: (None if v is None else v.to(DEV).contiguous()) for k, v in tensors.items()}


def _oracle(x, host, dequant=None):
    with np.errstate(over="ignore", invalid="ignore", under="ignore"):
        return oracle.moe_layer(bits(x), host, 8, dequant=dequant)


def _run(layer, x):
    out, idx, w = layer.forward(x.to(DEV).contiguous(), return_routing=True)
    torch.cuda.synchronize()
    assert layer.status() == lm.LING_MOE_OK
    return out, idx, w


@pytest.fixture(scope="module")
def reduced_layers():
    """The 32-expert layer without and with a Zipf(1.1) router bias."""
    lw = workloads.layer_weights(32, seed=0, device="cpu")
    host = lw.host_arrays()
    bias = workloads.zipf_router_bias(32, 1.1, seed=0)
    wb = dict(lw.tensors())
    wb["router_bias"] = bias
    host_b = dict(host)
    host_b["router_bias"] = bias.numpy()
    layers = {False: (host, lm.MoELayer(_cuda(lw.tensors()), top_k=8, max_tokens=64)),
              True: (host_b, lm.MoELayer(_cuda(wb), top_k=8, max_tokens=64))}
    yield layers
    for _, layer in layers.values():
        layer.close()


@pytest.mark.parametrize("bias", [False, True])
@pytest.mark.parametrize("kind", KINDS)
def test_decode_t1_token_of_each_kind(reduced_layers, kind, bias):
    host, layer = reduced_layers[bias]
    x = workloads.extreme_tokens([kind], seed=700 + KINDS.index(kind))
    out, idx, w = _run(layer, x)
    rep = compare_range(_oracle(x, host), out, idx, w, 8, f"decode T=1 {kind} bias={bias}")
    if kind in ("near_max", "all_max"):
        assert rep["inf"] == x.shape[0] * 2560  # every output overflows bf16, with the oracle's sign
    if kind in ("subnormal", "zeros"):
        assert torch.count_nonzero(out) == 0


@pytest.mark.parametrize("bias", [False, True])
@pytest.mark.parametrize("group", range(len(T4_GROUPS)))
def test_decode_t4_mixed_kinds(reduced_layers, group, bias):
    host, layer = reduced_layers[bias]
    x = workloads.extreme_tokens(T4_GROUPS[group], seed=800 + 10 * group)
    out, idx, w = _run(layer, x)
    compare_range(_oracle(x, host), out, idx, w, 8, f"decode T=4 {T4_GROUPS[group]} bias={bias}")


@pytest.mark.parametrize("bias", [False, True])
def test_decode_t8_mixed_kinds(reduced_layers, bias):
    host, layer = reduced_layers[bias]
    x = workloads.extreme_tokens(T4_GROUPS[0] + T4_GROUPS[1], seed=850)
    out, idx, w = _run(layer, x)
    compare_range(_oracle(x, host), out, idx, w, 8, f"decode T=8 bias={bias}")


@pytest.mark.parametrize("bias", [False, True])
def test_grouped_t37_every_kind(reduced_layers, bias):
    host, layer = reduced_layers[bias]
    kinds = [KINDS[i % len(KINDS)] for i in range(37)]
    x = workloads.extreme_tokens(kinds, seed=900)
    out, idx, w = _run(layer, x)
    counts = np.bincount(idx.cpu().numpy().reshape(-1), minlength=32)
    assert (counts > 8).any() and ((counts > 0) & (counts <= 8)).any()  # tiles and GEMV both run
    rep = compare_range(_oracle(x, host), out, idx, w, 8, f"grouped T=37 bias={bias}")
    print("grouped T=37", rep)


def test_full_layer_extreme_tokens():
    lw = workloads.layer_weights(512, seed=0, device=DEV)
    host = lw.host_arrays()
    layer = lm.MoELayer(lw.tensors(), top_k=8, max_tokens=64)
    del lw
    torch.cuda.empty_cache()
    try:
        for kind in ("big", "all_max", "tiny", "mixed", "tiny_huge"):
            x = workloads.extreme_tokens([kind], seed=1100 + KINDS.index(kind))
            out, idx, w = _run(layer, x)
            compare_range(_oracle(x, host), out, idx, w, 8, f"full T=1 {kind}")
        x = workloads.extreme_tokens(T4_GROUPS[1], seed=1200)
        out, idx, w = _run(layer, x)
        compare_range(_oracle(x, host), out, idx, w, 8, "full T=4")
        kinds = [KINDS[i % len(KINDS)] for i in range(20)]
        x = workloads.extreme_tokens(kinds, seed=1300)
        out, idx, w = _run(layer, x)
        compare_range(_oracle(x, host), out, idx, w, 8, "full grouped T=20")
    finally:
        layer.close()


@pytest.mark.parametrize("group", range(len(T4_GROUPS)))
def test_mxfp4_decode_mixed_kinds(group):
    _mxfp4_case(T4_GROUPS[group], 1400 + 10 * group, f"mxfp4 T=4 {T4_GROUPS[group]}")


def test_mxfp4_grouped_t37_every_kind():
    _mxfp4_case([KINDS[i % len(KINDS)] for i in range(37)], 1500, "mxfp4 grouped T=37")


def _mxfp4_case(kinds, seed, label):
    lw = workloads.layer_weights_mxfp4(32, seed=3, device="cpu")
    host = lw.host_arrays()
    layer = lm.MoELayer(_cuda(lw.tensors()), top_k=8, max_tokens=64, fmt="mxfp4")
    try:
        x = workloads.extreme_tokens(kinds, seed=seed)
        out, idx, w = _run(layer, x)
        with np.errstate(over="ignore", invalid="ignore", under="ignore"):
            ref = MX.moe_layer_mxfp4(bits(x), host, 8)
        compare_range(ref, out, idx, w, 8, label)
    finally:
        layer.close()
