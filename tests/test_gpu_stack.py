"""The 40-layer stack (independent full-shape layers, one token per call)
against the fp64 oracle (needs a B200 with room for all 40 layers, ~68 GB).

Every layer is checked on the first 4 tokens of the stack's input recipe and
layers 0, 13, 26 and 39 on the first 16; all 40 handles stay alive together,
as in the benchmark, and layer 0 is run again at the end to show that the
other 39 left it untouched.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import weight_only_int4_fp32_b200 as lm
from tests.parity import bits, compare

pytestmark = pytest.mark.gpu

DEV = "cuda"
TOKENS = 4
TOKENS_FULL = 16
FULL_LAYERS = (0, 13, 26, 39)


def _layer_inputs(layer_index: int) -> torch.Tensor:
    n = TOKENS_FULL if layer_index in FULL_LAYERS else TOKENS
    return torch.stack([workloads.tokens(1, seed=workloads.stack_token_seed(t, layer_index), device=DEV)[0]
                        for t in range(n)])


def _run_t1(layer, xs):
    outs, idxs, ws = [], [], []
    for t in range(xs.shape[0]):
        o, ix, w = layer.forward(xs[t:t + 1].contiguous(), return_routing=True)
        outs.append(o)
        idxs.append(ix)
        ws.append(w)
    torch.cuda.synchronize()
    return torch.cat(outs), torch.cat(idxs), torch.cat(ws)


def test_stack40_every_layer_against_the_oracle():
    wl = workloads.WORKLOADS["stack40_e512_t1"]
    layers = []
    first_out = None
    try:
        for l, seed in enumerate(wl["layer_seeds"]):
            lw = workloads.layer_weights(512, seed=seed, device=DEV)
            layer = lm.MoELayer(lw.tensors(), top_k=8, max_tokens=1)
            layers.append(layer)
            xs = _layer_inputs(l)
            out, idx, w = _run_t1(layer, xs)
            assert layer.status() == lm.LING_MOE_OK
            host = lw.host_arrays()
            del lw
            compare(oracle.moe_layer(bits(xs), host, 8), out, idx, w, 8, f"stack layer {l}")
            del host
            if l == 0:
                first_out = out.clone()
        assert len(layers) == 40
        again, _, _ = _run_t1(layers[0], _layer_inputs(0))
        assert torch.equal(again, first_out)
    finally:
        for layer in layers:
            layer.close()
        torch.cuda.empty_cache()
