"""The MoE layer with MXFP4 routed experts on the GPU (the decode path,
T <= 8) against the fp64 MXFP4 oracle, with the bar of tests/parity.py
(needs a B200)."""
import numpy as np
import pytest
import torch

import oracle
import oracle.mxfp4_ref as MX
import workloads
import weight_only_int4_fp32_b200 as lm
from tests.parity import bits, compare

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _calls(layer, xs, T):
    outs, idxs, ws = [], [], []
    for i in range(0, xs.shape[0], T):
        o, ix, w = layer.forward(xs[i:i + T].contiguous(), return_routing=True)
        outs.append(o)
        idxs.append(ix)
        ws.append(w)
    torch.cuda.synchronize()
    assert layer.status() == lm.LING_MOE_OK
    return torch.cat(outs), torch.cat(idxs), torch.cat(ws)


@pytest.mark.parametrize("T", [1, 2, 3, 4, 5, 8, 9, 17, 37, 200])
def test_mxfp4_reduced_layer_matches_the_oracle(T):
    """Decode path up to 8 tokens, the token-grouped path above (at T = 200
    the 32 experts hold ~50 tokens each: tensor-core tiles; at 9..37 both the
    GEMV kernels and the tiles run)."""
    lw = workloads.layer_weights_mxfp4(32, seed=3, device="cpu")
    host = lw.host_arrays()
    layer = lm.MoELayer({k: (None if v is None else v.to(DEV)) for k, v in lw.tensors().items()},
                        top_k=8, max_tokens=max(T, 8), fmt="mxfp4")
    try:
        assert "MXFP4" in layer.describe()
        xs = workloads.token_stream(range(300, 300 + (4 if T <= 8 else 1) * T))
        out, idx, w = _calls(layer, xs.to(DEV), T)
        compare(MX.moe_layer_mxfp4(bits(xs), host, 8), out, idx, w, 8, f"mxfp4 reduced T={T}")
    finally:
        layer.close()


def test_mxfp4_full_layer_matches_the_oracle_and_the_launch_count():
    lw = workloads.layer_weights_mxfp4(512, seed=0, device=DEV)
    host = lw.host_arrays()
    layer = lm.MoELayer(lw.tensors(), top_k=8, max_tokens=8, fmt="mxfp4")
    del lw
    torch.cuda.empty_cache()
    try:
        for T, seeds in ((1, range(1, 9)), (4, range(10000, 10008)), (8, range(20000, 20008))):
            xs = workloads.token_stream(seeds)
            n0 = layer.launch_count()
            out, idx, w = _calls(layer, xs.to(DEV), T)
            assert layer.launch_count() - n0 == len(seeds) // T  # one decode launch per call up to 8 tokens
            compare(MX.moe_layer_mxfp4(bits(xs), host, 8), out, idx, w, 8, f"mxfp4 full T={T}")
    finally:
        layer.close()


def test_mxfp4_equals_int4_on_weights_both_formats_hold():
    """The same weights stored both ways (int4 q = 2 v with bf16 scale
    2^(e-128); E2M1 v with E8M0 e) give the same outputs on the two paths,
    within the output bar, and the same routing."""
    rng = np.random.default_rng(7)
    E, H, I = 32, workloads.HIDDEN, workloads.INTER
    q_vals = np.array([0, 1, 2, 3, 4, 6, -1, -2, -3, -4, -6])
    e2m1_of_half = {0: 0x0, 1: 0x1, 2: 0x2, 3: 0x3, 4: 0x4, 6: 0x5, -1: 0x9, -2: 0xA, -3: 0xB, -4: 0xC, -6: 0xD}
    lw = workloads.layer_weights(E, seed=8, device="cpu")
    w4 = dict(lw.tensors())
    wm = dict(lw.tensors())
    for name, (rows, K) in (("gate", (I, H)), ("up", (I, H)), ("down", (H, I))):
        q = rng.choice(q_vals, size=(E, rows, K))
        e = rng.integers(116, 124, size=(E, rows, K // 32)).astype(np.uint8)
        w4[f"{name}_q"] = torch.from_numpy(oracle.pack_int4(q))
        w4[f"{name}_s"] = torch.from_numpy((((e.astype(np.uint32) - 1) << 23) >> 16).astype(np.uint16).view(np.int16)).view(torch.bfloat16)
        codes = np.vectorize(e2m1_of_half.get)(q).astype(np.uint8)
        wm[f"{name}_q"] = torch.from_numpy(MX.pack_e2m1(codes))
        wm[f"{name}_s"] = torch.from_numpy(e)
    to_dev = lambda d: {k: (None if v is None else v.to(DEV).contiguous()) for k, v in d.items()}
    a = lm.MoELayer(to_dev(w4), top_k=8, max_tokens=4)
    b = lm.MoELayer(to_dev(wm), top_k=8, max_tokens=4, fmt="mxfp4")
    try:
        xs = workloads.token_stream(range(500, 508)).to(DEV)
        oa, ia, _ = _calls(a, xs, 4)
        ob, ib, _ = _calls(b, xs, 4)
        assert torch.equal(ia, ib)
        diff = (oa.float() - ob.float()).abs()
        assert bool((diff <= 2e-2 * torch.clamp(oa.float().abs(), min=1.0)).all())
    finally:
        a.close()
        b.close()


def test_mxfp4_prefill_t2048_zipf_every_output():
    """The full MXFP4 layer with the Zipf(1.1) router bias at T = 2048 (the
    prefill workload's shape) against the MXFP4 oracle, every output."""
    lw = workloads.layer_weights_mxfp4(512, seed=0, device=DEV)
    host = lw.host_arrays()
    bias = workloads.zipf_router_bias(512, 1.1, seed=0)
    wb = dict(lw.tensors())
    wb["router_bias"] = bias.to(DEV)
    host["router_bias"] = bias.numpy()
    layer = lm.MoELayer(wb, top_k=8, max_tokens=2048, fmt="mxfp4")
    del lw, wb
    torch.cuda.empty_cache()
    try:
        xs = workloads.tokens(2048, seed=20000)
        n0 = layer.launch_count()
        out, idx, w = _calls(layer, xs.to(DEV), 2048)
        assert layer.launch_count() - n0 == 9  # the token-grouped path
        counts = np.bincount(idx.cpu().numpy().reshape(-1), minlength=512)
        assert counts.max() > 1000 and ((counts > 0) & (counts <= 8)).any()  # tiles and GEMV both run
        rep = compare(MX.moe_layer_mxfp4(bits(xs), host, 8), out, idx, w, 8, "mxfp4 prefill T=2048")
        print("mxfp4 prefill T=2048", rep)
    finally:
        layer.close()
