"""GPU library vs the fp64 oracle on the same seeded inputs (needs a B200).

Covers the five workloads (reduced 32-expert layer; full layer at T=1, at
T=4, and T=2048 with the Zipf router bias; the 40-layer stack is covered in
test_gpu_stack.py), both kernel paths (decode T<=4, grouped T>4), ragged
token counts, degenerate routing (all logits equal, k=1, k=E), argument
errors, determinism, CUDA-graph replay, the host-buffer entry point and the
bounded device-side wait.
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


def _cuda_weights(lw: workloads.LayerWeights) -> dict:
    return {k: (None if v is None else v.to(DEV).contiguous()) for k, v in lw.tensors().items()}


@pytest.fixture(scope="session")
def reduced():
    lw = workloads.layer_weights(32, seed=0, device="cpu")
    layer = lm.MoELayer(_cuda_weights(lw), top_k=8, max_tokens=64)
    yield lw.host_arrays(), layer
    layer.close()


@pytest.fixture(scope="session")
def full():
    lw = workloads.layer_weights(512, seed=0, device=DEV)
    host = lw.host_arrays()
    layer = lm.MoELayer(lw.tensors(), top_k=8, max_tokens=2048)
    bias = workloads.zipf_router_bias(512, 1.1, seed=0)
    wb = dict(lw.tensors())
    wb["router_bias"] = bias.to(DEV)
    layer_b = lm.MoELayer(wb, top_k=8, max_tokens=2048)
    host_b = dict(host)
    host_b["router_bias"] = bias.numpy()
    del lw, wb
    torch.cuda.empty_cache()
    yield host, layer, host_b, layer_b
    layer.close()
    layer_b.close()


def run_calls(layer, xs, T):
    outs, idxs, ws = [], [], []
    for i in range(0, xs.shape[0], T):
        o, ix, w = layer.forward(xs[i:i + T].contiguous(), return_routing=True)
        outs.append(o)
        idxs.append(ix)
        ws.append(w)
    torch.cuda.synchronize()
    assert layer.status() == lm.LING_MOE_OK
    return torch.cat(outs), torch.cat(idxs), torch.cat(ws)


# ------------------------------------------------------------------ workloads

def test_reduced_e32_t1_100_tokens(reduced):
    host, layer = reduced
    xs = workloads.token_stream(range(100), device="cpu")
    out, idx, w = run_calls(layer, xs.to(DEV), 1)
    ref = oracle.moe_layer(bits(xs), host, 8)
    rep = compare(ref, out, idx, w, 8, "reduced e32 T=1")
    print("reduced", rep)


def test_full_decode_t1(full):
    host, layer, _, _ = full
    xs = workloads.token_stream([1 + t for t in range(40)], device=DEV)
    out, idx, w = run_calls(layer, xs, 1)
    rep = compare(oracle.moe_layer(bits(xs), host, 8), out, idx, w, 8, "full T=1")
    print("decode", rep)


def test_full_verify_t4(full):
    host, layer, _, _ = full
    xs = torch.cat([workloads.tokens(4, seed=10000 + i, device=DEV) for i in range(10)])
    out, idx, w = run_calls(layer, xs, 4)
    rep = compare(oracle.moe_layer(bits(xs), host, 8), out, idx, w, 8, "full T=4")
    print("verify", rep)


def test_full_verify_t8_one_launch(full):
    """8-token verify windows: one decode launch per call, the expert union
    over all 8 tokens (about 60 distinct experts: phase 4 runs in two
    passes), bit-identical when repeated."""
    host, layer, _, _ = full
    xs = torch.cat([workloads.tokens(8, seed=20000 + i, device=DEV) for i in range(6)])
    n0 = layer.launch_count()
    out, idx, w = run_calls(layer, xs, 8)
    assert layer.launch_count() - n0 == 6
    rep = compare(oracle.moe_layer(bits(xs), host, 8), out, idx, w, 8, "full T=8")
    print("verify T=8", rep)
    again, _, _ = run_calls(layer, xs, 8)
    assert torch.equal(again, out)


@pytest.mark.parametrize("T", [2, 3, 5, 6, 7, 8, 9, 17, 37])
def test_full_ragged_token_counts(full, T):
    host, layer, _, _ = full
    xs = workloads.tokens(T, seed=500 + T, device=DEV)
    out, idx, w = layer.forward(xs, return_routing=True)
    torch.cuda.synchronize()
    compare(oracle.moe_layer(bits(xs), host, 8), out, idx, w, 8, f"full T={T}")


def test_prefill_t2048_zipf_every_output(full):
    _, _, host_b, layer_b = full
    T = 2048
    xs = workloads.tokens(T, seed=20000, device=DEV)
    out, idx, w = layer_b.forward(xs, return_routing=True)
    torch.cuda.synchronize()
    assert layer_b.status() == lm.LING_MOE_OK
    # routing of every token against the oracle's logits
    x64 = oracle.bf16_bits_to_f64(bits(xs))
    logits = oracle.router_logits(x64, oracle.bf16_bits_to_f64(host_b["router_w"]), host_b["router_bias"])
    ref_idx, ref_w = oracle.route(logits, 8)
    near = oracle.near_tie(logits, 8)
    gi = idx.cpu().numpy()
    for t in range(T):
        if not near[t]:
            assert set(gi[t].tolist()) == set(ref_idx[t].tolist()), t
    counts = np.bincount(gi.reshape(-1), minlength=512)
    print("prefill tokens per expert: max", counts.max(), "experts used", (counts > 0).sum(),
          "near ties", int(near.sum()))
    assert counts.max() > 1000  # the Zipf tilt makes a few experts very popular
    # every token's output (the oracle groups the 2048 tokens by expert: ~15 s)
    rep = compare(oracle.moe_layer(bits(xs), host_b, 8), out, idx, w, 8, "prefill T=2048")
    print("prefill T=2048", rep)


def test_mixed_gemv_and_tile_experts_t200(full):
    """One call whose experts split between the GEMV kernels (1..8 tokens)
    and the tensor-core tiles (more), every output compared."""
    _, _, host_b, layer_b = full
    T = 200
    xs = workloads.tokens(T, seed=31337, device=DEV)
    out, idx, w = layer_b.forward(xs, return_routing=True)
    torch.cuda.synchronize()
    counts = np.bincount(idx.cpu().numpy().reshape(-1), minlength=512)
    assert (counts > 8).any() and ((counts > 0) & (counts <= 8)).any()
    compare(oracle.moe_layer(bits(xs), host_b, 8), out, idx, w, 8, "mixed T=200")


# ------------------------------------------------------------------ degenerate routing

def _small_layer(E, k, seed, max_tokens=16, zero_router=False):
    lw = workloads.layer_weights(E, seed=seed, device="cpu")
    if zero_router:
        lw.router_w = torch.zeros_like(lw.router_w)
    return lw.host_arrays(), lm.MoELayer(_cuda_weights(lw), top_k=k, max_tokens=max_tokens)


def test_all_logits_equal_picks_lowest_indices():
    host, layer = _small_layer(16, 8, seed=3, zero_router=True)
    # experts 0..7 get exactly T tokens each: T = 8 is the largest expert the
    # GEMV kernels take, T = 9 the smallest tensor-core tile
    for T in (1, 4, 8, 9):
        xs = workloads.tokens(T, seed=40 + T, device="cpu")
        out, idx, w = layer.forward(xs.to(DEV), return_routing=True)
        torch.cuda.synchronize()
        assert (idx.cpu().numpy() == np.arange(8)[None, :]).all()
        assert torch.allclose(w.cpu(), torch.full((T, 8), 1 / 8))
        compare(oracle.moe_layer(bits(xs), host, 8), out, idx, w, 8, f"ties T={T}")
    layer.close()


@pytest.mark.parametrize("E,k", [(8, 1), (8, 8), (9, 8), (32, 3)])
def test_small_expert_counts_and_k(E, k):
    host, layer = _small_layer(E, k, seed=E * 10 + k)
    for T in (1, 3, 4, 6, 16):
        xs = workloads.tokens(T, seed=70 + T, device="cpu")
        out, idx, w = layer.forward(xs.to(DEV), return_routing=True)
        torch.cuda.synchronize()
        compare(oracle.moe_layer(bits(xs), host, k), out, idx, w, k, f"E={E} k={k} T={T}")
    layer.close()


# ------------------------------------------------------------------ API behaviour

def test_zero_tokens_is_a_noop(full):
    _, layer, _, _ = full
    n0 = layer.launch_count()
    x = torch.empty((0, 2560), dtype=torch.bfloat16, device=DEV)
    lm.ling_moe_forward(layer.handle, x.data_ptr() or 16, 0, 32, 0)
    assert layer.launch_count() == n0


def test_invalid_arguments_are_rejected(full):
    _, layer, _, _ = full
    x = workloads.tokens(4, seed=1, device=DEV)
    out = torch.empty_like(x)
    with pytest.raises(lm.LingMoEError) as e:
        lm.ling_moe_forward(layer.handle, x.data_ptr(), 2049, out.data_ptr())
    assert e.value.code == lm.LING_MOE_ERR_INVALID_ARG
    with pytest.raises(lm.LingMoEError):
        lm.ling_moe_forward(layer.handle, x.data_ptr() + 2, 1, out.data_ptr())
    with pytest.raises(lm.LingMoEError):
        lm.ling_moe_forward(layer.handle, x.data_ptr(), 4, x.data_ptr() + 5120)
    with pytest.raises(lm.LingMoEError):
        lm.ling_moe_forward(layer.handle, x.data_ptr(), -1, out.data_ptr())


def test_deterministic(full):
    _, layer, _, _ = full
    for T in (1, 4, 64):
        x = workloads.tokens(T, seed=900 + T, device=DEV)
        a = layer.forward(x).clone()
        b = layer.forward(x)
        torch.cuda.synchronize()
        assert torch.equal(a, b), T


def test_cuda_graph_replay_matches_eager(full):
    _, layer, _, _ = full
    for T in (1, 4, 32):
        x_static = workloads.tokens(T, seed=1, device=DEV)
        out_static = torch.empty_like(x_static)
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            layer.forward(x_static, out_static)  # warm
        torch.cuda.current_stream().wait_stream(s)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            layer.forward(x_static, out_static)
        for seed in (2, 3):
            x_new = workloads.tokens(T, seed=seed, device=DEV)
            x_static.copy_(x_new)
            g.replay()
            eager = layer.forward(x_new)
            torch.cuda.synchronize()
            assert torch.equal(out_static, eager), (T, seed)
        del g


def test_kernel_timing_reports_each_launch(full):
    _, layer, _, _ = full
    layer.set_kernel_timing(True)
    try:
        for T, names in ((1, ["decode"]), (64, ["route", "topk", "plan", "scatter", "gemv_gu", "tc_gu",
                                               "gemv_dn", "tc_dn", "combine"])):
            x = workloads.tokens(T, seed=5, device=DEV)
            timed = layer.forward(x)
            times = layer.kernel_times()
            assert [n for n, _ in times] == names
            assert all(ms > 0 for _, ms in times)
            layer.set_kernel_timing(False)
            plain = layer.forward(x)
            torch.cuda.synchronize()
            assert torch.equal(timed, plain)  # the events change nothing
            layer.set_kernel_timing(True)
    finally:
        layer.set_kernel_timing(False)


def test_forward_host_matches_device(full):
    _, layer, _, _ = full
    for T in (1, 4, 20):
        x = workloads.tokens(T, seed=77 + T, device="cpu").pin_memory()
        out_h = torch.empty_like(x).pin_memory()
        layer.forward_host(x, out_h)
        dev = layer.forward(x.to(DEV))
        torch.cuda.synchronize()
        assert torch.equal(out_h, dev.cpu()), T


def test_bounded_wait_reports_timeout_and_recovers(full):
    host, layer, _, _ = full
    x = workloads.tokens(1, seed=5, device=DEV)
    lm.ling_moe_test_set_wait(layer.handle, 0, 20_000_000)  # CTA 0 never arrives; 20 ms limit
    layer.forward(x)
    assert layer.status() == lm.LING_MOE_ERR_DEVICE_TIMEOUT
    lm.ling_moe_test_set_wait(layer.handle, -1, 0)
    out, idx, w = layer.forward(x, return_routing=True)
    assert layer.status() == lm.LING_MOE_OK
    compare(oracle.moe_layer(bits(x), host, 8), out, idx, w, 8, "after timeout")


def test_describe_and_launch_count(full):
    _, layer, _, _ = full
    d = layer.describe()
    assert "decode path" in d and "grouped path" in d and "E=512" in d
    n0 = layer.launch_count()
    layer.forward(workloads.tokens(1, seed=1, device=DEV))
    assert layer.launch_count() == n0 + 1
    layer.forward(workloads.tokens(8, seed=1, device=DEV))  # up to 8 tokens: one decode launch
    assert layer.launch_count() == n0 + 2
    layer.forward(workloads.tokens(9, seed=1, device=DEV))  # the token-grouped path: 9 kernels
    assert layer.launch_count() == n0 + 11
