"""The routing entry point that allocates nothing, against the normal path.

ling_moe_route_noalloc keeps its scratch in a static device array instead of
allocating it, for callers that cannot allocate device memory where they
route tokens.  Its routing is checked against the fp64 oracle's routing and
must equal what ling_moe_forward_ex reports for the
same router weights and tokens: the same fp32 accumulation order gives the
same logits, so indices and weights match exactly (well inside the 1e-5
weight tolerance of the other tests).  Two calls in a row on each token count
check that every call leaves the shared scratch ready for the next.
This file is collected last on purpose, and also runs alone in a fresh
process (the first call looks up the scratch address itself).
"""
import pytest
import torch

import workloads
import weight_only_int4_fp32_b200 as lm

pytestmark = pytest.mark.gpu


def _route_noalloc(x, router_w, bias, E, k):
    T = x.shape[0]
    idx = torch.full((T, k), -7, dtype=torch.int32, device=x.device)
    w = torch.full((T, k), -1.0, dtype=torch.float32, device=x.device)
    lm.ling_moe_route_noalloc(x.data_ptr(), T, router_w.data_ptr(), bias.data_ptr() if bias is not None else 0,
                              E, k, idx.data_ptr(), w.data_ptr(), torch.cuda.current_stream().cuda_stream)
    return idx, w


@pytest.mark.parametrize("E,with_bias", [(512, False), (512, True), (32, False)])
def test_route_noalloc_matches_forward_ex(E, with_bias):
    k = 8
    lw = workloads.layer_weights(E, seed=0, device="cuda")
    weights = dict(lw.tensors())
    bias = workloads.zipf_router_bias(E, 1.1).cuda() if with_bias else None
    weights["router_bias"] = bias
    layer = lm.MoELayer(weights, top_k=k, max_tokens=4)
    try:
        for T in (1, 4, 3):
            for call in range(2):  # two calls in a row share the static scratch
                x = workloads.tokens(T, seed=300 + 10 * T + call, device="cuda")
                _, idx_ref, w_ref = layer.forward(x, return_routing=True)
                idx, w = _route_noalloc(x, lw.router_w, bias, E, k)
                torch.cuda.synchronize()
                assert torch.equal(idx, idx_ref), (E, T, call, idx, idx_ref)
                assert torch.allclose(w, w_ref, rtol=0, atol=1e-5), (E, T, call)
    finally:
        layer.close()


@pytest.mark.parametrize("with_bias", [False, True])
def test_route_noalloc_against_the_oracle(with_bias):
    """The selection and weights straight against the fp64 oracle's routing,
    including tokens of extreme magnitude (the power-of-two token scale)."""
    import numpy as np
    import oracle
    from tests.parity import W_TOL, bits
    E, k = 512, 8
    lw = workloads.layer_weights(E, seed=0, device="cuda")
    bias = workloads.zipf_router_bias(E, 1.1) if with_bias else None
    wr64 = oracle.bf16_bits_to_f64(bits(lw.router_w))
    kinds = [["normal"], ["normal", "big", "tiny", "mixed"], ["near_max", "all_max", "subnormal"]]
    for seed, ks in enumerate(kinds):
        x = workloads.extreme_tokens(ks, seed=4000 + 10 * seed).cuda()
        idx, w = _route_noalloc(x, lw.router_w, bias.cuda() if bias is not None else None, E, k)
        torch.cuda.synchronize()
        logits = oracle.router_logits(oracle.bf16_bits_to_f64(bits(x)), wr64,
                                      bias.numpy() if bias is not None else None)
        ref_idx, ref_w = oracle.route(logits, k)
        srt = -np.sort(-logits, axis=1)
        near = np.abs(srt[:, k - 1] - srt[:, k]) <= 1e-5 * np.abs(logits).max(axis=1)
        gi, gw = idx.cpu().numpy(), w.cpu().numpy()
        for t in range(len(ks)):
            if near[t]:
                continue
            assert set(gi[t].tolist()) == set(ref_idx[t].tolist()), (ks[t], gi[t], ref_idx[t])
            ref = dict(zip(ref_idx[t].tolist(), ref_w[t].tolist()))
            for e, wv in zip(gi[t].tolist(), gw[t].tolist()):
                assert abs(wv - ref[e]) <= W_TOL, (ks[t], e, wv, ref[e])


def test_route_noalloc_rejects_sizes_beyond_its_scratch():
    x = torch.zeros((5, 2560), dtype=torch.bfloat16, device="cuda")
    wr = torch.zeros((16, 2560), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((5, 8), dtype=torch.int32, device="cuda")
    w = torch.empty((5, 8), dtype=torch.float32, device="cuda")
    for T, E, k in ((5, 16, 8), (1, 513, 8), (1, 16, 9), (1, 4, 8)):
        with pytest.raises(lm.LingMoEError) as e:
            lm.ling_moe_route_noalloc(x.data_ptr(), T, wr.data_ptr(), 0, E, k, idx.data_ptr(), w.data_ptr(), 0)
        assert e.value.code == lm.LING_MOE_ERR_INVALID_ARG
        assert "route_noalloc" in lm.ling_moe_last_error()


def _reduced_layer(k=8):
    lw = workloads.layer_weights(32, seed=0, device="cuda")
    return lw, lm.MoELayer(lw.tensors(), top_k=k, max_tokens=4)


def test_route_noalloc_wait_runs_out_then_next_call_is_correct():
    """A call whose CTA 5 withholds its logits gives up after the shortened
    wait: -1 indices, 0 weights, and the status call reports the time-out
    once.  The next call routes correctly (its fresh tag ignores the slots
    the cut-short call left behind)."""
    lw, layer = _reduced_layer()
    stream = torch.cuda.current_stream().cuda_stream
    try:
        assert lm.ling_moe_route_noalloc_status(stream) == lm.LING_MOE_OK
        x = workloads.tokens(2, seed=901, device="cuda")
        lm.ling_moe_route_noalloc_test_set_wait(5, 50_000_000)
        idx, w = _route_noalloc(x, lw.router_w, None, 32, 8)
        torch.cuda.synchronize()
        assert (idx == -1).all() and (w == 0).all(), (idx, w)
        assert lm.ling_moe_route_noalloc_status(stream) == lm.LING_MOE_ERR_DEVICE_TIMEOUT
        assert lm.ling_moe_route_noalloc_status(stream) == lm.LING_MOE_OK  # read once, then cleared
        lm.ling_moe_route_noalloc_test_set_wait(-1, 0)
        for T, seed in ((2, 902), (4, 903)):
            x = workloads.tokens(T, seed=seed, device="cuda")
            idx, w = _route_noalloc(x, lw.router_w, None, 32, 8)
            _, idx_ref, w_ref = layer.forward(x, return_routing=True)
            torch.cuda.synchronize()
            assert torch.equal(idx, idx_ref), (T, idx, idx_ref)
            assert torch.allclose(w, w_ref, rtol=0, atol=1e-5), T
        assert lm.ling_moe_route_noalloc_status(stream) == lm.LING_MOE_OK
    finally:
        lm.ling_moe_route_noalloc_test_set_wait(-1, 0)
        layer.close()


def test_route_noalloc_replayed_from_a_cuda_graph():
    """One call outside capture (it looks up the scratch address), one call
    captured into a CUDA graph on a side stream, then two replays with new
    tokens copied into the captured input: each replay's routing equals
    forward_ex on the same tokens."""
    lw, layer = _reduced_layer()
    T, E, k = 3, 32, 8
    try:
        x_static = workloads.tokens(T, seed=910, device="cuda")
        idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
        w = torch.empty((T, k), dtype=torch.float32, device="cuda")
        _route_noalloc(x_static, lw.router_w, None, E, k)
        torch.cuda.synchronize()
        side = torch.cuda.Stream()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            lm.ling_moe_route_noalloc(x_static.data_ptr(), T, lw.router_w.data_ptr(), 0, E, k, idx.data_ptr(),
                                      w.data_ptr(), side.cuda_stream)
        for replay in range(2):
            x = workloads.tokens(T, seed=911 + replay, device="cuda")
            x_static.copy_(x)
            graph.replay()
            torch.cuda.synchronize()
            _, idx_ref, w_ref = layer.forward(x, return_routing=True)
            torch.cuda.synchronize()
            assert torch.equal(idx, idx_ref), (replay, idx, idx_ref)
            assert torch.allclose(w, w_ref, rtol=0, atol=1e-5), replay
        del graph
        assert lm.ling_moe_route_noalloc_status(torch.cuda.current_stream().cuda_stream) == lm.LING_MOE_OK
    finally:
        layer.close()
