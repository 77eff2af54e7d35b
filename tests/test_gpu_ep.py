"""Expert-parallel handles on one B200 (needs a GPU): the ranks of a 2- and
4-way partition are emulated as separate handles on the same device, their
fp32 partial sums added in rank order and rounded once with
ling_moe_round_bf16, and the result compared with the fp64 oracle.  Covers the
decode kernel (T = 1, 4 and 8), the token-grouped path (T = 37 and 200), both
weight formats, a rank that holds none of a token's experts, and the
ExpertParallelMoE class over a one-rank NCCL group.  Multi-GPU runs (the NCCL
all-reduce between devices) are not covered: one GPU per run here.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

import oracle
import oracle.mxfp4_ref as MX
import workloads
import weight_only_int4_fp32_b200 as lm
from weight_only_int4_fp32_b200.ep import ExpertParallelMoE, expert_range, local_weights
from tests.parity import bits, compare

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _cuda(d: dict) -> dict:
    return {k: (None if v is None else v.to(DEV).contiguous()) for k, v in d.items()}


def _ranks(weights: dict, world: int, fmt: str, max_tokens: int):
    E = weights["router_w"].shape[0]
    out = []
    for r in range(world):
        b, n = expert_range(E, world, r)
        out.append(lm.MoELayer(local_weights(weights, b, n, with_shared=(r == 0)), top_k=8, max_tokens=max_tokens,
                               fmt=fmt, ep=(b, n, r == 0)))
    return out


def _combined(ranks, x):
    total, idx0, w0 = None, None, None
    for layer in ranks:
        part, idx, w = layer.forward_partial(x, return_routing=True)
        if idx0 is None:
            idx0, w0 = idx, w
        else:
            assert torch.equal(idx, idx0) and torch.equal(w, w0)  # the same selection on every rank
        total = part.clone() if total is None else total + part
    out = lm.round_bf16(total)
    torch.cuda.synchronize()
    for layer in ranks:
        assert layer.status() == lm.LING_MOE_OK
    return out, idx0, w0


@pytest.fixture(scope="module")
def reduced():
    lw = workloads.layer_weights(32, seed=0, device="cpu")
    bias = workloads.zipf_router_bias(32, 1.1, seed=0)
    t = dict(lw.tensors())
    t["router_bias"] = bias
    host = lw.host_arrays()
    host["router_bias"] = bias.numpy()
    return _cuda(t), host


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("T", [1, 4, 8, 37, 200])
def test_ep_ranks_sum_to_the_layer(reduced, world, T):
    weights, host = reduced
    ranks = _ranks(weights, world, "int4", max_tokens=max(T, 8))
    try:
        assert "expert parallel" in ranks[1].describe()
        x = workloads.token_stream(range(3000 + T, 3000 + 2 * T)).to(DEV)
        out, idx, w = _combined(ranks, x)
        compare(oracle.moe_layer(bits(x), host, 8), out, idx, w, 8, f"ep world={world} T={T}")
    finally:
        for layer in ranks:
            layer.close()


def test_ep_rank_without_selected_experts_and_forward_guards(reduced):
    """A rank none of whose experts a token selects contributes exactly zero
    (no shared expert there); an EP handle refuses the bf16 entry points."""
    weights, host = reduced
    x = workloads.token_stream([3100]).to(DEV)
    full = lm.MoELayer(weights, top_k=8, max_tokens=8)
    try:
        _, idx, _ = full.forward(x, return_routing=True)
        sel = set(idx[0].tolist())
        b = next(s for s in range(0, 32 - 2) if not ({s, s + 1} & sel))  # two experts the token does not use
        layer = lm.MoELayer(local_weights(weights, b, 2, with_shared=False), top_k=8, max_tokens=8, ep=(b, 2, False))
        try:
            part = layer.forward_partial(x)
            torch.cuda.synchronize()
            assert torch.count_nonzero(part) == 0
            with pytest.raises(lm.LingMoEError):
                layer.forward(x)
            with pytest.raises(lm.LingMoEError):
                layer.forward_host(x.cpu())
        finally:
            layer.close()
        # the partial entry point on an ordinary handle is the whole layer in fp32
        part = full.forward_partial(x)
        assert torch.equal(lm.round_bf16(part), full.forward(x))
    finally:
        full.close()


@pytest.mark.parametrize("T", [4, 37])
def test_ep_mxfp4(T):
    lw = workloads.layer_weights_mxfp4(32, seed=3, device="cpu")
    host = lw.host_arrays()
    ranks = _ranks(_cuda(lw.tensors()), 2, "mxfp4", max_tokens=max(T, 8))
    try:
        x = workloads.token_stream(range(3200, 3200 + T)).to(DEV)
        out, idx, w = _combined(ranks, x)
        compare(MX.moe_layer_mxfp4(bits(x), host, 8), out, idx, w, 8, f"ep mxfp4 T={T}")
    finally:
        for layer in ranks:
            layer.close()


def test_ep_full_layer_world4():
    lw = workloads.layer_weights(512, seed=0, device=DEV)
    host = lw.host_arrays()
    weights = lw.tensors()
    ranks = _ranks(weights, 4, "int4", max_tokens=64)
    del lw, weights
    torch.cuda.empty_cache()
    try:
        for T, seeds in ((1, [1]), (4, range(10000, 10004)), (64, range(3300, 3364))):
            x = workloads.token_stream(seeds).to(DEV)
            out, idx, w = _combined(ranks, x)
            compare(oracle.moe_layer(bits(x), host, 8), out, idx, w, 8, f"ep full world=4 T={T}")
    finally:
        for layer in ranks:
            layer.close()


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_expert_parallel_class_over_a_one_rank_nccl_group(reduced):
    import torch.distributed as dist
    weights, host = reduced
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        layer = ExpertParallelMoE.create(weights, top_k=8, max_tokens=16)
        try:
            x = workloads.token_stream(range(3400, 3416)).to(DEV)
            out, idx, w = layer.forward(x, return_routing=True)
            torch.cuda.synchronize()
            compare(oracle.moe_layer(bits(x), host, 8), out, idx, w, 8, "ExpertParallelMoE world=1")
        finally:
            layer.close()
    finally:
        dist.destroy_process_group()
