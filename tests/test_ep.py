"""Expert parallel on the CPU (gloo): the partition of the experts over the
ranks, the weights each rank's handle takes, and the combine (all-reduce of
fp32 partial sums, one bf16 rounding), against the fp64 oracle.

The per-rank partial sum is computed here by a stand-in built from the
oracle's own steps (router over all experts, top-k, the terms of the selected
experts the rank holds, the shared expert on one rank), fed with exactly the
tensors `local_weights` gives the rank's handle; the GPU kernels behind the
real handle are checked in tests/test_gpu_ep.py.  Multi-GPU runs of the NCCL
all-reduce are not part of this suite (one GPU per run here).
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import workloads  # noqa: E402
from weight_only_int4_fp32_b200.ep import ExpertParallelMoE, expert_range, local_weights  # noqa: E402


def test_expert_range_partitions_every_expert_once():
    for E in (8, 9, 32, 100, 511, 512):
        for world in range(1, 9):
            if world > E:
                continue
            seen = []
            prev_end = 0
            for r in range(world):
                b, n = expert_range(E, world, r)
                assert b == prev_end and n >= 1
                prev_end = b + n
                seen += list(range(b, b + n))
            assert seen == list(range(E))
            sizes = [expert_range(E, world, r)[1] for r in range(world)]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        expert_range(4, 8, 0)
    with pytest.raises(ValueError):
        expert_range(32, 2, 2)


def test_local_weights_slices_experts_and_keeps_the_router():
    lw = workloads.layer_weights(8, seed=1).tensors()
    loc = local_weights(lw, 3, 2, with_shared=False)
    assert loc["router_w"] is lw["router_w"]
    for name in ("gate_q", "gate_s", "up_q", "up_s", "down_q", "down_s"):
        assert torch.equal(loc[name], lw[name][3:5]) and loc[name].is_contiguous()
    assert loc["sh_gate"] is None and loc["sh_up"] is None and loc["sh_down"] is None
    assert local_weights(lw, 0, 8, with_shared=True)["sh_down"] is lw["sh_down"]


class OracleShard:
    """Stand-in for a rank's handle: the fp32 partial sum of the selected
    experts in [begin, begin + count) (indexed in the local tensors as
    e - begin) and, if present, the shared expert, from the oracle's steps."""

    def __init__(self, local: dict, begin: int, count: int):
        self.begin, self.count = begin, count
        self.h = {k: (None if v is None else
                      (v.contiguous().view(torch.int16).numpy().view(np.uint16) if v.dtype == torch.bfloat16
                       else v.numpy())) for k, v in local.items()}

    def forward_partial(self, x, return_routing=False):
        h = self.h
        xb = oracle.bf16_bits_to_f64(x.contiguous().view(torch.int16).numpy().view(np.uint16))
        logits = oracle.router_logits(xb, oracle.bf16_bits_to_f64(h["router_w"]), h.get("router_bias"))
        idx, w = oracle.route(logits, 8)
        out = np.zeros_like(xb)
        for t in range(xb.shape[0]):
            for s in range(idx.shape[1]):
                e = int(idx[t, s])
                if not self.begin <= e < self.begin + self.count:
                    continue
                el = e - self.begin
                y = oracle.expert_ffn(xb[t:t + 1], oracle.dequantize(h["gate_q"][el], h["gate_s"][el]),
                                      oracle.dequantize(h["up_q"][el], h["up_s"][el]),
                                      oracle.dequantize(h["down_q"][el], h["down_s"][el]))
                out[t] += w[t, s] * y[0]
        if h["sh_gate"] is not None:
            out += oracle.expert_ffn(xb, oracle.bf16_bits_to_f64(h["sh_gate"]), oracle.bf16_bits_to_f64(h["sh_up"]),
                                     oracle.bf16_bits_to_f64(h["sh_down"]))
        part = torch.from_numpy(out).float()
        return (part, torch.from_numpy(idx), torch.from_numpy(w)) if return_routing else part


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, bias, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        lw = workloads.layer_weights(32, seed=5).tensors()
        if bias:
            lw["router_bias"] = workloads.zipf_router_bias(32, 1.1, seed=2)
        b, n = expert_range(32, world, rank)
        shard = OracleShard(local_weights(lw, b, n, with_shared=(rank == 0)), b, n)
        layer = ExpertParallelMoE(shard, round_fn=lambda p: p.to(torch.bfloat16))
        x = workloads.token_stream(range(900, 906))
        out, idx, w = layer.forward(x, return_routing=True)
        q.put((rank, out.view(torch.int16).numpy().copy(), idx.numpy().copy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,bias", [(2, False), (3, True)])
def test_partition_and_combine_match_the_oracle(world, bias):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, bias, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict((r, (o, i)) for r, o, i in (q.get(timeout=300) for _ in procs))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    lw = workloads.layer_weights(32, seed=5)
    host = lw.host_arrays()
    if bias:
        host["router_bias"] = workloads.zipf_router_bias(32, 1.1, seed=2).numpy()
    x = workloads.token_stream(range(900, 906))
    ref = oracle.moe_layer(x.view(torch.int16).numpy().view(np.uint16), host, 8)
    outs = [got[r][0] for r in range(world)]
    for r in range(1, world):
        assert np.array_equal(outs[r], outs[0])  # every rank holds the same combined output
        assert np.array_equal(got[r][1], got[0][1])
    assert np.array_equal(got[0][1], ref["idx"])
    g = torch.from_numpy(outs[0]).view(torch.bfloat16).double().numpy()
    # the exact sum rounded through fp32 partials and one bf16 rounding
    assert np.all(np.abs(g - ref["out"]) <= 2.0 ** -7 * np.abs(ref["out"]) + 1e-30)
