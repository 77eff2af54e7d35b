"""Expert-parallel MoE layer: the routed experts partitioned over the GPUs of a
process group (one process per GPU), as the pages' TP4 + EP4 deployment runs
the model with vLLM's --enable-expert-parallel (vLLM recipe page
"inclusionAI/Ling-3.0-flash", section "Launching the Server").

Every rank holds the full router and a contiguous range of the experts
(`expert_range`); one rank also holds the shared expert.  Each rank's handle
(`ling_moe_create_ep`) scores all experts, selects the same top-k with the
same weights as every other rank, and computes in fp32 only the terms of the
selected experts it holds (plus the shared expert where it lives).  The
ranks' partial sums are added by one all-reduce over the process group (NCCL
on GPUs) and the total is rounded once to bf16 (`ling_moe_round_bf16`).

Argument marshalling and the collective only: the layer's arithmetic runs in
the library's kernels.
"""
from __future__ import annotations

ROUTED = ("gate_q", "gate_s", "up_q", "up_s", "down_q", "down_s")
SHARED = ("sh_gate", "sh_up", "sh_down")


def expert_range(num_experts: int, world: int, rank: int) -> tuple[int, int]:
    """(first expert, count) held by `rank` of `world`: contiguous ranges whose
    sizes differ by at most one, rank 0 first; together they cover every
    expert exactly once."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    if num_experts < world:
        raise ValueError(f"{num_experts} experts cannot give each of {world} ranks one")
    b = rank * num_experts // world
    e = (rank + 1) * num_experts // world
    return b, e - b


def local_weights(weights: dict, begin: int, count: int, with_shared: bool) -> dict:
    """The tensors a rank's handle takes: the full router (and bias), the
    routed tensors of experts [begin, begin + count) (contiguous slices along
    the expert dimension) and the shared expert only if `with_shared`."""
    out = {"router_w": weights["router_w"], "router_bias": weights.get("router_bias")}
    for name in ROUTED:
        out[name] = weights[name][begin:begin + count].contiguous()
    for name in SHARED:
        out[name] = weights[name] if with_shared else None
    return out


class ExpertParallelMoE:
    """The layer over a process group.  `partial_layer` computes this rank's
    fp32 partial sum (`forward_partial(x, return_routing=True)`, as
    `MoELayer` does for a handle from `ling_moe_create_ep`); `round_fn` turns
    the all-reduced fp32 total into the bf16 output (default: the library's
    `round_bf16`).  Build the usual GPU form with `create`."""

    def __init__(self, partial_layer, group=None, round_fn=None):
        self.layer = partial_layer
        self.group = group
        if round_fn is None:
            from . import round_bf16 as round_fn
        self.round = round_fn

    @classmethod
    def create(cls, weights: dict, top_k: int = 8, max_tokens: int = 1, fmt: str = "int4", group=None,
               shared_rank: int = 0):
        """Each rank calls this with the full layer's CUDA tensors (or with
        tensors that hold at least its own experts at their global indices);
        it copies only what its handle needs."""
        import torch.distributed as dist
        from . import MoELayer
        rank, world = dist.get_rank(group), dist.get_world_size(group)
        E = weights["router_w"].shape[0]
        begin, count = expert_range(E, world, rank)
        with_shared = rank == shared_rank
        layer = MoELayer(local_weights(weights, begin, count, with_shared), top_k=top_k, max_tokens=max_tokens,
                         fmt=fmt, ep=(begin, count, with_shared))
        return cls(layer, group)

    def forward(self, x, return_routing: bool = False):
        """bf16 [T, hidden] on every rank (x: the same tokens on every rank)."""
        import torch.distributed as dist
        partial, idx, w = self.layer.forward_partial(x, return_routing=True)
        dist.all_reduce(partial, op=dist.ReduceOp.SUM, group=self.group)
        out = self.round(partial)
        return (out, idx, w) if return_routing else out

    __call__ = forward

    def close(self):
        close = getattr(self.layer, "close", None)
        if close:
            close()
