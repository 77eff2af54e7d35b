"""Benchmark of the W4 g32 MoE layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode_e512_t1|verify_e512_t4|verify_e512_t8|stack40_e512_t1|prefill_e512_t2048_zipf|reduced_e32_t1
                               |lmhead_fp8_v157184_t1|lmhead_fp8_v157184_t8]

A step is one pass of the whole layer (router, top-k, routed gate/up, down,
shared expert, combine) over one batch of synthetic input: one token for the
default batch-1 decode workload, each step a new seeded token.  Inputs and
weights are resident in HBM when the timed region starts; L2 is flushed
(256 MiB write, then a 256 MiB read) before every step, outside the per-step
CUDA events.  The online-FP8 LM-head workloads stream 402 MB per call, over
three times the L2, and are not flushed.
Rank 0 prints one JSON line.  With N > 1 every rank runs its own independent
token stream on its own GPU: replicas, no collective on the data path; time is
the max over ranks.  Started with --gpus N > 1 outside a launcher, bench.py
starts the N ranks itself under torch.distributed.run.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer decode tokens/s and achieved HBM GB/s (W4 g32, 512e top-8, T=1)"
METRIC_MXFP4 = "MoE-layer decode tokens/s and achieved HBM GB/s (MXFP4 e2m1/e8m0, 512e top-8, T=1)"
# every other workload's line carries its own metric, so that no line claims another's
WORKLOAD_METRIC = {
    "decode_e512_t1": METRIC,
    "decode_e512_t1_mxfp4": METRIC_MXFP4,
    "reduced_e32_t1": "reduced MoE-layer decode tokens/s and achieved HBM GB/s (W4 g32, 32e top-8, T=1)",
    "verify_e512_t4": "MoE-layer verify tokens/s and achieved HBM GB/s (W4 g32, 512e top-8, T=4 per call)",
    "verify_e512_t8": "MoE-layer verify tokens/s and achieved HBM GB/s (W4 g32, 512e top-8, T=8 per call)",
    "stack40_e512_t1": "40-layer MoE-stack decode tokens/s and achieved HBM GB/s (W4 g32, 512e top-8, T=1)",
    "prefill_e512_t2048_zipf": "MoE-layer prefill tokens/s (W4 g32, 512e top-8, T=2048 per call, Zipf(1.1) routing)",
    "prefill_e512_t2048_zipf_mxfp4": "MoE-layer prefill tokens/s (MXFP4 e2m1/e8m0, 512e top-8, T=2048 per call, "
                                     "Zipf(1.1) routing)",
}


# The default run (no --workload) also times these, briefly, and attaches a
# compact record of each to the one JSON line under "secondary".
SECONDARY = ("verify_e512_t4", "verify_e512_t8", "decode_e512_t1_mxfp4", "stack40_e512_t1",
             "prefill_e512_t2048_zipf", "prefill_e512_t2048_zipf_mxfp4", "lmhead_fp8_v157184_t1")
_CAPTURE = None  # a list while secondary workloads run: lines are collected, not printed


def emit(line):
    if _CAPTURE is not None:
        _CAPTURE.append(line)
    else:
        print(json.dumps(line), flush=True)


def compact(line):
    """The figures of a workload line that the secondary record keeps."""
    r = line.get("roofline") or {}
    e = line.get("e2e") or {}
    return {"metric": line["metric"], "value": line["value"], "unit": line["unit"],
            "ms_per_step": line["ms_per_step"], "steps": line["steps"], "warmup": line["warmup"],
            "step_us_p10_p50_p90": line.get("step_us_p10_p50_p90"),
            "roofline": {k: r.get(k) for k in ("bound", "kernel", "achieved", "peak", "unit", "frac", "traffic")},
            "e2e": {k: e.get(k) for k in ("value", "unit")} if e else None,
            "config": line.get("config"), "clocks": line.get("clocks")}


def metric_for(workload):
    return WORKLOAD_METRIC.get(workload, f"MoE-layer tokens/s ({workload})")
H, I = 2560, 768
ROUTED_BYTES = 3_317_760        # per expert: int4 codes + bf16 scales
ROUTED_BYTES_MXFP4 = 3_133_440  # per expert: E2M1 codes + E8M0 scale bytes
SHARED_BYTES = 11_796_480       # bf16 shared expert
L2_FLUSH_BYTES = 256 << 20


# DRAM traffic per launch of the dominant kernel, from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum; profiles/ has the summary and
# the command), valid only while the kernel's sources are the ones captured:
# the sources are hashed and the figure is reported as null once they change.
TRAFFIC = {
    "decode_e512_t1": {"bytes": 41_048_320 + 1_280,
                       "sources": ('decode.cu', 'decode.h', 'common.cuh', 'layout.h'),
                       "sha256": "722bfd0b89f3542e928f71abd6a629ed2429a8e24c609c3c311ed185a0bb212a"},
    "verify_e512_t4": {"bytes": 132_140_288 + 2_912_768,
                       "sources": ('decode.cu', 'decode.h', 'common.cuh', 'layout.h'),
                       "sha256": "722bfd0b89f3542e928f71abd6a629ed2429a8e24c609c3c311ed185a0bb212a"},
    # one launch for the 8-token window (the union, ~62 experts, read once)
    "verify_e512_t8": {"bytes": 219_967_232 + 3_237_632,
                       "sources": ('decode.cu', 'decode.h', 'common.cuh', 'layout.h'),
                       "sha256": "722bfd0b89f3542e928f71abd6a629ed2429a8e24c609c3c311ed185a0bb212a"},
    # online-FP8 LM head: lmh_mma_kernel, the only kernel of a call
    "lmhead_fp8_v157184_t1": {"bytes": 403_095_296 + 3_477_504,
                              "sources": ('lmhead.cu', 'lmhead.h', 'common.cuh', 'layout.h'),
                              "sha256": "97b9d0faf1db3059f55fc99a28f7971773752ba535a85e10db5243403a1fbea5"},
    # MXFP4 routed experts (the decode kernel's E2M1 instantiation); the unit
    # layout keeps a bf16 scale per 32, so 8 experts read 3,317,760 B each
    "decode_e512_t1_mxfp4": {"bytes": 41_051_136 + 37_888,
                             "sources": ('decode.cu', 'decode.h', 'common.cuh', 'layout.h'),
                             "sha256": "722bfd0b89f3542e928f71abd6a629ed2429a8e24c609c3c311ed185a0bb212a"},
    # token-grouped: the dominant kernel, tc_grouped_kernel<0> (gate/up tiles)
    "prefill_e512_t2048_zipf": {"bytes": 459_126_272 + 52_561_920,
                                "sources": ('grouped_tc.cu', 'grouped_tc.h', 'common.cuh', 'layout.h'),
                                "sha256": "458c7407873c6c414b9498241e25dd17313a763852a163987dc634a7406c5806"},
}


def kernel_sources_sha(names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "weight_only_int4_fp32_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def traffic_for(workload):
    t = TRAFFIC.get(workload)
    if t is None or kernel_sources_sha(t["sources"]) != t["sha256"]:
        return None
    return t["bytes"]


def router_bytes(E):
    return E * H * 2


def decode_bytes(E, union, fmt="int4"):
    """Algorithmic bytes of one call: distinct routed experts + shared + router."""
    return union * (ROUTED_BYTES_MXFP4 if fmt == "mxfp4" else ROUTED_BYTES) + SHARED_BYTES + router_bytes(E)


def _layer_gen(wl):
    """The workload's weight generator and its oracle."""
    import oracle
    import workloads
    if wl.get("fmt") == "mxfp4":
        import oracle.mxfp4_ref as MX
        return workloads.layer_weights_mxfp4, MX.moe_layer_mxfp4
    return workloads.layer_weights, oracle.moe_layer


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def tensor_peak():
    """Burst bf16 dense TFLOP/s (fp16 inputs run at the same rate)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


class L2Flush:
    """Leaves L2 holding none of the layer's bytes, and no dirty lines.

    A 256 MiB write (over twice the 126 MB L2) evicts everything; the write
    would leave L2 full of dirty lines, whose write-back would then load the
    next timed call, so a 256 MiB read of another buffer follows and leaves
    L2 holding clean, unrelated lines.  Runs outside every timed region."""

    def __init__(self, device):
        import torch
        self.w = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
        self.r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
        self.s = torch.empty((), dtype=torch.float32, device=device)

    def __call__(self, i):
        import torch
        self.w.fill_(float(i))
        torch.sum(self.r, dim=0, out=self.s)


GEMV_MAX_TOKENS = 8  # experts with at most this many tokens take the GEMV kernels, not the tensor-core tiles


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.rows = []
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        while not self._stop.is_set():
            try:
                r = subprocess.run(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                    "--format=csv,noheader,nounits"], capture_output=True, text=True,
                                   timeout=5)
                if r.returncode == 0 and r.stdout.strip():
                    self.rows.append([c.strip() for c in r.stdout.strip().split(",")])
            except Exception:
                pass
            self._stop.wait(0.2)

    def __enter__(self):
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        self._t.join(timeout=10)

    def summary(self):
        sm = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4)
                          if len(r) > 5 + i and r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(self.rows)}


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(x, device=None):
    """Max of a float over all ranks of the process group (x itself without one).

    Every rank must call it, in the same order (it is a collective)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ reference arm (the oracle)

def cpu_oracle_rate(workload: str, seconds: float = 15.0, max_tokens: int = 64):
    """Time the fp64 oracle on a bounded sample of the workload (rank 0 only)."""
    import numpy as np
    import torch
    import oracle
    import workloads
    wl = workloads.WORKLOADS[workload]
    E = wl["num_experts"]
    gen, layer_fn = _layer_gen(wl)
    lw = gen(E, seed=wl.get("weight_seed", 100), device="cpu" if E <= 32 else
             ("cuda" if torch.cuda.is_available() else "cpu"))
    host = lw.host_arrays()
    if workload.startswith("prefill"):
        host["router_bias"] = workloads.zipf_router_bias(E, wl["zipf_s"]).numpy()
    T = min(wl["T"], 8)
    seeds = wl.get("token_seeds") or wl.get("call_seeds") or [1 + t for t in range(1000)]

    def timed(budget):
        n, calls, t0 = 0, 0, time.perf_counter()
        while calls < max_tokens and (time.perf_counter() - t0) < budget:
            x = workloads.tokens(T, seed=seeds[calls % len(seeds)], device="cpu")
            xb = x.view(torch.int16).numpy().view(np.uint16)
            layer_fn(xb, host, 8)
            n += T
            calls += 1
        return n, calls, time.perf_counter() - t0

    from threadpoolctl import threadpool_info, threadpool_limits
    blas = sum(i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas") or 1
    n, calls, dt = timed(seconds * 2 / 3)  # BLAS threads as configured (all cores by default)
    with threadpool_limits(limits=1, user_api="blas"):
        n1, calls1, dt1 = timed(seconds / 3)
    cores = len(os.sched_getaffinity(0))
    return {"value": n / dt, "unit": "tokens/s", "cores": cores, "threads": blas,
            "kind": "oracle",
            "sample": f"{calls} calls of T={T} of {workload} through the fp64 numpy oracle "
                      f"({dt:.1f} s of host time, {blas} BLAS threads)",
            "single_thread": {"value": n1 / dt1, "unit": "tokens/s", "threads": 1,
                              "sample": f"{calls1} calls, {dt1:.1f} s, one BLAS thread"}}


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    steps, warm = args.steps, args.warmup
    import numpy as np
    import torch
    import oracle
    import workloads
    wl = workloads.WORKLOADS[args.workload]
    E = wl["num_experts"]
    gen, layer_fn = _layer_gen(wl)
    lw = gen(E, seed=wl.get("weight_seed", 100), device="cuda" if torch.cuda.is_available() else "cpu")
    host = lw.host_arrays()
    del lw
    T = wl["T"] if wl["T"] <= 8 else 8
    seeds = wl.get("token_seeds") or wl.get("call_seeds") or [1 + t for t in range(1000)]
    def step(i):
        x = workloads.tokens(T, seed=seeds[i % len(seeds)], device="cpu")
        layer_fn(x.view(torch.int16).numpy().view(np.uint16), host, 8)
    for i in range(warm):
        step(i)
    t0 = time.perf_counter()
    for i in range(steps):
        step(warm + i)
    dt = time.perf_counter() - t0
    v = steps * T / dt
    line = {"metric": metric_for(args.workload), "value": v, "unit": "tokens/s",
            "n_gpus": ws, "steps": steps,
            "warmup": warm, "ms_per_step": dt * 1e3 / steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": args.workload, "T": T, "experts": E, "top_k": 8, "hidden": H,
                       "inter": I},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": len(os.sched_getaffinity(0)),
                             "kind": "oracle",
                             "sample": f"{steps} calls of T={T} through the fp64 numpy oracle"},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm

ROTATE_LAYERS = 12       # independent copies a single-layer workload rotates over (L2 not flushed)
ROTATE_SEED_STRIDE = 7919  # copy r > 0 of a layer draws its weights from seed + r times this


def build_layers(workload, device, rotate=1):
    import torch
    import workloads
    import weight_only_int4_fp32_b200 as lm
    wl = workloads.WORKLOADS[workload]
    E = wl["num_experts"]
    T = wl["T"]
    nlayers = wl.get("layers", 1)
    seeds = wl.get("layer_seeds") or [wl["weight_seed"]]
    if nlayers == 1 and rotate > 1:
        # the same workload on `rotate` independent layers: step i runs layer i % rotate
        nlayers = rotate
        seeds = [seeds[0] + r * ROTATE_SEED_STRIDE for r in range(rotate)]
    layers = []
    gen, _ = _layer_gen(wl)
    fmt = wl.get("fmt", "int4")
    for l in range(nlayers):
        lw = gen(E, seed=seeds[l], device=device)
        w = lw.tensors()
        if workload.startswith("prefill"):
            w = dict(w)
            w["router_bias"] = workloads.zipf_router_bias(E, wl["zipf_s"]).to(device)
        layers.append(lm.MoELayer(w, top_k=8, max_tokens=max(T, 1), fmt=fmt))
        del lw, w
        torch.cuda.empty_cache()
    return layers, E, T


def l2_mode(workload, requested):
    """'rotate' (single-layer decode-size workloads: steps rotate over independent
    layers, no flush) or 'flush' (an L2 flush before every step)."""
    if requested != "auto":
        return requested
    import workloads
    wl = workloads.WORKLOADS[workload]
    if wl.get("layers", 1) == 1 and wl["T"] <= 8 and wl["num_experts"] >= 512:
        return "rotate"
    return "flush"


def workloads_fmt(workload):
    import workloads
    return workloads.WORKLOADS[workload].get("fmt", "int4")


REPLICA_SEED_STRIDE = 1_000_003  # rank r > 0 draws its token stream from seeds shifted by r times this


def make_inputs(workload, n, T, device, rank=0):
    """The first n inputs of the workload's token stream; replica rank r > 0 runs its own stream."""
    import torch
    import workloads
    wl = workloads.WORKLOADS[workload]
    off = rank * REPLICA_SEED_STRIDE
    if workload.startswith("decode") or workload.startswith("reduced"):
        seeds = [1 + t for t in range(n)] if workload.startswith("decode") else list(range(n))
        return [workloads.tokens(1, seed=s + off, device=device) for s in seeds]
    if workload.startswith("verify"):
        seeds = wl["call_seeds"]
        return [workloads.tokens(T, seed=seeds[0] + i + off, device=device) for i in range(n)]
    if workload.startswith("stack"):
        return [torch.stack([workloads.tokens(1, seed=workloads.stack_token_seed(t, l) + off, device=device)[0]
                             for l in range(wl["layers"])]) for t in range(n)]
    return [workloads.tokens(T, seed=wl["token_seed"] + i + off, device=device) for i in range(n)]


def run_ours(args):
    import torch
    import torch.distributed as dist
    ws, rank, local = dist_env()
    if ws > 1:
        dist.init_process_group("nccl", init_method="env://", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import weight_only_int4_fp32_b200 as lm
    mode = l2_mode(args.workload, args.l2)
    stack = args.workload.startswith("stack")
    layers, E, T = build_layers(args.workload, dev, rotate=ROTATE_LAYERS if mode == "rotate" else 1)
    if args.tokens:
        # a verify window of fewer tokens on the same layers (verify-cost sweeps)
        if not args.workload.startswith("verify") or not 1 <= args.tokens <= T:
            raise SystemExit(f"--tokens applies to the verify workloads, 1..{T} tokens")
        T = args.tokens
    nsteps, nwarm = args.steps, args.warmup
    inputs = make_inputs(args.workload, nsteps + nwarm, T, dev, rank=rank)
    l2flush = L2Flush(dev)
    flush = l2flush if mode == "flush" else (lambda i: None)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    def one_step(x, i=0):
        if stack:
            for l, layer in enumerate(layers):
                layer.forward(x[l:l + 1], out)
        else:
            layers[i % len(layers)].forward(x, out)

    # union of routed experts per step (bytes the method must read), from the
    # routing; for token-grouped calls also the rows the tensor-core tiles take
    tc_rows = []

    def union_of(x, i=0):
        if stack:
            return [8] * len(layers)
        _, idx, _ = layers[i % len(layers)].forward(x, return_routing=True)
        cnt = torch.bincount(idx.flatten().long(), minlength=E)
        tc_rows.append(int(cnt[cnt > GEMV_MAX_TOKENS].sum()) + T)
        return [int(torch.unique(idx).numel())]

    for i in range(nwarm):
        flush(i)
        one_step(inputs[i], i)
    torch.cuda.synchronize()
    unions = [union_of(inputs[nwarm + i], nwarm + i) for i in range(nsteps)]
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(nsteps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(nsteps)]
    n0 = sum(l.launch_count() for l in layers)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall = time.perf_counter()
    with ClockSampler(local) as clk:
        g0 = torch.cuda.Event(enable_timing=True)
        g1 = torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for i in range(nsteps):
            flush(i)
            starts[i].record(stream)
            one_step(inputs[nwarm + i], nwarm + i)
            ends[i].record(stream)
        g1.record(stream)
        torch.cuda.synchronize()
    t_wall = time.perf_counter() - t_wall
    if ws > 1:
        dist.barrier()
    launches = sum(l.launch_count() for l in layers) - n0
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    kern_ms = max_over_ranks(sum(step_ms), dev)
    status = [l.status() for l in layers]
    if any(s != lm.LING_MOE_OK for s in status):
        raise RuntimeError(f"device status {status}")

    # the same steps as one CUDA graph per step (stack: the 40 layer calls
    # captured once and replayed; inputs copied into the captured buffer
    # before each step's start event)
    graph = None
    if stack:
        xs_static = torch.empty_like(inputs[0])
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            one_step(xs_static)  # warm-up outside the capture
        stream.wait_stream(side)
        torch.cuda.synchronize()
        cg = torch.cuda.CUDAGraph()
        n_cap0 = sum(l.launch_count() for l in layers)
        with torch.cuda.graph(cg):
            one_step(xs_static)
        per_replay = sum(l.launch_count() for l in layers) - n_cap0
        for i in range(nwarm):
            flush(i)
            xs_static.copy_(inputs[i])
            cg.replay()
        torch.cuda.synchronize()
        gs = [torch.cuda.Event(enable_timing=True) for _ in range(nsteps)]
        ge = [torch.cuda.Event(enable_timing=True) for _ in range(nsteps)]
        for i in range(nsteps):
            flush(i)
            xs_static.copy_(inputs[nwarm + i])
            gs[i].record(stream)
            cg.replay()
            ge[i].record(stream)
        torch.cuda.synchronize()
        g_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in zip(gs, ge)), dev)
        del cg
        graph = {"value": ws * nsteps * T / (g_ms * 1e-3), "unit": "tokens/s", "ms_per_step": g_ms / nsteps,
                 "us_per_layer": g_ms / nsteps / len(layers) * 1e3, "gpu_launches": per_replay * nsteps,
                 "note": "the step's layer calls captured once as one CUDA graph and replayed; "
                         "L2 flushed and inputs copied before each step's start event"}

    # warm: the same calls back to back with nothing in between (weights may
    # partly stay in L2 between calls: router and shared expert)
    warm = None
    if not stack:
        nw = min(nsteps, 100)
        for i in range(3):
            one_step(inputs[nwarm + i % nsteps])
        torch.cuda.synchronize()
        w0 = torch.cuda.Event(enable_timing=True)
        w1 = torch.cuda.Event(enable_timing=True)
        w0.record(stream)
        for i in range(nw):
            one_step(inputs[nwarm + i])
        w1.record(stream)
        torch.cuda.synchronize()
        w_ms = max_over_ranks(w0.elapsed_time(w1), dev)
        warm = {"value": ws * nw * T / (w_ms * 1e-3), "unit": "tokens/s", "us_per_layer": w_ms / nw * 1e3,
                "calls": nw, "note": "calls back to back, no L2 flush between them"}

    # per-kernel times of the token-grouped path (a separate pass: the events
    # around each launch are not in the timed steps above)
    ktimes = None
    if T > 8 and not stack:
        layers[0].set_kernel_timing(True)
        per = {}
        for i in range(nsteps):
            flush(i)
            one_step(inputs[nwarm + i])
            for name, ms in layers[0].kernel_times():
                per.setdefault(name, []).append(ms)
        layers[0].set_kernel_timing(False)
        ktimes = {n: sum(v) / len(v) for n, v in per.items()}

    status = [l.status() for l in layers]
    if any(s != lm.LING_MOE_OK for s in status):
        raise RuntimeError(f"device status after the graph / warm / timing runs {status}")

    # end to end through the host-buffer entry point (pinned buffers, copies timed)
    e2e = None
    if not stack:
        xh = [inputs[nwarm + i].cpu().pin_memory() for i in range(nsteps)]
        oh = torch.empty((T, H), dtype=torch.bfloat16).pin_memory()
        for i in range(min(nwarm, 5)):
            layers[i % len(layers)].forward_host(xh[i % nsteps], oh)
        torch.cuda.synchronize()
        if ws > 1:
            dist.barrier()
        te = 0.0
        for i in range(nsteps):
            flush(i)
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            layers[(nwarm + i) % len(layers)].forward_host(xh[i], oh)
            te += time.perf_counter() - t0
        te = max_over_ranks(te, dev)
        e2e = {"value": ws * nsteps * T / te, "unit": "tokens/s",
               "h2d_bytes_per_step": T * H * 2, "d2h_bytes_per_step": T * H * 2,
               "note": "ling_moe_forward_host per step (pinned H2D copy + layer + D2H copy + stream sync), "
                       "host wall clock summed over the calls; " + (
                           "steps rotate over the layers as in the timed steps" if mode == "rotate" else
                           "L2 flushed before each call, outside its clock")}

    # with rotation, the same steps on one layer with an L2 flush before each
    # (instruction and weight bytes both come from HBM), for comparison
    flushed = None
    if mode == "rotate":
        fs = [torch.cuda.Event(enable_timing=True) for _ in range(nsteps)]
        fe = [torch.cuda.Event(enable_timing=True) for _ in range(nsteps)]
        for i in range(nsteps):
            l2flush(i)
            fs[i].record(stream)
            layers[0].forward(inputs[nwarm + i], out)
            fe[i].record(stream)
        torch.cuda.synchronize()
        f_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in zip(fs, fe)), dev)
        flushed = {"value": ws * nsteps * T / (f_ms * 1e-3), "unit": "tokens/s", "us_per_step": f_ms / nsteps * 1e3,
                   "note": "one layer, L2 flushed (256 MiB write + 256 MiB read) before every step, outside its events"}

    fmt = workloads_fmt(args.workload)
    per_call_bytes = [sum(decode_bytes(E, u, fmt) for u in us) for us in unions]
    if args.workload.startswith("prefill"):
        per_call_bytes = [b + 2 * T * H * 2 for b in per_call_bytes]
    avg_bytes = sum(per_call_bytes) / len(per_call_bytes)
    calls_per_step = len(layers) if stack else 1
    avg_launch_ms = kern_ms / nsteps / calls_per_step
    achieved = (avg_bytes / calls_per_step) / (avg_launch_ms * 1e-3) / 1e9
    peak, peak_kind = peaks()
    roofline = {"bound": "hbm", "kernel": "whole layer (one launch per call at T <= 8)", "achieved": achieved,
                "peak": peak, "unit": "GB/s", "frac": achieved / peak, "traffic": traffic_for(args.workload),
                "peak_kind": peak_kind, "bytes_per_launch": avg_bytes / calls_per_step}
    if ktimes is not None and "tc_gu" in ktimes:
        # dominant kernel: the gate/up tiles; algorithmic FLOPs of the rows they take
        tpk, tpk_kind = tensor_peak()
        flops = sum(2.0 * r * H * 2 * I for r in tc_rows) / len(tc_rows)
        ach_t = flops / (ktimes["tc_gu"] * 1e-3) / 1e12
        roofline = {"bound": "tensor", "kernel": "tc_grouped_kernel<0> (gate/up tiles)", "achieved": ach_t,
                    "peak": tpk, "unit": "TFLOP/s", "frac": ach_t / tpk, "traffic": traffic_for(args.workload),
                    "peak_kind": tpk_kind + " (bf16 burst; fp16 x fp16 runs at the same rate)",
                    "flops_per_launch": flops, "kernel_ms": ktimes["tc_gu"],
                    "kernel_ms_by_name": ktimes, "layer_hbm_gbs": achieved}
    tokens = ws * nsteps * T
    value = tokens / (kern_ms * 1e-3)
    if rank == 0:
        cpu = cpu_oracle_rate(args.workload if not stack else "decode_e512_t1",
                              seconds=args.cpu_seconds) if ws == 1 and args.cpu_seconds > 0 else None
        line = {
            "metric": metric_for(args.workload) if not args.tokens else
                      f"MoE-layer verify tokens/s and achieved HBM GB/s (W4 g32, 512e top-8, T={T} per call)",
            "value": value, "unit": "tokens/s",
            "n_gpus": ws, "steps": nsteps,
            "warmup": nwarm, "ms_per_step": kern_ms / nsteps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": ("mxfp4 (e2m1, e8m0 per 32) x fp16" if fmt == "mxfp4" else "w4a16") + ", fp32 accumulate",
            "data": "synthetic (seeded weights and tokens drawn by workloads/synth.py)",
            "config": {"workload": args.workload, "T": T, "experts": E, "top_k": 8, "hidden": H,
                       "inter": I, "layers": len(layers),
                       "l2": (f"not flushed: step i runs layer i mod {len(layers)} of {len(layers)} independent "
                              f"full-shape layers, so the bytes a step reads were last read {len(layers)} steps "
                              f"(over {len(layers) - 1} x 40 MB of other weight traffic, above the 126 MB L2) before"
                              if mode == "rotate" else
                              "flushed before every step (256 MiB write, then a 256 MiB read of another buffer "
                              "so that no dirty lines are left), outside the per-step events"),
                       "parallelism": f"replicas x{ws}"},
            "us_per_layer": avg_launch_ms * 1e3,
            "achieved_gbs": achieved,
            "frac_of_8tbs": achieved / 8000.0,
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "warm": warm,
            "flushed": flushed,
            "graph": graph,
            "gpu_launches": launches,
            "clocks": clk.summary(),
            "wall_s_timed_region": t_wall,
            "step_us_p10_p50_p90": [sorted(step_ms)[int(q * (nsteps - 1))] * 1e3 for q in (0.1, 0.5, 0.9)],
            "tokens_per_s_median_step": ws * T / (statistics.median(step_ms) * 1e-3),
        }
        emit(line)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    for l in layers:
        l.close()
    return 0


# ------------------------------------------------------------------ online-FP8 LM head

LMHEAD_METRIC = "online-FP8 LM-head tokens/s and achieved HBM GB/s (157,184 x 2,560 e4m3, fp32 logits)"


def lmhead_bytes(V, T):
    """Algorithmic bytes of one call: e4m3 codes + row scales, the tokens, the fp32 logits."""
    return V * H + 4 * V + T * H * 2 + T * V * 4


def lmhead_oracle_rate(workload: str, seconds: float = 15.0, rows: int = 8192):
    """The oracle (quantise the head rows and the tokens, exact dot products)
    on a slice of the head, scaled to tokens/s of the whole vocabulary."""
    import numpy as np
    import torch
    import oracle.lmhead_ref as L
    import workloads
    wl = workloads.LMHEAD_WORKLOADS[workload]
    V, T = wl["vocab"], wl["T"]
    w = workloads.lm_head_weights(rows, H, seed=wl["weight_seed"], device="cpu")
    wb = w.view(torch.int16).numpy().view(np.uint16)
    n, dt, t0 = 0, 0.0, time.perf_counter()
    while dt < seconds and n < 64:
        x = workloads.tokens(T, H, seed=wl["token_seed"] + n, device="cpu")
        L.lm_head_fp8(x.view(torch.int16).numpy().view(np.uint16), wb)
        n += 1
        dt = time.perf_counter() - t0
    per_call_full = dt / n * (V / rows)
    return {"value": T / per_call_full, "unit": "tokens/s", "cores": len(os.sched_getaffinity(0)),
            "kind": "oracle",
            "sample": f"{n} calls of T={T} through the fp64 numpy oracle on {rows} of the {V} head rows "
                      f"(each call quantises those rows and the tokens), {dt:.1f} s, scaled by {V}/{rows}"}


def run_lmhead_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    import workloads
    wl = workloads.LMHEAD_WORKLOADS[args.workload]
    budget = max(10.0, min(60.0, 2.0 * (args.steps + args.warmup)))
    cpu = lmhead_oracle_rate(args.workload, seconds=budget)
    v = cpu["value"]
    line = {"metric": LMHEAD_METRIC, "value": v, "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": wl["T"] / v * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": args.workload, "T": wl["T"], "vocab": wl["vocab"], "hidden": H},
            "cpu_baseline": cpu,
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_lmhead(args):
    import torch
    import torch.distributed as dist
    ws, rank, local = dist_env()
    if ws > 1:
        dist.init_process_group("nccl", init_method="env://", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import workloads
    import weight_only_int4_fp32_b200 as lm
    wl = workloads.LMHEAD_WORKLOADS[args.workload]
    V, T = wl["vocab"], wl["T"]
    w = workloads.lm_head_weights(V, H, seed=wl["weight_seed"], device=dev)
    head = lm.LMHeadFP8(w)
    del w
    torch.cuda.empty_cache()
    nsteps, nwarm = args.steps, args.warmup
    off = rank * REPLICA_SEED_STRIDE
    inputs = [workloads.tokens(T, H, seed=wl["token_seed"] + i + off, device=dev) for i in range(nsteps + nwarm)]
    logits = torch.empty((T, V), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    for i in range(nwarm):
        head.forward(inputs[i], logits)
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(nsteps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(nsteps)]
    n0 = head.launch_count()
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall = time.perf_counter()
    with ClockSampler(local) as clk:
        for i in range(nsteps):
            starts[i].record(stream)
            head.forward(inputs[nwarm + i], logits)
            ends[i].record(stream)
        torch.cuda.synchronize()
    t_wall = time.perf_counter() - t_wall
    launches = head.launch_count() - n0
    step_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    kern_ms = max_over_ranks(sum(step_ms), dev)

    # end to end: pinned host tokens in, fp32 logits back to pinned host memory
    xh = [inputs[nwarm + i].cpu().pin_memory() for i in range(nsteps)]
    lh = torch.empty((T, V), dtype=torch.float32).pin_memory()
    for i in range(min(nwarm, 5)):
        head.forward_host(xh[i % nsteps], lh)
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    te = time.perf_counter()
    for i in range(nsteps):
        head.forward_host(xh[i], lh)
    te = max_over_ranks(time.perf_counter() - te, dev)
    e2e = {"value": ws * nsteps * T / te, "unit": "tokens/s", "h2d_bytes_per_step": T * H * 2,
           "d2h_bytes_per_step": T * V * 4,
           "note": "ling_moe_lmhead_forward_host per step: pinned H2D copy + head + D2H copy of the logits + "
                   "stream sync"}

    bytes_per_launch = lmhead_bytes(V, T)
    avg_ms = kern_ms / nsteps
    achieved = bytes_per_launch / (avg_ms * 1e-3) / 1e9
    peak, peak_kind = peaks()
    roofline = {"bound": "hbm", "kernel": "lmh_mma_kernel (one launch per call)", "achieved": achieved,
                "peak": peak, "unit": "GB/s", "frac": achieved / peak, "traffic": traffic_for(args.workload),
                "peak_kind": peak_kind, "bytes_per_launch": bytes_per_launch}
    if rank == 0:
        cpu = lmhead_oracle_rate(args.workload, seconds=args.cpu_seconds) \
            if ws == 1 and args.cpu_seconds > 0 else None
        line = {
            "metric": LMHEAD_METRIC, "value": ws * nsteps * T / (kern_ms * 1e-3), "unit": "tokens/s",
            "n_gpus": ws, "steps": nsteps, "warmup": nwarm, "ms_per_step": avg_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "e4m3 x e4m3, fp32 accumulate",
            "data": "synthetic (seeded head and tokens drawn by workloads/synth.py)",
            "config": {"workload": args.workload, "T": T, "vocab": V, "hidden": H,
                       "l2": "not flushed: every call streams 402 MB of codes, over 3x the 126 MB L2, "
                             "from the start of each CTA's range, so nothing of a call is left in L2 for the next",
                       "parallelism": f"replicas x{ws}"},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
            "clocks": clk.summary(), "wall_s_timed_region": t_wall,
            "step_us_p10_p50_p90": [sorted(step_ms)[int(q * (nsteps - 1))] * 1e3 for q in (0.1, 0.5, 0.9)],
        }
        emit(line)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    head.close()
    return 0


def spawn_ranks(n):
    """Run this same command as n ranks (one per GPU) under torch.distributed.run.

    Used when bench.py is started with --gpus N > 1 but not under a launcher
    (WORLD_SIZE unset): each rank reads RANK / LOCAL_RANK / WORLD_SIZE from the
    environment the launcher sets, rank 0 prints the one JSON line.  The
    launcher's exit code is returned."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__)] + sys.argv[1:]
    env = dict(os.environ)
    env.setdefault("OMP_NUM_THREADS", "4")
    return subprocess.call(cmd, env=env, timeout=3600)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode_e512_t1")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-secondary", dest="secondary", action="store_false",
                    help="default run: skip the short runs of the other workloads")
    ap.add_argument("--tokens", type=int, default=0,
                    help="verify workloads: calls of this many tokens (1..the workload's T) instead")
    ap.add_argument("--l2", default="auto", choices=["auto", "rotate", "flush"],
                    help="between steps: rotate over independent layers (decode-size workloads) or flush L2")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return spawn_ranks(args.gpus)
    ws, _, _ = dist_env()
    if ws != args.gpus and "WORLD_SIZE" in os.environ:
        print(f"bench.py: --gpus {args.gpus} under a launcher of WORLD_SIZE={ws}: running {ws} ranks",
              file=sys.stderr)
    lmhead = args.workload.startswith("lmhead")
    if args.impl == "reference":
        return run_lmhead_reference(args) if lmhead else run_reference(args)
    if args.secondary and ws == 1 and "--workload" not in sys.argv:
        return run_with_secondary(args)
    return run_lmhead(args) if lmhead else run_ours(args)


def run_with_secondary(args):
    """The headline workload as usual, then each SECONDARY workload for a
    short run (at most 50 steps, 3 warm-up, no CPU baseline); one JSON line,
    the headline's, with the others' compact records under "secondary"."""
    global _CAPTURE
    import copy
    import torch
    _CAPTURE = []
    try:
        rc = run_ours(args)
        line = _CAPTURE.pop()
        sec = {}
        for wl in SECONDARY:
            a = copy.copy(args)
            a.workload, a.steps, a.warmup, a.cpu_seconds, a.tokens = wl, min(args.steps, 50), 3, 0.0, 0
            try:
                (run_lmhead if wl.startswith("lmhead") else run_ours)(a)
                sec[wl] = compact(_CAPTURE.pop())
            except Exception as exc:  # a failing secondary workload does not lose the headline line
                sec[wl] = {"error": f"{type(exc).__name__}: {exc}"[:300]}
            torch.cuda.empty_cache()
        line["secondary"] = sec
    finally:
        _CAPTURE = None
    print(json.dumps(line), flush=True)
    return rc


if __name__ == "__main__":
    sys.exit(main())
