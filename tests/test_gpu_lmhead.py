"""The online-FP8 LM head on the GPU against the fp64 oracle.

Codes and scales (of the head and of the tokens) must be bit-exact: both
sides take every quantisation decision in the same fp32 steps.  Logits must
lie within the rounding bound of the GPU's arithmetic derived in
tests/parity.py; the largest measured error, as a fraction of that bound,
is printed.
"""
import numpy as np
import pytest
import torch

import oracle.lmhead_ref as L
import workloads
import weight_only_int4_fp32_b200 as lm
from tests.parity import lmhead_bound_ratio

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _check_logits(got, xq, xs, wq, ws, hidden, what):
    ratio = lmhead_bound_ratio(got, xq, xs, wq, ws, hidden, what)
    print(f"{what}: largest error {ratio:.3f} of the bound")


def _run(head, x):
    logits, xq, xs = head.forward(x, return_codes=True)
    assert head.status() == lm.LING_MOE_OK
    return logits.cpu().numpy(), xq.cpu().numpy(), xs.cpu().numpy()


# vocabularies from one tile per CTA (pieces of a tile on several warps) to
# several (tiles cut between two warps); hidden from 2 to 16 chunks per row
@pytest.mark.parametrize("vocab,hidden", [(3001, 2560), (777, 512), (777, 4096), (1, 2560), (2369, 1024),
                                          (20011, 2560), (9473, 1536)])
def test_lmhead_matches_the_oracle(vocab, hidden):
    w = workloads.lm_head_weights(vocab, hidden, seed=11, device=DEV)
    head = lm.LMHeadFP8(w)
    try:
        wq_ref, ws_ref = L.quantize_rows(_f32(_bits(w)))
        wq, ws = head.weights()
        assert np.array_equal(wq.cpu().numpy(), wq_ref), "head codes differ from the oracle"
        assert np.array_equal(ws.cpu().numpy(), ws_ref), "head scales differ from the oracle"
        for T in range(1, 9):
            x = workloads.tokens(T, hidden, seed=500 + T, device=DEV)
            logits, xq, xs = _run(head, x)
            xq_ref, xs_ref = L.quantize_rows(_f32(_bits(x)))
            assert np.array_equal(xq, xq_ref) and np.array_equal(xs, xs_ref), f"token codes T={T}"
            _check_logits(logits, xq_ref, xs_ref, wq_ref, ws_ref, hidden, f"V={vocab} H={hidden} T={T}")
    finally:
        head.close()


def test_lmhead_degenerate_rows_and_tokens():
    """All-zero rows and tokens (scale 1, codes 0, logits exactly 0), a row
    whose maximum dwarfs the rest (subnormal codes), a constant row, signs."""
    vocab, hidden = 700, 2560
    w = workloads.lm_head_weights(vocab, hidden, seed=12, device=DEV)
    w[3] = 0
    w[10] = 1e-4
    w[10, 17] = 30.0
    w[11] = -0.5
    w[699] = 0
    x = workloads.tokens(6, hidden, seed=13, device=DEV)
    x[2] = 0
    x[4] = x[4] * 1e-3
    x[5, 100] = 300.0
    head = lm.LMHeadFP8(w)
    try:
        wq_ref, ws_ref = L.quantize_rows(_f32(_bits(w)))
        wq, ws = head.weights()
        assert np.array_equal(wq.cpu().numpy(), wq_ref) and np.array_equal(ws.cpu().numpy(), ws_ref)
        assert ws_ref[3] == 1.0 and not wq_ref[3].any()
        logits, xq, xs = _run(head, x)
        xq_ref, xs_ref = L.quantize_rows(_f32(_bits(x)))
        assert np.array_equal(xq, xq_ref) and np.array_equal(xs, xs_ref)
        assert xs[2] == 1.0 and not logits[2].any()
        assert not logits[:, 3].any() and not logits[:, 699].any()
        _check_logits(logits, xq_ref, xs_ref, wq_ref, ws_ref, hidden, "degenerate")
    finally:
        head.close()


def test_lmhead_full_vocabulary_sampled():
    """157,184 x 2,560 (the benchmark's head and its launch): every token's
    codes, and the codes, scales and logits of sampled rows, which the oracle
    computes row by row."""
    wl = workloads.LMHEAD_WORKLOADS["lmhead_fp8_v157184_t8"]
    V, H = wl["vocab"], workloads.HIDDEN
    w = workloads.lm_head_weights(V, H, seed=wl["weight_seed"], device=DEV)
    head = lm.LMHeadFP8(w)
    try:
        rng = np.random.default_rng(14)
        rows = np.unique(np.concatenate([np.arange(64), np.arange(V - 64, V), rng.integers(0, V, 4096)]))
        wrows = _bits(w[torch.from_numpy(rows).to(DEV)])
        wq_ref, ws_ref = L.quantize_rows(_f32(wrows))
        wq, ws = head.weights()
        assert np.array_equal(wq[torch.from_numpy(rows).to(DEV)].cpu().numpy(), wq_ref)
        assert np.array_equal(ws.cpu().numpy()[rows], ws_ref)
        del wq
        for T, seed in ((1, 30000), (8, wl["token_seed"])):
            x = workloads.tokens(T, H, seed=seed, device=DEV)
            logits, xq, xs = _run(head, x)
            xq_ref, xs_ref = L.quantize_rows(_f32(_bits(x)))
            assert np.array_equal(xq, xq_ref) and np.array_equal(xs, xs_ref)
            _check_logits(logits[:, rows], xq_ref, xs_ref, wq_ref, ws_ref, H, f"full vocab T={T}")
            assert np.isfinite(logits).all()
    finally:
        head.close()


def test_lmhead_one_launch_per_call_deterministic_and_host_path():
    V, H = 5000, 2560
    w = workloads.lm_head_weights(V, H, seed=15, device=DEV)
    head = lm.LMHeadFP8(w)
    try:
        x = workloads.tokens(3, H, seed=16, device=DEV)
        n0 = head.launch_count()
        a = head.forward(x)
        b = head.forward(x)
        torch.cuda.synchronize()
        assert head.launch_count() - n0 == 2
        assert torch.equal(a, b)
        got = head.forward_host(x.cpu().pin_memory())
        assert torch.equal(got, a.cpu())
        assert head.forward(x[:0]).shape == (0, V)
        assert head.launch_count() - n0 == 3
        with pytest.raises(lm.LingMoEError):
            head.forward(workloads.tokens(9, H, seed=1, device=DEV))
    finally:
        head.close()


def test_lmhead_wait_that_runs_out_reports_an_error_and_the_next_call_is_clean():
    """One CTA withholds its copies: its consumers' bounded waits run out
    (50 ms), the launch ends with DEVICE_TIMEOUT instead of hanging, and the
    next call, with the hook off, is exact again."""
    V, H = 20011, 2560
    w = workloads.lm_head_weights(V, H, seed=17, device=DEV)
    head = lm.LMHeadFP8(w)
    try:
        x = workloads.tokens(2, H, seed=18, device=DEV)
        good = head.forward(x)
        assert head.status() == lm.LING_MOE_OK
        head.test_set_wait(5, 50_000_000)
        head.forward(x)
        assert head.status() == lm.LING_MOE_ERR_DEVICE_TIMEOUT
        head.test_set_wait(-1, 0)
        again = head.forward(x)
        assert head.status() == lm.LING_MOE_OK
        assert torch.equal(again, good)
    finally:
        head.close()


def test_lmhead_graph_capture_replays_the_call():
    V, H = 5000, 2560
    w = workloads.lm_head_weights(V, H, seed=19, device=DEV)
    head = lm.LMHeadFP8(w)
    try:
        x = workloads.tokens(4, H, seed=20, device=DEV)
        logits = torch.empty((4, V), dtype=torch.float32, device=DEV)
        ref = head.forward(x).clone()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            head.forward(x, logits)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            head.forward(x, logits)
        for _ in range(2):
            logits.zero_()
            g.replay()
            torch.cuda.synchronize()
            assert torch.equal(logits, ref)
        assert head.status() == lm.LING_MOE_OK
        del g
    finally:
        head.close()
