"""The magnitude-independent bar (tests.parity.compare_range) on the CPU: the
oracle's own outputs, rounded to bf16, pass it; planted mistakes in them
(a NaN, an infinity of the wrong sign, a finite value where bf16 overflows,
a 5 % error on a tiny token that compare()'s absolute floor would let
through, a wrong expert) do not."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.parity import bits, compare, compare_range

KINDS = ["normal", "near_max", "tiny", "mixed", "all_max", "subnormal"]


@pytest.fixture(scope="module")
def case():
    lw = workloads.layer_weights(32, seed=0, device="cpu")
    host = lw.host_arrays()
    x = workloads.extreme_tokens(KINDS, seed=123)
    with np.errstate(over="ignore", invalid="ignore", under="ignore"):
        ref = oracle.moe_layer(bits(x), host, 8)
    out = torch.from_numpy(ref["out"]).to(torch.bfloat16)
    return ref, out, torch.from_numpy(ref["idx"]), torch.from_numpy(ref["w"]).float()


def test_rounded_oracle_passes(case):
    ref, out, idx, w = case
    rep = compare_range(ref, out, idx, w, 8, "rounded oracle")
    assert rep["inf"] == 2 * 2560  # near_max and all_max overflow bf16 everywhere
    assert torch.isinf(out[1]).all() and torch.isinf(out[4]).all()
    assert torch.count_nonzero(out[5]) == 0  # subnormal tokens: outputs below bf16's range


def _planted(case, t, n, value):
    ref, out, idx, w = case
    bad = out.clone()
    bad[t, n] = value
    with pytest.raises(AssertionError):
        compare_range(ref, bad, idx, w, 8, "planted")


def test_nan_is_caught(case):
    _planted(case, 0, 5, float("nan"))


def test_wrong_infinity_sign_is_caught(case):
    ref = case[0]
    _planted(case, 1, 7, -float(np.sign(ref["out"][1, 7])) * float("inf"))


def test_finite_value_where_bf16_overflows_is_caught(case):
    _planted(case, 4, 3, 3.0e38)


def test_relative_error_on_a_tiny_token_is_caught(case):
    ref, out, idx, w = case
    bad = out.clone()
    bad[2] = (torch.from_numpy(ref["out"][2]) * 1.05).to(torch.bfloat16)
    row = {key: ref[key][2:3] for key in ("out", "idx", "w", "logits")}
    compare(row, bad[2:3], idx[2:3], w[2:3], 8, "absolute floor lets it through")  # |o| << 1 there
    with pytest.raises(AssertionError):
        compare_range(ref, bad, idx, w, 8, "planted")


def test_wrong_expert_is_caught(case):
    ref, out, idx, w = case
    bad_idx = idx.clone()
    row = set(bad_idx[3].tolist())
    bad_idx[3, 0] = next(e for e in range(32) if e not in row)
    with pytest.raises(AssertionError):
        compare_range(ref, out, bad_idx, w, 8, "planted")
