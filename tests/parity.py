"""Comparison of the GPU library against the fp64 oracle (test helper).

The bar, per token:
  * routing: the set of selected expert indices equals the oracle's, bit
    for bit, unless the oracle's k-th and (k+1)-th logits lie within 1e-5
    (a near tie: reported, and the token is exempt from both checks when the
    sets differ);
  * routing weights: within 1e-5 of the oracle's, matched by expert index;
  * output: |gpu - oracle| <= 2e-2 * max(1, |oracle|) elementwise, the oracle
    taken in fp64 before any rounding.

The online-FP8 LM head (lmhead_bound_ratio): codes and scales bit-exact;
logits within the rounding bound of the GPU's arithmetic.  Every product of
two e4m3 values is exact.  One m16n8k16 MMA adds 16 of them to its fp32
accumulator; the bound takes each MMA as its exact result rounded once to
fp32, possibly toward zero (error at most 2^-23 times the magnitude of the
chunk it belongs to) -- a model of the tensor core that the measurements fit
(the worst error seen is 7 * 2^-24 times the magnitude sum, 16 % of the bound
below), not a documented guarantee.  16 MMAs are chained per 256 codes, so
each such chunk may be off by 16 * 2^-23 = 32 * 2^-24 times its sum of
magnitudes; the chunk sums of a logit are added in fp32 (at most
ceil(hidden / 256) roundings, two more where a tile's K range is split
between two warps) and the total is multiplied by the two scales (two more).
So |gpu - exact| <= (32 + ceil(hidden / 256) + 4) * 2^-24 * sum_k |x_k w_k|
* s_x * s_w, 46 * 2^-24 at hidden = 2560.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

OUT_TOL = 2e-2
W_TOL = 1e-5
TIE_EPS = 1e-5


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def compare(ref: dict, out: torch.Tensor, idx: torch.Tensor | None, w: torch.Tensor | None, k: int,
            label: str = "") -> dict:
    """Raise AssertionError on a violation; return a small report."""
    o = ref["out"]
    g = out.detach().float().cpu().double().numpy()
    T = o.shape[0]
    near = oracle.near_tie(ref["logits"], k, TIE_EPS)
    exempt = np.zeros(T, dtype=bool)
    if idx is not None:
        gi = idx.detach().cpu().numpy()
        gw = w.detach().cpu().numpy() if w is not None else None
        for t in range(T):
            same = set(gi[t].tolist()) == set(ref["idx"][t].tolist())
            if not same:
                if near[t]:
                    exempt[t] = True
                    continue
                raise AssertionError(f"{label}: token {t} routed to {sorted(gi[t])}, "
                                     f"oracle {sorted(ref['idx'][t])}")
            if gw is not None:
                ref_w = dict(zip(ref["idx"][t].tolist(), ref["w"][t].tolist()))
                for e, wv in zip(gi[t].tolist(), gw[t].tolist()):
                    assert abs(wv - ref_w[e]) <= W_TOL, (label, t, e, wv, ref_w[e])
    err = np.abs(g - o)
    bound = OUT_TOL * np.maximum(1.0, np.abs(o))
    bad = (err > bound) & ~exempt[:, None]
    if bad.any():
        t, n = np.argwhere(bad)[0]
        raise AssertionError(f"{label}: {int(bad.sum())} outputs out of tolerance; first at "
                             f"token {t} col {n}: gpu {g[t, n]} oracle {o[t, n]}")
    rel = err / np.maximum(1.0, np.abs(o))
    return {"near_ties": int(near.sum()), "exempt": int(exempt.sum()),
            "max_scaled_err": float(rel[~exempt].max()) if (~exempt).any() else 0.0}


# bf16 rounds |v| >= (2 - 2^-8) * 2^127 to infinity (round to nearest even)
BF16_OVERFLOW = (2.0 - 2.0 ** -8) * 2.0 ** 127
BF16_SUBNORMAL = 2.0 ** -133


def compare_range(ref: dict, out: torch.Tensor, idx: torch.Tensor, w: torch.Tensor, k: int,
                  label: str = "") -> dict:
    """The bar of compare() made independent of each token's magnitude, for
    tokens of extreme range (|x| up to bf16's largest value, subnormals, both
    in one token):
      * routing: the selected set equals the oracle's unless its k-th and
        (k+1)-th logits lie within TIE_EPS times the token's largest |logit|;
        weights within W_TOL;
      * no output is NaN;
      * where bf16 rounds the oracle's output to +-inf, the GPU's is the same
        infinity (outputs within 2^-7 of that threshold are skipped);
      * elsewhere |gpu - oracle| <= OUT_TOL * max(|oracle|, rms_t / 32)
        + 2^-133, rms_t the root mean square of the token's oracle outputs
        (for an N(0, 1) token about 27, so rms_t / 32 stands where compare()
        puts 1) and 2^-133 bf16's subnormal spacing."""
    o = ref["out"]
    lg = np.asarray(ref["logits"], dtype=np.float64)
    g = out.detach().float().cpu().double().numpy()
    T = o.shape[0]
    gi = idx.detach().cpu().numpy()
    gw = w.detach().cpu().numpy()
    srt = -np.sort(-lg, axis=1)
    near = (np.abs(srt[:, k - 1] - srt[:, k]) <= TIE_EPS * np.abs(lg).max(axis=1)) if lg.shape[1] > k \
        else np.zeros(T, dtype=bool)
    exempt = np.zeros(T, dtype=bool)
    for t in range(T):
        if set(gi[t].tolist()) != set(ref["idx"][t].tolist()):
            if near[t]:
                exempt[t] = True
                continue
            raise AssertionError(f"{label}: token {t} routed to {sorted(gi[t])}, oracle {sorted(ref['idx'][t])}")
        ref_w = dict(zip(ref["idx"][t].tolist(), ref["w"][t].tolist()))
        for e, wv in zip(gi[t].tolist(), gw[t].tolist()):
            assert abs(wv - ref_w[e]) <= W_TOL, (label, t, e, wv, ref_w[e])
    assert not np.isnan(g).any(), f"{label}: NaN in the output"
    ovf = np.abs(o) >= BF16_OVERFLOW
    edge = np.abs(np.abs(o) / BF16_OVERFLOW - 1.0) < 2.0 ** -7
    fin = ~ovf & ~edge & ~exempt[:, None]
    inf_ok = np.isinf(g) & (np.sign(g) == np.sign(o))
    bad_inf = ovf & ~edge & ~exempt[:, None] & ~inf_ok
    if bad_inf.any():
        t, n = np.argwhere(bad_inf)[0]
        raise AssertionError(f"{label}: {int(bad_inf.sum())} outputs should be +-inf; first at token {t} col {n}: "
                             f"gpu {g[t, n]} oracle {o[t, n]}")
    rms = np.sqrt(np.mean(o * o, axis=1))
    bound = OUT_TOL * np.maximum(np.abs(o), rms[:, None] / 32) + BF16_SUBNORMAL
    err = np.where(fin, np.abs(g - o), 0.0)
    bad = fin & ~(err <= bound)
    if bad.any():
        t, n = np.argwhere(bad)[0]
        raise AssertionError(f"{label}: {int(bad.sum())} outputs out of tolerance; first at token {t} col {n}: "
                             f"gpu {g[t, n]} oracle {o[t, n]} bound {bound[t, n]}")
    with np.errstate(invalid="ignore", divide="ignore"):
        rel = np.where(fin, err / bound, 0.0)
    return {"near_ties": int(near.sum()), "exempt": int(exempt.sum()), "inf": int((ovf & ~edge).sum()),
            "max_err_over_bound": float(rel.max()) if fin.any() else 0.0}


def lmhead_bound_ratio(got: np.ndarray, xq, xs, wq, ws, hidden: int, label: str = "") -> float:
    """Check LM-head logits got [T, R] against the oracle's exact logits of the
    same codes (x codes/scales [T], head rows' codes/scales [R]); return the
    largest error as a fraction of the bound."""
    import oracle.lmhead_ref as L
    xd, wd = L.e4m3_decode(xq), L.e4m3_decode(wq)
    scale = xs.astype(np.float64)[:, None] * ws.astype(np.float64)[None, :]
    exact = (xd @ wd.T) * scale
    mag = (np.abs(xd) @ np.abs(wd).T) * scale
    u = 2.0 ** -24
    tol = (32 + (hidden + 255) // 256 + 4) * u * mag + 1e-37
    err = np.abs(np.asarray(got, dtype=np.float64) - exact)
    ratio = float((err / tol).max())
    bad = int((err > tol).sum())
    assert bad == 0, f"{label}: {bad} logits outside the bound; worst {ratio:.2f} x bound"
    return ratio
