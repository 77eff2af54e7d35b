"""Comparison of the GPU library against the fp64 oracle (test helper).

The bar, per token:
  * routing: the set of selected expert indices equals the oracle's, bit
    for bit, unless the oracle's k-th and (k+1)-th logits lie within 1e-5
    (a near tie: reported, and the token is exempt from both checks when the
    sets differ);
  * routing weights: within 1e-5 of the oracle's, matched by expert index;
  * output: |gpu - oracle| <= 2e-2 * max(1, |oracle|) elementwise, the oracle
    taken in fp64 before any rounding.

The online-FP8 LM head (compare_lmhead): codes and scales bit-exact; logits
within the rounding bound of the GPU's arithmetic.  Every product of two
e4m3 values is exact.  A tensor-core MMA adds 16 of them to its accumulator;
the bound allows that step an error of 2^-21 times (|accumulator| + the sum
of the 16 magnitudes) -- a model, not a documented guarantee: it grants the
tensor core's internal alignment a few guard bits' worth of truncation.  16
MMAs are chained per 256 codes, so each such chunk may be off by
16 * 2^-21 = 2^-17 times its sum of magnitudes; the hidden / 256 chunk sums
of a logit are added in fp32 (at most hidden / 256 roundings) and the total
is multiplied by the two scales (two more).  So
|gpu - exact| <= (2^-17 + (hidden / 256 + 2) * 2^-24) * sum_k |x_k w_k| * s_x * s_w.
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
    tol = (128 * u + (hidden // 256 + 2) * u) * mag + 1e-37
    err = np.abs(np.asarray(got, dtype=np.float64) - exact)
    ratio = float((err / tol).max())
    bad = int((err > tol).sum())
    assert bad == 0, f"{label}: {bad} logits outside the bound; worst {ratio:.2f} x bound"
    return ratio
