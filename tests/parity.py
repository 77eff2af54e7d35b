"""Comparison of the GPU library against the fp64 oracle (test helper).

The bar, per token:
  * routing: the set of selected expert indices equals the oracle's, bit
    for bit, unless the oracle's k-th and (k+1)-th logits lie within 1e-5
    (a near tie: reported, and the token is exempt from both checks when the
    sets differ);
  * routing weights: within 1e-5 of the oracle's, matched by expert index;
  * output: |gpu - oracle| <= 2e-2 * max(1, |oracle|) elementwise, the oracle
    taken in fp64 before any rounding.
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
