"""Margin enforcement for generated inputs (TEST INFRASTRUCTURE ONLY).

Index lists must match the CUDA path bit for bit, while the CUDA path scores
in fp32 and the oracle in fp64. Generated inputs are therefore nudged so that
no score lies within a relative 1e-3 of any selection boundary (threshold,
top-k cut, group cut). A token's change is scaled by lambda, cur = ref +
lambda * delta, which scales its relative-L1 score by lambda before bf16
rounding; the loop re-rounds, re-scores and repeats until every boundary has
its margin (at most 32 rounds, else it fails loudly).

This lives beside the oracle because it uses the oracle's score and rank
order; it is applied to inputs before either side sees them.
"""
from __future__ import annotations

import numpy as np
import torch

from .tps_oracle import _rank_order, f64, lipar_score

MARGIN = 1e-3     # required relative distance from every boundary
PUSH = 2e-3       # where a violating score is moved to

__all__ = ["MARGIN", "boundary_sides", "enforce_step_margin", "enforce_frame_margin", "margins_ok"]


def boundary_sides(s: np.ndarray, *, tau=None, ranks=()):
    """For each boundary return (t, above_mask): the cut value and which tokens
    must stay above it. Threshold: t = tau, above = s >= tau. Rank cut r: the
    first r tokens in rank order are above; t is the midpoint of the scores at
    ranks r-1 and r."""
    out = []
    if tau is not None:
        out.append((float(tau), s >= tau))
    if ranks:
        order = _rank_order(s)
        for r in ranks:
            if r <= 0 or r >= len(s):
                continue
            hi, lo = s[order[r - 1]], s[order[r]]
            if not (np.isfinite(hi) and np.isfinite(lo)):
                continue
            above = np.zeros(len(s), bool)
            above[order[:r]] = True
            out.append((0.5 * (hi + lo), above))
    return out


def _violations(s, bounds):
    """Per-token target ratio (target / s) for tokens inside a margin band."""
    scale = np.ones(len(s))
    bad = np.zeros(len(s), bool)
    for t, above in bounds:
        if t <= 0:
            continue
        fin = np.isfinite(s) & (s > 0)
        up = above & fin & (s < t * (1 + MARGIN))
        dn = ~above & fin & (s > t * (1 - MARGIN))
        scale[up] = t * (1 + PUSH) / s[up]
        scale[dn] = t * (1 - PUSH) / s[dn]
        bad |= up | dn
    return bad, scale


def margins_ok(s, bounds) -> bool:
    return not _violations(s, bounds)[0].any()


def enforce_step_margin(v_prev: torch.Tensor, delta: np.ndarray, *, tau=None, ranks=()):
    """Inter-step pair: returns v_cur (bf16) = RN(v_prev + lambda * delta) whose
    scores against v_prev keep the margin from every boundary."""
    ref = f64(v_prev)
    d = np.asarray(delta, np.float64)
    lam = np.ones(ref.shape[0])
    for _ in range(32):
        cur = torch.from_numpy(ref + lam[:, None] * d).to(torch.bfloat16)
        s = lipar_score(cur[None], v_prev[None])
        bad, scale = _violations(s, boundary_sides(s, tau=tau, ranks=ranks))
        if not bad.any():
            return cur
        lam[bad] *= scale[bad]
    raise RuntimeError("margin enforcement did not converge")


def enforce_frame_margin(x_bf16: torch.Tensor, *, tau=None, ranks=()):
    """Inter-frame video [F, HW, C]: scale per-token frame-to-frame changes so
    that every inter-frame score keeps the margin. A position whose change is
    rescaled at frame f is rebuilt from frame f on (frame f+1's reference
    moves with it); untouched positions stay bit-identical."""
    x0 = f64(x_bf16)
    F, HW, C = x0.shape
    d = np.zeros_like(x0)
    d[1:] = x0[1:] - x0[:-1]
    lam = np.ones((F, HW))
    x = x_bf16.clone()
    for _ in range(32):
        s = lipar_score(x)
        bad, scale = _violations(s, boundary_sides(s, tau=tau, ranks=ranks))
        if not bad.any():
            return x
        lam.reshape(-1)[bad] *= scale[bad]
        touched = np.cumsum(lam != 1.0, axis=0) > 0          # rebuilt from first change on
        xn = x0.copy()
        for f in range(1, F):
            t = touched[f]
            if t.any():
                row = xn[f - 1, t] + lam[f, t][:, None] * d[f, t]
                xn[f, t] = f64(torch.from_numpy(row).to(torch.bfloat16))
        x = torch.from_numpy(xn).to(torch.bfloat16)
    raise RuntimeError("margin enforcement did not converge")
