"""Per-config inputs for the parity tests (CPU tensors, margin-enforced).

The seeded generators (token_pruned_sparse_b200.synth) make the data; the
oracle's margin enforcement then keeps every score at least a relative 1e-3
away from each selection boundary, so index lists can be compared bit for bit.
"""
from __future__ import annotations

import functools

import numpy as np
import torch

import oracle as O
from oracle import margins as M
from token_pruned_sparse_b200 import synth


@functools.lru_cache(maxsize=None)
def frame_case(name: str):
    """Inter-frame configs (tiny, mid, block): bf16 video x [F, HW, C] and the
    boundary (tau or k)."""
    cfg = synth.CONFIGS[name]
    x, _ = synth.latent_video(cfg.video)
    xb = synth.to_bf16(x)
    if cfg.mode == "thresh":
        xb = M.enforce_frame_margin(xb, tau=cfg.tau)
        return cfg, xb, None
    k = synth.keep_count(cfg.video.N, cfg.keep[0])
    xb = M.enforce_frame_margin(xb, ranks=(k,))
    return cfg, xb, k


@functools.lru_cache(maxsize=None)
def step_case(name: str):
    """Inter-step configs (wan, hsa): (v_prev, v_cur) bf16 [N, C] and the cuts."""
    cfg = synth.CONFIGS[name]
    vp, delta = synth.velocity_pair(cfg.video)
    vpb = synth.to_bf16(vp)
    N = cfg.video.N
    if cfg.mode == "hsa":
        K = cfg.extra["K"]
        ranks = tuple((b + 1) * (N // K) for b in range(K - 1))
    else:
        ranks = tuple(synth.keep_count(N, r) for r in cfg.keep if synth.keep_count(N, r) < N)
    vc = M.enforce_step_margin(vpb, delta, ranks=ranks)
    return cfg, vpb, vc, ranks


@functools.lru_cache(maxsize=None)
def qkv(name: str, which: str = "cur"):
    """Q, K, V [N, H, d] bf16 projected from the config's tokens."""
    cfg = synth.CONFIGS[name]
    if cfg.score_kind == "frame":
        _, xb, _ = frame_case(name)
        tok = xb.reshape(-1, cfg.video.C)
    else:
        _, vpb, vc, _ = step_case(name)
        tok = vc if which == "cur" else vpb
    W = synth.projection_weights(cfg.video.C, cfg.H, cfg.d, cfg.video.seed)
    return tuple(synth.project(tok, w, cfg.H, cfg.d) for w in W)


def oracle_idx(name: str, ratio_index: int = 0):
    cfg = synth.CONFIGS[name]
    if cfg.score_kind == "frame":
        _, xb, k = frame_case(name)
        s = O.lipar_score(xb)
        return O.select_threshold(s, cfg.tau) if k is None else O.select_topk(s, k)
    _, vpb, vc, _ = step_case(name)
    s = O.lipar_score(vc[None], vpb[None])
    return O.select_topk(s, synth.keep_count(cfg.video.N, cfg.keep[ratio_index]))


def attn_tolerance_ok(o_gpu: np.ndarray, o_ref: np.ndarray):
    """Bar for bf16 inputs with fp32 accumulation: max-abs <= 2e-2 and
    mean-abs <= 2e-3; plus a scale-aware bound (2% of the largest reference
    magnitude, at least 4 bf16 ulps of it) so tiny outputs cannot hide errors."""
    err = np.abs(o_gpu.astype(np.float64) - o_ref)
    mx = float(np.abs(o_ref).max()) if o_ref.size else 0.0
    rel_bound = max(2e-2 * mx, 4 * 2.0 ** -8 * mx, 1e-6)
    return (err.max() <= 2e-2 and err.mean() <= 2e-3 and err.max() <= rel_bound,
            dict(max_abs=float(err.max()) if err.size else 0.0, mean_abs=float(err.mean()) if err.size else 0.0,
                 ref_max=mx))
