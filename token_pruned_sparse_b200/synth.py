"""Seeded synthetic inputs for the token-pruned attention path.

This module only *makes data*: latent videos, velocity pairs, projection
weights, caches, score arrays and key-block masks. It holds none of the
method's arithmetic (no scoring, selection, cache sync, attention or
scatter), so both the CUDA path and the fp64 oracle can consume exactly the
same inputs without sharing any computation.

The recipe stands in for the pages' workloads (DAVIS clips, Wan/HunyuanVideo
latents), which are not available offline:

* background: a static per-token N(0,1) field plus fresh N(0, 0.01^2)
  jitter every frame (static regions are what the latent inter-frame
  pruning of "Training-free Latent Inter-Frame Pruning with Attention
  Recovery", section 2.B, removes);
* moving objects: square patches that move one token per frame along a
  seeded axis direction, wrap toroidally, and carry fresh N(0,1) content;
* a pan strip: round(0.2 * W) full-height columns showing a per-row
  Gaussian texture that slides by half a token per frame (linear
  interpolation);
* inter-step velocities (the dynamic token selection of "Asignacion de
  Pasos Heterogenea (HSA)", section 2.1): v_prev is the latent, v_cur adds
  a step delta of N(0, 0.05^2) on background tokens and N(0,1) on
  object/pan tokens.

All draws use numpy's PCG64 ``default_rng(seed)`` in float32; tensors are
rounded to bf16 (round-to-nearest-even) by torch.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

__all__ = [
    "VideoSpec", "CONFIGS", "latent_video", "velocity_pair", "projection_weights",
    "project", "to_bf16", "random_scores", "block_mask_band_random", "gaussian_bf16",
    "timeripple_windows", "TR_THETA", "rope_dims",
]


@dataclass(frozen=True)
class VideoSpec:
    """Shape and content of one synthetic latent video."""
    F: int           # latent frames
    Hs: int          # latent grid height (tokens)
    Ws: int          # latent grid width (tokens)
    C: int           # latent channels
    n_obj: int       # moving square objects
    obj: int         # object side (tokens)
    pan: bool        # half-token-per-frame pan strip over 20% of the width
    seed: int

    @property
    def HW(self) -> int:
        return self.Hs * self.Ws

    @property
    def N(self) -> int:
        return self.F * self.HW


@dataclass(frozen=True)
class Config:
    """One workload: a video plus the attention geometry and the active-set rule."""
    name: str
    video: VideoSpec
    H: int
    d: int
    mode: str                     # "thresh" | "topk" | "hsa" | "block"
    score_kind: str               # "frame" (inter-frame) | "step" (inter-step)
    tau: float = 0.0
    keep: tuple = ()              # keep ratios for top-k configs
    extra: dict = field(default_factory=dict)


CONFIGS = {
    # 4 frames x 8x8 tokens, 2 heads, d=64; one 3x3 object; threshold 0.2.
    "tiny": Config("tiny", VideoSpec(4, 8, 8, 64, 1, 3, False, 1), 2, 64, "thresh", "frame", tau=0.2),
    # 13 x 30x52 = 20280 tokens, 12 heads, d=128; six 8x8 objects + pan; top-k 30%.
    "mid": Config("mid", VideoSpec(13, 30, 52, 128, 6, 8, True, 2), 12, 128, "topk", "frame", keep=(0.3,)),
    # 21 x 30x52 = 32760 tokens, 12 heads, d=128; inter-step score; keep 10/30/50/100%.
    "wan": Config("wan", VideoSpec(21, 30, 52, 128, 6, 8, True, 3), 12, 128, "topk", "step",
                  keep=(0.1, 0.3, 0.5, 1.0)),
    # 33 x 45x80 = 118800 tokens, 24 heads, d=128; K=3 groups, budgets T, T/2, T/4, T=40.
    "hsa": Config("hsa", VideoSpec(33, 45, 80, 128, 6, 8, True, 4), 24, 128, "hsa", "step",
                  extra={"K": 3, "T": 40, "budgets": (40, 20, 10), "m": 0}),
    # 118800 tokens, 24 heads; 40% active queries (top-k of inter-frame score); 139/929 key blocks.
    "block": Config("block", VideoSpec(33, 45, 80, 128, 6, 8, True, 5), 24, 128, "block", "frame",
                    keep=(0.4,), extra={"block": 128, "kept_per_row": 139}),
}


def timeripple_windows(d: int):
    """Channel windows (start, length) of the t, x and y similarity checks for a
    head of d channels, as cyclic ranges over the head dimension.

    Configuration, not arithmetic: the head's rotary channels are taken as three
    contiguous groups [t | x | y] of sizes (d - 4*(d//6), 2*(d//6), 2*(d//6)),
    each even so rotary pairs stay whole. A check along an axis uses the channels
    that axis does NOT rotate (they stay similar between neighbours on it): t ->
    the x and y groups; x -> the y and t groups (the window wraps); y -> the t
    and x groups."""
    g = 2 * (d // 6)
    dt = d - 2 * g
    return ((dt, 2 * g), (dt + g, dt + g), (0, dt + g))


def rope_dims(d: int):
    """Channel counts (t, x, y) of a head's rotary groups, contiguous in that
    order: (d - 4*(d//6), 2*(d//6), 2*(d//6)), each even (the same split as the
    Timeripple windows above). Configuration, not arithmetic."""
    g = 2 * (d // 6)
    return (d - 2 * g, g, g)


# Threshold schedule of the per-axis checks (t, x, y): theta rises from 0 at
# step 11 to these values at step 21. Background tokens of the synthetic video
# move by jitter only (RMS about 0.01 after projection), moving tokens by ~1.4.
TR_THETA = (0.05, 0.05, 0.05)


def keep_count(N: int, ratio: float) -> int:
    """Integer k for a keep ratio (all configured ratios give exact integers)."""
    return int(round(N * ratio))


def to_bf16(a) -> torch.Tensor:
    """fp32 array -> bf16 tensor, IEEE round-to-nearest-even (torch's conversion)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def _object_tracks(spec: VideoSpec, rng: np.random.Generator):
    dirs = np.array([(0, 1), (0, -1), (1, 0), (-1, 0)])
    starts = np.stack([rng.integers(0, spec.Hs, spec.n_obj), rng.integers(0, spec.Ws, spec.n_obj)], 1)
    moves = dirs[rng.integers(0, 4, spec.n_obj)]
    return starts, moves


def latent_video(spec: VideoSpec):
    """Latent video x [F, HW, C] float32 and its moving-token mask [F, HW].

    Frame f paints, in order: background + jitter, the pan strip, then the
    objects at (start + f * move) mod grid.
    """
    rng = np.random.default_rng(spec.seed)
    F, Hs, Ws, C = spec.F, spec.Hs, spec.Ws, spec.C
    bg = rng.standard_normal((Hs, Ws, C), dtype=np.float32)
    starts, moves = _object_tracks(spec, rng)
    pw = int(round(0.2 * Ws)) if spec.pan else 0
    c0 = int(rng.integers(0, Ws - pw + 1)) if spec.pan else 0
    tex_w = pw + int(math.ceil(0.5 * F)) + 2
    tex = rng.standard_normal((Hs, tex_w, C), dtype=np.float32) if spec.pan else None
    x = np.empty((F, Hs, Ws, C), np.float32)
    moving = np.zeros((F, Hs, Ws), bool)
    for f in range(F):
        x[f] = bg + np.float32(0.01) * rng.standard_normal((Hs, Ws, C), dtype=np.float32)
        if pw:
            u = np.arange(pw, dtype=np.float64) + 0.5 * f
            i0 = np.floor(u).astype(int)
            t = (u - i0).astype(np.float32)[None, :, None]
            x[f, :, c0:c0 + pw] = (1 - t) * tex[:, i0] + t * tex[:, i0 + 1]
            moving[f, :, c0:c0 + pw] = True
        for o in range(spec.n_obj):
            y = (starts[o, 0] + moves[o, 0] * f + np.arange(spec.obj)) % Hs
            xx = (starts[o, 1] + moves[o, 1] * f + np.arange(spec.obj)) % Ws
            x[f][np.ix_(y, xx)] = rng.standard_normal((spec.obj, spec.obj, C), dtype=np.float32)
            moving[f][np.ix_(y, xx)] = True
    return x.reshape(F, Hs * Ws, C), moving.reshape(F, Hs * Ws)


def velocity_pair(spec: VideoSpec, seed_offset: int = 1000):
    """Two consecutive velocity predictions (v_prev, delta) as float32 [N, C].

    v_prev is the latent video; the step delta is N(0, 0.05^2) on
    background tokens and N(0, 1) on object/pan tokens. v_cur = v_prev + delta
    (callers may rescale delta per token before forming v_cur).
    """
    x, moving = latent_video(spec)
    rng = np.random.default_rng(spec.seed + seed_offset)
    N, C = spec.N, spec.C
    sd = np.where(moving.reshape(N), np.float32(1.0), np.float32(0.05)).astype(np.float32)
    delta = rng.standard_normal((N, C), dtype=np.float32) * sd[:, None]
    return x.reshape(N, C), delta


def projection_weights(C: int, H: int, d: int, seed: int):
    """W_q, W_k, W_v in R^{C x H*d}, entries N(0, 1/d) (variance 1/d)."""
    rng = np.random.default_rng(seed + 77)
    s = np.float32(1.0 / math.sqrt(d))
    return tuple(rng.standard_normal((C, H * d), dtype=np.float32) * s for _ in range(3))


def project(x_bf16: torch.Tensor, W: np.ndarray, H: int, d: int) -> torch.Tensor:
    """bf16 tokens [N, C] @ W -> bf16 [N, H, d] (fp32 product, then RNE)."""
    y = x_bf16.float() @ torch.from_numpy(W)
    return y.to(torch.bfloat16).reshape(-1, H, d).contiguous()


def gaussian_bf16(shape, seed: int, std: float = 1.0) -> torch.Tensor:
    rng = np.random.default_rng(seed)
    return to_bf16(rng.standard_normal(shape, dtype=np.float32) * np.float32(std))


def random_scores(N: int, seed: int, *, ties: bool = False, specials: bool = False) -> torch.Tensor:
    """fp32 score arrays for selection tests (optionally with ties, +inf, 0)."""
    rng = np.random.default_rng(seed)
    s = rng.exponential(1.0, N).astype(np.float32)
    if ties:
        s = np.round(s * 4).astype(np.float32) / 4       # many exact duplicates
    if specials and N >= 8:
        pick = rng.choice(N, size=max(4, N // 16), replace=False)
        s[pick[: len(pick) // 2]] = np.inf
        s[pick[len(pick) // 2:]] = 0.0
    return torch.from_numpy(s)


def block_mask_band_random(spec: VideoSpec, block: int, kept_per_row: int, seed: int) -> torch.Tensor:
    """Key-block keep mask [nb, nb] uint8 (row = query block, column = key block).

    Row qb keeps the blocks that hold the same spatial start in every frame
    (which includes the diagonal) plus seeded uniform distinct others, so that
    exactly ``kept_per_row`` blocks are kept in every row.
    """
    N, HW = spec.N, spec.HW
    nb = -(-N // block)
    rng = np.random.default_rng(seed + 555)
    m = np.zeros((nb, nb), np.uint8)
    for qb in range(nb):
        s0 = (qb * block) % HW
        band = {(f * HW + s0) // block for f in range(spec.F)}
        band.add(qb)
        rest = np.setdiff1d(np.arange(nb), np.fromiter(band, int))
        extra = rng.choice(rest, size=kept_per_row - len(band), replace=False)
        m[qb, list(band)] = 1
        m[qb, extra] = 1
    return torch.from_numpy(m)
