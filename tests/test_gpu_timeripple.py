"""GPU parity: timeripple_score (Timeripple per-axis similarity check) vs the
fp64 oracle, through the C ABI.

Delta is compared element by element within the fp32 error bound of a sum of
at most d positive terms. Reuse bits follow from Delta < theta: they must equal
the oracle's decision wherever the oracle's Delta lies outside that error band
around theta (elsewhere both decisions are correct), and they must equal the
kernel's own fp32 decision on the Delta it reports, everywhere.
"""
import numpy as np
import pytest
import torch

import oracle as O
from token_pruned_sparse_b200 import synth
from token_pruned_sparse_b200 import tps

from workloads import qkv

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _tol(d):
    # fp32: d squared differences summed (<= d roundings), one division, one sqrt
    return (d + 4) * 2.0 ** -24


def _check(x, F, Hs, Ws, wins, theta, ref_delta=None, rows=None):
    """Run the kernel on x [N, H, d]; compare against the oracle on the rows
    `rows` of the flattened token index (all rows by default)."""
    N, H, d = x.shape
    reuse, delta, score = tps.timeripple_score(x.to(DEV), F, Hs, Ws, wins, theta, delta=True, score=True)
    tps.tps_check()
    g = delta.cpu().double().numpy()
    r = reuse.cpu().numpy()
    sc = score.cpu().numpy()
    D = O.timeripple_delta(x, F, Hs, Ws, wins) if ref_delta is None else ref_delta
    if rows is not None:
        g, r, sc = g[:, rows], r[rows], sc[rows]
    tol = _tol(d)
    assert np.array_equal(np.isinf(g), np.isinf(D))
    fin = np.isfinite(D)
    np.testing.assert_allclose(g[fin], D[fin], rtol=tol, atol=0)
    # bits: the kernel's own decision on its reported Delta, everywhere
    th = np.asarray(theta, np.float32)
    own = np.zeros_like(r)
    for a in range(3):
        own |= ((g[a].astype(np.float32) < th[a]).astype(np.uint8) << a)
    assert np.array_equal(r, own)
    # and the oracle's decision outside the rounding band around theta
    ref_bits = O.timeripple_reuse(D, theta)
    amb = np.zeros(r.shape, bool)
    for a in range(3):
        amb |= np.isfinite(D[a]) & (np.abs(D[a] - theta[a]) <= 2 * tol * abs(theta[a]))
    assert np.array_equal(r[~amb], ref_bits[~amb])
    assert amb.mean() < 1e-3
    # token score: heads with no bit set
    assert np.array_equal(sc, (r == 0).sum(axis=1).astype(np.float32))
    clean = ~amb.any(axis=1)
    assert np.array_equal(sc[clean], O.timeripple_token_score(ref_bits)[clean])
    return r, g, sc


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_timeripple_on_projected_video(name):
    cfg = synth.CONFIGS[name]
    q, k, _ = qkv(name)
    v = cfg.video
    wins = synth.timeripple_windows(cfg.d)
    for x in (q, k):
        r, _, sc = _check(x, v.F, v.Hs, v.Ws, wins, synth.TR_THETA)
        # the static background is reusable along t from frame 1 on; moving tokens are not
        assert 0.3 < (r[v.HW:] != 0).mean() < 0.95


@pytest.mark.parametrize("F,Hs,Ws,H,d,wins", [
    (1, 5, 37, 3, 128, ((5, 100), (120, 30), (0, 128))),     # one frame: t never passes
    (3, 1, 40, 2, 64, ((0, 64), (60, 10), (3, 0))),           # one row; zero-length y window
    (4, 9, 1, 2, 128, ((127, 1), (0, 0), (64, 64))),          # one column; one-channel window
    (40, 8, 16, 1, 128, ((44, 84), (86, 86), (0, 86))),       # many frames: runs with priming frames
    (6, 17, 33, 3, 64, ((24, 40), (44, 44), (0, 44))),        # ragged tiles in both directions
])
def test_timeripple_shapes_and_windows(F, Hs, Ws, H, d, wins):
    rng = np.random.default_rng(F * 1000 + Hs * 10 + Ws)
    base = rng.standard_normal((1, Hs, Ws, H, d)).astype(np.float32)
    x = base + 0.02 * rng.standard_normal((F, Hs, Ws, H, d)).astype(np.float32)
    x[:, ::3] = rng.standard_normal(x[:, ::3].shape)          # every third row changes fully
    xb = synth.to_bf16(x.reshape(-1, H, d))
    _check(xb, F, Hs, Ws, wins, (0.05, 0.5, 1.2))


def test_timeripple_theta_edges_and_optional_outputs():
    q, _, _ = qkv("tiny")
    v = synth.CONFIGS["tiny"].video
    wins = synth.timeripple_windows(64)
    xd = q.to(DEV)
    r0, _, _ = tps.timeripple_score(xd, v.F, v.Hs, v.Ws, wins, (0.0, -1.0, 0.0))
    assert not r0.any()                                       # theta <= 0 never passes
    rinf, _, _ = tps.timeripple_score(xd, v.F, v.Hs, v.Ws, wins, (float("inf"),) * 3)
    D = O.timeripple_delta(q, v.F, v.Hs, v.Ws, wins)
    assert np.array_equal(rinf.cpu().numpy(), O.timeripple_reuse(D, (np.inf,) * 3))
    # reuse alone (no delta, no score) is the same as with them
    r1, _, _ = tps.timeripple_score(xd, v.F, v.Hs, v.Ws, wins, synth.TR_THETA)
    r2, _, _ = tps.timeripple_score(xd, v.F, v.Hs, v.Ws, wins, synth.TR_THETA, delta=True, score=True)
    assert torch.equal(r1, r2)
    tps.tps_check()


def test_timeripple_hsa_size_sampled():
    """Full HSA size (33 x 45 x 80 tokens, 24 heads, d = 128) in the launch the
    bench times; the oracle checks crops, whose inner tokens have all their
    neighbours inside the crop."""
    cfg = synth.CONFIGS["hsa"]
    v = cfg.video
    F, Hs, Ws, H, d = v.F, v.Hs, v.Ws, cfg.H, cfg.d
    g = torch.Generator().manual_seed(9)
    base = torch.randn((1, Hs, Ws, H, d), generator=g)
    x = (base + 0.01 * torch.randn((F, Hs, Ws, H, d), generator=g)).to(torch.bfloat16)
    x[:, 20:28, 30:46] = torch.randn((F, 8, 16, H, d), generator=g).to(torch.bfloat16)   # a changing block
    wins = synth.timeripple_windows(d)
    reuse, delta, score = tps.timeripple_score(x.reshape(-1, H, d).to(DEV), F, Hs, Ws, wins, synth.TR_THETA,
                                               delta=True, score=True)
    tps.tps_check()
    r = reuse.cpu().numpy().reshape(F, Hs, Ws, H)
    gd = delta.cpu().double().numpy().reshape(3, F, Hs, Ws, H)
    sc = score.cpu().numpy().reshape(F, Hs, Ws)
    tol = _tol(d)
    # crops: corners, tile seams (rows 8k, columns 16k), the changing block, run seams in f
    for (fa, fb), (ya, yb), (xa, xb) in (((0, 3), (0, 10), (0, 20)), ((30, 33), (36, 45), (60, 80)),
                                         ((10, 14), (6, 18), (14, 50)), ((15, 19), (19, 29), (29, 47)),
                                         ((21, 25), (39, 45), (0, 18))):
        crop = x[fa:fb, ya:yb, xa:xb].reshape(-1, H, d)
        D = O.timeripple_delta(crop, fb - fa, yb - ya, xb - xa, wins).reshape(3, fb - fa, yb - ya, xb - xa, H)
        # inner tokens: the neighbour on every axis lies in the crop (or does not exist globally)
        fi = 1 if fa > 0 else 0
        yi = 1 if ya > 0 else 0
        xi = 1 if xa > 0 else 0
        Di = D[:, fi:, yi:, xi:]
        Gi = gd[:, fa + fi:fb, ya + yi:yb, xa + xi:xb]
        assert np.array_equal(np.isinf(Gi), np.isinf(Di))
        fin = np.isfinite(Di)
        np.testing.assert_allclose(Gi[fin], Di[fin], rtol=tol, atol=0)
        ref_bits = O.timeripple_reuse(Di.reshape(3, -1, H), synth.TR_THETA).reshape(Di.shape[1:])
        assert np.array_equal(r[fa + fi:fb, ya + yi:yb, xa + xi:xb], ref_bits)
        assert np.array_equal(sc[fa + fi:fb, ya + yi:yb, xa + xi:xb], (ref_bits == 0).sum(-1).astype(np.float32))
    # properties that hold everywhere: bits agree with the reported Delta; t never passes on frame 0
    th = np.asarray(synth.TR_THETA, np.float32)
    own = sum(((gd[a].astype(np.float32) < th[a]).astype(np.uint8) << a) for a in range(3))
    assert np.array_equal(r, own)
    assert np.isinf(gd[0, 0]).all() and np.isinf(gd[1, :, :, 0]).all() and np.isinf(gd[2, :, 0]).all()
    assert np.array_equal(sc, (r == 0).sum(-1).astype(np.float32))
