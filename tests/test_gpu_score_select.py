"""GPU parity: lipar_score, lipar_select, lipar_group, lipar_schedule vs the
fp64 oracle, through the C ABI (ctypes binding)."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from token_pruned_sparse_b200 import synth
from token_pruned_sparse_b200 import tps

from workloads import frame_case, oracle_idx, step_case

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _rtol(C):
    # fp32 sums of C terms from exact bf16 inputs, then one division
    return 4 * C * 2.0 ** -24


def _idx(idx, count):
    n = int(count.item())
    return idx[:n].cpu().numpy()


# ---------------------------------------------------------------- score -----
@pytest.mark.parametrize("name", ["tiny", "mid", "block"])
def test_score_interframe(name):
    cfg, xb, _ = frame_case(name)
    s = tps.lipar_score(xb.to(DEV)).cpu().numpy()
    ref = O.lipar_score(xb)
    assert np.array_equal(np.isinf(s), np.isinf(ref))
    fin = np.isfinite(ref)
    np.testing.assert_allclose(s[fin], ref[fin], rtol=_rtol(cfg.video.C), atol=0)


@pytest.mark.parametrize("name", ["wan", "hsa"])
def test_score_interstep(name):
    cfg, vpb, vc, _ = step_case(name)
    F, HW, C = cfg.video.F, cfg.video.HW, cfg.video.C
    s = tps.lipar_score(vc.reshape(F, HW, C).to(DEV), vpb.reshape(F, HW, C).to(DEV)).cpu().numpy()
    ref = O.lipar_score(vc[None], vpb[None])
    np.testing.assert_allclose(s, ref, rtol=_rtol(C), atol=0)


def test_score_prev_frame_zero_change_and_edges():
    x = synth.gaussian_bf16((5, 37, 24), 7)
    same = x[:1].expand(5, 37, 24).contiguous()
    s = tps.lipar_score(same.to(DEV), x_prev_frame=same[0].to(DEV)).cpu().numpy()
    assert not s.any()                                        # zero change -> all 0
    idx, cnt = tps.lipar_select(torch.from_numpy(s).to(DEV), tps.SELECT_THRESHOLD, tau=1e-6)
    assert int(cnt.item()) == 0
    # den = 0 rules and ragged C = 8
    z = torch.zeros((1, 3, 8), dtype=torch.bfloat16)
    cur = z.clone()
    cur[0, 1, 3] = 1.0
    s = tps.lipar_score(cur.to(DEV), z.to(DEV)).cpu().numpy()
    assert s[0] == 0 and s[1] == math.inf and s[2] == 0
    for C in (8, 16, 40, 64, 200):
        a = synth.gaussian_bf16((3, 11, C), C)
        b = synth.gaussian_bf16((3, 11, C), C + 1)
        np.testing.assert_allclose(tps.lipar_score(a.to(DEV), b.to(DEV)).cpu().numpy(),
                                   O.lipar_score(a, b), rtol=_rtol(C))
        np.testing.assert_allclose(tps.lipar_score(a.to(DEV), x_prev_frame=b[0].to(DEV)).cpu().numpy(),
                                   O.lipar_score(a, x_prev_frame=b[0]), rtol=_rtol(C))


# --------------------------------------------------------------- select -----
@pytest.mark.parametrize("N", [1, 7, 1023, 1024, 1025, 5000, 20280, 32768, 32769, 118800, 300001])
@pytest.mark.parametrize("ties", [False, True])
def test_select_threshold_and_topk(N, ties):
    s = synth.random_scores(N, N + int(ties), ties=ties, specials=True)
    sd = s.to(DEV)
    for tau in (0.0, 0.5, 1.0, math.inf):
        idx, cnt = tps.lipar_select(sd, tps.SELECT_THRESHOLD, tau=tau)
        assert np.array_equal(_idx(idx, cnt), O.select_threshold(s.numpy(), tau))
    for k in sorted({0, 1, N // 3, N // 2, N - 1, N} - {-1}):
        idx, cnt = tps.lipar_select(sd, tps.SELECT_TOPK, k=k)
        assert int(cnt.item()) == k
        assert np.array_equal(_idx(idx, cnt), O.select_topk(s.numpy(), k)), (N, k)


def test_select_special_values():
    s = torch.tensor([math.nan, -0.0, 0.0, 1.0, -math.inf, math.inf, -2.0, math.nan], dtype=torch.float32)
    for k in range(9):
        idx, cnt = tps.lipar_select(s.to(DEV), tps.SELECT_TOPK, k=k)
        assert np.array_equal(_idx(idx, cnt), O.select_topk(s.numpy(), k)), k
    idx, cnt = tps.lipar_select(s.to(DEV), tps.SELECT_THRESHOLD, tau=0.0)
    assert np.array_equal(_idx(idx, cnt), O.select_threshold(s.numpy(), 0.0))
    allsame = torch.full((3000,), 0.25)
    idx, cnt = tps.lipar_select(allsame.to(DEV), tps.SELECT_TOPK, k=1234)
    assert np.array_equal(_idx(idx, cnt), np.arange(1234))


@pytest.mark.parametrize("name", ["tiny", "mid", "block"])
def test_pipeline_interframe_bit_exact(name):
    cfg, xb, k = frame_case(name)
    s = tps.lipar_score(xb.to(DEV))
    if k is None:
        idx, cnt = tps.lipar_select(s, tps.SELECT_THRESHOLD, tau=cfg.tau)
    else:
        idx, cnt = tps.lipar_select(s, tps.SELECT_TOPK, k=k)
    assert np.array_equal(_idx(idx, cnt), oracle_idx(name))


def test_pipeline_interstep_keep_sweep():
    cfg, vpb, vc, _ = step_case("wan")
    F, HW, C = cfg.video.F, cfg.video.HW, cfg.video.C
    s = tps.lipar_score(vc.reshape(F, HW, C).to(DEV), vpb.reshape(F, HW, C).to(DEV))
    for i, r in enumerate(cfg.keep):
        k = synth.keep_count(cfg.video.N, r)
        idx, cnt = tps.lipar_select(s, tps.SELECT_TOPK, k=k)
        assert np.array_equal(_idx(idx, cnt), oracle_idx("wan", i))


# ---------------------------------------------------------- HSA groups -----
def test_group_and_schedule_hsa():
    cfg, vpb, vc, _ = step_case("hsa")
    F, HW, C = cfg.video.F, cfg.video.HW, cfg.video.C
    K, T, budgets = cfg.extra["K"], cfg.extra["T"], cfg.extra["budgets"]
    s = tps.lipar_score(vc.reshape(F, HW, C).to(DEV), vpb.reshape(F, HW, C).to(DEV))
    g = tps.lipar_group(s, K)
    g_ref = O.group_split(O.lipar_score(vc[None], vpb[None]), K)
    assert np.array_equal(g.cpu().numpy(), g_ref)
    for m in (0, 3):
        for step in range(T):
            idx, cnt = tps.lipar_schedule(g, K, budgets, T, step, m)
            assert np.array_equal(_idx(idx, cnt), O.schedule_active(g_ref, K, budgets, T, step, m)), (m, step)


@pytest.mark.parametrize("N,K", [(7, 3), (1000, 1), (1000, 2), (4097, 5), (50000, 8), (7, 7)])
def test_group_random_with_ties(N, K):
    s = synth.random_scores(N, 100 + K, ties=True, specials=True)
    g = tps.lipar_group(s.to(DEV), K).cpu().numpy()
    assert np.array_equal(g, O.group_split(s.numpy(), K))
    budgets = [12] + [12 // (2 ** min(i, 2)) for i in range(1, K)]
    gd = torch.from_numpy(g).to(DEV)
    for step in range(12):
        idx, cnt = tps.lipar_schedule(gd, K, budgets, 12, step, 1)
        assert np.array_equal(_idx(idx, cnt), O.schedule_active(g, K, budgets, 12, step, 1))


def test_schedule_ignores_out_of_range_groups():
    g = torch.tensor([0, 1, 2, -1, 5, 1, 0, 127], dtype=torch.int8)
    idx, cnt = tps.lipar_schedule(g.to(DEV), 3, [4, 2, 1], 4, 0, 0)
    assert np.array_equal(_idx(idx, cnt), O.schedule_active(g.numpy(), 3, [4, 2, 1], 4, 0, 0))


# -------------------------------------------------- motion-robust score -----
@pytest.mark.parametrize("name", ["tiny", "mid", "block"])
@pytest.mark.parametrize("L", [1, 3, 8])
def test_score_motion(name, L):
    cfg, xb, _ = frame_case(name)
    s = tps.lipar_score_motion(xb.to(DEV), L).cpu().numpy()
    ref = O.lipar_score_motion(xb, L)
    assert np.array_equal(np.isinf(s), np.isinf(ref))
    fin = np.isfinite(ref)
    np.testing.assert_allclose(s[fin], ref[fin], rtol=_rtol(cfg.video.C), atol=0)


@pytest.mark.parametrize("N", [1000, 118800, 600000])
def test_select_multi_launch_path_matches_oracle(N):
    """The multi-launch path (taken with the minimum workspace, and for N beyond
    one cooperative launch) gives the oracle's lists too."""
    s = synth.random_scores(N, 77 + N, ties=True, specials=True)
    sd = s.to(DEV)
    sn = s.numpy()
    for ws in (tps.workspace(tps.OP_SELECT, N, 0, DEV, minimal=True), tps.workspace(tps.OP_SELECT, N, 0, DEV)):
        for k in (0, 1, N // 7, N // 2, N):
            idx, cnt = tps.lipar_select(sd, tps.SELECT_TOPK, k=k, ws=ws)
            assert np.array_equal(_idx(idx, cnt), O.select_topk(sn, k)), (N, k, ws.numel())
        for tau in (0.25, 1.0):
            idx, cnt = tps.lipar_select(sd, tps.SELECT_THRESHOLD, tau=tau, ws=ws)
            assert np.array_equal(_idx(idx, cnt), O.select_threshold(sn, tau)), (N, tau, ws.numel())
    tps.tps_check()


@pytest.mark.parametrize("N,K", [(1000, 2), (118800, 3), (600000, 4)])
def test_group_cooperative_and_multi_launch_paths(N, K):
    """lipar_group runs as one cooperative launch with the recommended
    workspace (N within one launch) and as the multi-launch radix path with the
    minimum workspace; both equal the oracle's rank split, ties included."""
    s = synth.random_scores(N, 300 + N, ties=True, specials=True)
    ref = O.group_split(s.numpy(), K)
    sd = s.to(DEV)
    for ws in (tps.workspace(tps.OP_GROUP, N, K, DEV), tps.workspace(tps.OP_GROUP, N, K, DEV, minimal=True)):
        g = tps.lipar_group(sd, K, ws=ws).cpu().numpy()
        assert np.array_equal(g, ref), ws.numel()
    tps.tps_check()


# ------------------------------------------------- fused front end ----------
@pytest.mark.parametrize("name", ["tiny", "mid", "block"])
def test_front_interframe_matches_separate_stages(name):
    """lipar_front = lipar_score + lipar_select: the same scores bit for bit
    and the oracle's index list."""
    cfg, xb, k = frame_case(name)
    x = xb.to(DEV)
    ref_s = tps.lipar_score(x).cpu()
    s = torch.full((cfg.video.N,), 7.0, device=DEV)
    if k is None:
        idx, cnt = tps.lipar_front(x, tps.FRONT_THRESHOLD, tau=cfg.tau, score=s)
    else:
        idx, cnt = tps.lipar_front(x, tps.FRONT_TOPK, k=k, score=s)
    assert torch.equal(s.cpu(), ref_s)
    assert np.array_equal(_idx(idx, cnt), oracle_idx(name))
    tps.tps_check()


def test_front_interstep_keep_sweep_and_hsa_groups():
    cfg, vpb, vc, _ = step_case("wan")
    F, HW, C = cfg.video.F, cfg.video.HW, cfg.video.C
    cur, prev = vc.reshape(F, HW, C).to(DEV), vpb.reshape(F, HW, C).to(DEV)
    ws = tps.workspace(tps.OP_FRONT, cfg.video.N, 0, DEV)
    for i, r in enumerate(cfg.keep):
        k = synth.keep_count(cfg.video.N, r)
        idx, cnt = tps.lipar_front(cur, tps.FRONT_TOPK, x_ref=prev, k=k, ws=ws)
        assert np.array_equal(_idx(idx, cnt), oracle_idx("wan", i))
    cfg, vpb, vc, _ = step_case("hsa")
    F, HW, C = cfg.video.F, cfg.video.HW, cfg.video.C
    K = cfg.extra["K"]
    cur, prev = vc.reshape(F, HW, C).to(DEV), vpb.reshape(F, HW, C).to(DEV)
    s = torch.empty(cfg.video.N, device=DEV)
    g = tps.lipar_front(cur, tps.FRONT_GROUP, x_ref=prev, K=K, score=s).cpu().numpy()
    assert torch.equal(s.cpu(), tps.lipar_score(cur, prev).cpu())
    assert np.array_equal(g, O.group_split(O.lipar_score(vc[None], vpb[None]), K))
    tps.tps_check()


@pytest.mark.parametrize("F,HW,C", [(3, 700, 64), (2, 70000, 128), (5, 130000, 128), (4, 33, 96)])
def test_front_sizes_prev_frame_and_fallback(F, HW, C):
    """Both cooperative tilings (N <= 131072 and larger), the separate-kernel
    path (N beyond one cooperative launch, or C outside {64, 128}), the
    streaming case with a previous frame, and zero change."""
    x = synth.gaussian_bf16((F, HW, C), F * HW + C)
    prev = synth.gaussian_bf16((HW, C), 5)
    N = F * HW
    xd, pd = x.to(DEV), prev.to(DEV)
    for xp in (None, pd):
        s_ref = tps.lipar_score(xd, x_prev_frame=xp)
        for k in (1, N // 3, N):
            idx, cnt = tps.lipar_front(xd, tps.FRONT_TOPK, x_prev_frame=xp, k=k)
            ridx, rcnt = tps.lipar_select(s_ref, tps.SELECT_TOPK, k=k)
            n = int(rcnt.item())
            assert int(cnt.item()) == n and torch.equal(idx[:n], ridx[:n]), (xp is None, k)
        idx, cnt = tps.lipar_front(xd, tps.FRONT_THRESHOLD, x_prev_frame=xp, tau=1.0)
        ridx, rcnt = tps.lipar_select(s_ref, tps.SELECT_THRESHOLD, tau=1.0)
        n = int(rcnt.item())
        assert int(cnt.item()) == n and torch.equal(idx[:n], ridx[:n])
        for K in (1, 3):
            g = tps.lipar_front(xd, tps.FRONT_GROUP, x_prev_frame=xp, K=K)
            assert torch.equal(g, tps.lipar_group(s_ref, K))
    same = x[:1].expand(F, HW, C).contiguous().to(DEV)
    idx, cnt = tps.lipar_front(same, tps.FRONT_THRESHOLD, x_prev_frame=same[0], tau=1e-6)
    assert int(cnt.item()) == 0
    tps.tps_check()
