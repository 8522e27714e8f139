"""GPU parity: pruned attention (tcgen05 kernel and the legacy mma.sync
baseline) vs the fp64 oracle, through the C ABI; plus the whole per-layer path
on the configs, at full size with sampled rows."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from token_pruned_sparse_b200 import synth
from token_pruned_sparse_b200 import tps

from workloads import attn_tolerance_ok, frame_case, oracle_idx, qkv, step_case

pytestmark = pytest.mark.gpu
DEV = "cuda"
IMPLS = ["pruned_attn", "pruned_attn_mma", "pruned_attn_pair"]


def _supported(impl, d, bm):
    """pruned_attn_pair takes dense attention with d = 128 only."""
    if impl == "pruned_attn_pair" and (d != 128 or bm is not None):
        pytest.skip("pruned_attn_pair: dense d = 128 only")


def _run(impl, q, k, v, idx, scale, bm=None, with_lse=True, count=None, cap=None):
    _supported(impl, q.shape[-1], bm)
    fn = getattr(tps, impl)
    qd = q.to(DEV)
    di = torch.from_numpy(np.asarray(idx, np.int32)).to(DEV) if len(idx) else torch.zeros(1, dtype=torch.int32, device=DEV)
    dc = torch.tensor([len(idx) if count is None else count], dtype=torch.int32, device=DEV)
    cap = q.shape[0] if cap is None else cap
    o = torch.full_like(qd, 7.0)
    lse = torch.full((max(q.shape[0], 1), q.shape[1]), 7.0, device=DEV) if with_lse else None
    fn(qd, k.to(DEV), v.to(DEV), di, dc, scale, blockmask=None if bm is None else bm.to(DEV),
       o_act=o, lse=lse, cap=cap)
    tps.tps_check()
    return o.cpu(), (lse.cpu().numpy() if with_lse else None)


def _check(o_gpu, lse_gpu, o_ref, lse_ref, rows=None, v_absmax=None):
    """v_absmax (stress cases with score spikes): the largest |v| per head.
    Such spikes make single keys dominate, |o| reaches the size of |v| (4 and
    more), and the bound that the kernel's arithmetic fixes -- probabilities in
    bf16 (relative error <= 2^-8 each, so <= 2^-8 max|v| in o) plus the bf16
    output (<= 2^-9 |o|) -- exceeds the absolute 2e-2; those rows are held
    to that bound (mean-abs stays <= 2e-3)."""
    g = o_gpu.double().numpy()
    if rows is not None:
        g = g[rows]
        lse_gpu = None if lse_gpu is None else lse_gpu[rows]
    if v_absmax is None:
        ok, info = attn_tolerance_ok(g, o_ref)
        assert ok, info
    else:
        err = np.abs(g - o_ref)
        bound = np.maximum(2e-2, 2.0 ** -8 * np.asarray(v_absmax)[None, :, None] + 2.0 ** -9 * np.abs(o_ref) + 1e-4)
        assert np.all(err <= bound) and err.mean() <= 2e-3, dict(max_abs=float(err.max()), mean_abs=float(err.mean()))
    if lse_gpu is not None:
        fin = np.isfinite(lse_ref)
        assert np.array_equal(np.isneginf(lse_gpu), np.isneginf(lse_ref))
        np.testing.assert_allclose(lse_gpu[fin], lse_ref[fin], rtol=0, atol=2e-3)


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("N,A,H,d", [(256, 256, 2, 64), (300, 113, 2, 64), (517, 131, 3, 128), (1000, 1, 1, 128),
                                     (129, 129, 4, 128), (4099, 700, 2, 64), (2000, 1999, 1, 128)])
@pytest.mark.parametrize("sharp", [False, True])
def test_attn_random_dense(impl, N, A, H, d, sharp):
    q = synth.gaussian_bf16((A, H, d), N + A)
    k = synth.gaussian_bf16((N, H, d), N + A + 1)
    v = synth.gaussian_bf16((N, H, d), N + A + 2)
    idx = np.sort(np.random.default_rng(A).choice(N, A, replace=False))
    scale = (0.35 if sharp else 1.0 / math.sqrt(d))
    o, lse = _run(impl, q, k, v, idx, scale)
    o_ref, lse_ref = O.pruned_attn(q, k, v, idx, scale)
    _check(o, lse, o_ref, lse_ref)


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("growth", ["rising", "falling", "spike", "spike_lo", "spike_hi"])
def test_attn_running_max_moves(impl, growth):
    """Score scales that change along the keys: rising makes later key tiles
    dominate (tile sums far above 2^40 against the first tile's maximum, so the
    kernel must take the slow path, find the new maximum and rescale O);
    falling keeps the first tile's maximum; spike puts one huge tile mid-way;
    spike_lo / spike_hi put it on keys 0-63 / 64-127 of that tile only."""
    N, A, H, d = 1500, 200, 2, 128
    q = synth.gaussian_bf16((A, H, d), 11)
    k = synth.gaussian_bf16((N, H, d), 12).double()
    pos = torch.arange(N, dtype=torch.float64)[:, None, None] / N
    if growth == "rising":
        g = 1.0 + 24.0 * pos
    elif growth == "falling":
        g = 25.0 - 24.0 * pos
    else:
        g = torch.ones_like(pos)
        lo, hi = {"spike": (640, 768), "spike_lo": (640, 704), "spike_hi": (704, 768)}[growth]
        g[lo:hi] = 30.0
    k = (k * g).to(torch.bfloat16)
    v = synth.gaussian_bf16((N, H, d), 13)
    idx = np.sort(np.random.default_rng(5).choice(N, A, replace=False))
    scale = 1.0 / math.sqrt(d)
    o, lse = _run(impl, q, k, v, idx, scale)
    o_ref, lse_ref = O.pruned_attn(q, k, v, idx, scale)
    _check(o, lse, o_ref, lse_ref, v_absmax=v.double().abs().amax(dim=(0, 2)).numpy())


@pytest.mark.parametrize("impl", IMPLS)
def test_attn_constant_keys_mean_of_v(impl):
    N, H, d = 1500, 2, 128
    k = synth.gaussian_bf16((1, H, d), 1).expand(N, H, d).contiguous()
    v = synth.gaussian_bf16((N, H, d), 2)
    q = synth.gaussian_bf16((200, H, d), 3)
    o, _ = _run(impl, q, k, v, np.arange(200), 0.2)
    mean_v = v.double().mean(0).numpy()
    ok, info = attn_tolerance_ok(o.double().numpy(), np.broadcast_to(mean_v, (200, H, d)))
    assert ok, info


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("N,A", [(1000, 400), (1100, 1100), (129, 60)])
def test_attn_blockmask(impl, N, A):
    H, d = 2, 128
    q = synth.gaussian_bf16((A, H, d), 10)
    k = synth.gaussian_bf16((N, H, d), 11)
    v = synth.gaussian_bf16((N, H, d), 12)
    idx = np.sort(np.random.default_rng(13).choice(N, A, replace=False))
    nb = -(-N // 128)
    bm = torch.from_numpy((np.random.default_rng(14).random((nb, nb)) < 0.35).astype(np.uint8))
    bm[np.arange(nb), np.arange(nb)] = 1
    bm[idx[A // 2] // 128] = 0                     # one query block keeps nothing
    o, lse = _run(impl, q, k, v, idx, 0.3, bm=bm)
    o_ref, lse_ref = O.pruned_attn(q, k, v, idx, 0.3, blockmask=bm)
    _check(o, lse, o_ref, lse_ref)


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("d", [64, 128])
def test_attn_blockmask_query_block_edges(impl, d):
    """Masked mode runs one tile per original query block: full blocks (128
    active rows), single-row and empty blocks, key lists of very different
    lengths within one CTA (all blocks vs one), a block whose row keeps nothing,
    an odd number of blocks (the last CTA has one tile), a running-max spike in
    a kept tile, and a count below cap (rows past the count stay untouched)."""
    N, H = 2000, 2                                          # nb = 16
    rng = np.random.default_rng(40 + d)
    sel = [np.arange(0, 128), np.array([130]), np.arange(384, 512), np.arange(512, 640, 3),
           np.array([700, 701, 830]), np.arange(1920, 2000)]
    idx = np.unique(np.concatenate(sel + [rng.choice(np.arange(896, 1900), 300, replace=False)]))
    A = len(idx)
    q = synth.gaussian_bf16((A, H, d), 41)
    k = synth.gaussian_bf16((N, H, d), 42).double()
    k[1000:1100] *= 20.0                                    # spike inside key block 7
    k = k.to(torch.bfloat16)
    v = synth.gaussian_bf16((N, H, d), 43)
    nb = -(-N // 128)
    bm = torch.from_numpy((rng.random((nb, nb)) < 0.3).astype(np.uint8))
    bm[0] = 1                                               # block 0 keeps every key block
    bm[1] = 0
    bm[1, 15] = 1                                           # block 1 keeps only the ragged last one
    bm[3] = 0                                               # block 3 keeps nothing
    bm[:, 7] = 1
    vmax = v.double().abs().amax(dim=(0, 2)).numpy()
    o, lse = _run(impl, q, k, v, idx, 1 / math.sqrt(d), bm=bm)
    o_ref, lse_ref = O.pruned_attn(q, k, v, idx, 1 / math.sqrt(d), blockmask=bm)
    _check(o, lse, o_ref, lse_ref, v_absmax=vmax)
    c = A - 77
    o, lse = _run(impl, q, k, v, idx, 1 / math.sqrt(d), bm=bm, count=c)
    o_ref, lse_ref = O.pruned_attn(q, k, v, idx, 1 / math.sqrt(d), blockmask=bm, rows=np.arange(c))
    _check(o[:c], lse[:c], o_ref, lse_ref, v_absmax=vmax)
    assert torch.all(o[c:].float() == 7.0) and np.all(lse[c:] == 7.0)


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("d", [64, 128])
def test_attn_blockmask_unit_edges_and_rescales(impl, d):
    """Masked mode at the row counts where a query block's run splits into
    units of 64 (d = 128: 63, 64, 65 and 128 active rows, one row, none, and
    17 in the ragged last block), with keys that grow block by block (x(1 + 4 kb))
    so that later key tiles push the exponent arguments past the running
    references again and again (the rescale path, repeatedly, in both kernels)."""
    nb_full, tail = 6, 40
    N, H = 128 * nb_full + tail, 2
    rng = np.random.default_rng(70 + d)
    runs = {0: 64, 1: 65, 2: 63, 3: 128, 4: 1, 5: 0, 6: 17}
    idx = np.concatenate([np.sort(rng.choice(np.arange(128 * b, min(N, 128 * b + 128)), n, replace=False))
                          for b, n in runs.items() if n > 0])
    A = len(idx)
    q = synth.gaussian_bf16((A, H, d), 71)
    k = synth.gaussian_bf16((N, H, d), 72).double()
    ramp = 1.0 + 4.0 * (np.arange(N) // 128)
    k = (k * torch.from_numpy(ramp)[:, None, None]).to(torch.bfloat16)
    v = synth.gaussian_bf16((N, H, d), 73)
    nb = -(-N // 128)
    bm = torch.from_numpy((rng.random((nb, nb)) < 0.5).astype(np.uint8))
    bm[np.arange(nb), np.arange(nb)] = 1
    bm[3] = 1                                                   # the 128-row block keeps every key block
    vmax = v.double().abs().amax(dim=(0, 2)).numpy()
    o, lse = _run(impl, q, k, v, idx, 1 / math.sqrt(d), bm=bm)
    o_ref, lse_ref = O.pruned_attn(q, k, v, idx, 1 / math.sqrt(d), blockmask=bm)
    _check(o, lse, o_ref, lse_ref, v_absmax=vmax)
    o2, _ = _run(impl, q, k, v, idx, 1 / math.sqrt(d), bm=bm, with_lse=False)   # no log-sum-exp output
    assert torch.equal(o2, o)


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("d", [64, 128])
def test_attn_count_below_cap_leaves_tail(impl, d):
    N, A, H = 700, 300, 2
    q = synth.gaussian_bf16((A, H, d), 20)
    k = synth.gaussian_bf16((N, H, d), 21)
    v = synth.gaussian_bf16((N, H, d), 22)
    idx = np.arange(0, 600, 2)
    o, lse = _run(impl, q, k, v, idx, 0.125, count=150)
    o_ref, lse_ref = O.pruned_attn(q, k, v, idx, 0.125, rows=np.arange(150))
    _check(o[:150], lse[:150], o_ref, lse_ref)
    assert torch.all(o[150:].float() == 7.0) and np.all(lse[150:] == 7.0)
    o0, _ = _run(impl, q, k, v, idx, 0.125, count=0)
    assert torch.all(o0.float() == 7.0)


# ------------------------------------------------------ whole per-layer path ---
def _layer(impl, k_cache, v_cache, q_full, k_full, v_full, o_cache, idx_d, cnt_d, cap, scale, bm=None, renoise=None):
    _supported(impl, q_full.shape[-1], bm)
    """gather -> kv_sync -> attention -> scatter on the device."""
    H, d = q_full.shape[1], q_full.shape[2]
    q_act = torch.empty((cap, H, d), dtype=torch.bfloat16, device=DEV)
    k_new = torch.empty_like(q_act)
    v_new = torch.empty_like(q_act)
    tps.tps_gather_rows(q_act, q_full, idx_d, cnt_d, cap=cap)
    tps.tps_gather_rows(k_new, k_full, idx_d, cnt_d, cap=cap)
    tps.tps_gather_rows(v_new, v_full, idx_d, cnt_d, cap=cap)
    ke, ve = tps.kv_sync(k_cache, v_cache, k_new, v_new, idx_d, cnt_d, cap=cap, renoise=renoise)
    kk, vv = (k_cache, v_cache) if renoise is None else (ke, ve)
    o_act = torch.empty_like(q_act)
    lse = torch.empty((cap, H), dtype=torch.float32, device=DEV)
    getattr(tps, impl)(q_act, kk, vv, idx_d, cnt_d, scale, blockmask=bm, o_act=o_act, lse=lse, cap=cap)
    tps.scatter_out(o_cache, o_act, idx_d, cnt_d, cap=cap)
    tps.tps_check()
    return o_act, lse, kk, vv


@pytest.mark.parametrize("impl", IMPLS)
def test_path_tiny_full(impl):
    """tiny: threshold 0.2 on inter-frame scores, every output row checked."""
    cfg, xb, _ = frame_case("tiny")
    Q, K, V = qkv("tiny")
    N, H, d = Q.shape
    kc = synth.gaussian_bf16((N, H, d), 90)
    vc = synth.gaussian_bf16((N, H, d), 91)
    oc = synth.gaussian_bf16((N, H, d), 92)
    s = tps.lipar_score(xb.to(DEV))
    idx_d, cnt_d = tps.lipar_select(s, tps.SELECT_THRESHOLD, tau=cfg.tau)
    A = int(cnt_d.item())
    idx = oracle_idx("tiny")
    assert A == len(idx) and np.array_equal(idx_d[:A].cpu().numpy(), idx)
    kcd, vcd, ocd = kc.to(DEV), vc.to(DEV), oc.to(DEV)
    o_act, lse, _, _ = _layer(impl, kcd, vcd, Q.to(DEV), K.to(DEV), V.to(DEV), ocd, idx_d, cnt_d, N, 1 / math.sqrt(d))
    k2, v2, _, _ = O.kv_sync(kc, vc, K[idx], V[idx], idx)
    assert torch.equal(kcd.cpu(), k2) and torch.equal(vcd.cpu(), v2)
    o_ref, lse_ref = O.pruned_attn(Q[idx], k2, v2, idx, 1 / math.sqrt(d))
    _check(o_act[:A].cpu(), lse[:A].cpu().numpy(), o_ref, lse_ref)
    out = ocd.cpu()
    rest = np.setdiff1d(np.arange(N), idx)
    assert torch.equal(out[rest], oc[rest]) and torch.equal(out[idx], o_act[:A].cpu())


def _sample(A, n, seed):
    r = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, A - 1], r.choice(A, min(n, A), replace=False)]))


@pytest.mark.parametrize("impl", IMPLS)
def test_path_mid_topk_sampled(impl):
    """mid: top-k 30% of inter-frame scores; cached K/V = previous frame's
    projection; 384 sampled active rows x all heads vs the oracle."""
    cfg, xb, k = frame_case("mid")
    Q, K, V = qkv("mid")
    N, H, d = Q.shape
    HW = cfg.video.HW
    kc = torch.cat([K[:HW], K[:-HW]])            # previous frame's projection
    vc = torch.cat([V[:HW], V[:-HW]])
    oc = synth.gaussian_bf16((N, H, d), 93)
    s = tps.lipar_score(xb.to(DEV))
    idx_d, cnt_d = tps.lipar_select(s, tps.SELECT_TOPK, k=k)
    idx = oracle_idx("mid")
    assert np.array_equal(idx_d[:k].cpu().numpy(), idx)
    kcd, vcd, ocd = kc.to(DEV), vc.to(DEV), oc.to(DEV)
    o_act, lse, kk, vv = _layer(impl, kcd, vcd, Q.to(DEV), K.to(DEV), V.to(DEV), ocd, idx_d, cnt_d, k, 1 / math.sqrt(d))
    k2, v2, _, _ = O.kv_sync(kc, vc, K[idx], V[idx], idx)
    assert torch.equal(kcd.cpu(), k2) and torch.equal(vcd.cpu(), v2)
    rows = _sample(k, 384, 1)
    o_ref, lse_ref = O.pruned_attn(Q[idx], k2, v2, idx, 1 / math.sqrt(d), rows=rows)
    _check(o_act.cpu(), lse.cpu().numpy(), o_ref, lse_ref, rows=rows)


@pytest.mark.parametrize("impl", IMPLS)
def test_wan_keep100_is_dense_sampled(impl):
    """Wan-like layer at keep 100%: pruned attention == dense attention."""
    Q, K, V = qkv("wan")
    N, H, d = Q.shape
    idx = np.arange(N)
    o, lse = _run(impl, Q, K, V, idx, 1 / math.sqrt(d))
    rows = _sample(N, 256, 2)
    o_ref, lse_ref = O.pruned_attn(Q, K, V, idx, 1 / math.sqrt(d), rows=rows)
    _check(o, lse, o_ref, lse_ref, rows=rows)


@pytest.mark.parametrize("impl", IMPLS)
def test_block_sparse_config_sampled(impl):
    """block-sparse: 118800 tokens, 40% active queries, 139/929 key blocks
    kept per query block; sampled rows vs the oracle."""
    cfg, xb, k = frame_case("block")
    Q, K, V = qkv("block")
    N, H, d = Q.shape
    bm = synth.block_mask_band_random(cfg.video, 128, cfg.extra["kept_per_row"], cfg.video.seed)
    assert int(bm.sum(1).min()) == int(bm.sum(1).max()) == 139
    idx = oracle_idx("block")
    assert len(idx) == 47520
    o, lse = _run(impl, Q[idx], K, V, idx, 1 / math.sqrt(d), bm=bm)
    rows = _sample(len(idx), 160, 3)
    o_ref, lse_ref = O.pruned_attn(Q[idx], K, V, idx, 1 / math.sqrt(d), blockmask=bm, rows=rows)
    _check(o, lse, o_ref, lse_ref, rows=rows)


@pytest.mark.parametrize("impl", IMPLS)
def test_hsa_steps_with_renoise_sampled(impl):
    """HSA at full size: groups from the inter-step score, per-step active sets
    (steps 0, 1, 2 give |A| = N, N/3, 2N/3), re-noised pruned rows
    (a = 1 - sigma, b = sigma). Checked: bit-exact caches and index lists, the
    re-noised K/V of three heads over all rows, and sampled attention rows of
    those heads against the oracle's own fp64 K_eff / V_eff."""
    cfg, vpb, vc, _ = step_case("hsa")
    F, HW, C = cfg.video.F, cfg.video.HW, cfg.video.C
    K_, T, budgets = cfg.extra["K"], cfg.extra["T"], cfg.extra["budgets"]
    Q, Kp, Vp = qkv("hsa")
    N, H, d = Q.shape
    heads = np.array([0, 11, 23])
    s = tps.lipar_score(vc.reshape(F, HW, C).to(DEV), vpb.reshape(F, HW, C).to(DEV))
    g = tps.lipar_group(s, K_)
    g_ref = O.group_split(O.lipar_score(vc[None], vpb[None]), K_)
    assert np.array_equal(g.cpu().numpy(), g_ref)
    kcd, vcd = Kp.to(DEV), Vp.to(DEV)          # step 0 fills the cache
    kc, vc_ = Kp.clone(), Vp.clone()
    ocd = torch.zeros((N, H, d), dtype=torch.bfloat16, device=DEV)
    Qd, Kd, Vd = Q.to(DEV), Kp.to(DEV), Vp.to(DEV)
    for step in (0, 1, 2):
        sigma = 1.0 - step / T
        idx_d, cnt_d = tps.lipar_schedule(g, K_, budgets, T, step, 0)
        idx = O.schedule_active(g_ref, K_, budgets, T, step, 0)
        A = int(cnt_d.item())
        assert A == len(idx) and np.array_equal(idx_d[:A].cpu().numpy(), idx)
        rn = (1.0 - sigma, sigma, cfg.video.seed, step)
        o_act, lse, ke, ve = _layer(impl, kcd, vcd, Qd, Kd, Vd, ocd, idx_d, cnt_d, A, 1 / math.sqrt(d), renoise=rn)
        kc, vc_, ke_ref, ve_ref = O.kv_sync(kc, vc_, Kp[idx], Vp[idx], idx, renoise=rn, heads=heads)
        assert torch.equal(kcd.cpu(), kc) and torch.equal(vcd.cpu(), vc_)
        for got, ref in ((ke, ke_ref), (ve, ve_ref)):
            err = np.abs(got[:, torch.from_numpy(heads)].cpu().double().numpy() - ref)
            ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -126))) - 7)
            assert np.all(err <= ulp + 1e-5 * sigma + 1e-30)
        rows = _sample(A, 48, step)
        o_ref, lse_ref = O.pruned_attn(Q[idx][:, torch.from_numpy(heads)], ke_ref, ve_ref, idx,
                                       1 / math.sqrt(d), rows=rows)
        _check(o_act[:, torch.from_numpy(heads)].cpu(), lse[:, torch.from_numpy(heads)].cpu().numpy(),
               o_ref, lse_ref, rows=rows)


# ----------------------------------------------- attention-recovery merge ---
def test_lse_merge_parity_and_empty_parts():
    A, H, d = 777, 3, 128
    o1 = synth.gaussian_bf16((A, H, d), 81)
    o2 = synth.gaussian_bf16((A, H, d), 82)
    rng = np.random.default_rng(83)
    l1 = torch.from_numpy((rng.standard_normal((A, H)) * 3).astype(np.float32))
    l2 = torch.from_numpy((rng.standard_normal((A, H)) * 3).astype(np.float32))
    l1[::7] = -np.inf
    l2[::11] = -np.inf
    cnt = torch.tensor([A], dtype=torch.int32, device=DEV)
    lse = torch.empty((A, H), device=DEV)
    o = tps.attn_lse_merge(o1.to(DEV), l1.to(DEV), o2.to(DEV), l2.to(DEV), cnt, lse=lse)
    o_ref, l_ref = O.lse_merge(o1, l1, o2, l2)
    g = o.cpu().double().numpy()
    assert np.all(np.abs(g - o_ref) <= 2.0 ** -8 * np.abs(o_ref) + 1e-6)     # one bf16 rounding
    lg = lse.cpu().numpy()
    assert np.array_equal(np.isneginf(lg), np.isneginf(l_ref))
    fin = np.isfinite(l_ref)
    np.testing.assert_allclose(lg[fin], l_ref[fin], rtol=1e-6, atol=1e-6)


@pytest.mark.parametrize("impl", IMPLS)
def test_split_key_attention_merges_to_full(impl):
    """Attention over keys [0, M) and [M, N) by two calls, merged with
    attn_lse_merge, equals attention over all N keys (oracle)."""
    N, M, A, H, d = 3000, 1234, 500, 2, 128
    q = synth.gaussian_bf16((A, H, d), 91)
    k = synth.gaussian_bf16((N, H, d), 92)
    v = synth.gaussian_bf16((N, H, d), 93)
    idx = np.sort(np.random.default_rng(94).choice(N, A, replace=False))
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    di = torch.from_numpy(idx.astype(np.int32)).to(DEV)
    dc = torch.tensor([A], dtype=torch.int32, device=DEV)
    fn = getattr(tps, impl)
    o1, o2 = torch.empty_like(qd), torch.empty_like(qd)
    l1, l2 = torch.empty((A, H), device=DEV), torch.empty((A, H), device=DEV)
    fn(qd, kd[:M], vd[:M], di, dc, 0.25, o_act=o1, lse=l1)
    fn(qd, kd[M:], vd[M:], di, dc, 0.25, o_act=o2, lse=l2)
    lse = torch.empty((A, H), device=DEV)
    o = tps.attn_lse_merge(o1, l1, o2, l2, dc, lse=lse)
    tps.tps_check()
    o_ref, l_ref = O.pruned_attn(q, k, v, idx, 0.25)
    _check(o.cpu(), lse.cpu().numpy(), o_ref, l_ref)


# --------------------------------------------- split-key attention (ws) -----
@pytest.mark.parametrize("N,A,H,d", [(3000, 300, 2, 128), (2600, 200, 3, 64), (5000, 1, 1, 128)])
def test_attn_ws_split_matches_oracle(N, A, H, d):
    """Few query tiles x heads: pruned_attn_ws splits the key range (its
    workspace size is non-zero) and the merged result matches the oracle."""
    assert tps.lib().tps_attn_workspace_size(A, N, H, d) > 0
    q = synth.gaussian_bf16((A, H, d), N + 7)
    k = synth.gaussian_bf16((N, H, d), N + 8)
    v = synth.gaussian_bf16((N, H, d), N + 9)
    idx = np.sort(np.random.default_rng(A).choice(N, A, replace=False))
    for scale in (1 / math.sqrt(d), 0.35):
        qd = q.to(DEV)
        o = torch.full_like(qd, 7.0)
        lse = torch.full((A, H), 7.0, device=DEV)
        tps.pruned_attn_ws(qd, k.to(DEV), v.to(DEV), torch.from_numpy(idx.astype(np.int32)).to(DEV),
                           torch.tensor([A], dtype=torch.int32, device=DEV), scale, o_act=o, lse=lse)
        tps.tps_check()
        o_ref, lse_ref = O.pruned_attn(q, k, v, idx, scale)
        _check(o.cpu(), lse.cpu().numpy(), o_ref, lse_ref)


def test_attn_ws_wan_keep10_sampled():
    """The Wan-like layer at keep 10% (3276 x 32760 keys, 12 heads): split path
    vs the oracle on sampled rows."""
    Q, K, V = qkv("wan")
    N, H, d = Q.shape
    idx = oracle_idx("wan", 0)
    A = len(idx)
    assert tps.lib().tps_attn_workspace_size(A, N, H, d) > 0
    o = torch.empty((A, H, d), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((A, H), device=DEV)
    tps.pruned_attn_ws(Q[idx].to(DEV), K.to(DEV), V.to(DEV), torch.from_numpy(idx).to(DEV),
                       torch.tensor([A], dtype=torch.int32, device=DEV), 1 / math.sqrt(d), o_act=o, lse=lse)
    tps.tps_check()
    rows = _sample(A, 192, 5)
    o_ref, lse_ref = O.pruned_attn(Q[idx], K, V, idx, 1 / math.sqrt(d), rows=rows)
    _check(o.cpu(), lse.cpu().numpy(), o_ref, lse_ref, rows=rows)


def test_attn_ws_no_split_when_grid_is_full():
    # 24 x 12 = 288 CTAs fill 148 SMs twice at 97%: no split, no workspace
    assert tps.lib().tps_attn_workspace_size(6084, 20280, 12, 128) == 0


# ------------------------------- split-key attention merged inside a cluster -----
@pytest.mark.parametrize("N,S", [(1100, 2), (1600, 3), (2100, 4), (4099, 4)])
@pytest.mark.parametrize("d", [64, 128])
def test_attn_cluster_split_matches_oracle(N, S, d):
    """One query tile pair x one head fills one SM: pruned_attn splits the keys
    over a cluster of S CTAs (S bounded by 4 key tiles per split) that merge
    over distributed shared memory. A score spike confined to one split's key
    range gives the partials very different maxima; a count below cap leaves
    the tail rows untouched."""
    A, H = 200, 1
    assert tps.attn_split(A, N, H, d) == S
    q = synth.gaussian_bf16((A, H, d), N + S)
    k = synth.gaussian_bf16((N, H, d), N + S + 1).double()
    k[N - 300:N - 200] *= 25.0                              # inside the last split only
    k = k.to(torch.bfloat16)
    v = synth.gaussian_bf16((N, H, d), N + S + 2)
    idx = np.sort(np.random.default_rng(S).choice(N, A, replace=False))
    vmax = v.double().abs().amax(dim=(0, 2)).numpy()
    for scale in (1 / math.sqrt(d), 0.35):
        o, lse = _run("pruned_attn", q, k, v, idx, scale)
        o_ref, lse_ref = O.pruned_attn(q, k, v, idx, scale)
        _check(o, lse, o_ref, lse_ref, v_absmax=vmax)
    o, lse = _run("pruned_attn", q, k, v, idx, 0.2, count=150)
    o_ref, lse_ref = O.pruned_attn(q, k, v, idx, 0.2, rows=np.arange(150))
    _check(o[:150], lse[:150], o_ref, lse_ref, v_absmax=vmax)
    assert torch.all(o[150:].float() == 7.0) and np.all(lse[150:] == 7.0)


def test_attn_cluster_split_wan_keep10_sampled():
    """The Wan-like layer at keep 10% (3276 queries x 32760 keys, 12 heads:
    156 CTAs on 148 SMs) through pruned_attn: a cluster split is chosen (of the
    whole grid or of the tiles past its full wave) and matches the oracle on
    sampled rows."""
    Q, K, V = qkv("wan")
    N, H, d = Q.shape
    idx = oracle_idx("wan", 0)
    A = len(idx)
    split, _, tail = tps.attn_plan(A, N, H, d)
    assert split > 1 or tail > 1                            # the whole grid or its last tiles split
    o, lse = _run("pruned_attn", Q[idx], K, V, idx, 1 / math.sqrt(d))
    rows = _sample(A, 192, 6)
    o_ref, lse_ref = O.pruned_attn(Q[idx], K, V, idx, 1 / math.sqrt(d), rows=rows)
    _check(o, lse, o_ref, lse_ref, rows=rows)


def test_attn_no_cluster_split_when_grid_is_full():
    assert tps.attn_split(6084, 20280, 12, 128) == 1
    assert tps.attn_split(39600, 118800, 24, 128) == 1
    assert tps.attn_plan(6084, 20280, 12, 128) == (1, 6084, 1)


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def test_attn_plan_hsa_tail():
    """The HSA step's attention (155 tile pairs x 24 heads = 3720 units on 148
    SMs, 25.1 waves): the full waves run unsplit and the last tile pair of
    every head runs split 4 ways in a second launch."""
    if _sms() != 148:
        pytest.skip("plan figures are for 148 SMs")
    split, main_rows, tail = tps.attn_plan(39600, 118800, 24, 128)
    assert (split, main_rows, tail) == (1, 154 * 256, 4)


@pytest.mark.parametrize("d", [64, 128])
def test_attn_tail_split_matches_oracle(d):
    """A grid one wave and two tile pairs long (H = 1): the first launch takes
    the full wave unsplit, the second the remaining tile pairs split over a
    cluster. Sampled rows on both sides of the boundary and the ragged last
    tile match the oracle; counts below cap (inside the first launch and
    inside the tail) leave the rows past the count untouched."""
    P = _sms()
    H = 1
    A = (P + 2) * 256 - 50
    N = A + 1000
    split, main_rows, tail = tps.attn_plan(A, N, H, d)
    assert split == 1 and main_rows == P * 256 and tail > 1
    q = synth.gaussian_bf16((A, H, d), 71)
    k = synth.gaussian_bf16((N, H, d), 72).double()
    k[N - 300:N - 200] *= 25.0                              # a spike inside the last key split
    k = k.to(torch.bfloat16)
    v = synth.gaussian_bf16((N, H, d), 73)
    idx = np.sort(np.random.default_rng(d).choice(N, A, replace=False))
    vmax = v.double().abs().amax(dim=(0, 2)).numpy()
    b = main_rows
    rows = np.unique(np.concatenate([_sample(A, 96, 5), np.arange(b - 3, b + 3), np.arange(A - 4, A)]))
    o, lse = _run("pruned_attn", q, k, v, idx, 1 / math.sqrt(d))
    o_ref, lse_ref = O.pruned_attn(q, k, v, idx, 1 / math.sqrt(d), rows=rows)
    _check(o, lse, o_ref, lse_ref, rows=rows, v_absmax=vmax)
    for count in (b - 100, b + 100):
        o, lse = _run("pruned_attn", q, k, v, idx, 0.2, count=count)
        sub = rows[rows < count]
        o_ref, lse_ref = O.pruned_attn(q, k, v, idx, 0.2, rows=sub)
        _check(o, lse, o_ref, lse_ref, rows=sub, v_absmax=vmax)
        assert torch.all(o[count:].float() == 7.0) and np.all(lse[count:] == 7.0)


# -------------------------------------------------- CTA-pair kernel (d = 128) -----
@pytest.mark.parametrize("N,A,H", [(128, 1, 1), (300, 513, 2), (1000, 1024, 3), (4099, 700, 2), (2049, 2000, 1)])
def test_attn_pair_ragged_and_against_single_cta(N, A, H):
    """pruned_attn_pair: 512-row pair tiles with ragged tails (a pair whose
    second CTA or second tile has no rows), matched against the oracle and, to
    the attention tolerance, against the single-CTA kernel; A > N exercises
    repeated indices, which attention allows."""
    d = 128
    q = synth.gaussian_bf16((A, H, d), 500 + A)
    k = synth.gaussian_bf16((N, H, d), 501 + N)
    v = synth.gaussian_bf16((N, H, d), 502 + N)
    idx = np.sort(np.random.default_rng(A + N).choice(N, A, replace=A > N))
    o, lse = _run("pruned_attn_pair", q, k, v, idx, 1 / math.sqrt(d))
    o_ref, lse_ref = O.pruned_attn(q, k, v, idx, 1 / math.sqrt(d))
    _check(o, lse, o_ref, lse_ref)
    o1, _ = _run("pruned_attn", q, k, v, idx, 1 / math.sqrt(d))
    ok, info = attn_tolerance_ok(o.double().numpy(), o1.double().numpy())
    assert ok, info


def test_attn_pair_rejects_unsupported():
    F = tps.C.c_void_p(0x1000)
    l = tps.lib()
    assert l.pruned_attn_pair(F, F, F, F, F, 10, 100, 2, 64, 0.1, None, 128, F, None, None) == tps.INVALID_ARG
    assert l.pruned_attn_pair(F, F, F, F, F, 10, 100, 2, 128, 0.1, F, 128, F, None, None) == tps.INVALID_ARG
