"""Pins for the fp64 oracle (CPU only).

Every oracle function is tied to something other than itself: hand-worked
examples from the pages' definitions (tests/golden), closed forms, library
routines (torch SDPA, torch.logsumexp, scipy's KS test), invariants, and brute
force on tiny inputs. The last tests plant mistakes in the oracle and check
that a pin catches each of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
from oracle import margins as M
from token_pruned_sparse_b200 import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _num(v):
    return {"inf": math.inf, "ln3": math.log(3.0), "ln4": math.log(4.0)}.get(v, v) if isinstance(v, str) else v


# ----------------------------------------------------------------- score ---
def test_score_worked_examples():
    g = _gold("score_worked.json")
    for c in g["cases"]:
        s = O.lipar_score(np.array([[c["cur"]]], float), np.array([[c["ref"]]], float))
        assert s[0] == _num(c["score"])
    fr = g["interframe"]
    x = np.array(fr["x"], float)
    assert list(O.lipar_score(x)) == [_num(v) for v in fr["score_no_prev"]]
    assert list(O.lipar_score(x, x_prev_frame=np.array(fr["x_prev_frame"], float))) == \
        [_num(v) for v in fr["score_with_prev"]]


def test_score_linearity_and_zero_change():
    rng = np.random.default_rng(0)
    ref = rng.integers(-128, 129, (50, 1, 16)).astype(float) / 16
    delta = rng.integers(-64, 65, (50, 1, 16)).astype(float) / 16
    s1 = O.lipar_score(ref + delta, ref)
    for lam in (0.25, 2.0, 8.0):
        np.testing.assert_array_equal(O.lipar_score(ref + lam * delta, ref), lam * s1)
    assert not O.lipar_score(ref, ref).any()
    # zero change -> empty active set at any tau > 0 (inter-step and inter-frame)
    assert len(O.select_threshold(O.lipar_score(ref, ref), 1e-6)) == 0
    video = np.repeat(ref[:8].reshape(1, 8, 16), 5, axis=0)
    s = O.lipar_score(video, x_prev_frame=video[0])
    assert len(O.select_threshold(s, 1e-6)) == 0
    # without a previous frame, frame 0 is always active
    assert list(O.select_threshold(O.lipar_score(video), 1e-6)) == list(range(8))


def test_score_matches_torch_norms():
    """Relative L1 equals torch's vector 1-norm ratio (library witness)."""
    x = synth.gaussian_bf16((6, 40, 32), 3)
    r = synth.gaussian_bf16((6, 40, 32), 4)
    xt, rt = x.double().reshape(-1, 32), r.double().reshape(-1, 32)
    ref = (torch.linalg.vector_norm(xt - rt, ord=1, dim=1) / torch.linalg.vector_norm(rt, ord=1, dim=1)).numpy()
    np.testing.assert_allclose(O.lipar_score(x, r), ref, rtol=1e-13)


# ---------------------------------------------------------------- select ---
def test_topk_bruteforce_tiny():
    """The selected set is the unique k-subset whose every member beats every
    non-member by (score desc, index asc); checked by enumerating subsets."""
    rng = np.random.default_rng(1)
    for trial in range(60):
        n = int(rng.integers(1, 9))
        s = rng.integers(0, 4, n).astype(float)          # many ties
        if trial % 3 == 0:
            s[rng.integers(0, n)] = math.inf
        for k in range(n + 1):
            winners = [S for S in itertools.combinations(range(n), k)
                       if all((s[a] > s[b]) or (s[a] == s[b] and a < b)
                              for a in S for b in set(range(n)) - set(S))]
            assert len(winners) == 1
            assert list(O.select_topk(s, k)) == list(winners[0])


def test_topk_equals_threshold_at_kth_score():
    rng = np.random.default_rng(2)
    s = rng.exponential(size=1000)
    for k in (1, 10, 500, 999):
        kth = np.sort(s)[::-1][k - 1]
        assert list(O.select_topk(s, k)) == list(O.select_threshold(s, kth))
    assert list(O.select_topk(s, 1000)) == list(range(1000))
    assert len(O.select_topk(s, 0)) == 0


def test_topk_golden_and_specials():
    g = _gold("schedule_worked.json")
    s = np.array(g["group_split"]["scores"])
    assert list(O.select_topk(s, g["topk"]["k"])) == g["topk"]["idx"]
    s2 = np.array([math.nan, -0.0, 0.0, 1.0, -math.inf])
    assert list(O.select_topk(s2, 3)) == [1, 2, 3]         # -0 == +0, tie to lower index; NaN lowest
    assert list(O.select_topk(s2, 4)) == [1, 2, 3, 4]
    assert list(O.select_threshold(s2, 0.0)) == [1, 2, 3]


def test_group_split_golden_and_invariants():
    g = _gold("schedule_worked.json")["group_split"]
    assert list(O.group_split(np.array(g["scores"]), 3)) == g["groups"]
    rng = np.random.default_rng(3)
    for N, K in ((30, 3), (31, 3), (100, 4), (7, 7)):
        s = rng.integers(0, 5, N).astype(float)
        grp = O.group_split(s, K)
        sizes = np.bincount(grp, minlength=K)
        assert list(sizes[:-1]) == [N // K] * (K - 1) and sizes[-1] == N - (K - 1) * (N // K)
        for a in range(K - 1):                           # earlier groups change faster
            assert s[grp == a].min() >= s[grp == a + 1].max()
        # brute force: a token's group is fixed by how many tokens outrank it
        for n in range(N):
            rank = sum((s[m] > s[n]) or (s[m] == s[n] and m < n) for m in range(N))
            assert grp[n] == min(rank // (N // K), K - 1)


def test_schedule_golden_and_enumeration():
    g = _gold("schedule_worked.json")
    for m, key in ((0, "active_groups_m0"), (1, "active_groups_m1")):
        for i in range(g["T"]):
            assert list(O.schedule_groups(3, g["budgets"], g["T"], i, m).astype(int)) == g[key][i]
    # the configured HSA schedule: T=40, budgets (40, 20, 10), thirds of 118800
    T, budgets, N = 40, (40, 20, 10), 118800
    grp = np.repeat(np.arange(3, dtype=np.int8), N // 3)
    counts = np.zeros(3, int)
    total = 0
    for i in range(T):
        act = O.schedule_groups(3, budgets, T, i, 0)
        counts += act
        A = len(O.schedule_active(grp, 3, budgets, T, i, 0))
        total += A
        assert A == {0: N, 2: 2 * N // 3}.get(i % 4, N // 3)
    assert list(counts) == list(budgets)                 # each group runs exactly s_k steps
    assert total * 3 == 70 * N                           # sum |A_i| = 23 1/3 N
    for i in list(range(3)) + list(range(T - 3, T)):
        assert len(O.schedule_active(grp, 3, budgets, T, i, 3)) == N


# ---------------------------------------------------------- kv sync / RNG ---
def test_kv_sync_rows_and_identity_renoise():
    N, H, d, A = 50, 2, 8, 17
    kc, vc = synth.gaussian_bf16((N, H, d), 1), synth.gaussian_bf16((N, H, d), 2)
    kf, vf = synth.gaussian_bf16((A, H, d), 3), synth.gaussian_bf16((A, H, d), 4)
    idx = np.sort(np.random.default_rng(5).choice(N, A, replace=False)).astype(np.int32)
    k2, v2, ke, ve = O.kv_sync(kc, vc, kf, vf, idx, renoise=(1.0, 0.0, 9, 3))
    pruned = np.setdiff1d(np.arange(N), idx)
    assert torch.equal(k2[idx], kf) and torch.equal(v2[idx], vf)
    assert torch.equal(k2[pruned], kc[pruned]) and torch.equal(v2[pruned], vc[pruned])
    np.testing.assert_array_equal(ke, k2.double().numpy())   # a=1, b=0 -> bit-identical
    np.testing.assert_array_equal(ve, v2.double().numpy())


def test_renoise_statistics():
    """z = (eff - a*c)/b over pruned rows is i.i.d. N(0,1): moments, KS test
    (scipy), and K/V and step independence."""
    from scipy import stats
    N, H, d = 600, 4, 64
    kc = synth.gaussian_bf16((N, H, d), 11)
    vc = synth.gaussian_bf16((N, H, d), 12)
    idx = np.arange(0, N, 3, dtype=np.int32)
    a, b = 0.3, 0.7
    _, _, ke, ve = O.kv_sync(kc, vc, kc[idx], vc[idx], idx, renoise=(a, b, 1234, 5))
    pruned = np.setdiff1d(np.arange(N), idx)
    zk = ((ke[pruned] - a * kc[pruned].double().numpy()) / b).ravel()
    zv = ((ve[pruned] - a * vc[pruned].double().numpy()) / b).ravel()
    n = zk.size
    for z in (zk, zv):
        assert abs(z.mean()) < 5 / math.sqrt(n)
        assert abs(z.var() - 1) < 5 * math.sqrt(2 / n)
        assert stats.kstest(z, "norm").pvalue > 1e-4
    assert abs(np.corrcoef(zk, zv)[0, 1]) < 5 / math.sqrt(n)
    e = np.arange(4096)
    z5, z6 = O.renoise_normals(1234, 5, 0, e), O.renoise_normals(1234, 6, 0, e)
    assert abs(np.corrcoef(z5, z6)[0, 1]) < 5 / math.sqrt(4096)
    # active rows are the fresh rows, untouched by noise
    np.testing.assert_array_equal(ke[idx], kc[idx].double().numpy())


def _box_muller_pin_failures(normals):
    """Names of the Box-Muller pins that `normals(seed, step, tensor, e)` breaks.

    Box & Muller (1958): from two independent uniforms U1, U2 the pair
    Z0 = sqrt(-2 ln U1) cos(2 pi U2), Z1 = sqrt(-2 ln U1) sin(2 pi U2) is two
    independent N(0,1) deviates. The raw Philox words fix U1 (word 0 or 2 of
    a counter block) and U2 (word 1 or 3), so the pins read them back:
      radius  Z0^2 + Z1^2 = -2 ln U1 (fp64 rounding only),
      angle   atan2(Z1, Z0) = 2 pi U2 (mod 2 pi),
      pairing the two members of a pair, and the two pairs of a block, are
              uncorrelated (|r| < 5/sqrt(n) over n = 2^16 blocks)."""
    seed, step, tensor = 77, 3, 1
    nq = 1 << 16
    q = np.arange(nq)
    z = normals(seed, step, tensor, np.arange(4 * nq)).reshape(nq, 4)
    w = O.philox_words(seed, step, tensor, q).astype(np.float64)
    u = (np.floor(w / 512.0) + 0.5) * 2.0 ** -23          # the word -> (0, 1) map of the oracle's reading
    bad = []
    for a, b in ((0, 1), (2, 3)):
        r2 = z[:, a] ** 2 + z[:, b] ** 2
        if not np.allclose(r2, -2.0 * np.log(u[:, a]), rtol=1e-12, atol=1e-300):
            bad.append("radius")
        ang = np.mod(np.arctan2(z[:, b], z[:, a]), 2 * np.pi)
        err = np.abs(np.angle(np.exp(1j * (ang - 2 * np.pi * u[:, b]))))
        if err.max() > 1e-9:
            bad.append("angle")
        if abs(np.corrcoef(z[:, a], z[:, b])[0, 1]) >= 5 / math.sqrt(nq):
            bad.append("pairing")
    if abs(np.corrcoef(z[:, 0], z[:, 2])[0, 1]) >= 5 / math.sqrt(nq):
        bad.append("pairing")
    return sorted(set(bad))


def test_box_muller_pairing_radius_and_angle():
    """The oracle's normals follow the Box-Muller pairing exactly: word 0 (2)
    gives the radius, word 1 (3) the angle, cosine first, and the two deviates
    of a pair are independent."""
    assert _box_muller_pin_failures(O.renoise_normals) == []


def _bm_variant(kind):
    """The oracle's normals with one plausible Box-Muller slip planted."""
    def fn(seed, step, tensor, e):
        e = np.asarray(e, np.int64)
        j = e & 3
        w = O.philox_words(seed, step, tensor, (e >> 2).astype(np.uint64)).astype(np.float64)
        u = (np.floor(w / 512.0) + 0.5) * 2.0 ** -23
        pair = (j >> 1) * 2
        ua = np.take_along_axis(u, pair[:, None], 1)[:, 0]
        ub = np.take_along_axis(u, (pair + 1)[:, None], 1)[:, 0]
        if kind == "same_u":            # both members of a pair from one uniform
            ub = ua
        if kind == "swapped_words":     # radius from the second word, angle from the first
            ua, ub = ub, ua
        r = np.sqrt(-2.0 * np.log(ua))
        first = r * np.cos(2 * np.pi * ub)
        second = r * (np.cos(2 * np.pi * ub) if kind == "cos_twice" else np.sin(2 * np.pi * ub))
        if kind == "sin_first":
            first, second = second, first
        return np.where((j & 1) == 0, first, second)
    return fn


@pytest.mark.parametrize("kind", ["cos_twice", "same_u", "swapped_words", "sin_first"])
def test_box_muller_pins_catch_planted_mistakes(kind):
    """Each slip keeps N(0,1) marginals (or nearly), which the moment and KS
    pins cannot see; the pairing, radius and angle pins catch every one."""
    assert _box_muller_pin_failures(_bm_variant("none")) == []
    assert _box_muller_pin_failures(_bm_variant(kind)) != []


def test_philox_words_uniform_and_distinct():
    """Raw stream properties beyond the known-answer vectors: uniform bytes
    and distinct streams across counters, steps, tensors and seeds."""
    from scipy import stats
    w = O.philox_words(42, 0, 0, np.arange(1 << 14))
    assert len(np.unique(w.reshape(-1))) > 0.999 * w.size
    top = (w >> 24).ravel()
    assert stats.chisquare(np.bincount(top, minlength=256)).pvalue > 1e-4
    assert not np.array_equal(w, O.philox_words(42, 1, 0, np.arange(1 << 14)))
    assert not np.array_equal(w, O.philox_words(42, 0, 1, np.arange(1 << 14)))
    assert not np.array_equal(w, O.philox_words(43, 0, 0, np.arange(1 << 14)))


# -------------------------------------------------------------- attention ---
def _sdpa(q, k, v, scale, allowed=None):
    """torch SDPA in fp64 on CPU, one head at a time: [A,H,d] x [N,H,d]."""
    out = []
    for h in range(q.shape[1]):
        qq = q[:, h].double()[None, None]
        kk = k[:, h].double()[None, None]
        vv = v[:, h].double()[None, None]
        m = None if allowed is None else torch.from_numpy(allowed)[None, None]
        out.append(torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=m, scale=scale)[0, 0])
    return torch.stack(out, 1).numpy()


def test_attn_worked_example():
    g = _gold("attn_worked.json")
    q = torch.tensor([[[_num(g["q"])]]], dtype=torch.float64)
    k = torch.tensor([[[_num(x)]] for x in g["k"]], dtype=torch.float64)
    v = torch.tensor([[[x]] for x in g["v"]], dtype=torch.float64)
    o, lse = O.pruned_attn(q, k, v, [0], 1.0)
    assert abs(o[0, 0, 0] - g["o"]) < 1e-12 and abs(lse[0, 0] - _num(g["lse"])) < 1e-12


@pytest.mark.parametrize("N,A,H,d", [(300, 300, 2, 64), (517, 131, 3, 128)])
def test_attn_dense_matches_sdpa(N, A, H, d):
    """All-active (k = N) equals textbook dense softmax attention."""
    q = synth.gaussian_bf16((A, H, d), 21)
    k = synth.gaussian_bf16((N, H, d), 22)
    v = synth.gaussian_bf16((N, H, d), 23)
    idx = np.sort(np.random.default_rng(0).choice(N, A, replace=False))
    for scale in (1 / math.sqrt(d), 0.5):
        o, lse = O.pruned_attn(q, k, v, idx, scale)
        np.testing.assert_allclose(o, _sdpa(q, k, v, scale), rtol=1e-9, atol=1e-11)
        s = torch.einsum("ahd,nhd->ahn", q.double(), k.double()) * scale
        np.testing.assert_allclose(lse, torch.logsumexp(s, -1).numpy(), rtol=1e-12)


def test_attn_blockmask_matches_sdpa():
    N, H, d, blk = 700, 2, 64, 128
    A = 300
    q = synth.gaussian_bf16((A, H, d), 31)
    k = synth.gaussian_bf16((N, H, d), 32)
    v = synth.gaussian_bf16((N, H, d), 33)
    idx = np.sort(np.random.default_rng(1).choice(N, A, replace=False))
    nb = -(-N // blk)
    bm = (np.random.default_rng(2).random((nb, nb)) < 0.4).astype(np.uint8)
    bm[np.arange(nb), np.arange(nb)] = 1
    allowed = np.array([[bm[i // blk, n // blk] for n in range(N)] for i in idx], bool)
    o, _ = O.pruned_attn(q, k, v, idx, 0.125, blockmask=bm, block=blk)
    np.testing.assert_allclose(o, _sdpa(q, k, v, 0.125, allowed), rtol=1e-9, atol=1e-11)
    # a query whose mask row keeps nothing gets o = 0, lse = -inf
    bm2 = bm.copy()
    bm2[idx[0] // blk] = 0
    o2, l2 = O.pruned_attn(q, k, v, idx, 0.125, blockmask=bm2, block=blk, rows=[0])
    assert not o2.any() and np.all(np.isneginf(l2))


def test_attn_constant_keys_give_mean_of_v():
    N, H, d = 333, 2, 64
    k = synth.gaussian_bf16((1, H, d), 41).expand(N, H, d).contiguous()
    v = synth.gaussian_bf16((N, H, d), 42)
    q = synth.gaussian_bf16((20, H, d), 43)
    o, lse = O.pruned_attn(q, k, v, np.arange(20), 0.3)
    np.testing.assert_allclose(o, np.broadcast_to(v.double().mean(0).numpy(), o.shape), rtol=1e-12, atol=1e-13)
    blk = 128
    bm = np.zeros((3, 3), np.uint8)
    bm[:, 1] = 1
    o, _ = O.pruned_attn(q, k, v, np.arange(20), 0.3, blockmask=bm, block=blk)
    np.testing.assert_allclose(o, np.broadcast_to(v[128:256].double().mean(0).numpy(), o.shape), rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- scatter ---
def test_scatter_and_gather_rows():
    full = synth.gaussian_bf16((40, 2, 8), 51)
    act = synth.gaussian_bf16((9, 2, 8), 52)
    idx = np.array([0, 3, 4, 10, 11, 20, 30, 38, 39], np.int32)
    out = O.scatter_out(full, act, idx)
    assert torch.equal(out[idx], act)
    rest = np.setdiff1d(np.arange(40), idx)
    assert torch.equal(out[rest], full[rest])
    assert torch.equal(O.gather_rows(out, idx), act)
    assert torch.equal(O.scatter_out(full, act[:0], idx[:0]), full)


# ------------------------------------------------------------- margins ---
def test_margin_enforcement_keeps_selection_gap():
    spec = synth.VideoSpec(5, 10, 12, 32, 2, 3, True, 9)
    x, _ = synth.latent_video(spec)
    xb = M.enforce_frame_margin(synth.to_bf16(x), ranks=(300,))
    s = O.lipar_score(xb)
    srt = np.sort(s)[::-1]
    assert srt[299] >= srt[300] * (1 + M.MARGIN)
    vp, dl = synth.velocity_pair(spec)
    vpb = synth.to_bf16(vp)
    vc = M.enforce_step_margin(vpb, dl, ranks=(200, 400))
    s = np.sort(O.lipar_score(vc[None], vpb[None]))[::-1]
    assert s[199] >= s[200] * (1 + M.MARGIN) and s[399] >= s[400] * (1 + M.MARGIN)


# ------------------------------------------------------- planted mistakes ---
def test_pins_catch_planted_mistakes(monkeypatch):
    """Each plausible slip in the oracle fails at least one pin."""
    g = _gold("score_worked.json")["cases"][0]
    cur, ref = np.array([[g["cur"]]], float), np.array([[g["ref"]]], float)
    # dropped |.| in the denominator
    bad = lambda x, r: np.abs(x - r).sum(-1) / r.sum(-1)
    assert bad(cur, ref)[0, 0] != g["score"]
    # transposed operands (score against the current token instead of the reference)
    assert O.lipar_score(ref, cur)[0] != g["score"]
    # attention without the scale, or with keys/values swapped, breaks the SDPA pin
    q = synth.gaussian_bf16((8, 1, 64), 1)
    k = synth.gaussian_bf16((50, 1, 64), 2)
    v = synth.gaussian_bf16((50, 1, 64), 3)
    ref_o = _sdpa(q, k, v, 0.125)
    assert np.abs(O.pruned_attn(q, k, v, np.arange(8), 1.0)[0] - ref_o).max() > 1e-3
    assert np.abs(O.pruned_attn(q, v, k, np.arange(8), 0.125)[0] - ref_o).max() > 1e-3
    # ties to the HIGHER index would break the brute-force top-k pin
    s = np.array([1.0, 1.0, 0.0])
    assert list(O.select_topk(s, 1)) == [0]
    # a strict '>' threshold would select k-1 at tau = s_(k)
    assert len(O.select_threshold(np.array([3.0, 2.0, 1.0]), 2.0)) == 2


# ------------------------------------------------------- HSA cached Euler ---
def test_euler_worked_example():
    g = _gold("euler_worked.json")
    x = torch.tensor(g["x"], dtype=torch.float32)
    vc = torch.tensor(g["v_cache"], dtype=torch.bfloat16)
    vf = torch.tensor(g["v_fresh"], dtype=torch.bfloat16)
    xn, vcn = O.euler_update(x, vc, vf, g["idx"], g["dsigma"])
    assert xn.tolist() == g["x_new"]
    assert vcn.float().tolist() == g["v_cache_new"]


def test_euler_closed_forms():
    """dsigma = 0 leaves x unchanged; all-active is the plain Euler step with the
    fresh velocity; constant velocities telescope over a schedule:
    x_T = x_0 + (sigma_T - sigma_0) * v exactly (dyadic values)."""
    rng = np.random.default_rng(7)
    N, C = 40, 16
    x0 = torch.from_numpy(rng.integers(-64, 64, (N, C)).astype(np.float32) / 8)
    v = torch.from_numpy(rng.integers(-16, 16, (N, C)).astype(np.float32) / 4).to(torch.bfloat16)
    idx = np.array([3, 9, 20], np.int32)
    xn, vcn = O.euler_update(x0, v, v[idx] * 2, idx, 0.0)
    np.testing.assert_array_equal(xn, x0.double().numpy())
    assert torch.equal(vcn[idx], v[idx] * 2)
    xa, _ = O.euler_update(x0, v * 0, v, np.arange(N), -0.125)
    np.testing.assert_array_equal(xa, x0.double().numpy() - 0.125 * v.double().numpy())
    T = 8
    sig = [1 - i / T for i in range(T + 1)]
    x = x0.double()
    vc = v.clone()
    for i in range(T):
        act = np.arange(N)[np.arange(N) % (1 + i % 3) == 0]     # a varying active set
        xi, vc = O.euler_update(x, vc, v[act], act, sig[i + 1] - sig[i])
        x = torch.from_numpy(xi)
    np.testing.assert_array_equal(x.numpy(), x0.double().numpy() + (sig[T] - sig[0]) * v.double().numpy())


# --------------------------------------------- attention-recovery LSE merge ---
def test_lse_merge_equals_attention_over_all_keys():
    """Attention over keys [0, N) equals the merge of attention over [0, M) and
    [M, N) (the merge is checked against the attention definition, not itself)."""
    N, M, A, H, d = 300, 111, 40, 2, 64
    q = synth.gaussian_bf16((A, H, d), 61)
    k = synth.gaussian_bf16((N, H, d), 62)
    v = synth.gaussian_bf16((N, H, d), 63)
    idx = np.arange(A)
    o_all, l_all = O.pruned_attn(q, k, v, idx, 0.2)
    o1, l1 = O.pruned_attn(q, k[:M], v[:M], idx, 0.2)
    o2, l2 = O.pruned_attn(q, k[M:], v[M:], idx, 0.2)
    o, l = O.lse_merge(o1, l1, o2, l2)
    np.testing.assert_allclose(o, o_all, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(l, l_all, rtol=1e-13)
    # an empty part is the identity; two empty parts give 0 / -inf
    e_o, e_l = np.zeros_like(o1), np.full_like(l1, -np.inf)
    o3, l3 = O.lse_merge(o1, l1, e_o, e_l)
    np.testing.assert_array_equal(o3, o1)
    np.testing.assert_array_equal(l3, l1)
    o4, l4 = O.lse_merge(e_o, e_l, e_o, e_l)
    assert not o4.any() and np.all(np.isneginf(l4))


# ------------------------------------------------------ motion-robust score ---
def test_motion_score_worked_and_reductions():
    g = _gold("motion_worked.json")
    s = O.lipar_score_motion(np.array(g["x"], float), g["L"])
    assert list(s) == [_num(v) for v in g["score"]]
    x = synth.gaussian_bf16((6, 30, 16), 71)
    np.testing.assert_array_equal(O.lipar_score_motion(x, 1), O.lipar_score(x))   # L = 1: plain score
    assert np.all(O.lipar_score_motion(x, 3) >= O.lipar_score(x))                 # never below short-term


# ------------------------------------------------ Timeripple similarity ---
def _tr_case(g):
    gr = g["grid"]
    x = torch.tensor(g["x"], dtype=torch.bfloat16).reshape(-1, gr["H"], gr["d"])
    return x, gr["F"], gr["Hs"], gr["Ws"]


def test_timeripple_worked_example():
    g = _gold("timeripple_worked.json")
    x, F, Hs, Ws = _tr_case(g)
    D = O.timeripple_delta(x, F, Hs, Ws, g["windows"])
    for a, key in enumerate(("delta_t", "delta_x", "delta_y")):
        np.testing.assert_allclose(D[a][:, 0], [_num(v) for v in g[key]], rtol=1e-15, atol=0)
    reuse = O.timeripple_reuse(D, g["theta"])
    assert reuse[:, 0].tolist() == g["reuse"]
    assert O.timeripple_token_score(reuse).tolist() == g["token_score"]


def test_timeripple_axes_transpose_and_invariants():
    rng = np.random.default_rng(11)
    F, Hs, Ws, H, d = 3, 4, 5, 2, 8
    g = rng.standard_normal((F, Hs, Ws, H, d))
    x = torch.from_numpy(g.reshape(-1, H, d)).to(torch.bfloat16)
    wins = [(0, 8), (3, 4), (6, 5)]
    D = O.timeripple_delta(x, F, Hs, Ws, wins)
    # transposing the grid swaps the x and y axes (and their windows)
    xt = x.reshape(F, Hs, Ws, H, d).permute(0, 2, 1, 3, 4).reshape(-1, H, d)
    Dt = O.timeripple_delta(xt, F, Ws, Hs, [wins[0], wins[2], wins[1]])
    T = lambda a: a.reshape(F, Hs, Ws, H).transpose(0, 2, 1, 3).reshape(-1, H)
    assert np.array_equal(Dt[0], T(D[0]))
    assert np.array_equal(Dt[1], T(D[2])) and np.array_equal(Dt[2], T(D[1]))
    # a common offset cancels, a common scale multiplies (powers of two: exact in bf16)
    np.testing.assert_allclose(O.timeripple_delta(x.double() + 4.0, F, Hs, Ws, wins), D, rtol=1e-15)
    np.testing.assert_allclose(O.timeripple_delta(x * 2, F, Hs, Ws, wins), 2 * D, rtol=1e-15)
    # no neighbour -> +inf on exactly the first frame / column / row
    Dg = D.reshape(3, F, Hs, Ws, H)
    assert np.isinf(Dg[0, 0]).all() and np.isfinite(Dg[0, 1:]).all()
    assert np.isinf(Dg[1, :, :, 0]).all() and np.isfinite(Dg[1, :, :, 1:]).all()
    assert np.isinf(Dg[2, :, 0]).all() and np.isfinite(Dg[2, :, 1:]).all()
    # a window of the full head equals the RMS computed by torch over whole rows
    full = O.timeripple_delta(x, F, Hs, Ws, [(5, d)] * 3)
    xx = x.double().reshape(F, Hs, Ws, H, d)
    rms = torch.sqrt(torch.mean((xx[1:] - xx[:-1]) ** 2, dim=-1)).numpy().reshape(-1, H)
    np.testing.assert_allclose(full[0][Hs * Ws:], rms, rtol=1e-14)
    # a zero-length window disables its axis
    assert np.isinf(O.timeripple_delta(x, F, Hs, Ws, [(0, 0), (0, 0), (0, 0)])).all()


def test_timeripple_static_video_and_theta_ramp():
    F, Hs, Ws, H, d = 4, 3, 3, 2, 8
    one = synth.gaussian_bf16((1, Hs * Ws, H, d), 5)
    x = one.expand(F, -1, -1, -1).reshape(-1, H, d).contiguous()
    D = O.timeripple_delta(x, F, Hs, Ws, [(0, 8), (0, 8), (0, 8)])
    r = O.timeripple_reuse(D, (1e-3, 0.0, 0.0)).reshape(F, Hs * Ws, H)
    assert (r[0] == 0).all() and (r[1:] == 1).all()          # t-bit on every frame after the first
    assert O.timeripple_token_score(r.reshape(-1, H)).tolist() == [H] * (Hs * Ws) + [0] * ((F - 1) * Hs * Ws)
    # theta <= 0 never passes (Delta >= 0 and the test is strict)
    assert not O.timeripple_reuse(D, (0.0, 0.0, 0.0)).any()
    th = [O.timeripple_theta(i, 0.0, 0.05) for i in range(1, 41)]
    assert th[:11] == [0.0] * 11 and th[20:] == [0.05] * 20
    assert th[15] == pytest.approx(0.025, abs=1e-18)              # step 16, halfway
    assert all(b >= a for a, b in zip(th, th[1:]))
    assert O.timeripple_theta(12, 1.0, 3.0) == pytest.approx(1.2, abs=1e-15)


def test_timeripple_pins_catch_planted_mistakes():
    g = _gold("timeripple_worked.json")
    x, F, Hs, Ws = _tr_case(g)
    X = x.double().reshape(F, Hs, Ws, 4)
    # a sum instead of a mean over the window, or the NEXT token as neighbour
    assert math.sqrt(float(((X[1, 1, 1] - X[0, 1, 1]) ** 2).sum())) != _num(g["delta_t"][7])
    assert float(torch.sqrt(((X[0, 0, 1, 2:] - X[0, 1, 1, 2:]) ** 2).mean())) != _num(g["delta_x"][1])
    # a window that does not wrap (channels 3 only, or 3 and 4 clipped) changes Delta_y of token 3
    assert float(torch.sqrt(((X[0, 1, 1, 3:] - X[0, 0, 1, 3:]) ** 2).mean())) != _num(g["delta_y"][3])
    # '<=' instead of '<' would mark token 1 reusable on x (Delta_x = theta_x = 1)
    D = O.timeripple_delta(x, F, Hs, Ws, g["windows"])
    assert (D[1][1, 0] <= g["theta"][1]) and O.timeripple_reuse(D, g["theta"])[1, 0] == 0


def test_philox_known_answer_vectors():
    """The oracle's Philox4x32-10 against the published known-answer vectors."""
    g = _gold("philox_kat.json")
    for case in g["cases"]:
        c = [np.array([int(v, 16)], dtype=np.uint64) for v in case["counter"]]
        k = [int(v, 16) for v in case["key"]]
        out = O.philox4x32_10(*c, k[0], k[1])
        got = [int(np.asarray(o).reshape(-1)[0]) for o in out]
        assert got == [int(v, 16) for v in case["out"]]


# ------------------------------------------------- RoPE re-rotation ([LIPAR] 2.C) ---
def test_rope_worked_examples():
    for c in _gold("rope_worked.json")["cases"]:
        got = O.rope_rotate(np.array(c["k"], float), c["dims"], c["shift"], c["base"])
        np.testing.assert_allclose(got, np.array(c["out"], float), rtol=0, atol=1e-15)


def _rope_complex(k, dims, shift, base=10000.0):
    """The same offset as complex multiplication: pair (x, y) is z = x + iy and
    moves to z * exp(i phi) (numpy's complex arithmetic)."""
    x = np.asarray(k, float)
    out = x.copy()
    o = 0
    for a, da in enumerate(dims):
        j = np.arange(da // 2)
        z = x[..., o + 2 * j] + 1j * x[..., o + 2 * j + 1]
        z = z * np.exp(1j * shift[a] * base ** (-2.0 * j / da))
        out[..., o + 2 * j], out[..., o + 2 * j + 1] = z.real, z.imag
        o += da
    return out


def test_rope_complex_form_composition_norm_and_relative_offset():
    dims = synth.rope_dims(128)
    rng = np.random.default_rng(5)
    k = rng.standard_normal((64, 3, 128))
    q = rng.standard_normal((64, 3, 128))
    s1, s2 = (1, -2, 3), (4, 5, -1)
    r1 = O.rope_rotate(k, dims, s1)
    np.testing.assert_allclose(r1, _rope_complex(k, dims, s1), rtol=0, atol=1e-12)
    # R(a) R(b) = R(a + b)
    np.testing.assert_allclose(O.rope_rotate(r1, dims, s2), O.rope_rotate(k, dims, np.add(s1, s2)),
                               rtol=0, atol=1e-12)
    # every pair keeps its length
    pn = lambda x: np.hypot(x[..., 0::2], x[..., 1::2])                 # noqa: E731
    np.testing.assert_allclose(pn(r1), pn(k), rtol=1e-13)
    # (R(p) q) . (R(p + delta) k) depends on the offset delta only
    ref = np.sum(q * O.rope_rotate(k, dims, (1, 0, 0)), axis=-1)
    for p in ((0, 0, 0), (5, 0, 0), (-7, 3, 2)):
        got = np.sum(O.rope_rotate(q, dims, p) * O.rope_rotate(k, dims, np.add(p, (1, 0, 0))), axis=-1)
        np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-10)
    # no offset is the identity, bit for bit
    assert np.array_equal(O.rope_rotate(k, dims, (0, 0, 0)), k)


def test_kv_rerotate_rows():
    kc = synth.gaussian_bf16((40, 2, 64), 71)
    idx = np.array([0, 3, 4, 17, 39])
    dims = synth.rope_dims(64)
    ke = O.kv_rerotate(kc, idx, dims, (1, 0, 0))
    np.testing.assert_array_equal(ke[idx], kc[idx].double().numpy())      # active rows: the cache row
    pruned = np.setdiff1d(np.arange(40), idx)
    np.testing.assert_array_equal(ke[pruned], O.rope_rotate(kc[pruned], dims, (1, 0, 0)))
    assert not np.allclose(ke[pruned], kc[pruned].double().numpy())
    np.testing.assert_array_equal(O.kv_rerotate(kc, idx, dims, (0, 0, 0)), kc.double().numpy())


def _rope_variant(kind):
    """The oracle's rotation with one plausible slip planted."""
    def fn(k, dims, shift, base=10000.0):
        x = np.asarray(k, float)
        out = x.copy()
        o = 0
        order = (1, 2, 0) if kind == "groups_rotated" else (0, 1, 2)
        for a in order:
            da = int(dims[a])
            j = np.arange(da // 2)
            denom = x.shape[-1] if kind == "freq_over_d" else da
            phi = float(shift[a]) * base ** (-2.0 * j / denom) * (-1.0 if kind == "sign" else 1.0)
            if kind == "half_split":                   # pairs (j, j + d_a/2) instead of adjacent channels
                i0, i1 = o + j, o + da // 2 + j
            else:
                i0, i1 = o + 2 * j, o + 2 * j + 1
            c, s = np.cos(phi), np.sin(phi)
            out[..., i0] = x[..., i0] * c - x[..., i1] * s
            out[..., i1] = x[..., i0] * s + x[..., i1] * c
            o += da
        return out
    return fn


@pytest.mark.parametrize("kind", ["sign", "half_split", "freq_over_d", "groups_rotated"])
def test_rope_pins_catch_planted_mistakes(kind):
    """Composition, norm and relative-offset pins hold for any consistent
    rotation; the hand-worked examples fix the sign, the pairing, the
    frequencies and the group order."""
    def worked_ok(fn):
        return all(np.allclose(fn(np.array(c["k"], float), c["dims"], c["shift"], c["base"]),
                               np.array(c["out"], float), rtol=0, atol=1e-12)
                   for c in _gold("rope_worked.json")["cases"])
    assert worked_ok(_rope_variant("none"))
    assert not worked_ok(_rope_variant(kind))
