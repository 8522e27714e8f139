"""Plain, slow, fp64 reference for every step of the token-pruned attention path.

TEST INFRASTRUCTURE ONLY (see the package docstring): nothing on the product
path may import or call this module.

Inputs are bf16 tensors (or arrays of bf16 values); they are widened exactly
to float64 and every result is computed in float64 with numpy/torch CPU ops.
Library primitives (matmul, stable sort, exp, log) are used as single steps;
no blocking, fusion or reordering is introduced beyond processing query rows
independently.

Sources (gist.science summaries):
  [LIPAR]  "Training-free Latent Inter-Frame Pruning with Attention Recovery"
           (Spanish technical summary: 2.B LIF pruning, 2.C Attention Recovery;
           Dutch technical summary: 2.B, 2.C, 2.D Restauratie)
  [HSA]    "Resumen Tecnico: Asignacion de Pasos Heterogenea (HSA) para la
           Generacion Eficiente de Video" (2.1 partition/schedule, 2.2 KV-cache
           sync, 2.4 phase-aware window)
  [SVOO]   "Training-Free Sparse Attention for Fast Video Generation via Offline
           Layer-Wise Sparsity Profiling and Online Bidirectional Co-Clustering"
           (part 2, co-clustering -> key-block sparsity)
  [Philox] Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as
           1, 2, 3", SC'11 -- Philox4x32-10.
  [BM]     Box & Muller, "A Note on the Generation of Random Normal
           Deviates", Ann. Math. Stat. 29 (1958).
  [TR]     "Timeripple: Accelerating vDiTs by Understanding the Spatio-Temporal
           Correlations in Latent Space" (Metodologia 2: per-axis similarity
           checks; Metodologia 3: threshold schedule)
"""
from __future__ import annotations

import math

import numpy as np
import torch

__all__ = [
    "f64", "round_bf16", "lipar_score", "select_threshold", "select_topk", "group_split",
    "schedule_groups", "schedule_active", "compact", "kv_sync", "philox4x32_10",
    "philox_words", "renoise_normals", "pruned_attn", "scatter_out", "gather_rows",
    "attn_flops", "euler_update", "lse_merge", "lipar_score_motion",
    "timeripple_delta", "timeripple_reuse", "timeripple_token_score", "timeripple_theta",
    "rope_rotate", "kv_rerotate",
]


def f64(a) -> np.ndarray:
    """Exact widening of bf16 / fp32 data to float64."""
    if isinstance(a, torch.Tensor):
        return a.detach().to(torch.float64).cpu().numpy()
    return np.asarray(a, dtype=np.float64)


def round_bf16(a: np.ndarray) -> torch.Tensor:
    """float64 -> bf16 by torch's conversion (round-to-nearest-even through
    fp32). Used only to re-round generated inputs, never to decide parity."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64)).to(torch.bfloat16)


# ---------------------------------------------------------------------------
# Step 1: token score = relative L1 change
# ---------------------------------------------------------------------------
def lipar_score(x, x_ref=None, x_prev_frame=None) -> np.ndarray:
    """Relative-L1 change per latent token, float64 [F*HW].

    [LIPAR] 2.B compares latent patches at the same spatial location in
    consecutive frames by L1 norm; [HSA] 2.1 assigns tokens by the per-token
    relative L1 change of the velocity predictions. Relative form:

        s = sum_c |cur_c - ref_c| / sum_c |ref_c|

    * inter-frame (x_ref is None): x is [F, HW, C]; token (f, p) has
      cur = x[f, p], ref = x[f-1, p]. Frame 0 has no predecessor: its score is
      +inf (always active) unless x_prev_frame [HW, C] is given, which then
      serves as its reference.
    * inter-step (x_ref given, same shape as x): cur = x[n], ref = x_ref[n].
    * den = 0: the score is 0 when num = 0, else +inf.
    """
    x = f64(x)
    F, HW, C = x.shape
    if x_ref is not None:
        cur = x.reshape(F * HW, C)
        ref = f64(x_ref).reshape(F * HW, C)
        first_inf = False
    else:
        ref = np.empty_like(x)
        ref[1:] = x[:-1]
        first_inf = x_prev_frame is None
        ref[0] = 0.0 if first_inf else f64(x_prev_frame).reshape(HW, C)
        cur = x.reshape(F * HW, C)
        ref = ref.reshape(F * HW, C)
    num = np.abs(cur - ref).sum(axis=1)
    den = np.abs(ref).sum(axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        s = np.where(den > 0, num / np.where(den > 0, den, 1.0), np.where(num > 0, np.inf, 0.0))
    if first_inf:
        s[:HW] = np.inf
    return s


# ---------------------------------------------------------------------------
# Step 2/3: active set and its compaction into ascending indices
# ---------------------------------------------------------------------------
def compact(active: np.ndarray) -> np.ndarray:
    """Boolean active mask -> ascending int32 index list."""
    return np.nonzero(np.asarray(active, bool))[0].astype(np.int32)


def select_threshold(s, tau: float) -> np.ndarray:
    """[LIPAR] 2.B: a token is redundant (pruned) when its change is below tau;
    hence active iff s >= tau. NaN scores are never active."""
    s = np.asarray(s, np.float64)
    return compact(s >= tau)


def _rank_order(s) -> np.ndarray:
    """Token indices by score descending, ties by ascending index, NaN last.
    -0.0 and +0.0 are equal scores."""
    s = np.asarray(s, np.float64)
    nan = np.isnan(s)                                 # NaN ranks below every number, -inf included
    key = np.where(nan, 0.0, -s)
    key = np.where(key == 0.0, 0.0, key)             # fold -0.0 into +0.0
    return np.lexsort((np.arange(len(s)), key, nan))


def select_topk(s, k: int) -> np.ndarray:
    """The k highest-scoring tokens (ties to the lower index), as an ascending
    index list. k = len(s) keeps every token (the dense special case)."""
    order = _rank_order(s)
    return np.sort(order[:k]).astype(np.int32)


def group_split(s, K: int) -> np.ndarray:
    """[HSA] 2.1: partition the N tokens into K disjoint groups by relative-L1
    velocity change (dynamic token selection). Reading: rank by score
    descending (ties to the lower index); group g holds ranks
    [g*(N//K), (g+1)*(N//K)), the remainder going to the last group. Group 0
    (G_1, fastest changing) is the reference group. Returns int8 [N]."""
    N = len(s)
    order = _rank_order(s)
    size = N // K
    g = np.empty(N, np.int8)
    for r, n in enumerate(order):
        g[n] = min(r // size, K - 1)
    return g


def schedule_groups(K: int, budgets, T: int, step: int, m: int) -> np.ndarray:
    """[HSA] 2.1 and 2.4: which groups are active at global step i.
    Group k (budget s_k, a divisor of T) is active iff i mod (T / s_k) == 0;
    in the first and last m steps every token runs."""
    if step < m or step >= T - m:
        return np.ones(K, bool)
    return np.array([step % (T // budgets[k]) == 0 for k in range(K)], bool)


def schedule_active(group, K: int, budgets, T: int, step: int, m: int) -> np.ndarray:
    """Ascending active index list A_i for step i given the group table."""
    act = schedule_groups(K, budgets, T, step, m)
    g = np.asarray(group).astype(np.int64)
    ok = (g >= 0) & (g < K)
    mask = np.zeros(len(g), bool)
    mask[ok] = act[g[ok]]
    return compact(mask)


# ---------------------------------------------------------------------------
# Counter-based normals: Philox4x32-10 [Philox] + Box-Muller [BM]
# ---------------------------------------------------------------------------
_PHILOX_M = (0xD2511F53, 0xCD9E8D57)   # multipliers, [Philox] section 4
_PHILOX_W = (0x9E3779B9, 0xBB67AE85)   # Weyl key increments
_MASK32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(c0, c1, c2, c3, k0: int, k1: int):
    """Philox4x32 with 10 rounds on uint32 counters (numpy arrays) and key.

    One round: (hi0, lo0) = M0 * c0, (hi1, lo1) = M1 * c2 (64-bit products);
    new counter = (hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0). The key is bumped
    by the Weyl constants between rounds. Pinned by the published
    known-answer vectors (tests/golden/philox_kat.json)."""
    c = [np.asarray(v, np.uint64) & _MASK32 for v in (c0, c1, c2, c3)]
    k = [np.uint64(k0) & _MASK32, np.uint64(k1) & _MASK32]
    m0, m1 = np.uint64(_PHILOX_M[0]), np.uint64(_PHILOX_M[1])
    for r in range(10):
        p0 = m0 * c[0]
        p1 = m1 * c[2]
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK32
        c = [hi1 ^ c[1] ^ k[0], lo1, hi0 ^ c[3] ^ k[1], lo0]
        k = [(k[0] + np.uint64(_PHILOX_W[0])) & _MASK32, (k[1] + np.uint64(_PHILOX_W[1])) & _MASK32]
    return [v.astype(np.uint32) for v in c]


def philox_words(seed: int, step: int, tensor: int, q) -> np.ndarray:
    """The four 32-bit words for counter block q: counter = (q mod 2^32,
    q div 2^32, step, tensor), key = (seed mod 2^32, seed div 2^32).
    Returns uint32 [len(q), 4]."""
    q = np.asarray(q, np.uint64)
    w = philox4x32_10(q & _MASK32, q >> np.uint64(32), np.full(q.shape, step, np.uint64),
                      np.full(q.shape, tensor, np.uint64), seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF)
    return np.stack(w, axis=-1)


def renoise_normals(seed: int, step: int, tensor: int, e) -> np.ndarray:
    """N(0,1) deviate for flat element index e (float64).

    Element e uses word (e mod 4) of counter block q = e div 4. Each word w
    maps to u = (floor(w / 2^9) + 1/2) * 2^-23 in (0, 1), a value that is
    exact in fp32 as well as fp64. Words (0, 1) and (2, 3) form Box-Muller
    pairs: r = sqrt(-2 ln u_a), z_a = r cos(2 pi u_b), z_b = r sin(2 pi u_b).
    Pinned by the radius (z_a^2 + z_b^2 = -2 ln u_a) and angle
    (atan2(z_b, z_a) = 2 pi u_b) identities read back from the raw words, by
    within-pair independence, and by planted pairing slips
    (tests/test_oracle_pins.py)."""
    e = np.asarray(e, np.int64)
    q = (e >> 2).astype(np.uint64)
    j = e & 3
    w = philox_words(seed, step, tensor, q).astype(np.float64)
    u = (np.floor(w / 512.0) + 0.5) * 2.0 ** -23
    pair = (j >> 1) * 2                       # 0 for words 0/1, 2 for words 2/3
    ua = np.take_along_axis(u, pair[:, None], 1)[:, 0]
    ub = np.take_along_axis(u, (pair + 1)[:, None], 1)[:, 0]
    r = np.sqrt(-2.0 * np.log(ua))
    return np.where((j & 1) == 0, r * np.cos(2 * np.pi * ub), r * np.sin(2 * np.pi * ub))


# ---------------------------------------------------------------------------
# Step 4: KV-cache synchronisation (+ noise-aware duplication)
# ---------------------------------------------------------------------------
def kv_sync(k_cache, v_cache, k_fresh, v_fresh, idx, renoise=None, heads=None):
    """[HSA] 2.2: only active tokens produce fresh K/V; those rows overwrite the
    per-layer cache, the other rows stay stale but valid. Returns the updated
    caches (bf16, bit copies) and, when ``renoise`` is given, float64 K_eff /
    V_eff.

    ``renoise = (a, b, seed, step)``: [LIPAR] 2.C noise-aware duplication
    re-uses clean cached tokens with fresh noise. Reading: for pruned rows n,
    eff[n] = a * cache[n] + b * eps(n), eps drawn independently for K (tensor
    0) and V (tensor 1) at flat element (n*H + h)*d + c; active rows take the
    fresh row. The noised rows are not written back into the cache.

    ``heads`` restricts K_eff / V_eff to a subset of heads (shape [N, len(heads),
    d]) for sampled checks at full size.
    """
    kc = k_cache.clone()
    vc = v_cache.clone()
    idx_t = torch.as_tensor(np.asarray(idx, np.int64))
    if len(idx_t):
        kc[idx_t] = k_fresh[: len(idx_t)]
        vc[idx_t] = v_fresh[: len(idx_t)]
    if renoise is None:
        return kc, vc, None, None
    a, b, seed, step = renoise
    N, H, d = kc.shape
    heads = np.arange(H) if heads is None else np.asarray(heads, np.int64)
    pruned = np.setdiff1d(np.arange(N), np.asarray(idx, np.int64))
    cols = (heads[:, None] * d + np.arange(d)[None, :]).reshape(-1)      # flat (h, c) offsets
    out = []
    for t, cache in ((0, kc), (1, vc)):
        eff = f64(cache[:, torch.as_tensor(heads)])
        for p0 in range(0, len(pruned), 4096):
            rows = pruned[p0:p0 + 4096]
            e = (rows[:, None] * (H * d) + cols[None, :]).reshape(-1)
            z = renoise_normals(seed, step, t, e).reshape(len(rows), len(heads), d)
            eff[rows] = a * eff[rows] + b * z
        out.append(eff)
    return kc, vc, out[0], out[1]


# ---------------------------------------------------------------------------
# Step 5: attention of active queries over all N cached keys
# ---------------------------------------------------------------------------
def pruned_attn(q_act, k, v, idx, scale: float, blockmask=None, block: int = 128,
                rows=None, heads=None):
    """[HSA] 2.2 (3)-(4): active queries attend the full cached K/V, cost
    O(|A_i| * N). For every active j and head h

        o[j, h] = sum_n softmax_n(scale * q[j, h] . k[n, h]) v[n, h]

    over the allowed keys n: all N, or (key-block sparsity in the style of
    [SVOO] part 2) only keys whose 128-token block kb has
    blockmask[idx[j] // block, kb] = 1 -- the mask row is that of the query's
    ORIGINAL token block. Also returns lse = log sum_n exp(scale * q . k_n)
    (natural log). A query with no allowed key gets o = 0, lse = -inf.

    ``rows`` restricts to a subset of active rows (sampled checks at full
    size); ``heads`` to a subset of heads. Returns float64 (o [R, Hs, d],
    lse [R, Hs]).
    """
    A, H, d = q_act.shape
    N = k.shape[0]
    idx = np.asarray(idx, np.int64)
    rows = np.arange(A) if rows is None else np.asarray(rows, np.int64)
    heads = np.arange(H) if heads is None else np.asarray(heads, np.int64)
    o = np.zeros((len(rows), len(heads), d))
    lse = np.full((len(rows), len(heads)), -np.inf)
    if len(rows) == 0:
        return o, lse
    if blockmask is not None:
        bm = np.asarray(blockmask.cpu().numpy() if isinstance(blockmask, torch.Tensor) else blockmask) != 0
        key_block = np.arange(N) // block
    chunk = max(1, min(len(rows), (1 << 24) // max(N, 1)))
    for hi, h in enumerate(heads):
        Kh, Vh = f64(k[:, h]), f64(v[:, h])                        # one head in fp64
        for c0 in range(0, len(rows), chunk):
            r = rows[c0:c0 + chunk]
            S = (f64(q_act[r, h]) @ Kh.T) * scale                  # [c, N]
            if blockmask is not None:
                S = np.where(bm[idx[r] // block][:, key_block], S, -np.inf)
            mx = S.max(axis=1)
            ok = np.isfinite(mx)
            P = np.exp(S - np.where(ok, mx, 0.0)[:, None])
            P[~ok] = 0.0
            l = P.sum(axis=1)
            O = P @ Vh
            o[c0:c0 + len(r), hi] = np.where(ok[:, None], O / np.where(ok, l, 1.0)[:, None], 0.0)
            lse[c0:c0 + len(r), hi] = np.where(ok, mx + np.log(np.where(ok, l, 1.0)), -np.inf)
    return o, lse


def lse_merge(o1, lse1, o2, lse2):
    """[LIPAR] 2.C (Spanish summary, M-degree approximation): the attention of
    removed tokens is recovered through a log-sum-exp based combination. Reading:
    attention over a key set split into two disjoint parts is assembled exactly
    from the two partial results. With w_i = exp(lse_i):
        o = (w1 * o1 + w2 * o2) / (w1 + w2),   lse = log(w1 + w2).
    A part with lse = -inf (no key) contributes nothing; two empty parts give
    o = 0, lse = -inf. Returns float64 (o [A, H, d], lse [A, H])."""
    O1, O2 = f64(o1), f64(o2)
    L1, L2 = f64(lse1), f64(lse2)
    m = np.maximum(L1, L2)
    ok = np.isfinite(m)
    mm = np.where(ok, m, 0.0)
    a = np.where(ok, np.exp(L1 - mm), 0.0)
    b = np.where(ok, np.exp(L2 - mm), 0.0)
    den = np.where(ok, a + b, 1.0)
    o = (a[..., None] * O1 + b[..., None] * O2) / den[..., None]
    return np.where(ok[..., None], o, 0.0), np.where(ok, m + np.log(den), -np.inf)


def lipar_score_motion(x, L: int) -> np.ndarray:
    """[LIPAR] 2.B (both summaries): motion detection with short- and long-term
    differences makes the pruning mask robust. Reading: a token is pruned only
    when BOTH its short-term change (against frame f-1) and its long-term change
    (against the key frame max(f-L, 0)) are small, i.e. the score is
        s(f, p) = max(s_short(f, p), s_long(f, p)),
    each a relative L1 change as in lipar_score; frame 0 is +inf. L >= 1
    (L = 1 is the plain inter-frame score)."""
    X = f64(x)
    F, HW, C = X.shape
    s = np.full((F, HW), np.inf)
    for f in range(1, F):
        parts = []
        for r in (f - 1, max(f - L, 0)):
            num = np.abs(X[f] - X[r]).sum(axis=1)
            den = np.abs(X[r]).sum(axis=1)
            with np.errstate(divide="ignore", invalid="ignore"):
                parts.append(np.where(den > 0, num / np.where(den > 0, den, 1.0), np.where(num > 0, np.inf, 0.0)))
        s[f] = np.maximum(parts[0], parts[1])
    return s.reshape(-1)


def attn_flops(A: int, N: int, H: int, d: int, keys_per_query=None) -> float:
    """Algorithmic FLOPs: 2*d for q.k plus 2*d for p*v per (query, key, head)."""
    if keys_per_query is None:
        return 4.0 * d * H * A * N
    return 4.0 * d * H * float(np.sum(keys_per_query))


# ---------------------------------------------------------------------------
# Step 6: restoration of the full-length output
# ---------------------------------------------------------------------------
def scatter_out(o_full, o_act, idx):
    """[LIPAR] (Dutch summary) 2.D: pruned tokens are restored by duplication so
    the decoder sees a full-length sequence. Reading: active rows take the new
    output, every other row keeps its cached output bit-for-bit."""
    out = o_full.clone()
    idx_t = torch.as_tensor(np.asarray(idx, np.int64))
    if len(idx_t):
        out[idx_t] = o_act[: len(idx_t)]
    return out


def euler_update(x, v_cache, v_fresh, idx, dsigma: float):
    """[HSA] 2.3 cached Euler update: every token keeps the velocity predicted at
    its most recent active step; at each global step ALL tokens advance by the
    same Euler increment (sigma_{i+1} - sigma_i) -- active tokens with their
    fresh velocity, skipped tokens with the cached one -- as one operation over
    the N tokens. Reading: the sampler state x is float32, velocities bf16.

    Returns (x_new float64 [N, C], v_cache_new bf16 [N, C]) with
    v_cache_new[idx] = v_fresh (bit copies) and x_new = x + dsigma * v_cache_new."""
    vc = v_cache.clone()
    idx_t = torch.as_tensor(np.asarray(idx, np.int64))
    if len(idx_t):
        vc[idx_t] = v_fresh[: len(idx_t)]
    return f64(x) + float(dsigma) * f64(vc), vc


def gather_rows(src, idx):
    """Rows idx of src (the active tokens handed to the QKV projection,
    [HSA] 2.2 (1))."""
    return src[torch.as_tensor(np.asarray(idx, np.int64))].clone()


# ---------------------------------------------------------------------------
# Timeripple: per-axis similarity check of Q / K tokens
# ---------------------------------------------------------------------------
def timeripple_delta(x, F: int, Hs: int, Ws: int, windows) -> np.ndarray:
    """[TR] Metodologia 2 (similarity checks): for every Q (or K) token three
    independent checks run along the temporal, x and y axes, each measuring a
    standard error over a window of the token's channels.

    Readings: x is [N, H, d] with token n = (f * Hs + y) * Ws + x_col. The
    neighbour along an axis is the previous token on it: t -> n - Hs*Ws (f >= 1),
    x -> n - 1 (x_col >= 1), y -> n - Ws (y >= 1). windows[a] = (start, length)
    picks the head-dim channels (start + j) mod d, j < length (a cyclic window,
    0 <= length <= d). The standard error is the root-mean-square difference
    over the window,
        Delta_a(n, h) = sqrt( sum_{c in W_a} (x[n,h,c] - x[nb_a(n),h,c])^2 / length_a ),
    and +inf when the token has no neighbour on that axis or length_a = 0.
    Returns float64 [3, N, H] in axis order (t, x, y)."""
    X = f64(x)
    N, H, d = X.shape
    assert N == F * Hs * Ws
    G = X.reshape(F, Hs, Ws, H, d)
    out = np.full((3, F, Hs, Ws, H), np.inf)
    for a, (start, length) in enumerate(windows):
        if length == 0:
            continue
        ch = (int(start) + np.arange(int(length))) % d
        if a == 0:
            cur, nb, dst = G[1:], G[:-1], out[0, 1:]
        elif a == 1:
            cur, nb, dst = G[:, :, 1:], G[:, :, :-1], out[1, :, :, 1:]
        else:
            cur, nb, dst = G[:, 1:], G[:, :-1], out[2, :, 1:]
        diff = cur[..., ch] - nb[..., ch]
        dst[...] = np.sqrt((diff * diff).sum(axis=-1) / float(length))
    return out.reshape(3, N, H)


def timeripple_reuse(delta, theta) -> np.ndarray:
    """[TR] Metodologia 2 (reuse decision): a token is reusable when its
    Delta is below the threshold on ANY of the three axes (logical OR).
    Returns uint8 [N, H] with bit a set iff Delta_a < theta_a, so a
    (token, head) is reusable iff its byte is non-zero."""
    D = np.asarray(delta, np.float64)
    bits = np.zeros(D.shape[1:], np.uint8)
    for a in range(3):
        bits |= (D[a] < float(theta[a])).astype(np.uint8) << a
    return bits


def timeripple_token_score(reuse) -> np.ndarray:
    """Reading that joins the per-(token, head) decision to the token-level
    active set: score[n] = number of heads of token n that are NOT reusable
    (an integer, float64). Thresholding it at 1 (lipar_select, tau = 1)
    keeps every token that needs any head recomputed."""
    return (np.asarray(reuse) == 0).sum(axis=1).astype(np.float64)


def timeripple_theta(step: int, theta_lo: float, theta_hi: float, i0: int = 11, i1: int = 21) -> float:
    """[TR] Metodologia 3: thresholds rise linearly over the critical window of
    steps i0..i1 (11..21, steps counted as on the page) and stay fixed
    outside it: theta_lo up to i0, theta_hi from i1 on."""
    if step <= i0:
        return float(theta_lo)
    if step >= i1:
        return float(theta_hi)
    return float(theta_lo) + (float(theta_hi) - float(theta_lo)) * (step - i0) / float(i1 - i0)


# ---------------------------------------------------------------------------
# Attention recovery: re-rotation of keys duplicated across frames
# ---------------------------------------------------------------------------
def rope_rotate(k, dims, shift, base: float = 10000.0) -> np.ndarray:
    """Rotary position offset of keys ([LIPAR] 2.C, Dutch summary: the K/V of a
    pruned token are approximated from the previous frame's cache, taking the
    RoPE rotations into account; [TR] Metodologia 1: the rotary channels of a
    head form temporal, x and y groups).

    Reading: a head's d channels are the contiguous groups [t | x | y] of
    sizes dims = (d_t, d_x, d_y) (all even, summing to d). Inside group a
    (channel offset o_a, size d_a) the adjacent channels (o_a + 2j,
    o_a + 2j + 1) form pair j with frequency theta = base^(-2j / d_a); a
    position offset shift = (s_t, s_x, s_y) rotates that pair by phi = s_a *
    theta:  (x, y) -> (x cos phi - y sin phi, x sin phi + y cos phi).
    k is [..., d] (bf16 tensor or array); returns float64 of the same shape.
    Pinned by a hand-worked example (tests/golden/rope_worked.json), the
    complex-number form z * exp(i phi) (numpy), composition of offsets, norm
    preservation, relative-offset invariance of q . k, and planted slips."""
    x = f64(k)
    out = x.copy()
    o = 0
    for a in range(3):
        da = int(dims[a])
        j = np.arange(da // 2)
        phi = float(shift[a]) * base ** (-2.0 * j / da)
        c, s = np.cos(phi), np.sin(phi)
        ev, od = x[..., o + 2 * j], x[..., o + 2 * j + 1]
        out[..., o + 2 * j] = ev * c - od * s
        out[..., o + 2 * j + 1] = ev * s + od * c
        o += da
    return out


def kv_rerotate(k_cache, idx, dims, shift, base: float = 10000.0) -> np.ndarray:
    """K_eff for attention when pruned tokens reuse cached keys of the previous
    frame ([LIPAR] 2.C): the row of an active token (in idx) is its cache row
    (already the fresh key after kv_sync); the row of a pruned token is its
    cache row moved to the token's own position, rope_rotate(row, shift) --
    the configured reading is shift = (1, 0, 0), one frame later. k_cache is
    [N, H, d]; returns float64 [N, H, d]."""
    out = f64(k_cache)
    N = out.shape[0]
    pruned = np.setdiff1d(np.arange(N), np.asarray(idx, np.int64))
    if len(pruned):
        out[pruned] = rope_rotate(out[pruned], dims, shift, base)
    return out
