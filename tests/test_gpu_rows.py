"""GPU parity: kv_sync (plain and re-noised), scatter_out, tps_gather_rows and
the raw Philox stream vs the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle as O
from token_pruned_sparse_b200 import synth
from token_pruned_sparse_b200 import tps

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(N, H, d, A, seed):
    kc = synth.gaussian_bf16((N, H, d), seed)
    vc = synth.gaussian_bf16((N, H, d), seed + 1)
    kf = synth.gaussian_bf16((max(A, 1), H, d), seed + 2)[:A]
    vf = synth.gaussian_bf16((max(A, 1), H, d), seed + 3)[:A]
    idx = np.sort(np.random.default_rng(seed).choice(N, A, replace=False)).astype(np.int32)
    return kc, vc, kf, vf, idx


def _dev_idx(idx, cap=None):
    cap = len(idx) if cap is None else cap
    buf = torch.zeros(max(cap, 1), dtype=torch.int32)
    buf[: len(idx)] = torch.from_numpy(idx)
    return buf.to(DEV), torch.tensor([len(idx)], dtype=torch.int32, device=DEV)


@pytest.mark.parametrize("N,H,d,A", [(256, 2, 64, 100), (1000, 3, 128, 1000), (20280, 12, 128, 6084),
                                     (517, 24, 128, 0), (9, 1, 64, 1)])
def test_kv_sync_plain_bit_exact(N, H, d, A):
    kc, vc, kf, vf, idx = _case(N, H, d, A, N + A)
    kcd, vcd = kc.to(DEV), vc.to(DEV)
    di, dc = _dev_idx(idx)
    kfd = kf.to(DEV) if A else torch.empty((1, H, d), dtype=torch.bfloat16, device=DEV)
    vfd = vf.to(DEV) if A else torch.empty((1, H, d), dtype=torch.bfloat16, device=DEV)
    tps.kv_sync(kcd, vcd, kfd, vfd, di, dc, cap=A)
    k2, v2, _, _ = O.kv_sync(kc, vc, kf, vf, idx)
    assert torch.equal(kcd.cpu(), k2) and torch.equal(vcd.cpu(), v2)
    tps.tps_check()


def _renoise_tol(ref, b):
    # one bf16 rounding of the result (half an ulp each side, so one ulp of
    # slack) plus the fp32 Box-Muller error (|z| <= 6, log/sincos ~1e-6 abs)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -126))) - 7)
    return ulp + abs(b) * 1e-5 + 1e-30


@pytest.mark.parametrize("N,H,d,A,a,b", [(256, 2, 64, 100, 0.3, 0.7), (3001, 3, 128, 1234, 0.9, 0.1),
                                         (5000, 24, 128, 5000, 0.5, 0.5), (777, 4, 64, 0, 0.0, 1.0),
                                         (777, 4, 64, 300, 1.0, 0.0)])
def test_kv_sync_renoise(N, H, d, A, a, b):
    kc, vc, kf, vf, idx = _case(N, H, d, A, 3 * N + A)
    kcd, vcd = kc.to(DEV), vc.to(DEV)
    di, dc = _dev_idx(idx)
    kfd = kf.to(DEV) if A else torch.empty((1, H, d), dtype=torch.bfloat16, device=DEV)
    vfd = vf.to(DEV) if A else torch.empty((1, H, d), dtype=torch.bfloat16, device=DEV)
    seed, step = 0x123456789ABC, 17
    ke, ve = tps.kv_sync(kcd, vcd, kfd, vfd, di, dc, cap=A, renoise=(a, b, seed, step))
    k2, v2, ke_ref, ve_ref = O.kv_sync(kc, vc, kf, vf, idx, renoise=(a, b, seed, step))
    assert torch.equal(kcd.cpu(), k2) and torch.equal(vcd.cpu(), v2)       # cache: bit copies only
    for got, ref in ((ke, ke_ref), (ve, ve_ref)):
        g = got.cpu().double().numpy()
        assert np.array_equal(g[idx], ref[idx])                             # active rows: fresh, exact
        err = np.abs(g - ref)
        assert np.all(err <= _renoise_tol(ref, b)), float(err.max())
    if a == 1.0 and b == 0.0:
        assert torch.equal(ke.cpu(), k2) and torch.equal(ve.cpu(), v2)
    tps.tps_check()


def test_philox_stream_bit_exact():
    for seed, step, t, q0 in ((0, 0, 0, 0), (0xFFFFFFFFFFFFFFFF, 39, 1, 2 ** 32 - 5), (42, 7, 0, 123456789)):
        got = tps.tps_philox_fill(q0, 4099, seed, step, t).cpu().numpy().view(np.uint32).reshape(-1, 4)
        ref = O.philox_words(seed, step, t, np.arange(q0, q0 + 4099, dtype=np.uint64))
        assert np.array_equal(got, ref)


@pytest.mark.parametrize("N,H,d,A", [(256, 2, 64, 100), (20280, 12, 128, 6084), (1000, 1, 64, 0), (130, 24, 128, 130)])
def test_scatter_and_gather_bit_exact(N, H, d, A):
    full = synth.gaussian_bf16((N, H, d), N)
    act = synth.gaussian_bf16((max(A, 1), H, d), N + 1)[:max(A, 1)]
    idx = np.sort(np.random.default_rng(A).choice(N, A, replace=False)).astype(np.int32)
    di, dc = _dev_idx(idx)
    fd = full.to(DEV)
    tps.scatter_out(fd, act.to(DEV), di, dc, cap=A)
    assert torch.equal(fd.cpu(), O.scatter_out(full, act[:A], idx))
    g = torch.empty((max(A, 1), H, d), dtype=torch.bfloat16, device=DEV)
    tps.tps_gather_rows(g, fd, di, dc, cap=A)
    assert torch.equal(g[:A].cpu(), O.gather_rows(fd.cpu(), idx))
    tps.tps_check()


def test_count_below_cap_and_bounds_flag():
    N, H, d = 100, 2, 64
    full = synth.gaussian_bf16((N, H, d), 5)
    act = synth.gaussian_bf16((10, H, d), 6)
    idx = torch.tensor([1, 5, 9, 200, 11, 0, 0, 0, 0, 0], dtype=torch.int32)   # 200 is out of range
    fd = full.to(DEV)
    cnt = torch.tensor([5], dtype=torch.int32, device=DEV)
    tps.scatter_out(fd, act.to(DEV), idx.to(DEV), cnt, cap=10)
    with pytest.raises(tps.TPSError) as e:
        tps.tps_check()
    assert e.value.code == tps.BOUNDS
    ref = O.scatter_out(full, act[[0, 1, 2, 4]], np.array([1, 5, 9, 11]))
    assert torch.equal(fd.cpu(), ref)
    tps.tps_check()                                                         # flag was cleared


# ------------------------------------------------------- HSA cached Euler ---
def _ulp32(a):
    return np.spacing(np.abs(a).astype(np.float32)).astype(np.float64)


@pytest.mark.parametrize("N,C,A", [(256, 64, 100), (1001, 128, 333), (118800, 128, 39600), (50, 8, 50), (77, 16, 0)])
def test_euler_update_parity(N, C, A):
    rng = np.random.default_rng(N + C + A)
    x = torch.from_numpy(rng.standard_normal((N, C)).astype(np.float32))
    vc = synth.gaussian_bf16((N, C), N + 1)
    vf = synth.gaussian_bf16((max(A, 1), C), N + 2)[:max(A, 1)]
    idx = np.sort(rng.choice(N, A, replace=False)).astype(np.int32)
    di, dc = _dev_idx(idx)
    xd, vcd = x.to(DEV), vc.to(DEV)
    dsigma = -2.0 ** -5                                         # exact in fp32 and fp64
    x_ref, vc_ref = x, vc
    for step in range(1, 3):                                    # two steps in a row
        tps.hsa_euler_update(xd, vcd, vf.to(DEV), di, dc, dsigma, cap=A)
        x_ref, vc_ref = O.euler_update(x_ref, vc_ref, vf[:A], idx, dsigma)   # the oracle's own state
        assert torch.equal(vcd.cpu(), vc_ref)
        got = xd.cpu().double().numpy()
        # one fp32 rounding (fmaf) per step on the device, none in the fp64 oracle
        assert np.all(np.abs(got - x_ref) <= step * _ulp32(x_ref) + 1e-45)
    tps.tps_check()


def test_euler_update_flags_bad_index():
    N, C = 64, 8
    x = torch.zeros((N, C), device=DEV)
    vc = torch.zeros((N, C), dtype=torch.bfloat16, device=DEV)
    vf = torch.ones((3, C), dtype=torch.bfloat16, device=DEV)
    idx = torch.tensor([5, 5, 9], dtype=torch.int32, device=DEV)   # duplicate
    tps.hsa_euler_update(x, vc, vf, idx, torch.tensor([3], dtype=torch.int32, device=DEV), 1.0)
    with pytest.raises(tps.TPSError) as e:
        tps.tps_check()
    assert e.value.code == tps.BOUNDS


def test_bounded_wait_gives_up_and_context_survives():
    """The failure-detection path without a fault: a barrier nothing completes,
    waited on with a ~1 ms limit, must end in TPS_ERR_TIMEOUT from tps_check,
    once, and leave the context usable."""
    tps.tps_check()
    tps.tps_wait_probe(2_000_000)
    with pytest.raises(tps.TPSError) as e:
        tps.tps_check()
    assert e.value.code == tps.TIMEOUT
    tps.tps_check()                                                         # cleared
    full = synth.gaussian_bf16((64, 2, 64), 3).to(DEV)
    act = synth.gaussian_bf16((4, 2, 64), 4).to(DEV)
    di, dc = _dev_idx(np.array([1, 7, 30, 63], np.int32))
    tps.scatter_out(full, act, di, dc, cap=4)
    tps.tps_check()
    assert torch.equal(full.cpu()[[1, 7, 30, 63]], act.cpu())


def test_gather_and_scatter_through_pinned_host_memory():
    """Zero-copy use: gathers read rows straight from pinned host memory and
    scatter_out writes rows straight into it; results are the oracle's, bit
    for bit, and pageable memory is reported as not device-accessible."""
    N, H, d, A = 3000, 4, 128, 777
    full = synth.gaussian_bf16((N, H, d), 21).pin_memory()
    assert tps.pointer_is_device_accessible(full)
    assert not tps.pointer_is_device_accessible(torch.zeros(16))       # pageable
    idx = np.sort(np.random.default_rng(22).choice(N, A, replace=False)).astype(np.int32)
    di, dc = _dev_idx(idx)
    g = torch.empty((A, H, d), dtype=torch.bfloat16, device=DEV)
    tps.tps_gather_rows(g, full, di, dc, cap=A)
    tps.tps_check()
    assert torch.equal(g.cpu(), O.gather_rows(full, idx))
    out = synth.gaussian_bf16((N, H, d), 23).pin_memory()
    before = out.clone()
    act = synth.gaussian_bf16((A, H, d), 24)
    tps.scatter_out(out, act.to(DEV), di, dc, cap=A)
    tps.tps_check()
    assert torch.equal(out, O.scatter_out(before, act, idx))


def test_philox_known_answer_vectors_on_gpu():
    """The kernels' Philox4x32-10 against the published known-answer vectors:
    counter = (q mod 2^32, q div 2^32, step, tensor), key = (seed mod 2^32, seed div 2^32)."""
    import json
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "philox_kat.json")) as f:
        cases = json.load(f)["cases"]
    for case in cases:
        c = [int(v, 16) for v in case["counter"]]
        k = [int(v, 16) for v in case["key"]]
        words = tps.tps_philox_fill(c[0] | (c[1] << 32), 1, k[0] | (k[1] << 32), c[2], c[3])
        got = words.cpu().numpy().view(np.uint32).tolist()
        assert got == [int(v, 16) for v in case["out"]]


def _rope_tol(ref, src):
    # one bf16 rounding of the result (one ulp of slack) plus the fp32 table and
    # arithmetic (a few 2^-24 relative of the pair's magnitude)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -126))) - 7)
    pair = (np.abs(src[..., 0::2]) + np.abs(src[..., 1::2])).repeat(2, axis=-1)
    return ulp + 1e-6 * pair + 1e-30


@pytest.mark.parametrize("N,H,d,A,shift,base", [(256, 2, 64, 100, (1, 0, 0), 10000.0),
                                                (4099, 12, 128, 1500, (1, 0, 0), 10000.0),
                                                (3001, 3, 128, 1000, (-3, 2, 5), 500.0),
                                                (517, 24, 128, 0, (2, -1, 0), 10000.0),
                                                (777, 4, 64, 777, (1, 0, 0), 10000.0)])
def test_kv_rerotate_parity(N, H, d, A, shift, base):
    kc, _, _, _, idx = _case(N, H, d, A, 7 * N + A)
    dims = synth.rope_dims(d)
    di, dc = _dev_idx(idx)
    ke = tps.kv_rerotate(kc.to(DEV), di, dc, dims, shift, base, cap=max(A, 1)).cpu()
    ref = O.kv_rerotate(kc, idx, dims, shift, base)
    assert torch.equal(ke[torch.from_numpy(idx).long()], kc[torch.from_numpy(idx).long()])   # active: bit copies
    pruned = np.setdiff1d(np.arange(N), idx)
    got = ke[torch.from_numpy(pruned)].double().numpy()
    err = np.abs(got - ref[pruned])
    assert np.all(err <= _rope_tol(ref[pruned], kc[torch.from_numpy(pruned)].double().numpy()))
    tps.tps_check()


def test_kv_rerotate_zero_shift_in_place_and_full_size():
    # no offset: every row is copied bit for bit (cos 0 = 1, sin 0 = 0), here in place
    kc, _, _, _, idx = _case(1000, 3, 128, 400, 91)
    kcd = kc.to(DEV)
    di, dc = _dev_idx(idx)
    tps.kv_rerotate(kcd, di, dc, synth.rope_dims(128), (0, 0, 0), k_eff=kcd)
    assert torch.equal(kcd.cpu(), kc)
    # the HSA size with the step's schedule-like list: sampled rows against the oracle
    cfg = synth.CONFIGS["hsa"]
    N, H, d = cfg.video.N, cfg.H, cfg.d
    kc = synth.gaussian_bf16((N, H, d), 92)
    idx = np.arange(0, N, 3, dtype=np.int32)
    di, dc = _dev_idx(idx)
    dims = synth.rope_dims(d)
    ke = tps.kv_rerotate(kc.to(DEV), di, dc, dims, (1, 0, 0)).cpu()
    rows = np.sort(np.random.default_rng(93).choice(N, 3000, replace=False))
    ref = O.kv_rerotate(kc[torch.from_numpy(rows)], np.flatnonzero(rows % 3 == 0), dims, (1, 0, 0))
    got = ke[torch.from_numpy(rows)].double().numpy()
    assert np.all(np.abs(got - ref) <= _rope_tol(ref, kc[torch.from_numpy(rows)].double().numpy()))
    tps.tps_check()
