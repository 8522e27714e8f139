"""C ABI checks that need no GPU: the library loads, exports every function
include/tps.h declares, and rejects bad arguments on the host (before any CUDA
call) with the documented status codes and a message."""
import ctypes as C
import os
import re

import pytest

from token_pruned_sparse_b200 import tps

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tps.h")


def declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^TPS_API\s+[\w\s\*]+?\b(\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_path():
    names = declared()
    for n in ("lipar_score", "lipar_select", "lipar_group", "lipar_schedule", "kv_sync", "pruned_attn",
              "scatter_out", "tps_gather_rows", "tps_workspace_size", "tps_last_error", "tps_check"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = tps.lib()
    missing = [n for n in declared() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(tps.SIGNATURES) >= set(declared())
    assert "sm_100a" in tps.version()


F = C.c_void_p(0x1000)        # fake, 16-byte aligned, never dereferenced
MIS = C.c_void_p(0x1001)      # misaligned
NULL = None


def _err(code):
    return code, tps.lib().tps_last_error().decode()


def test_score_validation():
    l = tps.lib()
    assert _err(l.lipar_score(NULL, NULL, NULL, 2, 4, 64, F, NULL))[0] == tps.INVALID_ARG
    code, msg = _err(l.lipar_score(F, NULL, NULL, 2, 4, 60, F, NULL))
    assert code == tps.SHAPE and "C=60" in msg
    assert l.lipar_score(MIS, NULL, NULL, 2, 4, 64, F, NULL) == tps.ALIGN
    assert l.lipar_score(F, F, F, 2, 4, 64, F, NULL) == tps.INVALID_ARG
    assert l.lipar_score(F, NULL, NULL, 0, 4, 64, F, NULL) == tps.SHAPE


def test_select_validation_and_workspace():
    l = tps.lib()
    assert l.lipar_select(F, 10, 5, 0.0, 0, F, F, F, 1 << 20, NULL) == tps.INVALID_ARG
    code, msg = _err(l.lipar_select(F, 10, tps.SELECT_TOPK, 0.0, 11, F, F, F, 1 << 20, NULL))
    assert code == tps.INVALID_ARG and "k=11" in msg
    need = tps.workspace_size(tps.OP_SELECT, 100000)
    assert need > 0 and tps.workspace_size(tps.OP_SELECT, 200000) > need
    code, msg = _err(l.lipar_select(F, 100000, tps.SELECT_THRESHOLD, 0.0, 0, F, F, F, 1024, NULL))
    assert code == tps.WORKSPACE and "required" in msg
    assert l.lipar_select(F, 100000, tps.SELECT_THRESHOLD, 0.0, 0, F, F, NULL, need, NULL) == tps.WORKSPACE
    assert l.lipar_select(F, 100000, tps.SELECT_THRESHOLD, 0.0, 0, F, F, MIS, need, NULL) == tps.ALIGN
    assert tps.workspace_size(9, 10) == 0
    assert l.lipar_group(F, 10, 9, F, F, 1 << 20, NULL) == tps.INVALID_ARG
    assert l.lipar_group(F, 2, 3, F, F, 1 << 20, NULL) == tps.INVALID_ARG
    bad = (C.c_int32 * 3)(40, 20, 7)                     # 7 does not divide 40
    code, msg = _err(l.lipar_schedule(F, 10, 3, C.cast(bad, C.c_void_p), 40, 0, 0, F, F, F, 1 << 20, NULL))
    assert code == tps.INVALID_ARG and "divide" in msg
    good = (C.c_int32 * 3)(40, 20, 10)
    assert l.lipar_schedule(F, 10, 3, C.cast(good, C.c_void_p), 40, 40, 0, F, F, F, 1 << 20, NULL) == tps.INVALID_ARG


def test_rows_and_attention_validation():
    l = tps.lib()
    assert l.kv_sync(F, F, F, F, F, F, 10, 100, 2, 96, NULL, NULL, NULL, NULL) == tps.INVALID_ARG
    assert l.kv_sync(F, F, F, F, NULL, F, 10, 100, 2, 64, NULL, NULL, NULL, NULL) == tps.INVALID_ARG
    rn = tps.Renoise(0.5, 0.5, 1, 0, 0)
    assert l.kv_sync(F, F, F, F, F, F, 10, 100, 2, 64, C.cast(C.byref(rn), C.c_void_p), NULL, NULL, NULL) == \
        tps.INVALID_ARG
    assert l.kv_sync(MIS, F, F, F, F, F, 10, 100, 2, 64, NULL, NULL, NULL, NULL) == tps.ALIGN
    assert l.scatter_out(F, F, F, F, 10, 0, 2, 64, NULL) == tps.SHAPE
    assert l.tps_gather_rows(F, F, F, F, 10, 100, 24, NULL) == tps.SHAPE
    for fn in (l.pruned_attn, l.pruned_attn_mma):
        assert fn(F, F, F, F, F, 10, 100, 2, 80, 0.1, NULL, 128, F, NULL, NULL) == tps.INVALID_ARG
        assert fn(F, F, F, F, F, 10, 100, 0, 64, 0.1, NULL, 128, F, NULL, NULL) == tps.SHAPE
        assert fn(F, F, F, F, F, 10, 100, 2, 64, 0.1, F, 64, F, NULL, NULL) == tps.INVALID_ARG
        assert fn(F, F, F, F, F, 10, 4097 * 128, 2, 64, 0.1, F, 128, F, NULL, NULL) == tps.SHAPE
        assert fn(MIS, F, F, F, F, 10, 100, 2, 64, 0.1, NULL, 128, F, NULL, NULL) == tps.ALIGN
        assert fn(F, F, F, F, F, 10, 100, 2, 64, float("nan"), NULL, 128, F, NULL, NULL) == tps.INVALID_ARG
    assert l.tps_philox_fill(MIS, 0, 4, 1, 0, 0, NULL) == tps.ALIGN


def test_binding_raises_with_message():
    with pytest.raises(tps.TPSError) as e:
        tps._chk(tps.lib().lipar_score(NULL, NULL, NULL, 2, 4, 64, F, NULL))
    assert e.value.code == tps.INVALID_ARG and "non-null" in str(e.value)


def test_timeripple_validation_and_theta_ramp():
    import oracle as O
    l = tps.lib()
    win = (C.c_int32 * 6)(44, 84, 86, 86, 0, 86)
    th = (C.c_float * 3)(0.05, 0.05, 0.05)
    W, T = C.cast(win, C.c_void_p), C.cast(th, C.c_void_p)
    assert l.timeripple_score(NULL, 2, 4, 4, 2, 128, W, T, F, NULL, NULL, NULL) == tps.INVALID_ARG
    assert l.timeripple_score(F, 2, 4, 4, 2, 128, W, T, NULL, NULL, NULL, NULL) == tps.INVALID_ARG
    code, msg = _err(l.timeripple_score(F, 2, 4, 4, 2, 96, W, T, F, NULL, NULL, NULL))
    assert code == tps.INVALID_ARG and "d=96" in msg
    assert l.timeripple_score(F, 0, 4, 4, 2, 128, W, T, F, NULL, NULL, NULL) == tps.SHAPE
    assert l.timeripple_score(F, 2, 4, 4, 0, 128, W, T, F, NULL, NULL, NULL) == tps.SHAPE
    bad = (C.c_int32 * 6)(44, 84, 128, 1, 0, 86)           # start = d
    code, msg = _err(l.timeripple_score(F, 2, 4, 4, 2, 128, C.cast(bad, C.c_void_p), T, F, NULL, NULL, NULL))
    assert code == tps.INVALID_ARG and "window 1" in msg
    longw = (C.c_int32 * 6)(0, 65, 0, 64, 0, 64)           # longer than d = 64
    assert l.timeripple_score(F, 2, 4, 4, 2, 64, C.cast(longw, C.c_void_p), T, F, NULL, NULL, NULL) == \
        tps.INVALID_ARG
    nan = (C.c_float * 3)(0.05, float("nan"), 0.05)
    assert l.timeripple_score(F, 2, 4, 4, 2, 128, W, C.cast(nan, C.c_void_p), F, NULL, NULL, NULL) == \
        tps.INVALID_ARG
    assert l.timeripple_score(MIS, 2, 4, 4, 2, 128, W, T, F, NULL, NULL, NULL) == tps.ALIGN
    # the host-only threshold ramp against the oracle's (fp32 vs fp64)
    for lo, hi in ((0.0, 0.05), (0.2, 0.1), (1.0, 3.0)):
        for step in range(0, 45):
            assert tps.timeripple_theta(step, lo, hi) == pytest.approx(O.timeripple_theta(step, lo, hi),
                                                                       rel=1e-6, abs=1e-8)
    assert tps.timeripple_theta(5, 1.0, 2.0, 7, 7) == 1.0 and tps.timeripple_theta(8, 1.0, 2.0, 7, 7) == 2.0


def test_workspace_min_size_is_a_lower_bound():
    for op, K in ((tps.OP_SELECT, 0), (tps.OP_GROUP, 3), (tps.OP_SCHEDULE, 3)):
        for N in (1, 1000, 118800, 600000, 1 << 22):
            lo, rec = tps.workspace_min_size(op, N, K), tps.workspace_size(op, N, K)
            assert 0 < lo <= rec
    assert tps.workspace_min_size(9, 10, 0) == 0
    F = C.c_void_p(0x1000)
    need = tps.workspace_min_size(tps.OP_SELECT, 100000)
    assert tps.lib().lipar_select(F, 100000, tps.SELECT_TOPK, 0.0, 5, F, F, F, need - 1, NULL) == tps.WORKSPACE


def test_rerotate_validation():
    l = tps.lib()
    P = lambda r: C.cast(C.byref(r), C.c_void_p)               # noqa: E731
    good = tps.Rope((C.c_int32 * 3)(24, 20, 20), (C.c_int32 * 3)(1, 0, 0), 10000.0, 0)
    odd = tps.Rope((C.c_int32 * 3)(23, 21, 20), (C.c_int32 * 3)(1, 0, 0), 10000.0, 0)
    short = tps.Rope((C.c_int32 * 3)(24, 20, 18), (C.c_int32 * 3)(1, 0, 0), 10000.0, 0)
    far = tps.Rope((C.c_int32 * 3)(24, 20, 20), (C.c_int32 * 3)((1 << 20) + 1, 0, 0), 10000.0, 0)
    nobase = tps.Rope((C.c_int32 * 3)(24, 20, 20), (C.c_int32 * 3)(1, 0, 0), 0.0, 0)
    assert _err(l.kv_rerotate(F, F, F, 10, 100, 2, 64, P(odd), F, NULL))[0] == tps.INVALID_ARG
    code, msg = _err(l.kv_rerotate(F, F, F, 10, 100, 2, 64, P(short), F, NULL))
    assert code == tps.INVALID_ARG and "sum to 62" in msg
    assert l.kv_rerotate(F, F, F, 10, 100, 2, 64, P(far), F, NULL) == tps.INVALID_ARG
    assert l.kv_rerotate(F, F, F, 10, 100, 2, 64, P(nobase), F, NULL) == tps.INVALID_ARG
    assert l.kv_rerotate(F, F, F, 10, 100, 2, 64, NULL, F, NULL) == tps.INVALID_ARG
    assert l.kv_rerotate(F, F, F, 10, 100, 2, 96, P(good), F, NULL) == tps.INVALID_ARG
    assert l.kv_rerotate(MIS, F, F, 10, 100, 2, 64, P(good), F, NULL) == tps.ALIGN
    assert l.kv_rerotate(F, F, F, 10, 0, 2, 64, P(good), F, NULL) == tps.SHAPE


def test_attn_plan_validation():
    l = tps.lib()
    s, t = C.c_int(0), C.c_int(0)
    m = C.c_int64(0)
    args = lambda cap, N, H, d: (cap, N, H, d, C.byref(s), C.byref(m), C.byref(t))   # noqa: E731
    assert l.tps_attn_plan(*args(100, 0, 2, 128)) == tps.INVALID_ARG
    assert l.tps_attn_plan(*args(100, 10, 2, 96)) == tps.INVALID_ARG
    assert l.tps_attn_plan(*args(-1, 10, 2, 64)) == tps.INVALID_ARG
    assert l.tps_attn_plan(100, 10, 2, 64, NULL, C.byref(m), C.byref(t)) == tps.INVALID_ARG
    assert l.tps_attn_plan(*args(0, 10, 2, 64)) == tps.OK
    assert (s.value, m.value, t.value) == (1, 0, 1)


def test_front_validation():
    l = tps.lib()
    need = tps.workspace_min_size(tps.OP_FRONT, 100, 3)
    assert need >= 400 and tps.workspace_size(tps.OP_FRONT, 100, 3) >= need
    args = lambda mode, k=5, K=3, ws=F, nws=1 << 20, x=F: (x, NULL, NULL, 4, 25, 128, mode, 0.5, k, K, NULL,   # noqa: E731
                                                          F, F, F, ws, nws, NULL)
    assert l.lipar_front(*args(3)) == tps.INVALID_ARG
    assert l.lipar_front(*args(1, k=101)) == tps.INVALID_ARG
    assert l.lipar_front(*args(2, K=9)) == tps.INVALID_ARG
    assert l.lipar_front(*args(0, x=NULL)) == tps.INVALID_ARG
    assert l.lipar_front(*args(0, x=MIS)) == tps.ALIGN
    code, msg = _err(l.lipar_front(*args(1, nws=16)))
    assert code == tps.WORKSPACE and "required" in msg
    assert l.lipar_front(F, F, F, 4, 25, 128, 0, 0.5, 5, 3, NULL, F, F, F, F, 1 << 20, NULL) == tps.INVALID_ARG
    assert l.lipar_front(F, NULL, NULL, 4, 25, 100, 0, 0.5, 5, 3, NULL, F, F, F, F, 1 << 20, NULL) == tps.SHAPE
