"""Thin ctypes binding of libtps.so (C ABI in include/tps.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels. Tensors are torch CUDA tensors (device memory and streams are
PyTorch's); calls are enqueued on the current torch stream unless ``stream``
is given. A missing or unloadable library raises immediately -- there is no
fallback.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtps.so")
_lib = None

OK, INVALID_ARG, SHAPE, ALIGN, CUDA, TIMEOUT, BOUNDS, WORKSPACE = range(8)
SELECT_THRESHOLD, SELECT_TOPK = 0, 1
OP_SELECT, OP_GROUP, OP_SCHEDULE, OP_FRONT = 0, 1, 2, 3
FRONT_THRESHOLD, FRONT_TOPK, FRONT_GROUP = 0, 1, 2

_P = C.c_void_p
_I64 = C.c_int64
_INT = C.c_int

# name -> (restype, argtypes); mirrors include/tps.h
SIGNATURES = {
    "lipar_score": (_INT, [_P, _P, _P, _I64, _I64, _I64, _P, _P]),
    "lipar_select": (_INT, [_P, _I64, _INT, C.c_float, _I64, _P, _P, _P, C.c_size_t, _P]),
    "lipar_select_static": (_INT, [_P, _I64, _INT, C.c_float, _I64, _P, _P, _P]),
    "lipar_front": (_INT, [_P, _P, _P, _I64, _I64, _I64, _INT, C.c_float, _I64, _INT, _P, _P, _P, _P, _P,
                           C.c_size_t, _P]),
    "lipar_group": (_INT, [_P, _I64, _INT, _P, _P, C.c_size_t, _P]),
    "lipar_schedule": (_INT, [_P, _I64, _INT, _P, _INT, _INT, _INT, _P, _P, _P, C.c_size_t, _P]),
    "tps_gather_rows": (_INT, [_P, _P, _P, _P, _I64, _I64, _I64, _P]),
    "kv_sync": (_INT, [_P, _P, _P, _P, _P, _P, _I64, _I64, _INT, _INT, _P, _P, _P, _P]),
    "kv_rerotate": (_INT, [_P, _P, _P, _I64, _I64, _INT, _INT, _P, _P, _P]),
    "pruned_attn": (_INT, [_P, _P, _P, _P, _P, _I64, _I64, _INT, _INT, C.c_float, _P, _INT, _P, _P, _P]),
    "pruned_attn_ws": (_INT, [_P, _P, _P, _P, _P, _I64, _I64, _INT, _INT, C.c_float, _P, _INT, _P, _P, _P,
                              C.c_size_t, _P]),
    "tps_attn_workspace_size": (C.c_size_t, [_I64, _I64, _INT, _INT]),
    "tps_attn_split": (_INT, [_I64, _I64, _INT, _INT]),
    "tps_attn_plan": (_INT, [_I64, _I64, _INT, _INT, _P, _P, _P]),
    "pruned_attn_pair": (_INT, [_P, _P, _P, _P, _P, _I64, _I64, _INT, _INT, C.c_float, _P, _INT, _P, _P, _P]),
    "pruned_attn_mma": (_INT, [_P, _P, _P, _P, _P, _I64, _I64, _INT, _INT, C.c_float, _P, _INT, _P, _P, _P]),
    "scatter_out": (_INT, [_P, _P, _P, _P, _I64, _I64, _INT, _INT, _P]),
    "hsa_euler_update": (_INT, [_P, _P, _P, _P, _P, _I64, _I64, _I64, C.c_float, _P]),
    "lipar_score_motion": (_INT, [_P, _I64, _I64, _I64, _INT, _P, _P]),
    "attn_lse_merge": (_INT, [_P, _P, _P, _P, _P, _I64, _INT, _INT, _P, _P, _P]),
    "timeripple_score": (_INT, [_P, _I64, _I64, _I64, _INT, _INT, _P, _P, _P, _P, _P, _P]),
    "timeripple_theta": (C.c_float, [_INT, C.c_float, C.c_float, _INT, _INT]),
    "tps_workspace_size": (C.c_size_t, [_INT, _I64, _INT]),
    "tps_workspace_min_size": (C.c_size_t, [_INT, _I64, _INT]),
    "tps_last_error": (C.c_char_p, []),
    "tps_pointer_is_device_accessible": (_INT, [_P]),
    "tps_check": (_INT, [_P]),
    "tps_philox_fill": (_INT, [_P, C.c_uint64, _I64, C.c_uint64, C.c_uint32, C.c_uint32, _P]),
    "tps_wait_probe": (_INT, [_I64, _P]),
    "tps_debug_inject_launch_failures": (None, [_INT]),
    "tps_version": (C.c_char_p, []),
}


class TPSError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"[tps status {code}] {msg}")
        self.code = code


class Renoise(C.Structure):
    """tps_renoise: eff = a * cache + b * eps for pruned rows."""
    _fields_ = [("a", C.c_float), ("b", C.c_float), ("seed", C.c_uint64),
                ("step", C.c_uint32), ("pad_", C.c_uint32)]


def lib() -> C.CDLL:
    """Loads libtps.so once; raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"libtps.so is not built ({_LIB_PATH}); run "
                               "`python -m token_pruned_sparse_b200.build`")
        l = C.CDLL(_LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            if not hasattr(l, name):
                continue            # calling it raises AttributeError; the ABI test flags it
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _lib = l
    return _lib


def _chk(code: int):
    if code != OK:
        raise TPSError(code, lib().tps_last_error().decode())


def _ptr(t):
    return None if t is None else _P(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return _P(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def workspace_size(op: int, N: int, K: int = 0) -> int:
    return int(lib().tps_workspace_size(op, N, K))


def workspace_min_size(op: int, N: int, K: int = 0) -> int:
    return int(lib().tps_workspace_min_size(op, N, K))


def workspace(op: int, N: int, K: int = 0, device=None, minimal: bool = False) -> torch.Tensor:
    n = workspace_min_size(op, N, K) if minimal else workspace_size(op, N, K)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device or "cuda")


# ---- the path -----------------------------------------------------------------------
def lipar_score(x, x_ref=None, x_prev_frame=None, out=None, stream=None):
    """x [F, HW, C] bf16 -> float32 [F*HW] relative-L1 change."""
    F, HW, Cc = x.shape
    if out is None:
        out = torch.empty(F * HW, dtype=torch.float32, device=x.device)
    _chk(lib().lipar_score(_ptr(x), _ptr(x_ref), _ptr(x_prev_frame), F, HW, Cc, _ptr(out), _stream(stream)))
    return out


def lipar_select(score, mode, tau=0.0, k=0, idx=None, count=None, ws=None, stream=None):
    """Returns (idx int32, count int32[1]) on the device."""
    N = score.numel()
    if idx is None:
        idx = torch.empty(max(N if mode == SELECT_THRESHOLD else k, 1), dtype=torch.int32, device=score.device)
    if count is None:
        count = torch.empty(1, dtype=torch.int32, device=score.device)
    if ws is None:
        ws = workspace(OP_SELECT, N, 0, score.device)
    _chk(lib().lipar_select(_ptr(score), N, mode, float(tau), int(k), _ptr(idx), _ptr(count),
                            _ptr(ws), ws.numel(), _stream(stream)))
    return idx, count


def lipar_select_static(score, mode, tau=0.0, k=0, idx=None, count=None, stream=None):
    """lipar_select without a workspace: the library's own static scratch
    (N <= 4,194,304; calls on one device must not overlap on the GPU)."""
    N = score.numel()
    if idx is None:
        idx = torch.empty(max(N if mode == SELECT_THRESHOLD else k, 1), dtype=torch.int32, device=score.device)
    if count is None:
        count = torch.empty(1, dtype=torch.int32, device=score.device)
    _chk(lib().lipar_select_static(_ptr(score), N, mode, float(tau), int(k), _ptr(idx), _ptr(count),
                                   _stream(stream)))
    return idx, count


def lipar_front(x, mode, x_ref=None, x_prev_frame=None, tau=0.0, k=0, K=1, score=None, idx=None, count=None,
                group=None, ws=None, stream=None):
    """Score + selection (mode FRONT_THRESHOLD / FRONT_TOPK -> (idx, count)) or
    score + group split (FRONT_GROUP -> group), in one launch where it applies.
    x [F, HW, C] bf16. Pass a tensor as `score` to also receive the scores."""
    F, HW, Cc = x.shape
    N = F * HW
    dev = x.device
    if mode == FRONT_GROUP:
        if group is None:
            group = torch.empty(N, dtype=torch.int8, device=dev)
    else:
        if idx is None:
            idx = torch.empty(max(N if mode == FRONT_THRESHOLD else k, 1), dtype=torch.int32, device=dev)
        if count is None:
            count = torch.empty(1, dtype=torch.int32, device=dev)
    if ws is None:
        ws = workspace(OP_FRONT, N, K, dev)
    _chk(lib().lipar_front(_ptr(x), _ptr(x_ref), _ptr(x_prev_frame), F, HW, Cc, int(mode), float(tau), int(k),
                           int(K), _ptr(score), _ptr(idx), _ptr(count), _ptr(group), _ptr(ws), ws.numel(),
                           _stream(stream)))
    return group if mode == FRONT_GROUP else (idx, count)


def lipar_group(score, K, group=None, ws=None, stream=None):
    N = score.numel()
    if group is None:
        group = torch.empty(N, dtype=torch.int8, device=score.device)
    if ws is None:
        ws = workspace(OP_GROUP, N, K, score.device)
    _chk(lib().lipar_group(_ptr(score), N, K, _ptr(group), _ptr(ws), ws.numel(), _stream(stream)))
    return group


def lipar_schedule(group, K, budgets, T, step, m=0, idx=None, count=None, ws=None, stream=None):
    N = group.numel()
    b = (C.c_int32 * K)(*budgets)
    if idx is None:
        idx = torch.empty(max(N, 1), dtype=torch.int32, device=group.device)
    if count is None:
        count = torch.empty(1, dtype=torch.int32, device=group.device)
    if ws is None:
        ws = workspace(OP_SCHEDULE, N, K, group.device)
    _chk(lib().lipar_schedule(_ptr(group), N, K, C.cast(b, _P), T, step, m, _ptr(idx), _ptr(count),
                              _ptr(ws), ws.numel(), _stream(stream)))
    return idx, count


def tps_gather_rows(dst, src, idx, count, cap=None, stream=None):
    N = src.shape[0]
    row_bytes = src[0].numel() * src.element_size()
    cap = dst.shape[0] if cap is None else cap
    _chk(lib().tps_gather_rows(_ptr(dst), _ptr(src), _ptr(idx), _ptr(count), cap, N, row_bytes, _stream(stream)))
    return dst


def kv_sync(k_cache, v_cache, k_fresh, v_fresh, idx, count, cap=None, renoise=None, k_eff=None,
            v_eff=None, stream=None):
    """renoise = (a, b, seed, step) or None."""
    N, H, d = k_cache.shape
    cap = k_fresh.shape[0] if cap is None else cap
    rn = None
    if renoise is not None:
        a, b, seed, step = renoise
        rn = Renoise(float(a), float(b), int(seed), int(step), 0)
        if k_eff is None:
            k_eff = torch.empty_like(k_cache)
        if v_eff is None:
            v_eff = torch.empty_like(v_cache)
    _chk(lib().kv_sync(_ptr(k_cache), _ptr(v_cache), _ptr(k_fresh), _ptr(v_fresh), _ptr(idx), _ptr(count),
                       cap, N, H, d, None if rn is None else C.cast(C.byref(rn), _P), _ptr(k_eff), _ptr(v_eff),
                       _stream(stream)))
    return k_eff, v_eff


class Rope(C.Structure):
    """tps_rope: rotary groups (t, x, y), the offset given to pruned rows, base."""
    _fields_ = [("dims", C.c_int32 * 3), ("shift", C.c_int32 * 3), ("base", C.c_float), ("pad_", C.c_int32)]


def kv_rerotate(k_cache, idx, count, dims, shift, base=10000.0, k_eff=None, cap=None, stream=None):
    """k_eff [N, H, d]: active rows copied, pruned rows turned by `shift`."""
    N, H, d = k_cache.shape
    cap = idx.shape[0] if cap is None else cap
    if k_eff is None:
        k_eff = torch.empty_like(k_cache)
    r = Rope((C.c_int32 * 3)(*[int(v) for v in dims]), (C.c_int32 * 3)(*[int(v) for v in shift]), float(base), 0)
    _chk(lib().kv_rerotate(_ptr(k_cache), _ptr(idx), _ptr(count), cap, N, H, d, C.cast(C.byref(r), _P),
                           _ptr(k_eff), _stream(stream)))
    return k_eff


def _attn(fn, q_act, k, v, idx, count, scale, blockmask, block, o_act, lse, cap, stream):
    N, H, d = k.shape
    cap = q_act.shape[0] if cap is None else cap
    if o_act is None:
        o_act = torch.empty_like(q_act)
    _chk(fn(_ptr(q_act), _ptr(k), _ptr(v), _ptr(idx), _ptr(count), cap, N, H, d, float(scale),
            _ptr(blockmask), int(block), _ptr(o_act), _ptr(lse), _stream(stream)))
    return o_act


def pruned_attn(q_act, k, v, idx, count, scale, blockmask=None, block=128, o_act=None, lse=None,
                cap=None, stream=None):
    return _attn(lib().pruned_attn, q_act, k, v, idx, count, scale, blockmask, block, o_act, lse, cap, stream)


def attn_workspace(cap, N, H, d, device=None):
    n = int(lib().tps_attn_workspace_size(cap, N, H, d))
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device or "cuda"), n


def attn_split(cap, N, H, d) -> int:
    """Whole-grid key-range split a dense pruned_attn call of this shape uses (1 = none)."""
    return int(lib().tps_attn_split(int(cap), int(N), int(H), int(d)))


def attn_plan(cap, N, H, d):
    """(split, main_rows, tail_split) of a dense pruned_attn call of this shape."""
    split, tail = C.c_int(0), C.c_int(0)
    main = C.c_int64(0)
    _chk(lib().tps_attn_plan(int(cap), int(N), int(H), int(d), C.byref(split), C.byref(main), C.byref(tail)))
    return split.value, main.value, tail.value


def pruned_attn_ws(q_act, k, v, idx, count, scale, blockmask=None, block=128, o_act=None, lse=None, cap=None,
                   ws=None, stream=None):
    N, H, d = k.shape
    cap = q_act.shape[0] if cap is None else cap
    if o_act is None:
        o_act = torch.empty_like(q_act)
    if ws is None:
        ws, _ = attn_workspace(cap, N, H, d, q_act.device)
    _chk(lib().pruned_attn_ws(_ptr(q_act), _ptr(k), _ptr(v), _ptr(idx), _ptr(count), cap, N, H, d, float(scale),
                              _ptr(blockmask), int(block), _ptr(o_act), _ptr(lse), _ptr(ws), ws.numel(),
                              _stream(stream)))
    return o_act


def pruned_attn_pair(q_act, k, v, idx, count, scale, blockmask=None, block=128, o_act=None, lse=None,
                     cap=None, stream=None):
    return _attn(lib().pruned_attn_pair, q_act, k, v, idx, count, scale, blockmask, block, o_act, lse, cap,
                 stream)


def pruned_attn_mma(q_act, k, v, idx, count, scale, blockmask=None, block=128, o_act=None, lse=None,
                    cap=None, stream=None):
    return _attn(lib().pruned_attn_mma, q_act, k, v, idx, count, scale, blockmask, block, o_act, lse, cap,
                 stream)


def scatter_out(o_full, o_act, idx, count, cap=None, stream=None):
    N, H, d = o_full.shape
    cap = o_act.shape[0] if cap is None else cap
    _chk(lib().scatter_out(_ptr(o_full), _ptr(o_act), _ptr(idx), _ptr(count), cap, N, H, d, _stream(stream)))
    return o_full


def hsa_euler_update(x, v_cache, v_fresh, idx, count, dsigma, cap=None, stream=None):
    """x [N, C] float32 and v_cache [N, C] bf16 updated in place."""
    N, Cc = x.shape
    cap = v_fresh.shape[0] if cap is None else cap
    _chk(lib().hsa_euler_update(_ptr(x), _ptr(v_cache), _ptr(v_fresh), _ptr(idx), _ptr(count), cap, N, Cc,
                                float(dsigma), _stream(stream)))
    return x


def lipar_score_motion(x, L, out=None, stream=None):
    F, HW, Cc = x.shape
    if out is None:
        out = torch.empty(F * HW, dtype=torch.float32, device=x.device)
    _chk(lib().lipar_score_motion(_ptr(x), F, HW, Cc, int(L), _ptr(out), _stream(stream)))
    return out


def attn_lse_merge(o1, lse1, o2, lse2, count, o=None, lse=None, cap=None, stream=None):
    A, H, d = o1.shape
    cap = A if cap is None else cap
    if o is None:
        o = torch.empty_like(o1)
    _chk(lib().attn_lse_merge(_ptr(o1), _ptr(lse1), _ptr(o2), _ptr(lse2), _ptr(count), cap, H, d, _ptr(o),
                              _ptr(lse), _stream(stream)))
    return o


def timeripple_score(x, F, Hs, Ws, windows, theta, reuse=None, delta=False, score=False, stream=None):
    """x [F*Hs*Ws, H, d] bf16. windows: ((start, len),) * 3 for t, x, y; theta:
    3 floats. Returns (reuse uint8 [N, H], delta float32 [3, N, H] or None,
    score float32 [N] or None); pass tensors as delta/score to reuse buffers."""
    N, H, d = x.shape
    if reuse is None:
        reuse = torch.empty((N, H), dtype=torch.uint8, device=x.device)
    if delta is True:
        delta = torch.empty((3, N, H), dtype=torch.float32, device=x.device)
    if score is True:
        score = torch.empty(N, dtype=torch.float32, device=x.device)
    delta = delta if isinstance(delta, torch.Tensor) else None
    score = score if isinstance(score, torch.Tensor) else None
    win = (C.c_int32 * 6)(*[int(v) for w in windows for v in w])
    th = (C.c_float * 3)(*[float(v) for v in theta])
    _chk(lib().timeripple_score(_ptr(x), F, Hs, Ws, H, d, C.cast(win, _P), C.cast(th, _P), _ptr(reuse),
                                _ptr(delta), _ptr(score), _stream(stream)))
    return reuse, delta, score


def timeripple_theta(step, theta_lo, theta_hi, i0=11, i1=21) -> float:
    return float(lib().timeripple_theta(int(step), float(theta_lo), float(theta_hi), int(i0), int(i1)))


def pointer_is_device_accessible(t) -> bool:
    """True if library kernels may read/write tensor t in place (device memory,
    or pinned host memory mapped into the device address space)."""
    return bool(lib().tps_pointer_is_device_accessible(_P(t.data_ptr())))


def tps_check(stream=None):
    _chk(lib().tps_check(_stream(stream)))


def tps_philox_fill(q0, nq, seed, step, tensor, out=None, stream=None):
    if out is None:
        out = torch.empty(nq * 4, dtype=torch.int32, device="cuda")
    _chk(lib().tps_philox_fill(_ptr(out), q0, nq, seed, step, tensor, _stream(stream)))
    return out


def tps_wait_probe(limit_cycles, stream=None):
    _chk(lib().tps_wait_probe(int(limit_cycles), _stream(stream)))


def debug_inject_launch_failures(n: int):
    lib().tps_debug_inject_launch_failures(int(n))


def version() -> str:
    return lib().tps_version().decode()
