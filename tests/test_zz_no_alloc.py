"""lipar_select_static: the allocation-free variant of lipar_select.

Some callers cannot hand the library a workspace -- a host running the step
inside a fixed device-memory plan, or a denoising loop that must not call
cudaMalloc because it synchronises the device. lipar_select_static keeps its
scratch in a static device array inside libtps.so instead. These tests call
it through the C ABI and check that it returns exactly what lipar_select (with
a caller-provided workspace) returns, on two calls in a row (the second call
sees the scratch the first one left behind). This file is collected last so a
run that stops at the first failure has run every other test first.
"""
import numpy as np
import pytest
import torch

from token_pruned_sparse_b200 import synth, tps


def test_static_select_rejects_oversized_input_without_gpu():
    """Sizes beyond the static scratch are refused on the host."""
    F = tps.C.c_void_p(0x1000)
    code = tps.lib().lipar_select_static(F, (1 << 22) + 1, tps.SELECT_TOPK, 0.0, 5, F, F, None)
    assert code == tps.SHAPE
    assert "static scratch limit" in tps.lib().tps_last_error().decode()


@pytest.mark.gpu
@pytest.mark.parametrize("N", [1, 1025, 20280, 118800, 1 << 22])
def test_static_select_matches_workspace_select_twice(N):
    dev = "cuda"
    s = synth.random_scores(N, 4242 + N, ties=True, specials=True).to(dev)
    cases = [(tps.SELECT_THRESHOLD, 0.5, 0), (tps.SELECT_TOPK, 0.0, N // 3), (tps.SELECT_TOPK, 0.0, N)]
    for mode, tau, k in cases:
        ref_idx, ref_cnt = tps.lipar_select(s, mode, tau=tau, k=k)
        n_ref = int(ref_cnt.item())
        for call in range(2):
            idx, cnt = tps.lipar_select_static(s, mode, tau=tau, k=k)
            assert int(cnt.item()) == n_ref, (mode, k, call)
            assert torch.equal(idx[:n_ref], ref_idx[:n_ref]), (mode, k, call)
    tps.tps_check()


@pytest.mark.gpu
def test_static_select_allocates_nothing():
    """After one warm-up call (which looks up the scratch address), further
    calls into preallocated outputs leave both the device's free memory and
    torch's allocator untouched: the entry point itself allocates nothing."""
    dev = "cuda"
    N = 118800
    s = synth.random_scores(N, 99, ties=True, specials=True).to(dev)
    idx = torch.empty(N, dtype=torch.int32, device=dev)
    cnt = torch.empty(1, dtype=torch.int32, device=dev)
    ref_idx, ref_cnt = tps.lipar_select(s, tps.SELECT_TOPK, k=N // 3)
    tps.lipar_select_static(s, tps.SELECT_TOPK, k=N // 3, idx=idx, count=cnt)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    for mode, tau, k in [(tps.SELECT_TOPK, 0.0, N // 3), (tps.SELECT_THRESHOLD, 0.5, 0),
                         (tps.SELECT_TOPK, 0.0, N // 3)]:
        tps.lipar_select_static(s, mode, tau=tau, k=k, idx=idx, count=cnt)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == alloc0
    assert free1 == free0
    n = int(ref_cnt.item())
    assert int(cnt.item()) == n and torch.equal(idx[:n], ref_idx[:n])
    tps.tps_check()
