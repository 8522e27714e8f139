#!/usr/bin/env python
"""Benchmark of the token-pruned attention hot path on B200.

One step = one pass of the whole per-layer path over one synthetic batch, on
the largest configuration that fits one GPU: an HSA denoising step of a
33 x 45x80 = 118800-token latent video, 24 heads, d = 128, bf16 --

    lipar_score (inter-step relative L1 between two velocity tensors)
    -> lipar_group (rank split into K = 3 groups, budgets 40/20/10 of T = 40)
    -> lipar_schedule (step i = 1: the reference group only, |A| = N/3 = 39600)
    -> gather (Q, K, V rows of the active tokens)
    -> kv_sync (fresh rows into the K/V cache; pruned rows re-noised as
       a*cache + b*eps with a = 1 - sigma_i, b = sigma_i, Philox normals)
    -> pruned_attn (39600 active queries x all 118800 keys)
    -> scatter_out (active rows over the cached outputs).

The metric is pruned-attention TFLOP/s (algorithmic 4*d*H*A*N FLOPs per step
over the whole step's time) with active tokens/s per layer alongside. The mid
step (20280 tokens, 12 heads, top-k 30%) is reported as an extra key; a
keep-ratio sweep on the Wan-like layer (32760 tokens) and per-config kernel
numbers time the kernels alone.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun every rank runs an independent layer (seed + rank): weak
scaling, no collective on the data path; the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from token_pruned_sparse_b200 import synth  # noqa: E402

METRIC = "pruned-attention TFLOP/s & active tokens/s per layer vs keep ratio; % roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 512 << 20       # > 2x the 126 MB L2
ATTN_SOURCES = ("attn_tc.cu", "attn_common.cuh", "tc_ptx.cuh", "tps_internal.cuh", "tma_host.cuh", "trace.cuh")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def attn_source_hash() -> str:
    """Hash of the dense attention kernel's source files (the kernel and every
    header it includes)."""
    h = hashlib.sha256()
    for name in ATTN_SOURCES:
        p = os.path.join(ROOT, "token_pruned_sparse_b200", "csrc", name)
        if os.path.exists(p):
            with open(p, "rb") as f:
                h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(profile_file: str):
    """DRAM bytes per launch from a committed ncu record, or None if the kernel
    source changed since those counters were taken."""
    p = os.path.join(ROOT, "profiles", profile_file)
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    if d.get("source_hash") != attn_source_hash():
        return None
    return d.get("dram_bytes_per_launch")


# ---------------------------------------------------------------- clocks ------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.gpu = gpu_index

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.gpu)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------- workloads ------
HSA_STEP = 1          # an odd step: only the reference group is active, |A| = N/3


def hsa_config(world: int) -> dict:
    """The headline workload's description; both arms print this same dict."""
    cfg = synth.CONFIGS["hsa"]
    v = cfg.video
    K, T, budgets = cfg.extra["K"], cfg.extra["T"], cfg.extra["budgets"]
    A = v.N // K
    return {"workload": f"HSA step: {v.F}x{v.Hs}x{v.Ws} = {v.N} tokens, {cfg.H} heads, d={cfg.d}, inter-step "
                        f"rel-L1 score, K={K} rank groups (budgets {'/'.join(map(str, budgets))} of T={T}), "
                        f"step i={HSA_STEP} active set |A| = N/3 = {A}, re-noised K/V cache sync "
                        f"(a = 1-sigma_i, b = sigma_i, Philox normals), pruned attention of {A} queries x {v.N} "
                        f"keys; step = score+group+schedule+gather(Q,K,V)+kv_sync+pruned_attn+scatter_out",
            "N": v.N, "active": A, "heads": cfg.H, "head_dim": cfg.d, "latent_channels": v.C,
            "l2": "flushed between timed steps (512 MiB write, then 512 MiB read: L2 left clean)",
            "parallelism": f"replicas x{world}"}


def project_on(dev, tok: torch.Tensor, W: np.ndarray, H: int, d: int) -> torch.Tensor:
    """bf16 tokens [N, C] @ W -> bf16 [N, H, d] on `dev` (fp32 product, then
    RNE): input preparation, untimed."""
    y = tok.to(dev).float() @ torch.from_numpy(W).to(dev)
    return y.to(torch.bfloat16).reshape(-1, H, d).contiguous()


class PathStep:
    """A device-resident workload and one step of the path: `_pre` (the stages
    before attention), `_attn`, `_post` (scatter_out)."""

    def capture_graphs(self) -> bool:
        """Capture the stages before and after attention as two CUDA graphs,
        replayed each step; the attention launch stays outside so its own
        events time it. Returns False (eager launches) if capture fails."""
        try:
            self.g_pre, self.g_post = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
            with torch.cuda.graph(self.g_pre):
                self._pre()
            with torch.cuda.graph(self.g_post):
                self._post()
            torch.cuda.synchronize()
            self.graphs = True
        except Exception as e:        # noqa: BLE001 - report and run eagerly
            print(f"bench: CUDA graph capture unavailable ({e}); eager launches", file=sys.stderr)
            self.g_pre = self.g_post = None
            self.graphs = False
        return self.graphs

    def step(self, ev_attn=None):
        if getattr(self, "graphs", False):
            self.g_pre.replay()
        else:
            self._pre()
        if ev_attn:
            ev_attn[0].record()
        self._attn()
        if ev_attn:
            ev_attn[1].record()
        if getattr(self, "graphs", False):
            self.g_post.replay()
        else:
            self._post()


def attn_launches(tps, attn, cap, N, H, d) -> int:
    """Kernel launches of one dense attention call: one, or two when the
    launch plan runs the grid's last query tiles split in a second launch."""
    if attn != "tc":
        return 1
    return 2 if tps.attn_plan(cap, N, H, d)[2] > 1 else 1


class HsaStep(PathStep):
    """HSA step at |A| = N/3 (step i = 1 of T = 40) on the 118800-token video.

    Q/K/V are the projections of the current velocity tensor, the K/V cache
    holds the previous step's projections, and the output cache starts at
    zero (the step rewrites the active rows)."""

    # this library's kernels per step: score + group split 1 (one cooperative
    # launch); schedule 1 (cooperative); gathers 3; kv_sync with re-noise 1
    # (fresh rows and re-noised rows in one pass); attention 1 (2 when its launch
    # plan adds a split tail launch, counted in __init__); scatter 1
    LAUNCHES = {"score_group": 1, "schedule": 1, "gather": 3, "kv_sync": 1, "attn": 1, "scatter": 1}

    def __init__(self, seed_offset: int, dev, attn: str):
        from token_pruned_sparse_b200 import tps
        self.tps = tps
        cfg = synth.CONFIGS["hsa"]
        spec = cfg.video
        if seed_offset:
            spec = synth.VideoSpec(spec.F, spec.Hs, spec.Ws, spec.C, spec.n_obj, spec.obj, spec.pan,
                                   spec.seed + 1000 * seed_offset)
        self.cfg, self.spec = cfg, spec
        self.N, self.H, self.d, self.C = spec.N, cfg.H, cfg.d, spec.C
        self.K, self.T, self.budgets = cfg.extra["K"], cfg.extra["T"], tuple(cfg.extra["budgets"])
        self.m = cfg.extra["m"]
        self.i = HSA_STEP
        sigma = 1.0 - self.i / self.T
        self.renoise = (1.0 - sigma, sigma, spec.seed, self.i)
        self.A = self.N // self.K
        vp, delta = synth.velocity_pair(spec)
        vpb, vcb = synth.to_bf16(vp), synth.to_bf16(vp + delta)
        F, HW, C = spec.F, spec.HW, spec.C
        W = synth.projection_weights(C, self.H, self.d, spec.seed)
        self.q, self.kf, self.vf = (project_on(dev, vcb, w, self.H, self.d) for w in W)
        self.kc = project_on(dev, vpb, W[1], self.H, self.d)       # cache = the previous step's K/V
        self.vc = project_on(dev, vpb, W[2], self.H, self.d)
        self.host = {"vp": vpb.reshape(F, HW, C), "vc": vcb.reshape(F, HW, C)}
        self.v_prev, self.v_cur = self.host["vp"].to(dev), self.host["vc"].to(dev)
        self.ke, self.ve = torch.empty_like(self.kc), torch.empty_like(self.vc)
        self.o_full = torch.zeros((self.N, self.H, self.d), dtype=torch.bfloat16, device=dev)
        self.bufs = self.new_buffers(dev)
        self.scale = 1.0 / math.sqrt(self.d)
        self.attn_fn = tps.pruned_attn if attn == "tc" else tps.pruned_attn_mma
        self.flops = 4.0 * self.d * self.H * self.A * self.N
        self.units = self.A
        self.launches = sum(self.LAUNCHES.values()) - 1 + attn_launches(tps, attn, self.A, self.N, self.H, self.d)

    def new_buffers(self, dev):
        t = self.tps
        shp = (self.A, self.H, self.d)
        z = lambda: torch.empty(shp, dtype=torch.bfloat16, device=dev)    # noqa: E731
        return {"vp": torch.empty_like(self.v_prev), "vc": torch.empty_like(self.v_cur),
                "score": torch.empty(self.N, dtype=torch.float32, device=dev),
                "group": torch.empty(self.N, dtype=torch.int8, device=dev),
                "idx": torch.empty(self.N, dtype=torch.int32, device=dev),
                "cnt": torch.empty(1, dtype=torch.int32, device=dev),
                "ws_g": t.workspace(t.OP_FRONT, self.N, self.K, dev),
                "ws_s": t.workspace(t.OP_SCHEDULE, self.N, self.K, dev),
                "q": z(), "k": z(), "v": z(), "o": z()}

    def select(self, X, vp, vc):
        """score + group split (one launch) -> schedule, into buffer set X."""
        t = self.tps
        t.lipar_front(vc, t.FRONT_GROUP, x_ref=vp, K=self.K, group=X["group"], ws=X["ws_g"])
        t.lipar_schedule(X["group"], self.K, self.budgets, self.T, self.i, self.m, idx=X["idx"], count=X["cnt"],
                         ws=X["ws_s"])

    def gather(self, X, q, kf, vf):
        t = self.tps
        t.tps_gather_rows(X["q"], q, X["idx"], X["cnt"])
        t.tps_gather_rows(X["k"], kf, X["idx"], X["cnt"])
        t.tps_gather_rows(X["v"], vf, X["idx"], X["cnt"])

    def sync(self, X):
        self.tps.kv_sync(self.kc, self.vc, X["k"], X["v"], X["idx"], X["cnt"], renoise=self.renoise,
                         k_eff=self.ke, v_eff=self.ve)

    def attend(self, X):
        self.attn_fn(X["q"], self.ke, self.ve, X["idx"], X["cnt"], self.scale, o_act=X["o"])

    def _pre(self):
        X = self.bufs
        self.select(X, self.v_prev, self.v_cur)
        self.gather(X, self.q, self.kf, self.vf)
        self.sync(X)

    def _attn(self):
        self.attend(self.bufs)

    def _post(self):
        X = self.bufs
        self.tps.scatter_out(self.o_full, X["o"], X["idx"], X["cnt"])

    def active_count(self) -> int:
        return int(self.bufs["cnt"].item())

    # ---- end to end: the step's inputs in pinned host memory ------------------
    # End to end, the step's inputs (2.25 GB) cross PCIe whole on the copy
    # engines: about 40 ms, hidden under the 51 ms attention. Kernels that
    # gathered the active rows straight from host memory beside the attention
    # kernel were starved of SM time (14 ms alone, 62 ms beside it).
    E2E_COPIES = True

    def host_inputs(self):
        """Pinned host copies of the step's inputs: the two velocity tensors and
        the Q/K/V projections."""
        return {"vp": self.host["vp"].pin_memory(), "vc": self.host["vc"].pin_memory(),
                "q": self.q.cpu().pin_memory(), "k": self.kf.cpu().pin_memory(), "v": self.vf.cpu().pin_memory()}

    def e2e_bytes(self, host):
        # in: every input tensor whole; out: the whole output tensor, read on the copy engine
        return sum(t.numel() * t.element_size() for t in host.values()), self.N * self.H * self.d * 2

    def e2e_buffers(self, dev):
        X = self.new_buffers(dev)
        X.update({"qf": torch.empty_like(self.q), "kf": torch.empty_like(self.kf), "vf": torch.empty_like(self.vf)})
        return X

    def e2e_copy(self, X, host):
        X["vp"].copy_(host["vp"], non_blocking=True)
        X["vc"].copy_(host["vc"], non_blocking=True)
        for key in ("q", "k", "v"):
            X[key + "f"].copy_(host[key], non_blocking=True)

    def e2e_select(self, X):
        self.select(X, X["vp"], X["vc"])

    def e2e_gather(self, X, host):
        self.gather(X, X["qf"], X["kf"], X["vf"])             # rows of the device copies


class MidStep(PathStep):
    """Mid step: 13 x 30x52 = 20280 tokens, 12 heads, inter-frame score, top-k
    30% = 6084 active queries; the K/V cache holds the previous frame's
    projections."""

    LAUNCHES = {"score_topk": 1, "gather": 3, "kv_sync": 1, "attn": 1, "scatter": 1}

    def __init__(self, seed_offset: int, dev, attn: str):
        from token_pruned_sparse_b200 import tps
        self.tps = tps
        cfg = synth.CONFIGS["mid"]
        spec = cfg.video
        if seed_offset:
            spec = synth.VideoSpec(spec.F, spec.Hs, spec.Ws, spec.C, spec.n_obj, spec.obj, spec.pan,
                                   spec.seed + 1000 * seed_offset)
        self.cfg, self.spec = cfg, spec
        self.N, self.H, self.d, self.C = spec.N, cfg.H, cfg.d, spec.C
        self.k = synth.keep_count(self.N, cfg.keep[0])
        self.A = self.k
        x, _ = synth.latent_video(spec)
        xb = synth.to_bf16(x)
        W = synth.projection_weights(self.C, self.H, self.d, spec.seed)
        tok = xb.reshape(-1, self.C)
        q, kf, vf = (synth.project(tok, w, self.H, self.d) for w in W)
        HW = spec.HW
        kc = torch.cat([kf[:HW], kf[:-HW]])       # cache = previous frame's projection
        vc = torch.cat([vf[:HW], vf[:-HW]])
        self.host = {"x": xb, "q": q, "k": kf, "v": vf}
        self.x = xb.to(dev)
        self.q, self.kf, self.vf = q.to(dev), kf.to(dev), vf.to(dev)
        self.kc, self.vc = kc.to(dev), vc.to(dev)
        self.o_full = torch.zeros((self.N, self.H, self.d), dtype=torch.bfloat16, device=dev)
        self.bufs = self.new_buffers(dev)
        self.scale = 1.0 / math.sqrt(self.d)
        self.attn_fn = tps.pruned_attn if attn == "tc" else tps.pruned_attn_mma
        self.flops = 4.0 * self.d * self.H * self.k * self.N
        self.units = self.k
        self.launches = sum(self.LAUNCHES.values()) - 1 + attn_launches(tps, attn, self.k, self.N, self.H, self.d)

    def new_buffers(self, dev):
        t = self.tps
        shp = (self.k, self.H, self.d)
        z = lambda: torch.empty(shp, dtype=torch.bfloat16, device=dev)    # noqa: E731
        return {"x": torch.empty_like(self.x), "score": torch.empty(self.N, dtype=torch.float32, device=dev),
                "idx": torch.empty(self.k, dtype=torch.int32, device=dev),
                "cnt": torch.empty(1, dtype=torch.int32, device=dev),
                "ws": t.workspace(t.OP_FRONT, self.N, 0, dev), "q": z(), "k": z(), "v": z(), "o": z()}

    def select(self, X, x):
        t = self.tps
        t.lipar_front(x, t.FRONT_TOPK, k=self.k, idx=X["idx"], count=X["cnt"], ws=X["ws"])

    def gather(self, X, q, kf, vf):
        t = self.tps
        t.tps_gather_rows(X["q"], q, X["idx"], X["cnt"])
        t.tps_gather_rows(X["k"], kf, X["idx"], X["cnt"])
        t.tps_gather_rows(X["v"], vf, X["idx"], X["cnt"])

    def sync(self, X):
        self.tps.kv_sync(self.kc, self.vc, X["k"], X["v"], X["idx"], X["cnt"])

    def attend(self, X):
        self.attn_fn(X["q"], self.kc, self.vc, X["idx"], X["cnt"], self.scale, o_act=X["o"])

    def _pre(self):
        X = self.bufs
        self.select(X, self.x)
        self.gather(X, self.q, self.kf, self.vf)
        self.sync(X)

    def _attn(self):
        self.attend(self.bufs)

    def _post(self):
        X = self.bufs
        self.tps.scatter_out(self.o_full, X["o"], X["idx"], X["cnt"])

    def active_count(self) -> int:
        return int(self.bufs["cnt"].item())

    # End to end the gathers read only the active rows straight from pinned
    # host memory (61 MB per step): whole-tensor copies (250 MB) would take
    # longer than the 0.7 ms step.
    E2E_COPIES = False

    def host_inputs(self):
        return {k: v.pin_memory() for k, v in self.host.items()}

    def e2e_bytes(self, host):
        R = self.H * self.d * 2
        return host["x"].numel() * host["x"].element_size() + 3 * self.k * R, self.k * R

    def e2e_buffers(self, dev):
        return self.new_buffers(dev)

    def e2e_copy(self, X, host):
        X["x"].copy_(host["x"], non_blocking=True)

    def e2e_select(self, X):
        self.select(X, X["x"])

    def e2e_gather(self, X, host):
        self.gather(X, host["q"], host["k"], host["v"])       # active rows over PCIe


# ---------------------------------------------------------------- timing ------
def rank_seed_offset(rank: int) -> int:
    """Each rank runs an independent layer: rank r shifts the video seed by r."""
    return rank


def max_over_ranks(values, world: int, device):
    """Element-wise max of per-rank timings (the slowest rank sets the job's
    time); a no-op at world size 1. Works with any initialised backend."""
    if world <= 1:
        return [float(v) for v in values]
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(per_rank_units: float, world: int, steps: int, total_ms_max: float) -> float:
    """Whole-job rate: the units every rank processed over the max-over-ranks time."""
    return world * per_rank_units * steps / (total_ms_max * 1e-3)


class L2Flush:
    """Flushes L2 between timed calls: writes a 512 MiB buffer (4x the 126 MB
    L2), then reads a second 512 MiB buffer, so L2 is left holding clean lines
    of unrelated data. Timed kernels then read their inputs from DRAM without
    also paying the write-back of dirty flush lines."""

    def __init__(self, dev):
        self.w = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        self.r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        self.sink = torch.zeros((), dtype=torch.float32, device=dev)

    def __call__(self):
        self.w.add_(1)
        torch.sum(self.r, dim=0, out=self.sink)


def timed_steps(fn, steps, flush, with_attn=False):
    """Per-step CUDA events on the launching stream, L2 flushed between steps."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    attn_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush()
        evs[i][0].record()
        fn(attn_evs[i] if with_attn else None)
        evs[i][1].record()
    torch.cuda.synchronize()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    attn_ms = [a.elapsed_time(b) for a, b in attn_evs] if with_attn else None
    return step_ms, attn_ms


def _time(fn, flush, reps=5, warm=2):
    ms = []
    for i in range(warm + reps):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        if i >= warm:
            ms.append(a.elapsed_time(b))
    return float(np.median(ms))


def run_path(st, steps, warmup, world, use_graphs, flush, dev):
    """Warm-up, then `steps` timed steps of a PathStep; returns (total ms and
    mean attention ms, both max over ranks)."""
    st.step()                     # first eager step: one-time setup (status word, occupancy queries)
    torch.cuda.synchronize()
    if use_graphs:
        st.capture_graphs()
    for _ in range(warmup):
        st.step()
    torch.cuda.synchronize()
    st.tps.tps_check()
    if st.active_count() != st.units:          # correctness guard on the timed configuration
        raise RuntimeError(f"active count {st.active_count()} != {st.units}")
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    step_ms, attn_ms = timed_steps(st.step, steps, flush, with_attn=True)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    st.tps.tps_check()
    total_ms, attn_avg = max_over_ranks([np.sum(step_ms), np.mean(attn_ms)], world, dev)
    return total_ms, attn_avg


# ------------------------------------------------------------------ e2e -------
def e2e_leg(st, dev, steps, world):
    """The same metric through the C ABI with the step's data in pinned host
    memory and the result written back into host memory.

    The library's kernels address pinned host memory directly (unified
    addressing, checked with tps_pointer_is_device_accessible). The data
    moves in one of two ways, per workload (E2E_COPIES): every input tensor
    whole on the copy engines, gathered on the device, and the output scattered
    into a device-side full output that one copy-engine transfer reads back
    whole (no kernel touches PCIe, so nothing competes with the attention for
    SMs); or the velocity / latent tensors whole, the active rows of Q/K/V
    gathered straight from host memory and scatter_out writing only the active
    rows of the caller's host-side output. Three buffer sets rotate so that,
    while step i's attention runs on the compute stream, step i+2's copies (and,
    in the second way, step i+1's gathers) run on a second stream and step i-1's
    read-back (or scatter_out) on a third. Step i+1's selection (one cooperative launch that wants every SM)
    runs on the compute stream between step i's kv_sync and its attention, so
    it never waits behind a long attention kernel."""
    tps = st.tps
    host = st.host_inputs()
    o_host = torch.zeros((st.N, st.H, st.d), dtype=torch.bfloat16).pin_memory()
    if not all(tps.pointer_is_device_accessible(t) for t in list(host.values()) + [o_host]):
        return {"unavailable": "pinned host memory is not device-accessible here"}
    h2d, d2h = st.e2e_bytes(host)
    sets = [st.e2e_buffers(dev) for _ in range(3)]
    copies = bool(getattr(st, "E2E_COPIES", False))
    comp = torch.cuda.current_stream()
    s_pre, s_post = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()           # noqa: E731
    copied, selected, gathered, attended, free = ([ev() for _ in range(3)] for _ in range(5))
    for e in free:
        e.record(comp)
    # copies: the full output lives on the device (scattered into in place) and is read back whole
    o_dev = torch.zeros_like(o_host, device=dev) if copies else None
    read_done = ev()
    read_done.record(comp)

    def copy_in(i):                            # s_pre: whole-tensor copy of step i's inputs
        b = i % 3
        with torch.cuda.stream(s_pre):
            s_pre.wait_event(free[b])
            st.e2e_copy(sets[b], host)
            copied[b].record(s_pre)

    def select(i):                             # compute stream: selection of step i
        b = i % 3
        comp.wait_event(copied[b])
        st.e2e_select(sets[b])
        selected[b].record(comp)

    def gather(i):                             # active rows of step i
        b = i % 3
        if copies:                             # from the device copies, on the compute stream
            st.e2e_gather(sets[b], host)
            gathered[b].record(comp)
            return
        with torch.cuda.stream(s_pre):         # over PCIe, beside the attention
            s_pre.wait_event(selected[b])
            st.e2e_gather(sets[b], host)
            gathered[b].record(s_pre)

    def run(n):
        copy_in(0)
        select(0)
        gather(0)
        if n > 1:
            copy_in(1)
        for i in range(n):
            b = i % 3
            X = sets[b]
            comp.wait_event(gathered[b])
            st.sync(X)
            if i + 1 < n:
                select(i + 1)
                if copies:
                    gather(i + 1)
            st.attend(X)
            if copies:
                comp.wait_event(read_done)                                # step i-1's read-back is done
                tps.scatter_out(o_dev, X["o"], X["idx"], X["cnt"])
                attended[b].record(comp)
                free[b].record(comp)
                with torch.cuda.stream(s_post):
                    s_post.wait_event(attended[b])
                    o_host.copy_(o_dev, non_blocking=True)               # whole output, copy engine
                    read_done.record(s_post)
            else:
                attended[b].record(comp)
                with torch.cuda.stream(s_post):
                    s_post.wait_event(attended[b])
                    tps.scatter_out(o_host, X["o"], X["idx"], X["cnt"])  # rows written over PCIe
                    free[b].record(s_post)
            if i + 1 < n and not copies:
                gather(i + 1)
            if i + 2 < n:
                copy_in(i + 2)
        comp.wait_stream(s_post)

    run(3)
    torch.cuda.synchronize()
    tps.tps_check()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(comp)
    s_pre.wait_event(a)
    run(steps)
    b.record(comp)
    torch.cuda.synchronize()
    tps.tps_check()
    ms = max_over_ranks([a.elapsed_time(b)], world, dev)[0]
    # the host-side output must equal the device-resident path's (same inputs, same kernels)
    st.step()
    torch.cuda.synchronize()
    if not torch.equal(o_host, st.o_full.cpu()):
        raise RuntimeError("e2e: host-side output differs from the device-resident step")
    return {"value": round(job_throughput(st.flops, world, steps, ms) / 1e12, 2), "unit": "TFLOP/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": steps,
            "ms_per_step": round(ms / steps, 4),
            "mode": ("pinned host data; all inputs copied whole on the copy engines and gathered on the device; "
                     "scatter_out into the device-side full output, read back whole on the copy engine; three "
                     "rotating buffer sets: step i+2's copies and step i-1's read-back overlap step i's "
                     "attention") if copies else
                    ("pinned host data; whole latent tensors copied in, gathers read and scatter_out writes only "
                     "the active rows over PCIe; three rotating buffer sets: step i+1's gathers and step i-1's "
                     "scatter overlap step i's attention")}


# ------------------------------------------------------- kernel sweeps --------
def keep_sweep(dev, attn, reps=5):
    """Wan-like layer (32760 tokens, 12 heads): attention kernel alone per keep ratio."""
    from token_pruned_sparse_b200 import tps
    cfg = synth.CONFIGS["wan"]
    N, H, d = cfg.video.N, cfg.H, cfg.d
    fn = tps.pruned_attn if attn == "tc" else tps.pruned_attn_mma
    k = synth.gaussian_bf16((N, H, d), 301).to(dev)
    v = synth.gaussian_bf16((N, H, d), 302).to(dev)
    flush = L2Flush(dev)
    out = []
    for r in cfg.keep:
        A = synth.keep_count(N, r)
        q = synth.gaussian_bf16((A, H, d), 303).to(dev)
        idx = torch.from_numpy(np.sort(np.random.default_rng(304).choice(N, A, replace=False)).astype(np.int32)).to(dev)
        cnt = torch.tensor([A], dtype=torch.int32, device=dev)
        o = torch.empty_like(q)
        t = _time(lambda: fn(q, k, v, idx, cnt, 1 / math.sqrt(d), o_act=o), flush, reps=reps)
        fl = 4.0 * d * H * A * N
        # the same call through pruned_attn_ws (key-range splits when the grid is thin)
        ws, nws = tps.attn_workspace(A, N, H, d, dev)
        tw = _time(lambda: tps.pruned_attn_ws(q, k, v, idx, cnt, 1 / math.sqrt(d), o_act=o, ws=ws), flush,
                   reps=reps)
        out.append({"keep": r, "active": A, "attn_ms": round(t, 4), "tflops": round(fl / t / 1e9, 1),
                    "active_tokens_per_s": round(A / t * 1e3, 1), "attn_ws_ms": round(tw, 4),
                    "tflops_ws": round(fl / tw / 1e9, 1), "ws_bytes": nws})
    return out
def executed_flops(idx: np.ndarray, N: int, H: int, d: int, nb_mask=None) -> float:
    """FLOPs the attention kernel executes, padding rows and whole 128-key
    tiles included. Dense: ceil(A/256) CTAs of two 128-row tiles, every key
    tile. Masked, d = 128: one 64-row unit per 64 active rows (or fewer) of an
    original query block (the transposed products' N), the key tiles that block
    keeps. Masked, d = 64: one 128-row tile per query block holding an active
    row."""
    nkt = -(-N // 128)
    A = len(idx)
    if nb_mask is None:
        return 4.0 * d * H * 256 * 128 * (-(-A // 256)) * nkt
    blocks, rows = np.unique(np.asarray(idx) // 128, return_counts=True)
    kept = nb_mask[blocks].astype(np.int64).sum(axis=1)
    if d == 128:
        return 4.0 * d * H * 64 * 128 * float(np.sum(-(-rows // 64) * kept))
    return 4.0 * d * H * 128 * 128 * float(kept.sum())


def config_sweep(dev, peak_tflops, hbm_gbs, stages_once=False):
    """Kernel-level numbers on the larger configs (inputs resident in HBM, L2
    flushed before every timed call). Attention: algorithmic FLOPs (4*d per
    query-key-head pair over allowed keys) and executed FLOPs (padded 256-row
    query tiles x whole 128-key tiles that the kernel runs). Memory-bound
    stages: algorithmic bytes / time against the measured HBM copy peak.
    stages_once: each HSA stage runs exactly once and attention is skipped
    (the launch sequence a per-kernel DRAM-counter capture wants)."""
    from token_pruned_sparse_b200 import tps
    g = torch.Generator(device=dev)
    g.manual_seed(4)
    flush = L2Flush(dev)
    out = {}
    timer = (lambda fn, fl, reps=1, warm=0: _time(fn, fl, reps=1, warm=0)) if stages_once else _time
    # ---- HSA: 33 x 45x80 = 118800 tokens, 24 heads, d = 128 -----------------------------
    cfg = synth.CONFIGS["hsa"]
    N, H, d, C = cfg.video.N, cfg.H, cfg.d, cfg.video.C
    R = H * d * 2                       # bytes of one K/V/Q/O row
    rnd = lambda *shape: torch.randn(*shape, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    v_prev, v_cur = rnd(cfg.video.F, cfg.video.HW, C), rnd(cfg.video.F, cfg.video.HW, C)
    score = torch.empty(N, dtype=torch.float32, device=dev)
    stages = {}
    t = timer(lambda: tps.lipar_score(v_cur, v_prev, out=score), flush)
    stages["score_interstep"] = (t, N * (4 * C + 4))
    x_frames = rnd(cfg.video.F, cfg.video.HW, C)
    t = timer(lambda: tps.lipar_score(x_frames, out=score), flush)
    stages["score_interframe"] = (t, N * (2 * C + 4))
    t = timer(lambda: tps.lipar_score_motion(x_frames, 4, out=score), flush)
    stages["score_motion_L4"] = (t, N * (2 * C + 4))
    ws = tps.workspace(tps.OP_SELECT, N, 0, dev)
    idx_all = torch.empty(N, dtype=torch.int32, device=dev)
    cnt = torch.empty(1, dtype=torch.int32, device=dev)
    k3 = N // 3
    t = timer(lambda: tps.lipar_select(score, tps.SELECT_TOPK, k=k3, idx=idx_all, count=cnt, ws=ws), flush)
    stages["select_topk"] = (t, N * 4 + k3 * 4)
    t = timer(lambda: tps.lipar_select(score, tps.SELECT_THRESHOLD, tau=1.0, idx=idx_all, count=cnt, ws=ws), flush)
    stages["select_threshold"] = (t, N * 4 + int(cnt.item()) * 4)
    K = cfg.extra["K"]
    wsg = tps.workspace(tps.OP_GROUP, N, K, dev)
    grp = torch.empty(N, dtype=torch.int8, device=dev)
    t = timer(lambda: tps.lipar_group(score, K, group=grp, ws=wsg), flush)
    stages["group"] = (t, N * 4 + N)
    wss = tps.workspace(tps.OP_SCHEDULE, N, K, dev)
    t = timer(lambda: tps.lipar_schedule(grp, K, cfg.extra["budgets"], cfg.extra["T"], 1, 0, idx=idx_all, count=cnt,
                                         ws=wss), flush)
    A = int(cnt.item())
    stages["schedule"] = (t, N + A * 4)
    # fused front end: score + top-k N/3, and score + group split, one cooperative launch each
    wsf = tps.workspace(tps.OP_FRONT, N, K, dev)
    idx_f = torch.empty(N, dtype=torch.int32, device=dev)
    cnt_f = torch.empty(1, dtype=torch.int32, device=dev)
    grp_f = torch.empty(N, dtype=torch.int8, device=dev)
    t = timer(lambda: tps.lipar_front(v_cur, tps.FRONT_TOPK, x_ref=v_prev, k=k3, idx=idx_f, count=cnt_f, ws=wsf),
              flush)
    stages["front_score_topk"] = (t, N * (4 * C + 4) + k3 * 4)
    t = timer(lambda: tps.lipar_front(v_cur, tps.FRONT_GROUP, x_ref=v_prev, K=K, group=grp_f, ws=wsf), flush)
    stages["front_score_group"] = (t, N * (4 * C + 1))
    idx = idx_all[:A].clone()
    kc, vc = rnd(N, H, d), rnd(N, H, d)
    kf, vf = rnd(A, H, d), rnd(A, H, d)
    ke, ve = torch.empty_like(kc), torch.empty_like(vc)
    t = timer(lambda: tps.tps_gather_rows(kf, kc, idx, cnt), flush)
    stages["gather"] = (t, 2 * R * A)
    t = timer(lambda: tps.kv_sync(kc, vc, kf, vf, idx, cnt), flush)
    stages["kv_sync"] = (t, 4 * R * A + 4 * A)
    t = timer(lambda: tps.kv_sync(kc, vc, kf, vf, idx, cnt, renoise=(0.025, 0.975, 4, 1), k_eff=ke, v_eff=ve), flush)
    stages["kv_sync_renoise"] = (t, 6 * R * A + 4 * R * (N - A) + 4 * A)
    o_full, o_act = rnd(N, H, d), rnd(A, H, d)
    t = timer(lambda: tps.scatter_out(o_full, o_act, idx, cnt), flush)
    stages["scatter_out"] = (t, 2 * R * A)
    # keys of the pruned rows turned one frame forward (RoPE re-rotation), active rows copied
    rope_dims = synth.rope_dims(d)
    t = timer(lambda: tps.kv_rerotate(kc, idx, cnt, rope_dims, (1, 0, 0), k_eff=ke), flush)
    stages["kv_rerotate"] = (t, 2 * R * N + 4 * A)
    # attention-recovery merge of two partial results for the A active rows
    lse_a, lse_b, lse_o = (torch.randn(A, H, generator=g, device=dev) for _ in range(3))
    o_b = rnd(A, H, d)
    t = timer(lambda: tps.attn_lse_merge(o_act, lse_a, o_b, lse_b, cnt, o=o_act, lse=lse_o), flush)
    stages["lse_merge"] = (t, 3 * R * A + 3 * 4 * H * A)
    # cached Euler update (HSA 2.3): fp32 state [N, C], bf16 velocity cache
    xs = torch.randn(N, C, generator=g, device=dev, dtype=torch.float32)
    vcache = rnd(N, C)
    vfresh = rnd(A, C)
    t = timer(lambda: tps.hsa_euler_update(xs, vcache, vfresh, idx, cnt, -0.025), flush)
    stages["euler_update"] = (t, A * (2 * C + 2 * C + 8 * C) + (N - A) * (2 * C + 8 * C) + 4 * A)
    # Timeripple per-axis check of all N query rows: reuse byte per (token, head) + token score
    tr_reuse = torch.empty((N, H), dtype=torch.uint8, device=dev)
    tr_score = torch.empty(N, dtype=torch.float32, device=dev)
    wins = synth.timeripple_windows(d)
    t = timer(lambda: tps.timeripple_score(kc, cfg.video.F, cfg.video.Hs, cfg.video.Ws, wins, synth.TR_THETA,
                                           reuse=tr_reuse, score=tr_score), flush)
    stages["timeripple_score"] = (t, N * R + 2 * N * H + 4 * N)
    # size ceiling: a plain device copy moving the score kernels' byte counts (read + write), same
    # flush and timing; at tens of MB launch, ramp-up and tail cap any kernel well below the peak
    for mb in (31, 61):
        n = mb * 1000000 // 4                         # bf16 elements per direction
        src = torch.empty(n, dtype=torch.bfloat16, device=dev).normal_()
        dst = torch.empty_like(src)
        t = timer(lambda: dst.copy_(src), flush)
        stages[f"copy_ceiling_{mb}MB"] = (t, 4 * n)
        del src, dst
    out["stages_hsa"] = {k: {"ms": round(v[0], 4), "bytes": int(v[1]), "GBps": round(v[1] / v[0] / 1e6, 1),
                             "frac_hbm": round(v[1] / v[0] / 1e6 / hbm_gbs, 3)} for k, v in stages.items()}
    if stages_once:
        return out
    # ---- HSA attention per step size --------------------------------------------------
    att = {}
    scale = 1 / math.sqrt(d)
    for name, Aq in (("hsa_A_N/3", N // 3), ("hsa_A_2N/3", 2 * N // 3), ("hsa_A_N", N)):
        q = rnd(Aq, H, d)
        ii = torch.arange(0, N, N // Aq if Aq < N else 1, device=dev, dtype=torch.int32)[:Aq].contiguous()
        cc = torch.tensor([Aq], dtype=torch.int32, device=dev)
        o = torch.empty_like(q)
        t = timer(lambda: tps.pruned_attn(q, ke, ve, ii, cc, scale, o_act=o), flush, reps=3, warm=1)
        alg = 4.0 * d * H * Aq * N
        exe = executed_flops(np.arange(Aq), N, H, d)
        att[name] = {"ms": round(t, 3), "tflops_alg": round(alg / t / 1e9, 1), "tflops_exec": round(exe / t / 1e9, 1),
                     "frac_peak_exec": round(exe / t / 1e9 / peak_tflops, 3)}
        del q, o
    # ---- block-sparse: 40% active queries, 139 of 929 key blocks per query block --------
    bcfg = synth.CONFIGS["block"]
    xv, _ = synth.latent_video(bcfg.video)
    xb = synth.to_bf16(xv).to(dev)
    sc = tps.lipar_score(xb)
    kb_ = synth.keep_count(N, bcfg.keep[0])
    bidx, bcnt = tps.lipar_select(sc, tps.SELECT_TOPK, k=kb_)
    bm = synth.block_mask_band_random(bcfg.video, 128, bcfg.extra["kept_per_row"], bcfg.video.seed)
    bmd = bm.to(dev)
    q = rnd(kb_, H, d)
    o = torch.empty_like(q)
    t = timer(lambda: tps.pruned_attn(q, kc, vc, bidx, bcnt, scale, blockmask=bmd, o_act=o), flush, reps=3, warm=1)
    bidx_h = bidx.cpu().numpy()
    bm_h = bm.numpy()
    alg = 4.0 * d * H * 128 * float(bm_h[bidx_h // 128].sum())
    alg -= 4.0 * d * H * float(np.sum(bm_h[bidx_h // 128][:, -1])) * (128 - (N - (bm_h.shape[0] - 1) * 128))
    exe = executed_flops(bidx_h, N, H, d, bm_h)
    # the transposed block kernel is bound by the shared-memory port: per (unit of <= 64 rows, key
    # tile) it moves 176 KB (TMA writes of K and V 64 KB; MMA operand reads of K 32, Q 16, V 32 and
    # P^T 16 KB; P^T stores 16 KB) against 128 bytes a clock per SM
    blocks, rows_b = np.unique(bidx_h // 128, return_counts=True)
    unit_tiles = float(np.sum(-(-rows_b // 64) * bm_h[blocks].astype(np.int64).sum(axis=1))) * H
    smem_bytes = unit_tiles * 176 * 1024
    smem_peak = 128.0 * torch.cuda.get_device_properties(dev).multi_processor_count * 1965e6   # B/s at the max clock
    att["block_sparse"] = {"ms": round(t, 3), "tflops_alg": round(alg / t / 1e9, 1),
                           "tflops_exec": round(exe / t / 1e9, 1), "frac_peak_exec": round(exe / t / 1e9 / peak_tflops, 3),
                           "exec_over_alg": round(exe / alg, 2),
                           "smem_TBps": round(smem_bytes / t / 1e9, 2),
                           "smem_frac": round(smem_bytes / (t * 1e-3) / smem_peak, 3)}
    out["attention"] = att
    return out




def kernel_case(name, dev):
    """One self-contained launch sequence of a single kernel for a counter
    capture (inputs larger than L2, at most a few GB on the device): a warm-up
    launch, then the launch to capture.

    attn_mid: one mid-size attention launch (6084 queries x 20280 keys, 12
    heads). attn_hsa_h8: the HSA step's attention (39600 queries x 118800
    keys) on 8 of its 24 heads: the grid still fills the GPU, so the call runs
    like the full one, its full waves unsplit and its remaining query tiles
    split in a second launch (capture both launches of the second call);
    heads are independent units of the grid, so a full call moves about 3x
    these bytes. attn_block_h2: the block-sparse config's attention on 2 of
    its 24 heads (one launch of the transposed block kernel). overlap_hsa is
    not a capture case:
    it times the HSA step's host transfers alone and beside the attention."""
    from token_pruned_sparse_b200 import tps
    g = torch.Generator(device=dev)
    g.manual_seed(4)
    rnd = lambda *shape: torch.randn(*shape, generator=g, device=dev).to(torch.bfloat16)   # noqa: E731
    if name == "timeripple":
        cfg = synth.CONFIGS["hsa"]
        v = cfg.video
        x = rnd(v.N, cfg.H, cfg.d)                                      # 730 MB
        reuse = torch.empty((v.N, cfg.H), dtype=torch.uint8, device=dev)
        score = torch.empty(v.N, dtype=torch.float32, device=dev)
        for _ in range(2):
            tps.timeripple_score(x, v.F, v.Hs, v.Ws, synth.timeripple_windows(cfg.d), synth.TR_THETA,
                                 reuse=reuse, score=score)
    elif name == "renoise":
        # HSA step at |A| = N/3: K/V caches, fresh rows and K_eff/V_eff (3.4 GB in all)
        cfg = synth.CONFIGS["hsa"]
        N, H, d = cfg.video.N, cfg.H, cfg.d
        A = N // 3
        idx = torch.sort(torch.randperm(N, device=dev, generator=g)[:A])[0].to(torch.int32)
        cnt = torch.tensor([A], dtype=torch.int32, device=dev)
        kc, vc = rnd(N, H, d), rnd(N, H, d)
        kf, vf = rnd(A, H, d), rnd(A, H, d)
        ke, ve = torch.empty_like(kc), torch.empty_like(vc)
        for _ in range(2):
            tps.kv_sync(kc, vc, kf, vf, idx, cnt, renoise=(0.025, 0.975, 4, 1), k_eff=ke, v_eff=ve)
    elif name == "front_hsa":
        # fused score + top-k N/3 on the HSA step's velocity tensors (61 MB read)
        cfg = synth.CONFIGS["hsa"]
        v = cfg.video
        cur, prev = rnd(v.F, v.HW, v.C), rnd(v.F, v.HW, v.C)
        ws = tps.workspace(tps.OP_FRONT, v.N, cfg.extra["K"], dev)
        for _ in range(2):
            tps.lipar_front(cur, tps.FRONT_TOPK, x_ref=prev, k=v.N // 3, ws=ws)
    elif name == "overlap_hsa":
        return overlap_probe(dev)
    elif name == "attn_block_h2":
        # the block-sparse config (118800 tokens, 40% active rows, 139 of 929 key blocks kept per
        # query block) on 2 of its 24 heads: 465 x 2 x 2 CTAs of the transposed kernel
        cfg = synth.CONFIGS["block"]
        N, H, d = cfg.video.N, 2, cfg.d
        A = synth.keep_count(N, cfg.keep[0])
        idx = torch.sort(torch.randperm(N, device=dev, generator=g)[:A])[0].to(torch.int32)
        cnt = torch.tensor([A], dtype=torch.int32, device=dev)
        q, k, v = rnd(A, H, d), rnd(N, H, d), rnd(N, H, d)
        bm = synth.block_mask_band_random(cfg.video, 128, cfg.extra["kept_per_row"], cfg.video.seed).to(dev)
        o = torch.empty_like(q)
        for _ in range(2):
            tps.pruned_attn(q, k, v, idx, cnt, 1 / math.sqrt(d), blockmask=bm, o_act=o)
    elif name in ("attn_mid", "attn_hsa_h8"):
        if name == "attn_mid":
            cfg = synth.CONFIGS["mid"]
            N, H, d, A = cfg.video.N, cfg.H, cfg.d, synth.keep_count(cfg.video.N, cfg.keep[0])
        else:
            cfg = synth.CONFIGS["hsa"]
            N, H, d, A = cfg.video.N, 8, cfg.d, cfg.video.N // 3
            assert tps.attn_split(A, N, H, d) == 1
        idx = torch.sort(torch.randperm(N, device=dev, generator=g)[:A])[0].to(torch.int32)
        cnt = torch.tensor([A], dtype=torch.int32, device=dev)
        q, k, v = rnd(A, H, d), rnd(N, H, d), rnd(N, H, d)
        o = torch.empty_like(q)
        for _ in range(2):
            tps.pruned_attn(q, k, v, idx, cnt, 1 / math.sqrt(d), o_act=o)
    else:
        raise SystemExit(f"unknown kernel case {name}")
    torch.cuda.synchronize()
    tps.tps_check()
    return {"kernel_case": name, "ok": True}


def overlap_probe(dev):
    """How the HSA step's host transfers share the GPU with its attention:
    CUDA-event times of the attention launch (39600 x 118800 keys, 24 heads),
    of the three row gathers straight from pinned host memory, of scatter_out
    into pinned host memory, of whole-tensor copies of Q/K/V on the copy
    engines, each alone and each beside the attention on a second stream."""
    from token_pruned_sparse_b200 import tps
    cfg = synth.CONFIGS["hsa"]
    N, H, d = cfg.video.N, cfg.H, cfg.d
    A = N // 3
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    rnd = lambda *s: torch.randn(*s, generator=g, device=dev).to(torch.bfloat16)   # noqa: E731
    q, k, v = rnd(A, H, d), rnd(N, H, d), rnd(N, H, d)
    idx = torch.arange(A, device=dev, dtype=torch.int32) * 3
    cnt = torch.tensor([A], dtype=torch.int32, device=dev)
    o = torch.empty_like(q)
    hq = torch.randn(N, H, d).to(torch.bfloat16).pin_memory()
    hk, hv = hq.clone().pin_memory(), hq.clone().pin_memory()
    ho = torch.zeros(N, H, d, dtype=torch.bfloat16).pin_memory()
    rows = [torch.empty_like(q) for _ in range(3)]
    whole = torch.empty(N, H, d, dtype=torch.bfloat16, device=dev)
    side = torch.cuda.Stream()
    comp = torch.cuda.current_stream()

    def attn():
        tps.pruned_attn(q, k, v, idx, cnt, 1 / math.sqrt(d), o_act=o)

    def gathers():
        for dst, src in zip(rows, (hq, hk, hv)):
            tps.tps_gather_rows(dst, src, idx, cnt)

    def scatter():
        tps.scatter_out(ho, o, idx, cnt)

    def copies():
        for t in (hq, hk, hv):
            whole.copy_(t, non_blocking=True)

    def timed(main, beside=None, reps=3):
        out = []
        for _ in range(reps + 1):
            torch.cuda.synchronize()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            ev[0].record(comp)
            if beside:
                side.wait_event(ev[0])
                with torch.cuda.stream(side):
                    ev[2].record(side)
                    beside()
                    ev[3].record(side)
            main()
            ev[1].record(comp)
            torch.cuda.synchronize()
            out.append((ev[0].elapsed_time(ev[1]), ev[2].elapsed_time(ev[3]) if beside else None))
        out = sorted(out[1:])
        mid = out[len(out) // 2]
        return {"ms": round(mid[0], 3), "beside_ms": None if mid[1] is None else round(mid[1], 3)}
    res = {"attention": timed(attn), "row_gathers_from_host": timed(gathers),
           "scatter_to_host": timed(scatter), "whole_qkv_copies": timed(copies),
           "attention_with_row_gathers": timed(attn, gathers), "attention_with_scatter": timed(attn, scatter),
           "attention_with_whole_copies": timed(attn, copies)}
    tps.tps_check()
    return {"kernel_case": "overlap_hsa", "ok": True, "times": res}


# -------------------------------------------------------- CPU oracle leg ------
def _threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # pragma: no cover
        return 1


class OracleHsaSlice:
    """The fp64 oracle on the HSA step, timed as proportional slices.

    Setup (untimed): the step's inputs; the full score, group and schedule (the
    step's active set; those two global rank steps take about 0.05 s of a full
    step that takes tens of minutes, and are not part of the slices); head 0's
    projections and its re-noised K_eff/V_eff (the oracle's kv_sync with
    re-noise, that head only), widened once to fp64.

    slice(r) runs one bounded sample holding the share phi = r / (A*H) of every
    per-row and per-token stage of the step: attention of r sampled active rows
    of head 0 against all N keys, the score of ceil(phi*N) tokens, kv_sync with
    re-noise over ceil(phi*N) rows of all heads, and the gather and scatter of
    ceil(phi*A) active rows. It returns its own seconds; the attention FLOPs it
    performs are 4*d*r*N."""

    def __init__(self):
        import oracle as O
        self.O = O
        self.threads = _threads()
        cfg = synth.CONFIGS["hsa"]
        spec = cfg.video
        self.N, self.H, self.d, self.C = spec.N, cfg.H, cfg.d, spec.C
        K, T, budgets = cfg.extra["K"], cfg.extra["T"], cfg.extra["budgets"]
        sigma = 1.0 - HSA_STEP / T
        self.renoise = (1.0 - sigma, sigma, spec.seed, HSA_STEP)
        vp, delta = synth.velocity_pair(spec)
        self.vpb, self.vcb = synth.to_bf16(vp), synth.to_bf16(vp + delta)
        s = O.lipar_score(self.vcb[None], self.vpb[None])
        g = O.group_split(s, K)
        self.idx = O.schedule_active(g, K, budgets, T, HSA_STEP, cfg.extra["m"])
        self.A = len(self.idx)
        W = synth.projection_weights(self.C, self.H, self.d, spec.seed)
        d = self.d
        # head 0 over all tokens (embedded in full-width tensors, so the re-noise
        # element indices are those of the full layer)
        def head0(tok, w):
            out = torch.zeros((self.N, self.H, d), dtype=torch.bfloat16)
            out[:, 0] = (tok.float() @ torch.from_numpy(np.ascontiguousarray(w[:, :d]))).to(torch.bfloat16)
            return out
        q0, kf0, vf0 = (head0(self.vcb, w) for w in W)
        kc0, vc0 = head0(self.vpb, W[1]), head0(self.vpb, W[2])
        _, _, ke, ve = O.kv_sync(kc0, vc0, kf0[self.idx], vf0[self.idx], self.idx, renoise=self.renoise,
                                 heads=[0])
        self.ke, self.ve = ke, ve                                      # fp64 [N, 1, d]
        self.q0 = O.f64(q0[torch.as_tensor(self.idx)][:, :1])          # fp64 [A, 1, d]
        del q0, kf0, vf0, kc0, vc0
        # all heads for a pool of tokens (the O(N) slices)
        self.pool = 4096
        tok_c, tok_p = self.vcb[: self.pool], self.vpb[: self.pool]
        self.pq, self.pkf, self.pvf = (synth.project(tok_c, w, self.H, d) for w in W)
        self.pkc, self.pvc = synth.project(tok_p, W[1], self.H, d), synth.project(tok_p, W[2], self.H, d)
        self.rng = np.random.default_rng(7)
        self.flops_per_row = 4.0 * d * self.N

    def slice(self, r: int) -> float:
        O = self.O
        phi = r / (self.A * self.H)
        n = min(self.pool, max(1, math.ceil(phi * self.N)))
        m = min(n, max(1, math.ceil(phi * self.A)))
        t0n = int(self.rng.integers(0, self.N - n + 1))
        rows = self.rng.choice(self.A, r, replace=False)
        local = np.arange(0, n, 3)[:m]                                 # active rows inside the token slice
        t0 = time.perf_counter()
        O.lipar_score(self.vcb[t0n:t0n + n][None], self.vpb[t0n:t0n + n][None])
        fresh = [O.gather_rows(t, local) for t in (self.pq, self.pkf, self.pvf)]
        O.kv_sync(self.pkc[:n], self.pvc[:n], fresh[1], fresh[2], local, renoise=self.renoise)
        O.pruned_attn(self.q0, self.ke, self.ve, self.idx, 1 / math.sqrt(self.d), rows=rows)
        O.scatter_out(self.pq[:n], fresh[0], local)
        return time.perf_counter() - t0

    def describe(self, r: int) -> str:
        phi = r / (self.A * self.H)
        return (f"HSA step (N={self.N}, |A|={self.A}, {self.H} heads): proportional slice phi = r/(A*H) with "
                f"r = {r} sampled active rows of one head attending all {self.N} keys, plus phi of every O(N) "
                f"stage (score of ceil(phi*N) tokens, re-noised kv_sync of ceil(phi*N) rows x all heads, gather "
                f"and scatter of ceil(phi*A) rows); phi = {phi:.2e}; fp64 numpy/BLAS. The group and schedule "
                f"rank steps (about 0.05 s per full step) run once at setup")


def oracle_baseline(rows: int = 8192):
    """cpu_baseline of the GPU arm: one proportional slice of the HSA step
    through the fp64 oracle on the host cores (about 10 s)."""
    o = OracleHsaSlice()
    o.slice(64)                                                        # warm
    t = o.slice(rows)
    return {"value": round(o.flops_per_row * rows / t / 1e12, 6), "unit": "TFLOP/s", "cores": o.threads,
            "kind": "oracle", "sample": o.describe(rows), "seconds": round(t, 2)}


def attn_cost_fit(O, q, k, v, idx, scale, bm=None, counts=(32, 128, 512), reps=3, seed=11):
    """The oracle's attention cost on one config, fitted once: head 0's Q/K/V
    are widened to fp64 once, then t(rows) = a + b*rows is fitted by least
    squares to the median of `reps` timings at each row count. Returns
    (a seconds per head-call, b seconds per (row, head), worst relative residual)."""
    rng = np.random.default_rng(seed)
    qh, kh, vh = O.f64(q[:, :1]), O.f64(k[:, :1]), O.f64(v[:, :1])
    counts = [min(c, len(idx)) for c in counts]
    med = []
    for c in counts:
        ts = []
        for _ in range(reps):
            r = rng.choice(len(idx), c, replace=False)
            t0 = time.perf_counter()
            O.pruned_attn(qh, kh, vh, idx, scale, blockmask=bm, rows=r)
            ts.append(time.perf_counter() - t0)
        med.append(float(np.median(ts)))
    if len(set(counts)) > 1:
        b, a = np.polyfit(np.asarray(counts, float), np.asarray(med), 1)
    else:
        a, b = 0.0, med[0] / counts[0]
    a, b = max(float(a), 0.0), max(float(b), 1e-12)
    resid = max(abs(m - (a + b * c)) / m for m, c in zip(med, counts))
    return a, b, resid


def oracle_config_baselines():
    """The fp64 oracle on the other configs, reported beside the GPU numbers (a
    baseline, not a target). The O(N) stages (score, selection, gather,
    kv_sync, scatter) run over all tokens; the attention cost per (row, head)
    is fitted once per config (attn_cost_fit: it depends on N, d and the mask,
    not on |A|) and the step is extrapolated as O(N) stages + H * (a + b*|A|)."""
    import oracle as O
    out = {}

    def tm(fn):
        t0 = time.perf_counter()
        r = fn()
        return time.perf_counter() - t0, r

    def report(name, t_lin, fit, A, H, N, flops):
        a, b, resid = fit
        step = t_lin + H * (a + b * A)
        out[name] = {"seconds_per_step_extrapolated": round(step, 3), "tflops_alg": round(flops / step / 1e12, 6),
                     "active_tokens_per_s": round(A / step, 1), "o_n_stages_seconds": round(t_lin, 3),
                     "attn_fit": {"per_head_s": round(a, 5), "per_row_head_s": round(b, 7),
                                  "worst_rel_residual": round(resid, 3)},
                     "active": int(A), "tokens": int(N)}

    def qkv(tok, cfg):
        W = synth.projection_weights(cfg.video.C, cfg.H, cfg.d, cfg.video.seed)
        return [synth.project(tok, w, cfg.H, cfg.d) for w in W]

    # tiny: the complete step, all rows and heads
    cfg = synth.CONFIGS["tiny"]
    x, _ = synth.latent_video(cfg.video)
    xb = synth.to_bf16(x)
    q, kf, vf = qkv(xb.reshape(-1, cfg.video.C), cfg)
    t_all, idx = tm(lambda: O.select_threshold(O.lipar_score(xb), cfg.tau))
    t_att, _ = tm(lambda: O.pruned_attn(q[idx], kf, vf, idx, 1 / math.sqrt(cfg.d)))
    out["tiny"] = {"seconds_per_step": round(t_all + t_att, 4), "active": int(len(idx)), "tokens": cfg.video.N,
                   "tflops_alg": round(O.attn_flops(len(idx), cfg.video.N, cfg.H, cfg.d) / (t_all + t_att) / 1e12, 6),
                   "sample": "the complete step"}

    # mid: inter-frame top-k 30%
    cfg = synth.CONFIGS["mid"]
    x, _ = synth.latent_video(cfg.video)
    xb = synth.to_bf16(x)
    N, H, d = cfg.video.N, cfg.H, cfg.d
    q, kf, vf = qkv(xb.reshape(-1, cfg.video.C), cfg)
    k = synth.keep_count(N, cfg.keep[0])
    t_lin, idx = tm(lambda: O.select_topk(O.lipar_score(xb), k))
    t_rows, _ = tm(lambda: (O.gather_rows(q, idx), O.kv_sync(kf, vf, kf[idx], vf[idx], idx),
                            O.scatter_out(q, q[idx], idx)))
    report("mid", t_lin + t_rows, attn_cost_fit(O, q[idx], kf, vf, idx, 1 / math.sqrt(d)), k, H, N,
           O.attn_flops(k, N, H, d))

    # Wan, inter-step score, keep 10/30/50/100%: one attention fit for all ratios
    cfg = synth.CONFIGS["wan"]
    vp, delta = synth.velocity_pair(cfg.video)
    vpb, vcb = synth.to_bf16(vp), synth.to_bf16(vp + delta)
    N, H, d = cfg.video.N, cfg.H, cfg.d
    q, kf, vf = qkv(vcb, cfg)
    t_score, s = tm(lambda: O.lipar_score(vcb[None], vpb[None]))
    fit = None
    for ratio in cfg.keep:
        k = synth.keep_count(N, ratio)
        t_sel, idx = tm(lambda: O.select_topk(s, k))
        t_rows, _ = tm(lambda: (O.gather_rows(q, idx), O.kv_sync(kf, vf, kf[idx], vf[idx], idx),
                                O.scatter_out(q, q[idx], idx)))
        if fit is None:
            fit = attn_cost_fit(O, q[idx], kf, vf, idx, 1 / math.sqrt(d))
        report(f"wan_keep{int(ratio * 100)}", t_score + t_sel + t_rows, fit, k, H, N, O.attn_flops(k, N, H, d))

    # block-sparse: inter-frame top-k 40%, 139 of 929 key blocks per query block
    cfg = synth.CONFIGS["block"]
    x, _ = synth.latent_video(cfg.video)
    xb = synth.to_bf16(x)
    N, H, d = cfg.video.N, cfg.H, cfg.d
    q, kf, vf = qkv(xb.reshape(-1, cfg.video.C), cfg)
    kk = synth.keep_count(N, cfg.keep[0])
    t_lin, idx = tm(lambda: O.select_topk(O.lipar_score(xb), kk))
    bm = synth.block_mask_band_random(cfg.video, 128, cfg.extra["kept_per_row"], cfg.video.seed)
    keys = bm.numpy()[np.asarray(idx) // 128].sum(axis=1) * 128.0
    report("block_sparse", t_lin, attn_cost_fit(O, q[idx], kf, vf, idx, 1 / math.sqrt(d), bm=bm), kk, H, N,
           O.attn_flops(kk, N, H, d, keys))
    for v in out.values():
        v.setdefault("sample", "O(N) stages over all tokens; attention cost per (row, head) fitted once per config "
                               "from 32, 128 and 512 sampled rows of head 0 (median of 3 timings each) and "
                               "extrapolated to all rows and heads")
    return out


# ------------------------------------------------------------- reference ------
def reference_arm(a, rank, world):
    """The reference arm is the fp64 CPU oracle (the pages ship no code), timed
    on the host cores on the headline workload, metric and unit. Every step is
    one proportional slice of the HSA step (OracleHsaSlice: r sampled active
    rows of one head plus the same share of every O(N) stage); the line reports
    the slices' own measured time and the attention FLOPs they perform. Under
    torchrun only rank 0 runs."""
    if rank != 0:
        return 0
    rows = 256
    o = OracleHsaSlice()
    for _ in range(a.warmup):
        o.slice(rows)
    times = [o.slice(rows) for _ in range(a.steps)]
    per_step = float(np.mean(times))
    value = o.flops_per_row * rows / per_step / 1e12
    line = {"metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": round(per_step * 1e3, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference", "config": hsa_config(world),
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": o.threads, "kind": "oracle",
                             "sample": "each step: " + o.describe(rows)},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ main ------
def roofline_block(flops, attn_ms, peak, peak_kind, traffic, kernel):
    achieved = flops / (attn_ms * 1e-3) / 1e12
    return {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "peak_kind": peak_kind, "traffic": traffic, "kernel": kernel,
            "flops_per_launch": flops, "avg_launch_ms": round(attn_ms, 4)}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--attn", choices=["tc", "mma"], default="tc", help="attention kernel (mma = legacy baseline)")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-mid", action="store_true", help="skip the mid step")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline leg")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-config kernel sweep")
    ap.add_argument("--no-graph", action="store_true", help="launch the step's stages eagerly (no CUDA graphs)")
    ap.add_argument("--kernel-case", choices=["timeripple", "renoise", "attn_mid", "attn_hsa_h8", "attn_block_h2", "front_hsa",
                                              "overlap_hsa"],
                    default=None,
                    help="run one kernel's small capture case (warm-up + one launch) and exit")
    ap.add_argument("--stages-once", action="store_true",
                    help="run each HSA-size stage kernel once, print its table and exit (for counter captures)")
    a = ap.parse_args()
    if a.warmup < 3:
        a.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if a.impl == "reference":
        return reference_arm(a, rank, world)

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    from token_pruned_sparse_b200 import tps
    tps.lib()
    if a.kernel_case:
        print(json.dumps(kernel_case(a.kernel_case, dev)), flush=True)
        return 0
    if a.stages_once:
        pk, _ = peaks()
        res = config_sweep(dev, float(pk["bf16_tflops"]), float(pk["hbm_gbs"]), stages_once=True)
        torch.cuda.synchronize()
        tps.tps_check()
        print(json.dumps(res["stages_hsa"]), flush=True)
        return 0
    pk, pk_kind = peaks()
    flush = L2Flush(dev)

    # ---- headline: the HSA step ------------------------------------------------------
    st = HsaStep(rank_seed_offset(rank), dev, a.attn)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    total_ms, attn_avg = run_path(st, a.steps, a.warmup, world, not a.no_graph, flush, dev)
    clocks = sampler.stop()
    ms_per_step = total_ms / a.steps
    value = job_throughput(st.flops, world, a.steps, total_ms) / 1e12
    tok_s = job_throughput(st.units, world, a.steps, total_ms)
    kernel = "pruned_attn" if a.attn == "tc" else "pruned_attn_mma"
    roofline = roofline_block(st.flops, attn_avg, float(pk["bf16_tflops_sustained"]),
                              f"bf16 dense sustained ({pk_kind}; the launch runs ~{attn_avg:.0f} ms inside a long "
                              f"step)", recorded_traffic("pruned_attn_hsa.json") if a.attn == "tc" else None, kernel)
    roofline["frac_of_burst"] = round(roofline["achieved"] / float(pk["bf16_tflops"]), 4)
    e2e = None if a.no_e2e else e2e_leg(st, dev, max(3, min(a.steps, 20)), world)
    graphs = bool(getattr(st, "graphs", False))
    launches = st.launches
    del st
    torch.cuda.empty_cache()

    # ---- extra: the mid step -----------------------------------------------------------
    mid = None
    if not a.no_mid:
        ms = MidStep(rank_seed_offset(rank), dev, a.attn)
        msteps = max(a.steps, 100)
        msampler = ClockSampler(local)
        msampler.start()
        time.sleep(0.3)
        m_total, m_attn = run_path(ms, msteps, a.warmup, world, not a.no_graph, flush, dev)
        mclocks = msampler.stop()
        mid = {"workload": "mid: 13x30x52 = 20280 tokens, 12 heads, d=128, inter-frame rel-L1 score, top-k 30% = "
                           "6084 active queries x 20280 keys; step = score+select+gather+kv_sync+pruned_attn+"
                           "scatter_out",
               "steps": msteps, "ms_per_step": round(m_total / msteps, 4),
               "value": round(job_throughput(ms.flops, world, msteps, m_total) / 1e12, 2), "unit": "TFLOP/s",
               "active_tokens_per_s": round(job_throughput(ms.units, world, msteps, m_total), 1),
               "roofline": roofline_block(ms.flops, m_attn, float(pk["bf16_tflops"]), f"bf16 dense burst ({pk_kind})",
                                          recorded_traffic("pruned_attn_mid.json") if a.attn == "tc" else None,
                                          kernel),
               "clocks": mclocks}
        # the 0.6 ms launches run back to back for the whole timed region: the sustained figure, beside
        mid["roofline"]["frac_of_sustained"] = round(mid["roofline"]["achieved"] / float(pk["bf16_tflops_sustained"]), 4)
        if not a.no_e2e:
            mid["e2e"] = e2e_leg(ms, dev, max(3, min(msteps, 50)), world)
        del ms
        torch.cuda.empty_cache()

    sweep = None if (a.no_sweep or world > 1) else keep_sweep(dev, a.attn)
    configs = None if (a.no_configs or world > 1) else config_sweep(dev, float(pk["bf16_tflops"]),
                                                                   float(pk["hbm_gbs"]))
    cpu = cpu_configs = None
    if rank == 0 and world == 1 and not a.no_cpu:
        cpu = oracle_baseline()
        cpu_configs = oracle_config_baselines()

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded velocity pair of a latent video: static background + jitter, moving objects, "
                "pan strip; step delta N(0,0.05) on background, N(0,1) on moving tokens)",
        "config": hsa_config(world),
        "impl_details": {"attn_kernel": kernel, "cuda_graphs": graphs},
        "active_tokens_per_s": round(tok_s, 1),
        "gpu_launches": launches * a.steps,
        "e2e": e2e, "roofline": roofline, "cpu_baseline": cpu, "clocks": clocks,
        "mid": mid, "keep_sweep_wan": sweep, "configs": configs, "cpu_baseline_configs": cpu_configs,
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
