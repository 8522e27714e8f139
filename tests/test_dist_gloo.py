"""Multi-rank host logic of bench.py on CPU: two gloo ranks (world size 2).

The GPU path has no exchange step: ranks are independent replicas (weak
scaling). What crosses ranks is the timing: the job's step time is the max
over ranks and the throughput counts every rank's work. These tests run that
logic on two real processes with the gloo backend."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    from token_pruned_sparse_b200 import synth
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        per_rank = [10.0 + 5 * rank, 1.0 + rank]                  # rank 1 is the slower one
        mx = bench.max_over_ranks(per_rank, world, "cpu")
        # replicas are independent problems: different seeds give different inputs
        spec = synth.CONFIGS["tiny"].video
        spec_r = synth.VideoSpec(spec.F, spec.Hs, spec.Ws, spec.C, spec.n_obj, spec.obj, spec.pan,
                                 spec.seed + 1000 * bench.rank_seed_offset(rank))
        x, _ = synth.latent_video(spec_r)
        digest = torch.tensor([float(np.abs(x).sum())], dtype=torch.float64)
        all_d = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(all_d, digest)
        q.put((rank, mx, [float(t) for t in all_d]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_timing_and_distinct_replicas():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, digests in out:
        assert mx == [15.0, 2.0]                                # element-wise max over ranks
        assert digests[0] != digests[1]                          # independent replica inputs


def test_job_throughput_counts_every_rank():
    import bench
    assert bench.job_throughput(100.0, 1, 10, 1000.0) == pytest.approx(1000.0)
    # two ranks, each 100 units x 10 steps, the slower finishing in 2 s
    assert bench.job_throughput(100.0, 2, 10, 2000.0) == pytest.approx(1000.0)
    assert bench.max_over_ranks([3.0, 4.0], 1, "cpu") == [3.0, 4.0]
