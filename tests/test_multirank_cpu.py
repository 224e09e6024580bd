"""The benchmark's multi-rank path on CPU: two gloo ranks (no GPU).

The operator has no exchange step, so N GPUs run N independent batches; what
must hold across ranks is the timing plumbing: each rank draws a different
batch, the reported time is the slowest rank's, and the whole-job value counts
the work of every rank.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from sequence_depth_attention_moda_b200 import inputs as I
        w = I.TINY_FP32
        x = I.make_inputs(w, device="cpu", seed=bench.rank_seed(w, rank))
        local_ms = 2.0 + 3.0 * rank             # rank 1 is the slow one
        bench.barrier(world)
        ms = bench.max_over_ranks(local_ms, world)
        value = bench.job_value(w.fwd_flops(), ms, world)
        out[rank] = (ms, value, float(x["Q"].double().sum()))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_time_max_and_distinct_batches():
    world = 2
    mgr = mp.get_context("spawn").Manager()   # no fork of a threaded process
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    (ms0, v0, q0), (ms1, v1, q1) = out[0], out[1]
    assert ms0 == ms1 == 5.0                  # both report the slowest rank's time
    assert v0 == v1
    from sequence_depth_attention_moda_b200 import inputs as I
    assert abs(v0 - 2 * I.TINY_FP32.fwd_flops() / 5e-3 / 1e12) < 1e-12
    assert q0 != q1                            # different batches per rank


@pytest.mark.timeout(300)
def test_bench_gpus_flag_starts_one_rank_per_gpu():
    """`python bench.py --gpus 2` outside torchrun starts two ranks itself
    (torch.distributed.run on this node); both join one group and rank 0
    reports them (gloo, no GPU work)."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    res = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2", "--launch-check"],
                         capture_output=True, text=True, timeout=240, env=env, cwd=root)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, res.stdout
    rep = json.loads(lines[0])
    assert rep["n_gpus"] == 2 and rep["ranks"] == [0, 1] and rep["parallelism"] == "dp2"
