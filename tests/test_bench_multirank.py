"""Host logic of bench.py's N > 1 path, on CPU: two `gloo` ranks, no GPU.

N GPUs run independent replicas (no data-path collective); the job's time is
the slowest rank's, obtained with one all_reduce MAX, and the value is all
ranks' bytes over that time.  The reference arm runs on rank 0 only; other
ranks exit 0 without output.
"""
from __future__ import annotations

import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        mine = [3.0, 5.5][rank]                       # this rank's elapsed ms
        t = bench.max_over_ranks(mine, world, torch.device("cpu"))
        v = bench.job_throughput(world, 1e6, 100, t)  # 1 MB per step, 100 steps
        out[rank] = (t, v)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_time_is_the_max_and_value_aggregates_all_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(2, _free_port(), out), nprocs=2, join=True, start_method="spawn")
        res = dict(out)
    assert res[0][0] == res[1][0] == 5.5
    # 2 replicas x 1 MB x 100 steps over 5.5 ms
    assert abs(res[0][1] - 2 * 1e6 * 100 / 5.5e-3 / 1e9) < 1e-9 and res[0][1] == res[1][1]


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.0, 1, None) == 7.0
    assert bench.job_throughput(1, 2e9, 10, 1000.0) == 20.0


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "3", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_e2e_runtime_wrapper_resolves_the_loaded_cuda_runtime():
    """bench.py's end-to-end loop issues its copies and event calls through the
    CUDA runtime library torch loaded; without a device the wrapper still
    resolves it and reports runtime errors by name."""
    sys.path.insert(0, ROOT)
    import bench
    rt = bench.CudaRuntime()
    assert "libcudart" in rt._loaded_path()
    for f in (rt.memcpy, rt.record, rt.wait):
        assert f.argtypes is not None and f.restype is not None
    rt.check(0, "no error")
    with pytest.raises(RuntimeError, match="cudaEventRecord"):
        rt.check(1, "cudaEventRecord")  # cudaErrorInvalidValue
