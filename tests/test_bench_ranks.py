"""Multi-rank logic of bench.py on CPU: two gloo ranks, no GPU.

Each rank reports its own time; the job time is the max over ranks and the
job throughput counts every rank's bytes (weak scaling, replicas with no
data-path collective).
"""

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms_local = 10.0 + 5.0 * rank  # rank 1 is slower
        ms = bench.reduce_max_ms(ms_local, world, dist, "cpu")
        dist.barrier()
        out[rank] = (ms, bench.job_throughput(1e9, 4, world, ms))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_throughput():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    assert out[0][0] == out[1][0] == 15.0
    # 2 ranks x 4 steps x 1 GB in 15 ms
    assert out[0][1] == pytest.approx(2 * 4 * 1.0 / 0.015)
    assert out[0][1] == out[1][1]


def test_single_rank_is_identity():
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench

    assert bench.reduce_max_ms(7.5, 1) == 7.5
    assert bench.job_throughput(2e9, 10, 1, 1000.0) == pytest.approx(20.0)


def _run_reference_arm(env_extra):
    import json
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, **env_extra)
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3"],
                       cwd=root, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    return [json.loads(ln) for ln in lines]


def test_reference_arm_line_matches_the_gpu_arm_contract():
    """The oracle arm prints one line with the GPU arm's metric, unit,
    direction and workload, a cpu_baseline describing itself and an e2e of
    its own value with no host-device bytes."""
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench

    (line,) = _run_reference_arm({"RANK": "0", "WORLD_SIZE": "1"})
    assert line["impl"] == "reference"
    assert line["metric"].startswith("encode/decode GB/s") and line["unit"] == "GB/s"
    assert line["higher_is_better"] is True and line["steps"] == 1 and line["warmup"] == 3
    assert line["config"]["workload"] == bench.LLAMA_WORKLOAD
    assert line["value"] > 0 and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    # the oracle arm maps none of the library's shared objects
    assert line["native_libs_loaded"] == []


def test_reference_arm_other_ranks_exit_quietly():
    """Under a multi-rank launch only rank 0 runs the oracle and prints."""
    assert _run_reference_arm({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}) == []
