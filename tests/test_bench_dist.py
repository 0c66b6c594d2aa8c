"""The multi-rank plumbing of bench.py (barrier, max over ranks, whole-job
throughput, reference arm on rank 0 only) on two gloo ranks on the CPU."""
import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import torch
    dist = bench.init_dist(world, "gloo")
    bench.barrier(world)
    ms = 10.0 + 5.0 * rank                       # rank 1 is the slow one
    mx = bench.max_over_ranks(ms, world, torch.device("cpu"))
    val = bench.whole_job_throughput(1e12, 4, world, mx)
    q.put((rank, mx, val))
    bench.barrier(world)
    dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, val in res:
        assert mx == 15.0
        # 2 ranks x 4 steps x 1 TFLOP over 15 ms
        assert abs(val - 2 * 4 * 1.0 / 15e-3) < 1e-9


def test_single_rank_helpers():
    assert bench.max_over_ranks(3.5, 1, None) == 3.5
    assert abs(bench.whole_job_throughput(2e12, 10, 1, 100.0) - 200.0) < 1e-9


def test_reference_arm_prints_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--gpus", "2"], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and r.stdout.strip() == ""
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--reference-rows", "8"], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    # the full-workload time extrapolated from the step time (an upper bound: each step also pays
    # the head's table and key rotation once): step time x B*H*N / rows per step
    w = bench.W.WORKLOADS[bench.WORKLOAD]
    expect = line["ms_per_step"] / 1e3 * w.B * w.H * w.N / 8
    assert abs(line["cpu_baseline"]["extrapolated_full_s"] - expect) <= 1e-9 * expect
    assert "extrapolated" in line["cpu_baseline"]["extrapolated_note"]
