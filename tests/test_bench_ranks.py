"""Multi-rank logic of bench.py on CPU (gloo): the job time is the slowest rank's, the value is the
whole job's tokens per second (weak scaling), and under a two-rank launch only rank 0 prints.

The GPU arm runs one replica per GPU with no data exchange; these tests cover the host-side parts
that make N ranks one measurement, without a GPU.
"""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_job_rate_is_whole_job_tokens_per_second():
    ms_per_step, value = bench.job_rate(tokens_per_rank=1000, world=4, job_ms=20.0, steps=10)
    assert ms_per_step == pytest.approx(2.0)
    assert value == pytest.approx(4 * 1000 / 2.0e-3)
    assert bench.max_over_ranks([3.5, 1.0], world=1) == [3.5, 1.0]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r pretends its timed steps took (r + 1) * 10 ms in total and its e2e step 7 - r ms
        got = bench.max_over_ranks([(rank + 1) * 10.0, 7.0 - rank], world)
        q.put((rank, got, bench.job_rate(500, world, got[0], 5)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_takes_the_slowest_rank_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, (ms_per_step, value) in results:
        assert got == [20.0, 7.0]                # element-wise maxima over both ranks
        assert ms_per_step == pytest.approx(4.0)  # 20 ms over 5 steps
        assert value == pytest.approx(2 * 500 / 4.0e-3)


def test_reference_arm_under_two_ranks_prints_one_line_from_rank0():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "1", "--gpus", "2",
           "--steps", "1", "--warmup", "3"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"
