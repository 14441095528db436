"""Host logic of bench.py's N>1 replica path, run as two gloo ranks on the CPU: every rank
joins the group from the torchrun environment, the timing each rank reports is the max
over ranks, the whole-job rate counts every replica's tokens, and the reference arm runs
on rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    dist = bench.dist_init("gloo")
    try:
        got_rank, got_world, _ = bench.rank_env()
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        m = bench.max_over_ranks(dist, ms, "cpu")
        dist.barrier()
        q.put((got_rank, got_world, m, bench.whole_job_rate(got_world, 8, 100, m)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [r[0] for r in res] == [0, 1]
    assert all(r[1] == world for r in res)
    assert all(r[2] == 15.0 for r in res)  # both ranks see the slowest rank's time
    # 2 replicas x 100 steps x 8 tokens in 15 ms
    assert all(r[3] == pytest.approx(2 * 8 * 100 / 0.015) for r in res)


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    env = {k: os.environ.pop(k) for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK") if k in os.environ}
    try:
        assert bench.rank_env() == (0, 1, 0)
        assert bench.dist_init("gloo") is None
        assert bench.max_over_ranks(None, 3.5, "cpu") == 3.5
    finally:
        os.environ.update(env)


@pytest.mark.timeout(600)
def test_reference_arm_rank0_only():
    """`--impl reference` under two ranks: rank 1 prints nothing and exits 0, rank 0 prints
    one JSON line with the contract's keys (a one-step oracle sample)."""
    outs = []
    for rank in (1, 0):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT="1")
        r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                            "--gpus", "2", "--steps", "1", "--warmup", "3", "--T", "1",
                            "--cpu-steps", "1"], env=env, capture_output=True, text=True,
                           timeout=600, cwd=ROOT)
        assert r.returncode == 0, r.stderr[-2000:]
        outs.append(r.stdout.strip())
    assert outs[0] == ""
    line = json.loads(outs[1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["steps"] == 1
    for key in ("metric", "value", "unit", "higher_is_better", "config", "cpu_baseline", "e2e"):
        assert key in line
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
