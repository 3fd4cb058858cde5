"""The N > 1 launch path of bench.py on CPU: two gloo ranks.

The hot path has no exchange step, so the multi-GPU form is weak scaling of
independent batches; what has to be right is the rank plumbing around it: the
barrier, the max-over-ranks reduction of the step time, the whole-job rate and
the one-line output of rank 0 (the reference arm runs on rank 0 alone).
"""
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


def _rank_main(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench

    r = bench.Ranks("gloo", "cpu", timeout_s=60)
    try:
        assert (r.rank, r.world) == (rank, world)
        local_ms = 2.0 + 3.0 * rank  # rank 1 is the slow one
        r.barrier()
        ms = r.max(local_ms)
        rate = bench.job_rate(1000, r.world, ms)
        # a second reduction in the same order on every rank
        ms2 = r.max(-float(rank))
        out.put((rank, ms, rate, ms2))
    finally:
        r.close()


def test_two_gloo_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(i, world, port, q)) for i in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, ms, rate, ms2 in got:
        assert ms == 5.0                        # max over ranks, seen by every rank
        assert rate == pytest.approx(2 * 1000 / 5e-3)  # all ranks' units over the slowest time
        assert ms2 == 0.0


def test_single_rank_needs_no_process_group(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    sys.path.insert(0, ROOT)
    import bench

    r = bench.Ranks("gloo", "cpu")
    assert (r.world, r.rank) == (1, 0)
    assert r.max(3.5) == 3.5
    assert bench.job_rate(10, 1, 1000.0) == pytest.approx(10.0)
    r.barrier()
    r.close()


def test_reference_arm_under_torchrun_prints_one_line_from_rank_0():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3", "--ref-sample", "256"]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, res.stdout
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["n_gpus"] == 2 and j["value"] > 0
    for key in ("metric", "unit", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling", "vs_baseline",
                "dtype", "data", "config"):
        assert key in j, key
    assert j["steps"] == 1 and j["warmup"] == 3 and j["higher_is_better"] is True
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["value"] == j["value"]
    assert j["cpu_baseline"]["cores"] >= 1 and j["cpu_baseline"]["sample"]
    assert j["e2e"]["h2d_bytes_per_step"] == 0 and j["e2e"]["d2h_bytes_per_step"] == 0
    assert j["e2e"]["value"] == j["value"] and j["e2e"]["unit"] == j["unit"]
