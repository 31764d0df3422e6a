"""Multi-rank host logic of bench.py on CPU: two gloo ranks (world size 2).

Covers what the N-GPU launch relies on without needing GPUs: the process
group comes up from the torchrun environment, the timed region is bracketed
by barriers, every rank reports the slowest rank's time, the job throughput
is the weak-scaling aggregate, and the reference arm runs on rank 0 only.
"""
import io
import json
import os
import socket
import sys
import time
from contextlib import redirect_stdout

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_q):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    d = bench.Dist("gloo")
    d.init()
    # every rank sees the slowest rank's figure
    got_max = d.max(float(rank + 1))
    # timed(): barrier-bracketed region, max over ranks; rank 1 is slower
    sleep_s = 0.02 * (1 + 2 * rank)
    ms = bench.timed(None, lambda: time.sleep(sleep_s), 3, 3, d, torch.device("cpu"))
    d.barrier()
    d.close()
    out_q.put((rank, got_max, ms))


def test_two_gloo_ranks_barrier_and_max():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    assert [r[1] for r in res] == [2.0, 2.0]
    # both ranks report the same (maximum) time, that of the slower rank:
    # 3 steps of 60 ms sleeps at least
    assert res[0][2] == res[1][2]
    assert res[0][2] >= 3 * 60.0 * 0.95


def test_job_throughput_weak_scaling():
    # 4 ranks x 32768 tokens per step, 10 steps, slowest rank 2 s
    assert bench.job_throughput(32768, 10, 2000.0, 4) == pytest.approx(4 * 32768 * 10 / 2.0)
    # one rank: plain tokens per second
    assert bench.job_throughput(100, 5, 1000.0, 1) == pytest.approx(500.0)


def test_reference_arm_other_ranks_do_no_work(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    buf = io.StringIO()
    with redirect_stdout(buf):
        rc = bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"])
    assert rc == 0 and buf.getvalue() == ""


def test_reference_arm_rank0_prints_one_line(monkeypatch):
    import oracle
    oracle.build()
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "2")
    buf = io.StringIO()
    with redirect_stdout(buf):
        rc = bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3", "--ref-budget", "2"])
    assert rc == 0
    lines = [l for l in buf.getvalue().splitlines() if l.strip()]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2
    assert rec["value"] > 0 and rec["unit"] == "tokens/s" and rec["higher_is_better"] is True
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["cpu_baseline"]["cores"] >= 1
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["e2e"]["value"] == rec["value"]


def test_warmup_below_three_rejected():
    with pytest.raises(SystemExit):
        bench.main(["--steps", "1", "--warmup", "2"])
