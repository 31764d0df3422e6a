"""Sequence parallelism across ranks, failure paths on the host: three gloo ranks
on CPU run linear_attention_13_b200.seqpar's exchange with the fp64 oracle as
the per-rank compute, and one rank misbehaves.  Every rank must end with an
error within a bounded time (never a hang), and every process must exit.

  * a rank whose local step raises before the exchange: every rank raises
    SequenceParallelError at once (the agreement all-gather carries the
    failure), naming that rank;
  * a rank whose shard has another head count or dtype: every rank raises
    before any state is exchanged;
  * a rank that leaves the group between two calls: the others' next call
    fails when the process group's timeout expires (or sooner, when gloo sees
    the closed connection).
"""
import datetime
import os
import socket
import sys
import time

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

B, H, N, D, R = 1, 2, 48, 8, 3
PG_TIMEOUT_S = 6


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    rng = np.random.default_rng(9)
    return [rng.standard_normal((B, H, N, D)) / np.sqrt(D) for _ in range(3)]


def _compute(fail_increment: bool):
    import oracle
    from linear_attention_13_b200.seqpar import ShardCompute

    def increment(k, v):
        if fail_increment:
            raise RuntimeError("injected failure in the local K^T V step")
        _, s = oracle.prefill_recurrent(np.zeros_like(k.numpy()), k.numpy(), v.numpy())
        return torch.from_numpy(s)

    def prefix(gathered, rank):
        return gathered[:rank].sum(dim=0) if rank > 0 else torch.zeros_like(gathered[0])

    def prefill(q, k, v, state_in):
        o, s = oracle.prefill_recurrent(q.numpy(), k.numpy(), v.numpy(), state_in.numpy())
        return torch.from_numpy(o), torch.from_numpy(s)

    return ShardCompute(increment, prefix, prefill)


def _report(out_q, item):
    # flush the queue's feeder thread: the process ends with os._exit
    out_q.put(item)
    out_q.close()
    out_q.join_thread()


def _rank_main(rank, port, out_q, scenario):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(R), "MASTER_ADDR": "127.0.0.1",
                       "MASTER_PORT": str(port)})
    import torch.distributed as dist
    from linear_attention_13_b200.seqpar import SequenceParallelError, prefill_sequence_parallel

    dist.init_process_group("gloo", rank=rank, world_size=R,
                            timeout=datetime.timedelta(seconds=PG_TIMEOUT_S))
    q, k, v = _inputs()
    cuts = [0, 16, 32, 48]
    shard = [torch.from_numpy(np.ascontiguousarray(x[:, :, cuts[rank]:cuts[rank + 1]])) for x in (q, k, v)]
    outcome = "ok"
    t0 = time.monotonic()
    try:
        if scenario == "local_failure":
            prefill_sequence_parallel(*shard, compute=_compute(fail_increment=rank == 1))
        elif scenario == "shape_mismatch":
            if rank == 2:
                shard = [x[:, :1].contiguous() for x in shard]    # one head instead of two
            prefill_sequence_parallel(*shard, compute=_compute(False))
        elif scenario == "dtype_mismatch":
            if rank == 0:
                shard = [x.to(torch.float32) for x in shard]
            prefill_sequence_parallel(*shard, compute=_compute(False))
        elif scenario == "rank_leaves":
            prefill_sequence_parallel(*shard, compute=_compute(False))
            if rank == 2:
                _report(out_q, (rank, "left", "", 0.0))
                os._exit(0)                      # leaves between calls, without a word
            prefill_sequence_parallel(*shard, compute=_compute(False))
    except SequenceParallelError as e:
        outcome = f"SequenceParallelError:{e.rank}"
    except Exception as e:  # noqa: BLE001 - the test checks that an error surfaced
        outcome = f"{type(e).__name__}"
    _report(out_q, (rank, outcome, "", time.monotonic() - t0))
    if scenario != "rank_leaves":
        try:
            dist.destroy_process_group()
        except Exception:  # noqa: BLE001
            pass
    os._exit(0)


def _run(scenario):
    import oracle
    oracle.build()
    port = _free_port()
    ctx = mp.get_context("spawn")
    q_ = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, port, q_, scenario)) for r in range(R)]
    for p in procs:
        p.start()
    res = {}
    try:
        for _ in range(R):
            rank, outcome, _, dt = q_.get(timeout=60 + 4 * PG_TIMEOUT_S)
            res[rank] = (outcome, dt)
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.is_alive():
                p.kill()
                p.join()
    for p in procs:
        assert p.exitcode == 0, (scenario, p.exitcode)
    return res


def test_local_failure_on_one_rank_fails_every_rank_at_once():
    res = _run("local_failure")
    for rank in range(R):
        outcome, dt = res[rank]
        assert outcome == "SequenceParallelError:1", (rank, outcome)
        assert dt < PG_TIMEOUT_S, (rank, dt)        # the agreement, not a timeout


@pytest.mark.parametrize("scenario,culprit", [("shape_mismatch", 2), ("dtype_mismatch", 0)])
def test_mismatched_shard_fails_every_rank_before_the_exchange(scenario, culprit):
    res = _run(scenario)
    for rank in range(R):
        outcome, dt = res[rank]
        assert outcome.startswith("SequenceParallelError"), (rank, outcome)
        assert dt < PG_TIMEOUT_S, (rank, dt)
    # every rank names the same culprit (rank 0's shard is the reference, so
    # a rank-0 mismatch is reported against the first rank that differs)
    culprits = {res[r][0] for r in range(R)}
    assert len(culprits) == 1
    if scenario == "shape_mismatch":
        assert culprits == {f"SequenceParallelError:{culprit}"}


def test_rank_leaving_between_calls_fails_the_others_within_the_timeout():
    res = _run("rank_leaves")
    assert res[2][0] == "left"
    for rank in (0, 1):
        outcome, dt = res[rank]
        assert outcome != "ok", (rank, outcome)
        assert dt < 3 * PG_TIMEOUT_S + 10, (rank, dt)
