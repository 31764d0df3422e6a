"""Sequence parallelism across ranks, host side: three gloo ranks on CPU run
the exchange of linear_attention_13_b200.seqpar with the fp64 oracle as the
per-rank compute, and the pieces must reassemble the single-sequence result
(outputs of every rank's tokens; the last rank's final state)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

B, H, N, D, R = 2, 2, 96, 8, 3


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _global_inputs():
    rng = np.random.default_rng(5)
    q = rng.standard_normal((B, H, N, D)) / np.sqrt(D)
    k = rng.standard_normal((B, H, N, D)) / np.sqrt(D)
    v = rng.standard_normal((B, H, N, D))
    return q, k, v


def _oracle_compute():
    import oracle
    from linear_attention_13_b200.seqpar import ShardCompute

    def increment(k, v):
        z = np.zeros_like(k.numpy())
        _, s = oracle.prefill_recurrent(z, k.numpy(), v.numpy())
        return torch.from_numpy(s)

    def prefix(gathered, rank):
        return gathered[:rank].sum(dim=0) if rank > 0 else torch.zeros_like(gathered[0])

    def prefill(q, k, v, state_in):
        o, s = oracle.prefill_recurrent(q.numpy(), k.numpy(), v.numpy(), state_in.numpy())
        return torch.from_numpy(o), torch.from_numpy(s)

    return ShardCompute(increment, prefix, prefill)


def _rank_main(rank, port, out_q, cuts):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(R), "MASTER_ADDR": "127.0.0.1",
                       "MASTER_PORT": str(port)})
    import torch.distributed as dist
    from linear_attention_13_b200.seqpar import prefill_sequence_parallel

    dist.init_process_group("gloo", rank=rank, world_size=R)
    q, k, v = _global_inputs()
    lo, hi = cuts[rank], cuts[rank + 1]
    shard = [torch.from_numpy(np.ascontiguousarray(x[:, :, lo:hi])) for x in (q, k, v)]
    o, s = prefill_sequence_parallel(*shard, compute=_oracle_compute())
    dist.barrier()
    dist.destroy_process_group()
    out_q.put((rank, o.numpy(), s.numpy()))


@pytest.mark.parametrize("cuts", [[0, 32, 64, 96], [0, 7, 61, 96]], ids=["even", "uneven"])
def test_three_rank_sequence_split_reassembles_the_sequence(cuts):
    # shards of any lengths: only the d x d states cross ranks
    import oracle
    oracle.build()
    port = _free_port()
    ctx = mp.get_context("spawn")
    q_ = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, port, q_, cuts)) for r in range(R)]
    for p in procs:
        p.start()
    res = sorted([q_.get(timeout=120) for _ in range(R)], key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    q, k, v = _global_inputs()
    o_ref, s_ref = oracle.prefill_recurrent(q, k, v)
    o = np.concatenate([r[1] for r in res], axis=2)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-10)
    np.testing.assert_allclose(res[-1][2], s_ref, rtol=0, atol=1e-10)
    # rank r's state is the state after its last token
    for rank, _, s in res:
        hi = cuts[rank + 1]
        _, s_hi = oracle.prefill_recurrent(q[:, :, :hi], k[:, :, :hi], v[:, :, :hi])
        np.testing.assert_allclose(s, s_hi, rtol=0, atol=1e-10)
