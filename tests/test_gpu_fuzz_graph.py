"""Seeded random shapes and schedules against the oracle, and CUDA-graph
capture / replay of the library calls (stream-ordered workspaces make the
prefill capturable)."""
import numpy as np
import pytest
import torch

import linear_attention_13_b200 as la
from linear_attention_13_b200 import inputs
import oracle
from _util import TOL_O_BF16, TOL_STATE, host64, per_head_rel_err, per_seq_head_rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"

FLAGS = [0, la.LA_FLAG_FUSED, la.LA_FLAG_THREE_PASS, la.LA_FLAG_FUSED | la.LA_FLAG_SPLIT_V,
         la.LA_FLAG_FUSED | la.LA_FLAG_NO_SPLIT_V, la.LA_FLAG_THREE_PASS | la.LA_FLAG_SPLIT_V]


@pytest.mark.parametrize("case", range(24))
def test_random_dense(case):
    rng = np.random.default_rng(1000 + case)
    B, H = int(rng.integers(1, 4)), int(rng.integers(1, 6))
    N = int(rng.integers(1, 3000))
    blk = int(rng.choice([64, 128]))
    flags = int(rng.choice(FLAGS)) if blk == 128 else int(rng.choice([0, la.LA_FLAG_THREE_PASS]))
    chunk = int(rng.choice([0, 128, 256, 640, 1024]))
    with_state_in = bool(rng.integers(0, 2))
    q, k, v = inputs.qkv((B, H, N, 128), dtype=torch.bfloat16, device=DEV, seed=case)
    s_in = None
    if with_state_in:
        s_in = (torch.randn((B, H, 128, 128), generator=torch.Generator().manual_seed(case)) * 4).to(DEV)
    o, st = la.prefill(q, k, v, blk=blk, chunk_tokens=chunk, flags=flags, state_in=s_in)
    assert la.la_get_last_error() == la.LA_OK
    o_ref, s_ref = oracle.prefill_recurrent(host64(q), host64(k), host64(v),
                                            host64(s_in) if s_in is not None else None)
    assert per_head_rel_err(host64(o), o_ref) <= TOL_O_BF16, (B, H, N, blk, flags, chunk)
    assert per_head_rel_err(host64(st), s_ref) <= TOL_STATE, (B, H, N, blk, flags, chunk)


@pytest.mark.parametrize("case", range(8))
def test_random_varlen(case):
    rng = np.random.default_rng(2000 + case)
    S = int(rng.integers(1, 12))
    lens = [int(x) for x in rng.integers(0, 1500, size=S)]
    H = int(rng.integers(1, 4))
    flags = int(rng.choice([0, la.LA_FLAG_THREE_PASS, la.LA_FLAG_SPLIT_V]))
    cu = torch.from_numpy(inputs.cu_seqlens_from_lengths(lens)).to(DEV)
    T = sum(lens)
    q, k, v = inputs.qkv((H, max(T, 1), 128), dtype=torch.bfloat16, device=DEV, seed=case)
    q, k, v = q[:, :T].contiguous(), k[:, :T].contiguous(), v[:, :T].contiguous()
    if T == 0:
        pytest.skip("all sequences empty")
    o, st = la.prefill_varlen(q, k, v, cu, blk=128, flags=flags)
    assert la.la_get_last_error() == la.LA_OK
    o_ref, s_ref = oracle.prefill_varlen(host64(q), host64(k), host64(v), cu.cpu().numpy())
    assert per_seq_head_rel_err(host64(o), o_ref, cu) <= TOL_O_BF16, (lens, flags)
    assert per_head_rel_err(host64(st), s_ref) <= TOL_STATE, (lens, flags)


@pytest.mark.parametrize("flags", [0, la.LA_FLAG_THREE_PASS, la.LA_FLAG_FUSED | la.LA_FLAG_NO_SPLIT_V])
def test_prefill_graph_capture_replay(flags):
    B, H, N = 2, 4, 5000
    q, k, v = inputs.qkv((B, H, N, 128), dtype=torch.bfloat16, device=DEV, seed=3)
    o = torch.empty_like(q)
    st = torch.empty((B, H, 128, 128), device=DEV)
    la.prefill(q, k, v, out=o, state_out=st, flags=flags, chunk_tokens=1024)   # warm up (setup)
    torch.cuda.synchronize()
    o_eager, st_eager = o.clone(), st.clone()
    s = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            la.prefill(q, k, v, out=o, state_out=st, flags=flags, chunk_tokens=1024, stream=s)
    o.zero_()
    st.zero_()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert la.la_get_last_error() == la.LA_OK
    assert torch.equal(o, o_eager) and torch.equal(st, st_eager)
    # new inputs in the same buffers: the replay recomputes
    q.copy_(inputs.qkv((B, H, N, 128), dtype=torch.bfloat16, device=DEV, seed=4)[0])
    graph.replay()
    torch.cuda.synchronize()
    o_ref, _ = oracle.prefill_recurrent(host64(q), host64(k), host64(v))
    assert per_head_rel_err(host64(o), o_ref) <= TOL_O_BF16


def test_decode_graph_capture_replay():
    Bq, H = 4, 8
    S0 = torch.randn((Bq, H, 128, 128), device=DEV)
    S = S0.clone()
    qq, kk, vv = inputs.decode_step_inputs(Bq, H, 128, 1, device=DEV)
    od = torch.empty_like(qq)
    la.decode_step(qq, kk, vv, S, out=od)     # warm up
    torch.cuda.synchronize()
    S.copy_(S0)
    s = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            la.decode_step(qq, kk, vv, S, out=od, stream=s)
    S.copy_(S0)
    for _ in range(5):
        graph.replay()
    torch.cuda.synchronize()
    # five replays = five steps with the same token
    ref_S = host64(S0)
    for _ in range(5):
        ref_o, ref_S = oracle.decode_step(host64(qq), host64(kk), host64(vv), ref_S)
    assert per_head_rel_err(host64(S), ref_S) <= TOL_STATE
    assert per_head_rel_err(host64(od), ref_o) <= TOL_O_BF16
