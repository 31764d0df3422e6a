"""GPU parity of the continuation entry points (la_prefill_from_state,
la_prefill_varlen_from_state) against the fp64 oracle started from the same
state: o_t = q_t (S_in + sum_{s<=t} k_s^T v_s), final state S_in + K^T V.

Starting states are those a real prefix produces (the oracle's final state of
a random prefix), or small integers for the bit-exact cases.
"""
import numpy as np
import pytest
import torch

import linear_attention_13_b200 as la
from linear_attention_13_b200 import inputs
import oracle
from _util import TOL_O_BF16, TOL_O_F32, TOL_STATE, host64, per_head_rel_err, per_seq_head_rel_err, round_like

pytestmark = pytest.mark.gpu
DEV = "cuda"

SCHEDULES = [
    pytest.param(0, 128, id="default"),
    pytest.param(la.LA_FLAG_FUSED | la.LA_FLAG_NO_SPLIT_V, 128, id="single-pass"),
    pytest.param(la.LA_FLAG_FUSED | la.LA_FLAG_SPLIT_V, 128, id="single-pass-splitv"),
    pytest.param(la.LA_FLAG_THREE_PASS | la.LA_FLAG_NO_SPLIT_V, 128, id="three-pass"),
    pytest.param(la.LA_FLAG_THREE_PASS | la.LA_FLAG_SPLIT_V, 128, id="three-pass-splitv"),
    pytest.param(0, 64, id="blk64"),
    pytest.param(la.LA_FLAG_THREE_PASS, 64, id="blk64-three-pass"),
    pytest.param(la.LA_FLAG_SPLIT_V, 64, id="blk64-splitv"),
    pytest.param(la.LA_FLAG_FUSED | la.LA_FLAG_NO_SPLIT_V, 64, id="blk64-whole-rows"),
]


def _prefix_state(shape_bhd, n_prefix, seed):
    """Final state of a random prefix of n_prefix tokens (fp64 oracle), fp32."""
    B, H, d = shape_bhd
    qp, kp, vp = inputs.qkv((B, H, n_prefix, d), dtype=torch.bfloat16, device="cpu", seed=seed)
    _, s = oracle.prefill_recurrent(host64(qp), host64(kp), host64(vp))
    return torch.from_numpy(s).to(torch.float32)


@pytest.mark.parametrize("flags,blk", SCHEDULES)
@pytest.mark.parametrize("N,chunk", [(1, 0), (300, 0), (1000, 256), (2049, 384)])
def test_bf16_from_state(N, chunk, flags, blk):
    B, H, d = 2, 3, 128
    q, k, v = inputs.qkv((B, H, N, d), dtype=torch.bfloat16, device=DEV, seed=N + 5)
    s_in = _prefix_state((B, H, d), 700, seed=N).to(DEV)
    o, st = la.prefill(q, k, v, blk=blk, chunk_tokens=chunk, flags=flags, state_in=s_in)
    assert la.la_get_last_error() == la.LA_OK
    o_ref, s_ref = oracle.prefill_recurrent(host64(q), host64(k), host64(v), host64(s_in))
    assert per_head_rel_err(host64(o), o_ref) <= TOL_O_BF16
    assert per_head_rel_err(host64(st), s_ref) <= TOL_STATE


@pytest.mark.parametrize("flags,blk", SCHEDULES)
@pytest.mark.parametrize("chunk", [0, 128, 1024])
def test_bf16_from_state_onehot_bit_exact(chunk, flags, blk):
    # one-hot keys, ternary q/v and an integer starting state in [-4, 4]:
    # every intermediate is a small integer, so every schedule is exact
    B, H, N, d = 1, 4, 4096, 128
    q, k, v = inputs.onehot_k_qkv((B, H, N, d), dtype=torch.bfloat16, device=DEV, seed=chunk + blk)
    g = torch.Generator().manual_seed(chunk)
    s_in = torch.randint(-4, 5, (B, H, d, d), generator=g).to(torch.float32).to(DEV)
    o, st = la.prefill(q, k, v, blk=blk, chunk_tokens=chunk, flags=flags, state_in=s_in)
    assert la.la_get_last_error() == la.LA_OK
    o_ref, s_ref = oracle.prefill_recurrent(host64(q), host64(k), host64(v), host64(s_in))
    assert np.array_equal(host64(o), round_like(o_ref, torch.bfloat16))
    assert np.array_equal(host64(st), s_ref)


@pytest.mark.parametrize("flags", [0, la.LA_FLAG_THREE_PASS, la.LA_FLAG_SPLIT_V])
def test_bf16_continuation_equals_one_call(flags):
    # prefill(A) then prefill_from_state(B, state(A)) reproduces prefill(A ++ B)
    B, H, N, d = 2, 8, 3000, 128
    split = 1111
    q, k, v = inputs.qkv((B, H, N, d), dtype=torch.bfloat16, device=DEV, seed=41)
    o_all, s_all = la.prefill(q, k, v, flags=flags)
    a = [x[:, :, :split].contiguous() for x in (q, k, v)]
    b = [x[:, :, split:].contiguous() for x in (q, k, v)]
    _, s_a = la.prefill(*a, flags=flags)
    o_b, s_b = la.prefill(*b, flags=flags, state_in=s_a)
    assert la.la_get_last_error() == la.LA_OK
    # same values up to the bf16 rounding of the state copies at other block
    # boundaries, and both within the bar of the oracle
    assert per_head_rel_err(host64(o_b), host64(o_all[:, :, split:])) <= TOL_O_BF16
    assert per_head_rel_err(host64(s_b), host64(s_all)) <= 1e-5
    o_ref, s_ref = oracle.prefill_recurrent(host64(q), host64(k), host64(v))
    assert per_head_rel_err(host64(o_b), o_ref[:, :, split:]) <= TOL_O_BF16
    assert per_head_rel_err(host64(s_b), s_ref) <= TOL_STATE


@pytest.mark.parametrize("flags", [0, la.LA_FLAG_THREE_PASS])
def test_bf16_state_in_may_alias_state_out(flags):
    B, H, N, d = 1, 4, 1500, 128
    q, k, v = inputs.qkv((B, H, N, d), dtype=torch.bfloat16, device=DEV, seed=7)
    s_in = _prefix_state((B, H, d), 300, seed=7).to(DEV)
    s_inout = s_in.clone()
    o, st = la.prefill(q, k, v, flags=flags, chunk_tokens=512, state_in=s_inout, state_out=s_inout)
    assert la.la_get_last_error() == la.LA_OK and st.data_ptr() == s_inout.data_ptr()
    o_ref, s_ref = oracle.prefill_recurrent(host64(q), host64(k), host64(v), host64(s_in))
    assert per_head_rel_err(host64(o), o_ref) <= TOL_O_BF16
    assert per_head_rel_err(host64(st), s_ref) <= TOL_STATE


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("blk", [1, 64, 100])
def test_fp32_from_state(d, blk):
    q, k, v = inputs.qkv((1, 3, 300, d), dtype=torch.float32, device=DEV, seed=blk + d)
    s_in = _prefix_state((1, 3, d), 200, seed=blk).to(DEV)
    o, st = la.prefill(q, k, v, blk=blk, state_in=s_in)
    assert la.la_get_last_error() == la.LA_OK
    o_ref, s_ref = oracle.prefill_recurrent(host64(q), host64(k), host64(v), host64(s_in))
    assert per_head_rel_err(host64(o), o_ref) <= TOL_O_F32
    assert per_head_rel_err(host64(st), s_ref) <= TOL_STATE


def _varlen_ref(q, k, v, cu, s_in):
    """Per-sequence oracle from each sequence's own starting state."""
    H, T, d = q.shape
    S = len(cu) - 1
    o = np.zeros((H, T, d))
    st = np.zeros((S, H, d, d))
    hq, hk, hv, hs = host64(q), host64(k), host64(v), host64(s_in)
    for j in range(S):
        a, b = int(cu[j]), int(cu[j + 1])
        if b == a:
            st[j] = hs[j]
            continue
        oj, sj = oracle.prefill_recurrent(hq[None, :, a:b], hk[None, :, a:b], hv[None, :, a:b], hs[j][None])
        o[:, a:b] = oj[0]
        st[j] = sj[0]
    return o, st


VARLEN_SCHEDULES = [
    pytest.param(0, 128, id="default"),
    pytest.param(la.LA_FLAG_THREE_PASS, 128, id="three-pass"),
    pytest.param(la.LA_FLAG_SPLIT_V, 128, id="split-v"),
    pytest.param(0, 64, id="blk64"),
    pytest.param(la.LA_FLAG_SPLIT_V, 64, id="blk64-split-v"),
]


@pytest.mark.parametrize("flags,blk", VARLEN_SCHEDULES)
@pytest.mark.parametrize("chunk", [0, 256])
def test_varlen_bf16_from_state(chunk, flags, blk):
    lens = [300, 0, 1000, 1, 129, 2500]
    cu = torch.from_numpy(inputs.cu_seqlens_from_lengths(lens)).to(DEV)
    H, T, d = 3, sum(lens), 128
    q, k, v = inputs.qkv((H, T, d), dtype=torch.bfloat16, device=DEV, seed=chunk + blk)
    s_in = torch.stack([_prefix_state((1, H, d), 400, seed=j)[0] for j in range(len(lens))]).to(DEV)
    o = torch.full_like(q, 3.0)
    st = torch.full((len(lens), H, d, d), 3.0, device=DEV)
    o, st = la.prefill_varlen(q, k, v, cu, blk=blk, out=o, state_out=st, chunk_tokens=chunk,
                              flags=flags, state_in=s_in)
    assert la.la_get_last_error() == la.LA_OK
    o_ref, s_ref = _varlen_ref(q, k, v, cu.cpu().numpy(), s_in)
    assert per_seq_head_rel_err(host64(o), o_ref, cu) <= TOL_O_BF16
    assert per_head_rel_err(host64(st), s_ref) <= TOL_STATE
    # an empty sequence hands its starting state through unchanged
    assert torch.equal(st[1], s_in[1])


@pytest.mark.parametrize("d", [64, 128])
def test_varlen_fp32_from_state(d):
    lens = [17, 0, 300, 64]
    cu = torch.from_numpy(inputs.cu_seqlens_from_lengths(lens)).to(DEV)
    H, T = 2, sum(lens)
    q, k, v = inputs.qkv((H, T, d), dtype=torch.float32, device=DEV, seed=d)
    s_in = torch.stack([_prefix_state((1, H, d), 100, seed=j)[0] for j in range(len(lens))]).to(DEV)
    o, st = la.prefill_varlen(q, k, v, cu, blk=64, state_in=s_in)
    assert la.la_get_last_error() == la.LA_OK
    o_ref, s_ref = _varlen_ref(q, k, v, cu.cpu().numpy(), s_in)
    assert per_seq_head_rel_err(host64(o), o_ref, cu) <= TOL_O_F32
    assert per_head_rel_err(host64(st), s_ref) <= TOL_STATE
