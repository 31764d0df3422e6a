"""Sequence parallelism on one GPU: the ranks of a sequence split are run one
after another (no collective; the gathered increments are stacked), through
la_state_increment, la_state_prefix and la_prefill_from_state, and must
reproduce the single-sequence oracle."""
import numpy as np
import pytest
import torch

import linear_attention_13_b200 as la
from linear_attention_13_b200 import inputs
import oracle
from _util import TOL_O_BF16, TOL_STATE, host64, per_head_rel_err, round_like

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _split_run(q, k, v, R, flags=0):
    N = q.shape[2]
    bounds = [r * N // R for r in range(R + 1)]
    shards = [[x[:, :, bounds[r]:bounds[r + 1]].contiguous() for x in (q, k, v)] for r in range(R)]
    gathered = torch.stack([la.state_increment(s[1], s[2]) for s in shards])
    outs, states = [], []
    for r in range(R):
        s_in = la.state_prefix(gathered, r)
        o, st = la.prefill(*shards[r], flags=flags, state_in=s_in)
        outs.append(o)
        states.append(st)
    assert la.la_get_last_error() == la.LA_OK
    return torch.cat(outs, dim=2), states


@pytest.mark.parametrize("R", [2, 4, 7])
@pytest.mark.parametrize("flags", [0, la.LA_FLAG_THREE_PASS])
def test_sequence_split_matches_oracle(R, flags):
    q, k, v = inputs.qkv((2, 4, 5000, 128), dtype=torch.bfloat16, device=DEV, seed=R)
    o, states = _split_run(q, k, v, R, flags)
    o_ref, s_ref = oracle.prefill_recurrent(host64(q), host64(k), host64(v))
    assert per_head_rel_err(host64(o), o_ref) <= TOL_O_BF16
    assert per_head_rel_err(host64(states[-1]), s_ref) <= TOL_STATE


@pytest.mark.parametrize("R", [3, 8])
def test_sequence_split_onehot_bit_exact(R):
    q, k, v = inputs.onehot_k_qkv((1, 4, 8192, 128), dtype=torch.bfloat16, device=DEV, seed=R)
    o, states = _split_run(q, k, v, R)
    o_ref, s_ref = oracle.prefill_recurrent(host64(q), host64(k), host64(v))
    assert np.array_equal(host64(o), round_like(o_ref, torch.bfloat16))
    assert np.array_equal(host64(states[-1]), s_ref)


@pytest.mark.parametrize("N", [1, 127, 129, 3000])
def test_state_increment(N):
    k = inputs.qkv((2, 3, N, 128), dtype=torch.bfloat16, device=DEV, seed=N)[1]
    v = inputs.qkv((2, 3, N, 128), dtype=torch.bfloat16, device=DEV, seed=N + 1)[2]
    d = la.state_increment(k, v)
    ref = np.einsum("bhnk,bhnv->bhkv", host64(k), host64(v))
    assert per_head_rel_err(host64(d), ref) <= TOL_STATE
    _, kk, vv = inputs.onehot_k_qkv((1, 2, N, 128), dtype=torch.bfloat16, device=DEV, seed=N)
    d = la.state_increment(kk, vv)
    assert np.array_equal(host64(d), np.einsum("bhnk,bhnv->bhkv", host64(kk), host64(vv)))


def test_state_prefix_exact():
    g = torch.Generator().manual_seed(3)
    states = torch.randint(-8, 9, (5, 2, 3, 128, 128), generator=g).to(torch.float32).to(DEV)
    for rank in range(6):
        got = la.state_prefix(states, rank)
        want = states[:rank].sum(dim=0) if rank else torch.zeros_like(states[0])
        assert torch.equal(got, want)
