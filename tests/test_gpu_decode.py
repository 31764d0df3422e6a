"""GPU parity of la_decode_step (through the C ABI) against the fp64 oracle:
S <- S + k^T v ; o = q S, update before read, so prefill(N) + step ==
prefill(N+1)."""
import numpy as np
import pytest
import torch

import linear_attention_13_b200 as la
from linear_attention_13_b200 import inputs
import oracle
from _util import TOL_O_BF16, TOL_O_F32, TOL_STATE, host64, per_head_rel_err, round_like

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32])
def test_decode_one_step(d, dt):
    B, H = 4, 8
    g = torch.Generator(device=DEV).manual_seed(1)
    S = torch.randn((B, H, d, d), generator=g, device=DEV, dtype=torch.float32)
    q, k, v = inputs.decode_step_inputs(B, H, d, step=1, dtype=dt, device=DEV)
    S0 = host64(S)
    o = la.decode_step(q, k, v, S)
    assert la.la_get_last_error() == la.LA_OK
    o_ref, s_ref = oracle.decode_step(host64(q), host64(k), host64(v), S0)
    tol = TOL_O_BF16 if dt == torch.bfloat16 else TOL_O_F32
    assert per_head_rel_err(host64(o), o_ref, head_dims=1) <= tol
    assert per_head_rel_err(host64(S), s_ref) <= 1e-6


def test_decode_ternary_exact():
    B, H, d = 3, 5, 128
    g = torch.Generator(device=DEV).manual_seed(2)
    S = torch.randint(-50, 51, (B, H, d, d), generator=g, device=DEV).to(torch.float32)
    q, k, v = inputs.ternary_qkv((B, H, d), dtype=torch.bfloat16, device=DEV, seed=4)
    S0 = host64(S)
    o = la.decode_step(q, k, v, S)
    o_ref, s_ref = oracle.decode_step(host64(q), host64(k), host64(v), S0)
    assert np.array_equal(host64(S), s_ref)
    assert np.array_equal(host64(o), round_like(o_ref, torch.bfloat16))


def test_decode_continues_prefill():
    B, H, N, d = 2, 4, 777, 128
    q, k, v = inputs.qkv((B, H, N + 1, d), dtype=torch.bfloat16, device=DEV, seed=8)
    _, st = la.prefill(q[:, :, :N].contiguous(), k[:, :, :N].contiguous(), v[:, :, :N].contiguous(),
                       blk=128, chunk_tokens=256)
    o_step = la.decode_step(q[:, :, N].contiguous(), k[:, :, N].contiguous(), v[:, :, N].contiguous(), st)
    o_full, s_full = la.prefill(q, k, v, blk=128, chunk_tokens=256)
    assert la.la_get_last_error() == la.LA_OK
    o_ref, s_ref = oracle.prefill_recurrent(host64(q), host64(k), host64(v))
    assert per_head_rel_err(host64(o_step), o_ref[:, :, N], head_dims=1) <= TOL_O_BF16
    assert per_head_rel_err(host64(st), s_ref) <= TOL_STATE
    assert per_head_rel_err(host64(o_full[:, :, N]), o_ref[:, :, N], head_dims=1) <= TOL_O_BF16


def test_decode_config_sampled_trajectories_and_all_heads():
    # 128 sequences x 64 heads, d = 128; state from a prefill of 4096 tokens;
    # 256 steps.  (i) every head: one step from the GPU's own state; (ii) 16
    # sampled (sequence, head) pairs: the whole trajectory in fp64.
    n_seq, H, d, N0, steps = 128, 64, 128, 4096, 256
    q0, k0, v0 = inputs.qkv((n_seq, H, N0, d), dtype=torch.bfloat16, device=DEV, seed=0)
    _, S = la.prefill(q0, k0, v0, blk=128)
    assert la.la_get_last_error() == la.LA_OK
    rng = np.random.default_rng(0)
    picks = [(int(rng.integers(n_seq)), int(rng.integers(H))) for _ in range(16)]
    seqs = [p[0] for p in picks]
    heads = [p[1] for p in picks]
    tq = [host64(q0[s, h]) for s, h in picks]
    tk = [host64(k0[s, h]) for s, h in picks]
    tv = [host64(v0[s, h]) for s, h in picks]
    del q0, k0, v0
    torch.cuda.empty_cache()
    gpu_o = []
    step_q = []
    for step in range(1, steps + 1):
        q, k, v = inputs.decode_step_inputs(n_seq, H, d, step, device=DEV)
        if step == steps:
            S_before = host64(S)
            last_qkv = (host64(q), host64(k), host64(v))
        o = la.decode_step(q, k, v, S)
        gpu_o.append(host64(o[seqs, heads]))
        step_q.append((host64(q[seqs, heads]), host64(k[seqs, heads]), host64(v[seqs, heads])))
    assert la.la_get_last_error() == la.LA_OK
    # (i) all heads, last step, from the GPU state before it
    o_ref, s_ref = oracle.decode_step(*last_qkv, S_before)
    o_last = host64(o)
    assert per_head_rel_err(o_last, o_ref, head_dims=1) <= TOL_O_BF16
    assert per_head_rel_err(host64(S), s_ref) <= TOL_STATE
    # (ii) full fp64 trajectories of the sampled pairs
    q_all = np.stack([np.concatenate([tq[i], np.stack([sq[0][i] for sq in step_q])]) for i in range(16)])
    k_all = np.stack([np.concatenate([tk[i], np.stack([sq[1][i] for sq in step_q])]) for i in range(16)])
    v_all = np.stack([np.concatenate([tv[i], np.stack([sq[2][i] for sq in step_q])]) for i in range(16)])
    o_traj, s_traj = oracle.prefill_recurrent(q_all, k_all, v_all)
    got = np.stack(gpu_o, axis=1)                       # [16, steps, d]
    assert per_head_rel_err(got, o_traj[:, N0:]) <= TOL_O_BF16
    assert per_head_rel_err(host64(S[seqs, heads]), s_traj) <= TOL_STATE
