"""GPU parity of la_prefill_backward (and the autograd wrapper) with the fp64
oracle's gradients of sum(dO * o)."""
import numpy as np
import pytest
import torch

import linear_attention_13_b200 as la
from linear_attention_13_b200 import inputs
import oracle
from _util import TOL_O_BF16, TOL_O_F32, grads_via_recurrent, host64, per_head_rel_err, round_like

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _grads_ref(q, k, v, do):
    return oracle.prefill_backward(host64(q), host64(k), host64(v), host64(do))


@pytest.mark.parametrize("blk", [128, 64])
@pytest.mark.parametrize("N", [1, 129, 1000, 2049])
def test_bf16_backward(N, blk):
    q, k, v = inputs.qkv((2, 3, N, 128), dtype=torch.bfloat16, device=DEV, seed=N)
    do = inputs.qkv((2, 3, N, 128), dtype=torch.bfloat16, device=DEV, seed=N + 99)[2]
    dq, dk, dv = la.prefill_backward(q, k, v, do, blk=blk)
    assert la.la_get_last_error() == la.LA_OK
    for got, ref in zip((dq, dk, dv), _grads_ref(q, k, v, do)):
        assert per_head_rel_err(host64(got), ref) <= TOL_O_BF16


def test_bf16_backward_many_tiles_ragged():
    # 24 tiles per sequence with a ragged last one: dk and dv come from the
    # anti-causal pass, which walks the tiles from the last (partial) one back
    q, k, v = inputs.qkv((1, 4, 3000, 128), dtype=torch.bfloat16, device=DEV, seed=31)
    do = inputs.qkv((1, 4, 3000, 128), dtype=torch.bfloat16, device=DEV, seed=32)[2]
    dq, dk, dv = la.prefill_backward(q, k, v, do)
    assert la.la_get_last_error() == la.LA_OK
    for got, ref in zip((dq, dk, dv), _grads_ref(q, k, v, do)):
        assert per_head_rel_err(host64(got), ref) <= TOL_O_BF16


@pytest.mark.parametrize("d", [64, 128])
def test_fp32_backward(d):
    q, k, v = inputs.qkv((1, 3, 300, d), dtype=torch.float32, device=DEV, seed=d)
    do = inputs.qkv((1, 3, 300, d), dtype=torch.float32, device=DEV, seed=d + 1)[2]
    dq, dk, dv = la.prefill_backward(q, k, v, do, blk=64)
    assert la.la_get_last_error() == la.LA_OK
    for got, ref in zip((dq, dk, dv), _grads_ref(q, k, v, do)):
        assert per_head_rel_err(host64(got), ref) <= TOL_O_F32


@pytest.mark.parametrize("N", [100, 256])
def test_bf16_backward_ternary_bit_exact(N):
    q, k, v = inputs.ternary_qkv((1, 4, N, 128), dtype=torch.bfloat16, device=DEV, seed=N)
    do = inputs.ternary_qkv((1, 4, N, 128), dtype=torch.bfloat16, device=DEV, seed=N + 1)[0]
    dq, dk, dv = la.prefill_backward(q, k, v, do)
    for got, ref in zip((dq, dk, dv), _grads_ref(q, k, v, do)):
        assert np.array_equal(host64(got), round_like(ref, torch.bfloat16))


def test_autograd_matches_oracle():
    from linear_attention_13_b200.autograd import lightning_attention
    q, k, v = inputs.qkv((1, 2, 700, 128), dtype=torch.bfloat16, device=DEV, seed=8)
    w = inputs.qkv((1, 2, 700, 128), dtype=torch.bfloat16, device=DEV, seed=9)[2]
    q, k, v = (x.clone().requires_grad_(True) for x in (q, k, v))
    o = lightning_attention(q, k, v)
    (o.float() * w.float()).sum().backward()
    o_ref, _ = oracle.prefill_recurrent(host64(q.detach()), host64(k.detach()), host64(v.detach()))
    assert per_head_rel_err(host64(o.detach()), o_ref) <= TOL_O_BF16
    refs = _grads_ref(q.detach(), k.detach(), v.detach(), w)
    for x, ref in zip((q, k, v), refs):
        assert per_head_rel_err(host64(x.grad), ref) <= TOL_O_BF16


def test_bf16_backward_long_context_sampled_heads():
    # B=1, H=64, N=262144 (the long-context shape): one CTA pair per head fills
    # the GPU, so dk and dv run as anti-causal passes without reversal copies;
    # 4 sampled heads against the recurrent-form reference
    B, H, N = 1, 64, 262144
    q, k, v = inputs.qkv((B, H, N, 128), dtype=torch.bfloat16, device=DEV, seed=41)
    do = inputs.qkv((B, H, N, 128), dtype=torch.bfloat16, device=DEV, seed=42)[2]
    la.la_timing_enable(64)
    dq, dk, dv = la.prefill_backward(q, k, v, do)
    torch.cuda.synchronize()
    _, _, n_aux = la.la_timing_read(la.LA_KERNEL_AUX)
    la.la_timing_enable(0)
    assert la.la_get_last_error() == la.LA_OK
    assert n_aux == 0                      # no token-reversal copies were made
    rng = np.random.default_rng(1)
    heads = [0, H - 1] + sorted(rng.choice(np.arange(1, H - 1), 2, replace=False).tolist())
    hq, hk, hv, hg = (host64(x[0, heads]) for x in (q, k, v, do))
    ref = grads_via_recurrent(oracle._get(), hq, hk, hv, hg)
    for got, r in zip((dq, dk, dv), ref):
        assert per_head_rel_err(host64(got[0, heads]), r) <= TOL_O_BF16
