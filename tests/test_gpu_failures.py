"""Failure paths on the GPU, in the forms that fault, trap or hang nothing: an
allocation that fails on the host (injected), the bounded-wait limit, and the
code-object version of the loaded kernels."""
import numpy as np
import pytest
import torch

import linear_attention_13_b200 as la
from linear_attention_13_b200 import inputs
import oracle
from _util import TOL_O_BF16, TOL_STATE, host64, per_head_rel_err, per_seq_head_rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_kernels_are_built_for_sm100():
    assert la.la_binary_version() == 100


def test_wait_limit_can_be_set_and_restored():
    st, prev = la.la_set_wait_limit_ns(5_000_000)
    assert st == la.LA_OK and prev == 2_000_000_000
    st, prev = la.la_set_wait_limit_ns(0)
    assert st == la.LA_OK and prev == 5_000_000
    st, prev = la.la_set_wait_limit_ns(0)
    assert st == la.LA_OK and prev == 2_000_000_000


def _dense_call(flags):
    # B=1, H=4, N=4096: split value columns and several chunks, so both the
    # single pass (look-back chain) and the three-pass schedule need a workspace
    q, k, v = inputs.qkv((1, 4, 4096, 128), dtype=torch.bfloat16, device=DEV, seed=11)
    o = torch.full_like(q, 7.0)
    st = torch.full((1, 4, 128, 128), 7.0, device=DEV)
    return (q, k, v), o, st, (lambda: la.prefill(q, k, v, out=o, state_out=st, flags=flags,
                                                 chunk_tokens=512))


@pytest.mark.parametrize("flags", [0, la.LA_FLAG_THREE_PASS], ids=["single-pass", "three-pass"])
def test_failed_workspace_allocation_launches_nothing_and_the_next_call_works(flags):
    (q, k, v), o, st, call = _dense_call(flags)
    assert la.la_debug_fail_allocations(2) == la.LA_OK
    try:
        for _ in range(2):
            with pytest.raises(la.LightningError) as e:
                call()
            assert e.value.status == la.LA_ERR_ALLOC
        torch.cuda.synchronize()
        # nothing was launched: the outputs still hold the fill value
        assert torch.all(o == 7.0) and torch.all(st == 7.0)
        assert la.la_get_last_error() == la.LA_OK
    finally:
        la.la_debug_fail_allocations(0)
    call()
    torch.cuda.synchronize()
    assert la.la_get_last_error() == la.LA_OK
    o_ref, s_ref = oracle.prefill_recurrent(host64(q), host64(k), host64(v))
    assert per_head_rel_err(host64(o), o_ref) <= TOL_O_BF16
    assert per_head_rel_err(host64(st), s_ref) <= TOL_STATE


def test_failed_packed_workspace_allocation_launches_nothing():
    lens = [700, 0, 2000, 5]
    cu = torch.from_numpy(inputs.cu_seqlens_from_lengths(lens)).to(DEV)
    q, k, v = inputs.qkv((2, sum(lens), 128), dtype=torch.bfloat16, device=DEV, seed=12)
    o = torch.full_like(q, 7.0)
    st = torch.full((len(lens), 2, 128, 128), 7.0, device=DEV)
    la.la_debug_fail_allocations(1)
    try:
        with pytest.raises(la.LightningError) as e:
            la.prefill_varlen(q, k, v, cu, out=o, state_out=st)
        assert e.value.status == la.LA_ERR_ALLOC
        torch.cuda.synchronize()
        assert torch.all(o == 7.0) and torch.all(st == 7.0)
    finally:
        la.la_debug_fail_allocations(0)
    la.prefill_varlen(q, k, v, cu, out=o, state_out=st)
    assert la.la_get_last_error() == la.LA_OK
    o_ref, s_ref = oracle.prefill_varlen(host64(q), host64(k), host64(v), cu.cpu().numpy())
    assert per_seq_head_rel_err(host64(o), o_ref, cu) <= TOL_O_BF16
    assert per_head_rel_err(host64(st), s_ref) <= TOL_STATE
