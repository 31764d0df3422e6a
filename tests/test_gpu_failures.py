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


LOOKBACK_CASES = [
    pytest.param((1, 4, 4096), 128, la.LA_FLAG_FUSED, id="split-v"),
    pytest.param((1, 4, 4096), 128, la.LA_FLAG_FUSED | la.LA_FLAG_NO_SPLIT_V, id="whole-rows"),
    pytest.param((1, 4, 4096), 64, la.LA_FLAG_FUSED, id="blk64"),
]


@pytest.mark.parametrize("shape,blk,flags", LOOKBACK_CASES)
def test_lookback_wait_runs_out_with_timeout_and_the_next_call_works(shape, blk, flags):
    # The first work item is skipped, so the chunk after it waits for a state
    # prefix that is never published: its bounded wait (5 ms here) runs out,
    # LA_ERR_TIMEOUT is recorded, every role of the kernel leaves and TMEM is
    # released -- the next call on the same context is correct.
    B, H, N = shape
    q, k, v = inputs.qkv((B, H, N, 128), dtype=torch.bfloat16, device=DEV, seed=13)
    la.prefill(q, k, v, blk=blk, chunk_tokens=512, flags=flags)      # set-up outside the test
    torch.cuda.synchronize()
    assert la.la_get_last_error() == la.LA_OK
    st, _ = la.la_set_wait_limit_ns(5_000_000)
    assert st == la.LA_OK
    try:
        assert la.la_debug_skip_lookback_items(1) == la.LA_OK
        la.prefill(q, k, v, blk=blk, chunk_tokens=512, flags=flags)
        torch.cuda.synchronize()
        assert la.la_get_last_error() == la.LA_ERR_TIMEOUT
    finally:
        la.la_debug_skip_lookback_items(0)
        la.la_set_wait_limit_ns(0)
    o, s = la.prefill(q, k, v, blk=blk, chunk_tokens=512, flags=flags)
    torch.cuda.synchronize()
    assert la.la_get_last_error() == la.LA_OK
    o_ref, s_ref = oracle.prefill_recurrent(host64(q), host64(k), host64(v))
    assert per_head_rel_err(host64(o), o_ref) <= TOL_O_BF16
    assert per_head_rel_err(host64(s), s_ref) <= TOL_STATE


def test_packed_lookback_wait_runs_out_with_timeout_and_the_next_call_works():
    lens = [3000, 5, 2600]
    cu = torch.from_numpy(inputs.cu_seqlens_from_lengths(lens)).to(DEV)
    q, k, v = inputs.qkv((2, sum(lens), 128), dtype=torch.bfloat16, device=DEV, seed=15)
    la.prefill_varlen(q, k, v, cu, chunk_tokens=512, flags=la.LA_FLAG_FUSED)
    torch.cuda.synchronize()
    assert la.la_get_last_error() == la.LA_OK
    la.la_set_wait_limit_ns(5_000_000)
    try:
        la.la_debug_skip_lookback_items(1)
        la.prefill_varlen(q, k, v, cu, chunk_tokens=512, flags=la.LA_FLAG_FUSED)
        torch.cuda.synchronize()
        assert la.la_get_last_error() == la.LA_ERR_TIMEOUT
    finally:
        la.la_debug_skip_lookback_items(0)
        la.la_set_wait_limit_ns(0)
    o, s = la.prefill_varlen(q, k, v, cu, chunk_tokens=512, flags=la.LA_FLAG_FUSED)
    torch.cuda.synchronize()
    assert la.la_get_last_error() == la.LA_OK
    o_ref, s_ref = oracle.prefill_varlen(host64(q), host64(k), host64(v), cu.cpu().numpy())
    assert per_seq_head_rel_err(host64(o), o_ref, cu) <= TOL_O_BF16
    assert per_head_rel_err(host64(s), s_ref) <= TOL_STATE


@pytest.mark.parametrize("flags", [la.LA_FLAG_FUSED, la.LA_FLAG_FUSED | la.LA_FLAG_NO_SPLIT_V],
                         ids=["split-v", "whole-rows"])
def test_lookback_progresses_while_another_kernel_holds_most_sms(flags):
    # Another kernel holds all but 8 SMs for 150 ms while the single-pass
    # prefill (16 chunks per head, look-back between them) runs on the rest.
    # Work items are taken in ticket order by running CTAs, so no CTA waits for
    # a chunk owned by a CTA that has not started: the call finishes well
    # inside a 50 ms wait limit and is correct.
    q, k, v = inputs.qkv((1, 8, 16384, 128), dtype=torch.bfloat16, device=DEV, seed=14)
    la.prefill(q, k, v, chunk_tokens=1024, flags=flags)
    torch.cuda.synchronize()
    assert la.la_get_last_error() == la.LA_OK
    sms = la.la_device_sm_count()
    side = torch.cuda.Stream()
    la.la_set_wait_limit_ns(50_000_000)
    try:
        assert la.la_debug_occupy_sms(sms - 8, 150_000_000, stream=side) == la.LA_OK
        o, s = la.prefill(q, k, v, chunk_tokens=1024, flags=flags)
        torch.cuda.synchronize()
        assert la.la_get_last_error() == la.LA_OK
    finally:
        la.la_set_wait_limit_ns(0)
    o_ref, s_ref = oracle.prefill_recurrent(host64(q), host64(k), host64(v))
    assert per_head_rel_err(host64(o), o_ref) <= TOL_O_BF16
    assert per_head_rel_err(host64(s), s_ref) <= TOL_STATE


@pytest.mark.parametrize("blk,kernel", [(128, "prefill_seq_kernel"), (64, "prefill_seq64_kernel")])
def test_split_kernel_wait_runs_out_with_timeout_and_the_next_call_works(blk, kernel):
    # The split kernels (value columns over two CTAs, one chunk per head): the
    # loads of every CTA's fourth tile are left unissued, so the MMA issuers'
    # bounded waits (5 ms here) run out, LA_ERR_TIMEOUT is recorded, and each
    # role leaves after letting its own loads and MMAs land -- the next call on
    # the same context is correct.
    q, k, v = inputs.qkv((1, 2, 2048, 128), dtype=torch.bfloat16, device=DEV, seed=16)
    la.prefill(q, k, v, blk=blk, chunk_tokens=2048, flags=la.LA_FLAG_SPLIT_V)
    torch.cuda.synchronize()
    assert la.la_get_last_error() == la.LA_OK
    assert la.la_prefill_main_kernel() == kernel
    la.la_set_wait_limit_ns(5_000_000)
    try:
        assert la.la_debug_stall_split_load(3) == la.LA_OK
        la.prefill(q, k, v, blk=blk, chunk_tokens=2048, flags=la.LA_FLAG_SPLIT_V)
        torch.cuda.synchronize()
        assert la.la_get_last_error() == la.LA_ERR_TIMEOUT
    finally:
        la.la_debug_stall_split_load(-1)
        la.la_set_wait_limit_ns(0)
    o, s = la.prefill(q, k, v, blk=blk, chunk_tokens=2048, flags=la.LA_FLAG_SPLIT_V)
    torch.cuda.synchronize()
    assert la.la_get_last_error() == la.LA_OK
    o_ref, s_ref = oracle.prefill_recurrent(host64(q), host64(k), host64(v))
    assert per_head_rel_err(host64(o), o_ref) <= TOL_O_BF16
    assert per_head_rel_err(host64(s), s_ref) <= TOL_STATE


def test_debug_hooks_validate_their_arguments():
    assert la.la_debug_stall_split_load(-2) == la.LA_ERR_INVALID_ARG
    assert la.la_debug_skip_lookback_items(-1) == la.LA_ERR_INVALID_ARG
    assert la.la_debug_occupy_sms(0, 1000) == la.LA_ERR_INVALID_ARG
    assert la.la_debug_occupy_sms(1, 2_000_000_000) == la.LA_ERR_INVALID_ARG
