"""la_prefill_noalloc: the bf16 prefill for callers that cannot allocate device
memory (for example inside a framework that has reserved almost all of the
GPU's memory for its own pool, where any allocation made by a library fails).
Its chunk states live in a fixed array inside the library instead of an
allocated workspace.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test; it also passes on its own in a
fresh process.
"""
import pytest
import torch

import linear_attention_13_b200 as la
from linear_attention_13_b200 import inputs
from _util import TOL_O_BF16, TOL_STATE, host64, per_head_rel_err

DEV = "cuda"


def _noalloc(q, k, v):
    B, H, N, d = q.shape
    o = torch.empty_like(q)
    st = torch.empty((B, H, d, d), dtype=torch.float32, device=q.device)
    status = la.la_prefill_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                   st.data_ptr(), B, H, N, d, 128, la.LA_BF16,
                                   torch.cuda.current_stream().cuda_stream)
    return status, o, st


@pytest.mark.gpu
def test_noalloc_matches_prefill_on_two_calls_in_a_row():
    # Two consecutive calls with different inputs (the second finds the first
    # call's chunk states left in the shared scratch); each is compared with
    # la_prefill on the same inputs.  B=4, H=16, N=8192 is split into chunks,
    # so the scratch is used.
    for seed in (0, 1):
        q, k, v = inputs.qkv((4, 16, 8192, 128), dtype=torch.bfloat16, device=DEV, seed=seed)
        o_ref, s_ref = la.prefill(q, k, v, blk=128)
        status, o, st = _noalloc(q, k, v)
        assert status == la.LA_OK, la.status_string(status)
        torch.cuda.synchronize()
        assert la.la_get_last_error() == la.LA_OK
        assert per_head_rel_err(host64(o), host64(o_ref)) <= TOL_O_BF16
        assert per_head_rel_err(host64(st), host64(s_ref)) <= TOL_STATE


@pytest.mark.gpu
def test_noalloc_rejects_work_beyond_its_scratch():
    # 64 heads of 262144 tokens are split into many chunks whose states need
    # more room than the fixed scratch holds: the call is refused before
    # anything is launched.
    q = torch.empty((1, 64, 262144, 128), dtype=torch.bfloat16, device=DEV)
    status, o, _ = _noalloc(q, q, q)
    assert status == la.LA_ERR_UNSUPPORTED
