"""la_prefill_noalloc: the bf16 prefill for callers that cannot allocate device
memory -- for example code running inside a framework that has already
reserved nearly all of the GPU's memory for its own pool, where any allocation
made by a library fails.  Its chunk states live in one fixed array inside the
library instead of an allocated workspace.

Each call is checked against the fp64 oracle (the same bar as la_prefill),
for 128- and 64-token blocks, on a case split into chunks (the fixed array is
used, which the test confirms from the launch counts) and on a case of one
chunk (no scratch), two calls in a row with different inputs: the second call
finds the first one's chunk states left in the shared array.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test; it also passes on its own in a
fresh process.
"""
import numpy as np
import pytest
import torch

import linear_attention_13_b200 as la
from linear_attention_13_b200 import inputs
import oracle
from _util import TOL_O_BF16, TOL_STATE, host64, per_head_rel_err

DEV = "cuda"


def _noalloc(q, k, v, blk):
    B, H, N, d = q.shape
    o = torch.empty_like(q)
    st = torch.empty((B, H, d, d), dtype=torch.float32, device=q.device)
    la.la_timing_enable(64)
    status = la.la_prefill_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                   st.data_ptr(), B, H, N, d, blk, la.LA_BF16,
                                   torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    _, _, n_chunk_state = la.la_timing_read(la.LA_KERNEL_CHUNK_STATE)
    la.la_timing_enable(0)
    return status, o, st, n_chunk_state


@pytest.mark.gpu
@pytest.mark.parametrize("blk", [128, 64])
@pytest.mark.parametrize("shape,chunked", [((4, 16, 8192, 128), True), ((1, 3, 500, 128), False)],
                         ids=["B4H16N8192-chunked", "B1H3N500-one-chunk"])
def test_noalloc_matches_the_oracle_on_two_calls_in_a_row(shape, chunked, blk):
    B, H = shape[:2]
    heads = [0, H - 1] if H > 2 else list(range(H))
    if H > 4:
        heads += sorted(np.random.default_rng(blk).choice(np.arange(1, H - 1), 2, replace=False).tolist())
    for seed in (0, 1):
        q, k, v = inputs.qkv(shape, dtype=torch.bfloat16, device=DEV, seed=seed)
        status, o, st, n_chunk_state = _noalloc(q, k, v, blk)
        assert status == la.LA_OK, la.status_string(status)
        assert la.la_get_last_error() == la.LA_OK
        # the chunked case goes through the fixed scratch (chunk states computed
        # there); one chunk needs none
        assert (n_chunk_state > 0) == chunked
        for b in range(B):
            o_ref, s_ref = oracle.prefill_recurrent(*(host64(x[b:b + 1, heads]) for x in (q, k, v)))
            assert per_head_rel_err(host64(o[b:b + 1, heads]), o_ref) <= TOL_O_BF16
            assert per_head_rel_err(host64(st[b:b + 1, heads]), s_ref) <= TOL_STATE


@pytest.mark.gpu
def test_noalloc_rejects_work_beyond_its_scratch():
    # 64 heads of 262144 tokens are split into many chunks whose states need
    # more room than the fixed scratch holds: the call is refused before
    # anything is launched.
    q = torch.empty((1, 64, 262144, 128), dtype=torch.bfloat16, device=DEV)
    B, H, N, d = q.shape
    status = la.la_prefill_noalloc(q.data_ptr(), q.data_ptr(), q.data_ptr(), q.data_ptr(), None,
                                   B, H, N, d, 128, la.LA_BF16,
                                   torch.cuda.current_stream().cuda_stream)
    assert status == la.LA_ERR_UNSUPPORTED
