"""GPU parity of la_prefill_varlen (packed sequences, state reset at every
sequence start) and its device-side cu_seqlens check."""
import numpy as np
import pytest
import torch

import linear_attention_13_b200 as la
from linear_attention_13_b200 import inputs
import oracle
from _util import TOL_O_F32, TOL_STATE, host64, per_head_rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _cu(lengths):
    return torch.from_numpy(inputs.cu_seqlens_from_lengths(lengths)).to(DEV)


@pytest.mark.parametrize("d", [64, 128])
def test_varlen_fp32(d):
    lens = [5, 0, 130, 1, 64, 257]
    cu = _cu(lens)
    H, T = 3, sum(lens)
    q, k, v = inputs.qkv((H, T, d), dtype=torch.float32, device=DEV, seed=2)
    o, st = la.prefill_varlen(q, k, v, cu, blk=64)
    assert la.la_get_last_error() == la.LA_OK
    o_ref, s_ref = oracle.prefill_varlen(host64(q), host64(k), host64(v), cu.cpu().numpy())
    assert per_head_rel_err(host64(o), o_ref) <= TOL_O_F32
    assert per_head_rel_err(host64(st), s_ref) <= TOL_STATE
    assert not torch.any(st[1])          # the empty sequence has a zero state


@pytest.mark.parametrize("bad", [[0, 5, 3, 10], [1, 5, 10], [0, 5, 9], [0, -1, 10]])
def test_bad_seqlens_detected_on_device(bad):
    H, T, d = 2, 10, 64
    q, k, v = inputs.qkv((H, T, d), dtype=torch.float32, device=DEV, seed=1)
    cu = torch.tensor(bad, dtype=torch.int32, device=DEV)
    o = torch.full_like(q, 3.0)
    st = torch.full((len(bad) - 1, H, d, d), 3.0, device=DEV)
    la.prefill_varlen(q, k, v, cu, blk=64, out=o, state_out=st)
    assert la.la_get_last_error() == la.LA_ERR_BAD_SEQLENS
    assert torch.all(o == 3.0) and torch.all(st == 3.0)
    assert la.la_get_last_error() == la.LA_OK   # cleared after reading
