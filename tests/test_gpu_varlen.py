"""GPU parity of la_prefill_varlen (packed sequences, state reset at every
sequence start) and its device-side cu_seqlens check."""
import numpy as np
import pytest
import torch

import linear_attention_13_b200 as la
from linear_attention_13_b200 import inputs
import oracle
from _util import TOL_O_F32, TOL_STATE, host64, per_head_rel_err, per_seq_head_rel_err

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
    assert per_seq_head_rel_err(host64(o), o_ref, cu) <= TOL_O_F32
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


# ---------------------------------------------------------------- bf16 tensor-core path
from _util import TOL_O_BF16, round_like  # noqa: E402


SCHEDULES = [pytest.param(0, id="default"), pytest.param(la.LA_FLAG_FUSED, id="single-pass"),
             pytest.param(la.LA_FLAG_THREE_PASS, id="three-pass"),
             pytest.param(la.LA_FLAG_SPLIT_V, id="split-v")]


@pytest.mark.parametrize("blk", [128, 64])
@pytest.mark.parametrize("flags", SCHEDULES)
@pytest.mark.parametrize("chunk", [0, 256])
@pytest.mark.parametrize("lens", [
    [5, 0, 130, 1, 64, 257],
    [128, 127, 129, 1, 0, 0, 1000],
    [3000, 1, 2049, 5000],
    [0, 0, 7],
])
def test_varlen_bf16(lens, chunk, flags, blk):
    cu = _cu(lens)
    H, T = 3, sum(lens)
    q, k, v = inputs.qkv((H, T, 128), dtype=torch.bfloat16, device=DEV, seed=len(lens))
    o = torch.full_like(q, 5.0)
    st = torch.full((len(lens), H, 128, 128), 5.0, device=DEV)
    o, st = la.prefill_varlen(q, k, v, cu, blk=blk, out=o, state_out=st, chunk_tokens=chunk,
                              flags=flags)
    assert la.la_get_last_error() == la.LA_OK
    o_ref, s_ref = oracle.prefill_varlen(host64(q), host64(k), host64(v), cu.cpu().numpy())
    assert per_seq_head_rel_err(host64(o), o_ref, cu) <= TOL_O_BF16
    assert per_head_rel_err(host64(st), s_ref) <= TOL_STATE
    for j, n in enumerate(lens):
        if n == 0:
            assert not torch.any(st[j])


@pytest.mark.parametrize("blk", [128, 64])
@pytest.mark.parametrize("flags", SCHEDULES)
@pytest.mark.parametrize("chunk", [0, 128, 640])
def test_varlen_bf16_onehot_bit_exact(chunk, flags, blk):
    # one-hot keys keep all intermediates small integers: the packed path,
    # including sequences longer than one chunk and ragged tails, is exact.
    lens = [2500, 1, 4097, 0, 1300, 128, 9000]
    cu = _cu(lens)
    H, T = 2, sum(lens)
    q, k, v = inputs.onehot_k_qkv((H, T, 128), dtype=torch.bfloat16, device=DEV, seed=21)
    o, st = la.prefill_varlen(q, k, v, cu, blk=blk, chunk_tokens=chunk, flags=flags)
    assert la.la_get_last_error() == la.LA_OK
    o_ref, s_ref = oracle.prefill_varlen(host64(q), host64(k), host64(v), cu.cpu().numpy())
    assert np.array_equal(host64(o), round_like(o_ref, torch.bfloat16))
    assert np.array_equal(host64(st), s_ref)


@pytest.mark.parametrize("lens", [
    [300, 7000, 1, 0, 129, 5000, 0, 2048, 128, 4097, 77],
    [0, 0, 0, 5],
    [1] * 40 + [3000],
])
@pytest.mark.parametrize("blk,kernel", [(128, "prefill_seq_kernel"), (64, "prefill_seq64_kernel")])
def test_varlen_bf16_split_longest_first_exact(lens, blk, kernel):
    # split value columns, longest sequence first: every sequence and head is
    # produced exactly once with its own state (one-hot keys: exact)
    cu = _cu(lens)
    H, T = 3, sum(lens)
    q, k, v = inputs.onehot_k_qkv((H, T, 128), dtype=torch.bfloat16, device=DEV, seed=len(lens))
    o = torch.full_like(q, 3.0)
    st = torch.full((len(lens), H, 128, 128), 3.0, device=DEV)
    o, st = la.prefill_varlen(q, k, v, cu, blk=blk, out=o, state_out=st, flags=la.LA_FLAG_SPLIT_V)
    assert la.la_get_last_error() == la.LA_OK
    assert la.la_prefill_main_kernel() == kernel
    o_ref, s_ref = oracle.prefill_varlen(host64(q), host64(k), host64(v), cu.cpu().numpy())
    assert np.array_equal(host64(o), round_like(o_ref, torch.bfloat16))
    assert np.array_equal(host64(st), s_ref)


@pytest.mark.parametrize("flags", SCHEDULES)
def test_varlen_bf16_bad_seqlens_detected(flags):
    H, T = 2, 300
    q, k, v = inputs.qkv((H, T, 128), dtype=torch.bfloat16, device=DEV, seed=1)
    cu = torch.tensor([0, 200, 100, 300], dtype=torch.int32, device=DEV)
    o = torch.full_like(q, 3.0)
    st = torch.full((3, H, 128, 128), 3.0, device=DEV)
    la.prefill_varlen(q, k, v, cu, blk=128, out=o, state_out=st, flags=flags)
    assert la.la_get_last_error() == la.LA_ERR_BAD_SEQLENS
    assert torch.all(o == 3.0) and torch.all(st == 3.0)


@pytest.mark.parametrize("flags,chunk", [pytest.param(0, 0, id="default"),
                                         pytest.param(la.LA_FLAG_SPLIT_V, 0, id="split-v"),
                                         pytest.param(la.LA_FLAG_FUSED, 8192, id="single-pass-8k")])
def test_varlen_bf16_packed_config_sampled_heads(flags, chunk):
    # 2^20 packed tokens, lengths uniform in [1024, 65536] (seeded, last
    # trimmed), H = 64, d = 128: every sequence of 8 sampled heads.
    T, H = 1 << 20, 64
    lens = inputs.varlen_lengths(T, 1024, 65536, seed=0)
    cu = _cu(lens)
    q, k, v = inputs.qkv((H, T, 128), dtype=torch.bfloat16, device=DEV, seed=0)
    o, st = la.prefill_varlen(q, k, v, cu, blk=128, flags=flags, chunk_tokens=chunk)
    assert la.la_get_last_error() == la.LA_OK
    rng = np.random.default_rng(0)
    heads = [0, H - 1] + sorted(rng.choice(np.arange(1, H - 1), 6, replace=False).tolist())
    hq, hk, hv = (host64(x[heads]) for x in (q, k, v))
    o_ref, s_ref = oracle.prefill_varlen(hq, hk, hv, cu.cpu().numpy())
    assert per_seq_head_rel_err(host64(o[heads]), o_ref, cu) <= TOL_O_BF16
    assert per_head_rel_err(host64(st[:, heads]), s_ref) <= TOL_STATE
