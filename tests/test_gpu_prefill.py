"""GPU parity of la_prefill (called through the C ABI) against the fp64 oracle.

Inputs are the seeded synthetic draws of linear_attention_13_b200.inputs; the
oracle consumes the same rounded values.  Bars: per-head relative error of o
<= 1e-4 (fp32) / 2e-2 (bf16), of the final state <= 1e-3; bit-exact equality
on small-integer inputs where every intermediate is exactly representable.
"""
import numpy as np
import pytest
import torch

import linear_attention_13_b200 as la
from linear_attention_13_b200 import inputs
import oracle
from _util import TOL_O_BF16, TOL_O_F32, TOL_STATE, host64, per_head_rel_err, round_like

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run(q, k, v, blk, **kw):
    o, st = la.prefill(q, k, v, blk=blk, **kw)
    assert la.la_get_last_error() == la.LA_OK
    return o, st


def test_tiny_fp32_config():
    # B=1, H=2, N=256, d=64, blk=64, fp32, seed 0
    q, k, v = inputs.qkv((1, 2, 256, 64), dtype=torch.float32, device=DEV, seed=0)
    o, st = _run(q, k, v, 64)
    o_ref, s_ref = oracle.prefill_recurrent(host64(q), host64(k), host64(v))
    assert per_head_rel_err(host64(o), o_ref) <= TOL_O_F32
    assert per_head_rel_err(host64(st), s_ref) <= TOL_STATE


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("blk", [1, 7, 64, 100, 256, 1000])
def test_fp32_block_sizes(d, blk):
    q, k, v = inputs.qkv((1, 3, 300, d), dtype=torch.float32, device=DEV, seed=blk)
    o, st = _run(q, k, v, blk)
    o_ref, s_ref = oracle.prefill_recurrent(host64(q), host64(k), host64(v))
    assert per_head_rel_err(host64(o), o_ref) <= TOL_O_F32
    assert per_head_rel_err(host64(st), s_ref) <= TOL_STATE


def test_fp32_ternary_exact():
    q, k, v = inputs.ternary_qkv((2, 2, 200, 64), dtype=torch.float32, device=DEV, seed=3)
    o, st = _run(q, k, v, 64)
    o_ref, s_ref = oracle.prefill_quadratic(host64(q), host64(k), host64(v)), None
    _, s_ref = oracle.prefill_recurrent(host64(q), host64(k), host64(v))
    assert np.array_equal(host64(o), o_ref)
    assert np.array_equal(host64(st), s_ref)


SCHEDULES = [
    pytest.param(0, id="default"),
    pytest.param(la.LA_FLAG_FUSED | la.LA_FLAG_NO_SPLIT_V, id="single-pass"),
    pytest.param(la.LA_FLAG_FUSED | la.LA_FLAG_SPLIT_V, id="single-pass-splitv"),
    pytest.param(la.LA_FLAG_THREE_PASS | la.LA_FLAG_NO_SPLIT_V, id="three-pass"),
    pytest.param(la.LA_FLAG_THREE_PASS | la.LA_FLAG_SPLIT_V, id="three-pass-splitv"),
]


@pytest.mark.parametrize("flags", SCHEDULES)
@pytest.mark.parametrize("N", [1, 2, 127, 128, 129, 255, 300, 1000, 2049])
@pytest.mark.parametrize("chunk", [0, 128, 384])
def test_bf16_ragged_lengths_and_chunks(N, chunk, flags):
    q, k, v = inputs.qkv((2, 3, N, 128), dtype=torch.bfloat16, device=DEV, seed=N + chunk)
    o, st = _run(q, k, v, 128, chunk_tokens=chunk, flags=flags)
    o_ref, s_ref = oracle.prefill_recurrent(host64(q), host64(k), host64(v))
    assert per_head_rel_err(host64(o), o_ref) <= TOL_O_BF16
    assert per_head_rel_err(host64(st), s_ref) <= TOL_STATE


@pytest.mark.parametrize("N,chunk", [(100, 0), (256, 0), (256, 128), (200, 128)])
def test_bf16_ternary_bit_exact(N, chunk):
    # |q.k| <= 128 and |S| <= N <= 256 are exact in bf16; fp32 sums are exact;
    # only the final o conversion rounds, with round-to-nearest-even.
    q, k, v = inputs.ternary_qkv((1, 4, N, 128), dtype=torch.bfloat16, device=DEV, seed=N)
    o, st = _run(q, k, v, 128, chunk_tokens=chunk)
    o_ref = oracle.prefill_quadratic(host64(q), host64(k), host64(v))
    _, s_ref = oracle.prefill_recurrent(host64(q), host64(k), host64(v))
    assert np.array_equal(host64(o), round_like(o_ref, torch.bfloat16))
    assert np.array_equal(host64(st), s_ref)


@pytest.mark.parametrize("flags", SCHEDULES)
@pytest.mark.parametrize("chunk", [0, 128, 1024, 8192])
def test_bf16_onehot_long_bit_exact(chunk, flags):
    # one nonzero per key row keeps every state entry a small integer, so even
    # the multi-chunk paths (look-back chain, or chunk states + scan) are exact.
    q, k, v = inputs.onehot_k_qkv((1, 4, 8192, 128), dtype=torch.bfloat16, device=DEV, seed=11)
    o, st = _run(q, k, v, 128, chunk_tokens=chunk, flags=flags)
    o_ref, s_ref = oracle.prefill_recurrent(host64(q), host64(k), host64(v))
    assert np.max(np.abs(s_ref)) <= 256
    assert np.array_equal(host64(o), round_like(o_ref, torch.bfloat16))
    assert np.array_equal(host64(st), s_ref)


@pytest.mark.parametrize("blk", [128, 64])
def test_bf16_prefill_config_all_heads(blk):
    # B=4, H=16, N=8192, d=128: every head against the oracle, in the launch
    # configuration the benchmark times (library-chosen chunking).
    q, k, v = inputs.qkv((4, 16, 8192, 128), dtype=torch.bfloat16, device=DEV, seed=0)
    o, st = _run(q, k, v, blk)
    o_ref, s_ref = oracle.prefill_recurrent(host64(q), host64(k), host64(v))
    assert per_head_rel_err(host64(o), o_ref) <= TOL_O_BF16
    assert per_head_rel_err(host64(st), s_ref) <= TOL_STATE


@pytest.mark.parametrize("flags", [0, la.LA_FLAG_FUSED | la.LA_FLAG_NO_SPLIT_V, la.LA_FLAG_THREE_PASS],
                         ids=["default", "single-pass", "three-pass"])
def test_bf16_long_context_sampled_heads(flags):
    # B=1, H=64, N=262144, d=128: 4 sampled heads (first, last, two seeded), in
    # the default schedule (value columns split, one chunk per head) and in the
    # chunked ones.
    B, H, N, d = 1, 64, 262144, 128
    q, k, v = inputs.qkv((B, H, N, d), dtype=torch.bfloat16, device=DEV, seed=0)
    o, st = _run(q, k, v, 128, flags=flags)
    rng = np.random.default_rng(0)
    heads = [0, H - 1] + sorted(rng.choice(np.arange(1, H - 1), 2, replace=False).tolist())
    hq, hk, hv = (host64(x[0, heads]) for x in (q, k, v))
    o_ref, s_ref = oracle.prefill_recurrent(hq, hk, hv)
    assert per_head_rel_err(host64(o[0, heads]), o_ref) <= TOL_O_BF16
    assert per_head_rel_err(host64(st[0, heads]), s_ref) <= TOL_STATE


@pytest.mark.parametrize("blk", [128, 64])
def test_bf16_many_items_per_cta_sampled_heads(blk):
    # The split kernels with many multi-tile work items per CTA (three-pass
    # output pass, 1024-token chunks of B1 H64 N32768: about 28 items per CTA).
    # Every item starts from a prefix state written into shared memory by eight
    # epilogue warps while the previous item is still in flight, so a barrier
    # hand-off that lets one warp's arrival stand in for another's shows up as a
    # wrong first tile of some chunk.  Three calls, eight sampled heads.
    B, H, N, d = 1, 64, 32768, 128
    q, k, v = inputs.qkv((B, H, N, d), dtype=torch.bfloat16, device=DEV, seed=21)
    heads = [0, H - 1] + sorted(np.random.default_rng(blk).choice(np.arange(1, H - 1), 6, replace=False).tolist())
    hq, hk, hv = (host64(x[0, heads]) for x in (q, k, v))
    o_ref, s_ref = oracle.prefill_recurrent(hq, hk, hv)
    for _ in range(3):
        o, st = _run(q, k, v, blk, chunk_tokens=1024, flags=la.LA_FLAG_THREE_PASS | la.LA_FLAG_SPLIT_V)
        assert la.la_prefill_main_kernel() == ("prefill_seq_kernel" if blk == 128 else "prefill_seq64_kernel")
        assert per_head_rel_err(host64(o[0, heads]), o_ref) <= TOL_O_BF16
        assert per_head_rel_err(host64(st[0, heads]), s_ref) <= TOL_STATE


# ---------------------------------------------------------------- 64-token blocks
# blk = 64 runs each 128-row tile as two blocks of 64 tokens (M = 64 MMAs):
# with the value columns split (prefill_seq64_kernel) when every sequence is
# one chunk or in the three-pass output pass, otherwise with whole value rows
# (prefill_tc_kernel<128,64>).
SCHEDULES_64 = [
    pytest.param(0, id="default"),
    pytest.param(la.LA_FLAG_FUSED, id="single-pass"),
    pytest.param(la.LA_FLAG_THREE_PASS, id="three-pass"),
    pytest.param(la.LA_FLAG_SPLIT_V, id="split-v"),
    pytest.param(la.LA_FLAG_NO_SPLIT_V, id="whole-rows"),
    pytest.param(la.LA_FLAG_THREE_PASS | la.LA_FLAG_SPLIT_V, id="three-pass-splitv"),
]


@pytest.mark.parametrize("flags", SCHEDULES_64)
@pytest.mark.parametrize("N", [1, 63, 64, 65, 127, 128, 129, 191, 192, 193, 300, 1000, 2049])
@pytest.mark.parametrize("chunk", [0, 128, 384])
def test_bf16_blk64_ragged_lengths_and_chunks(N, chunk, flags):
    q, k, v = inputs.qkv((2, 3, N, 128), dtype=torch.bfloat16, device=DEV, seed=N + chunk + 7)
    o, st = _run(q, k, v, 64, chunk_tokens=chunk, flags=flags)
    o_ref, s_ref = oracle.prefill_recurrent(host64(q), host64(k), host64(v))
    assert per_head_rel_err(host64(o), o_ref) <= TOL_O_BF16
    assert per_head_rel_err(host64(st), s_ref) <= TOL_STATE


def test_bf16_blk64_is_its_own_rounding_path():
    # The bf16 path rounds P and the state copy S̄ once per block: 64-token
    # blocks take a different rounding path from 128-token blocks (so the
    # block size is really honoured) and stay within the bf16 bar.
    q, k, v = inputs.qkv((1, 8, 1024, 128), dtype=torch.bfloat16, device=DEV, seed=31)
    o64, _ = _run(q, k, v, 64, chunk_tokens=1024)
    o128, _ = _run(q, k, v, 128, chunk_tokens=1024)
    o_ref, _ = oracle.prefill_recurrent(host64(q), host64(k), host64(v))
    assert per_head_rel_err(host64(o64), o_ref) <= TOL_O_BF16
    # different block sizes give different rounding paths, not the same bits
    assert not torch.equal(o64, o128)


@pytest.mark.parametrize("N,chunk", [(100, 0), (256, 0), (256, 128), (200, 128), (65, 0)])
def test_bf16_blk64_ternary_bit_exact(N, chunk):
    q, k, v = inputs.ternary_qkv((1, 4, N, 128), dtype=torch.bfloat16, device=DEV, seed=N + 1)
    o, st = _run(q, k, v, 64, chunk_tokens=chunk)
    o_ref = oracle.prefill_quadratic(host64(q), host64(k), host64(v))
    _, s_ref = oracle.prefill_recurrent(host64(q), host64(k), host64(v))
    assert np.array_equal(host64(o), round_like(o_ref, torch.bfloat16))
    assert np.array_equal(host64(st), s_ref)


@pytest.mark.parametrize("flags", SCHEDULES_64)
@pytest.mark.parametrize("chunk", [0, 128, 1024])
def test_bf16_blk64_onehot_long_bit_exact(chunk, flags):
    q, k, v = inputs.onehot_k_qkv((1, 4, 8192, 128), dtype=torch.bfloat16, device=DEV, seed=12)
    o, st = _run(q, k, v, 64, chunk_tokens=chunk, flags=flags)
    o_ref, s_ref = oracle.prefill_recurrent(host64(q), host64(k), host64(v))
    assert np.array_equal(host64(o), round_like(o_ref, torch.bfloat16))
    assert np.array_equal(host64(st), s_ref)


def test_bf16_blk64_split_flag_ignored_when_chunked():
    # chunked single pass keeps whole value rows at blk 64
    q, k, v = inputs.qkv((1, 2, 700, 128), dtype=torch.bfloat16, device=DEV, seed=8)
    o1, s1 = _run(q, k, v, 64, chunk_tokens=256, flags=la.LA_FLAG_FUSED)
    o2, s2 = _run(q, k, v, 64, chunk_tokens=256, flags=la.LA_FLAG_FUSED | la.LA_FLAG_SPLIT_V)
    assert la.la_prefill_main_kernel() == "prefill_tc_kernel<128,64>"
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


@pytest.mark.parametrize("flags,kernel", [
    (0, "prefill_seq64_kernel"),
    (la.LA_FLAG_NO_SPLIT_V, "prefill_tc_kernel<128,64>"),
    (la.LA_FLAG_THREE_PASS | la.LA_FLAG_SPLIT_V, "prefill_seq64_kernel"),
], ids=["default", "whole-rows", "three-pass-splitv"])
def test_bf16_blk64_kernels_agree_with_the_oracle(flags, kernel):
    # the two 64-token-block kernels on B4 H16 N8192 (every head): each within
    # the bar, and each is the kernel the dispatch names
    q, k, v = inputs.qkv((4, 16, 8192, 128), dtype=torch.bfloat16, device=DEV, seed=3)
    o, st = _run(q, k, v, 64, flags=flags)
    assert la.la_prefill_main_kernel() == kernel
    o_ref, s_ref = oracle.prefill_recurrent(host64(q), host64(k), host64(v))
    assert per_head_rel_err(host64(o), o_ref) <= TOL_O_BF16
    assert per_head_rel_err(host64(st), s_ref) <= TOL_STATE


def test_bf16_scaling_is_exact():
    q, k, v = inputs.qkv((1, 2, 700, 128), dtype=torch.bfloat16, device=DEV, seed=5)
    o1, s1 = _run(q, k, v, 128, chunk_tokens=256)
    o2, s2 = _run(q * 2, k, v, 128, chunk_tokens=256)
    o3, s3 = _run(q, k, v * 2, 128, chunk_tokens=256)
    assert torch.equal(o2, o1 * 2) and torch.equal(s2, s1)
    assert torch.equal(o3, o1 * 2) and torch.equal(s3, s1 * 2)


def test_no_writes_outside_outputs():
    B, H, N, d = 1, 3, 333, 128
    q, k, v = inputs.qkv((B, H, N, d), dtype=torch.bfloat16, device=DEV, seed=9)
    pad = 4096
    o_buf = torch.full((pad + B * H * N * d + pad,), 7.0, dtype=torch.bfloat16, device=DEV)
    s_buf = torch.full((pad + B * H * d * d + pad,), 7.0, dtype=torch.float32, device=DEV)
    o = o_buf[pad:pad + B * H * N * d].view(B, H, N, d)
    s = s_buf[pad:pad + B * H * d * d].view(B, H, d, d)
    la.prefill(q, k, v, blk=128, out=o, state_out=s, chunk_tokens=128)
    assert la.la_get_last_error() == la.LA_OK
    assert torch.all(o_buf[:pad] == 7.0) and torch.all(o_buf[-pad:] == 7.0)
    assert torch.all(s_buf[:pad] == 7.0) and torch.all(s_buf[-pad:] == 7.0)
    o_ref, _ = oracle.prefill_recurrent(host64(q), host64(k), host64(v))
    assert per_head_rel_err(host64(o), o_ref) <= TOL_O_BF16


def test_without_state_output():
    q, k, v = inputs.qkv((1, 2, 600, 128), dtype=torch.bfloat16, device=DEV, seed=6)
    o, st = la.prefill(q, k, v, blk=128, want_state=False, chunk_tokens=256)
    assert st is None and la.la_get_last_error() == la.LA_OK
    o_ref, _ = oracle.prefill_recurrent(host64(q), host64(k), host64(v))
    assert per_head_rel_err(host64(o), o_ref) <= TOL_O_BF16


@pytest.mark.parametrize("split", [la.LA_FLAG_NO_SPLIT_V, la.LA_FLAG_SPLIT_V])
@pytest.mark.parametrize("BH,N", [(1, 16384), (3, 5000), (200, 1000)])
def test_bf16_single_pass_long_chains(BH, N, split):
    # 128-token chunks: every chunk waits for its predecessor's published
    # prefix, the chains run through many CTAs (one head: 128 links).
    q, k, v = inputs.onehot_k_qkv((1, BH, N, 128), dtype=torch.bfloat16, device=DEV, seed=BH)
    o, st = _run(q, k, v, 128, chunk_tokens=128, flags=la.LA_FLAG_FUSED | split)
    o_ref, s_ref = oracle.prefill_recurrent(host64(q), host64(k), host64(v))
    assert np.array_equal(host64(o), round_like(o_ref, torch.bfloat16))
    assert np.array_equal(host64(st), s_ref)


def test_bf16_schedules_agree():
    q, k, v = inputs.qkv((2, 8, 6000, 128), dtype=torch.bfloat16, device=DEV, seed=17)
    o1, s1 = _run(q, k, v, 128, chunk_tokens=1024, flags=la.LA_FLAG_THREE_PASS | la.LA_FLAG_NO_SPLIT_V)
    for fl in (la.LA_FLAG_FUSED | la.LA_FLAG_NO_SPLIT_V, la.LA_FLAG_FUSED | la.LA_FLAG_SPLIT_V,
               la.LA_FLAG_THREE_PASS | la.LA_FLAG_SPLIT_V):
        o2, s2 = _run(q, k, v, 128, chunk_tokens=1024, flags=fl)
        # same chunking: the starting states agree up to fp32 summation order
        assert per_head_rel_err(host64(o2), host64(o1)) <= 1e-2
        assert per_head_rel_err(host64(s2), host64(s1)) <= 1e-5


@pytest.mark.parametrize("flags", SCHEDULES)
def test_bf16_prefill_config_all_heads_schedules(flags):
    # B=4, H=16, N=8192 in every schedule, all heads
    q, k, v = inputs.qkv((4, 16, 8192, 128), dtype=torch.bfloat16, device=DEV, seed=3)
    o, st = _run(q, k, v, 128, flags=flags)
    o_ref, s_ref = oracle.prefill_recurrent(host64(q), host64(k), host64(v))
    assert per_head_rel_err(host64(o), o_ref) <= TOL_O_BF16
    assert per_head_rel_err(host64(st), s_ref) <= TOL_STATE
