"""Run-to-run determinism of the warp-specialised prefill kernels, as a race
detector.

Every kernel here is deterministic by construction: each output element and
each state element is produced by a fixed sequence of MMAs and adds, whatever
the timing of the warps.  A barrier that lets a warp read a buffer before it
is written, or overwrite one still being read, makes the result depend on that
timing.  So each case repeats the same call many times on the same inputs and
requires every repetition to be bit-identical to the first, with no device
error.  The cases cover the split-value-column kernels at both block sizes with
one tile sequence per CTA, with many work items per CTA (the buffers' phases
carry across items), with a starting state, packed sequences with ragged
tails, and the anti-causal passes of the backward.  Parity with the oracle is
tested elsewhere; this file checks only that the result does not vary."""
import pytest
import torch

import linear_attention_13_b200 as la
from linear_attention_13_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _repeat_identical(call, reps):
    ref = [x.clone() for x in call()]
    mismatches = 0
    for _ in range(reps):
        out = call()
        if not all(torch.equal(a, b) for a, b in zip(out, ref)):
            mismatches += 1
    torch.cuda.synchronize()
    assert la.la_get_last_error() == la.LA_OK
    return mismatches


@pytest.mark.parametrize("blk", [128, 64])
def test_one_item_per_cta_repeats_bit_identical(blk):
    q, k, v = inputs.qkv((4, 16, 8192, 128), dtype=torch.bfloat16, device=DEV, seed=1)
    o = torch.empty_like(q)
    st = torch.empty((4, 16, 128, 128), dtype=torch.float32, device=DEV)

    def call():
        la.prefill(q, k, v, blk=blk, out=o, state_out=st)
        return o, st

    assert _repeat_identical(call, 300) == 0
    assert la.la_prefill_main_kernel() == ("prefill_seq_kernel" if blk == 128 else "prefill_seq64_kernel")


@pytest.mark.parametrize("with_state_in", [False, True])
@pytest.mark.parametrize("blk", [128, 64])
def test_many_items_per_cta_repeat_bit_identical(blk, with_state_in):
    # 32 chunks of 1024 tokens per head, 64 heads, two value halves: 4096 items
    # over at most one CTA per SM, so every CTA carries its barriers' phases
    # through many items
    q, k, v = inputs.qkv((1, 64, 32768, 128), dtype=torch.bfloat16, device=DEV, seed=2)
    o = torch.empty_like(q)
    st = torch.empty((1, 64, 128, 128), dtype=torch.float32, device=DEV)
    s_in = None
    if with_state_in:
        g = torch.Generator(device=DEV).manual_seed(7)
        s_in = torch.randn((1, 64, 128, 128), dtype=torch.float32, device=DEV, generator=g) * 0.1
    flags = la.LA_FLAG_THREE_PASS | la.LA_FLAG_SPLIT_V

    def call():
        la.prefill(q, k, v, blk=blk, chunk_tokens=1024, flags=flags, out=o, state_out=st, state_in=s_in)
        return o, st

    assert _repeat_identical(call, 100) == 0


@pytest.mark.parametrize("blk", [128, 64])
def test_packed_sequences_repeat_bit_identical(blk):
    lens = inputs.varlen_lengths(1 << 18, 100, 20000, seed=3)
    cu = torch.as_tensor(inputs.cu_seqlens_from_lengths(lens), dtype=torch.int32).to(DEV)
    T = int(cu[-1])
    q, k, v = inputs.qkv((1, 16, T, 128), dtype=torch.bfloat16, device=DEV, seed=4)
    q, k, v = q[0], k[0], v[0]

    def call():
        return la.prefill_varlen(q, k, v, cu, blk=blk, flags=la.LA_FLAG_SPLIT_V)

    assert _repeat_identical(call, 60) == 0


def test_backward_repeats_bit_identical():
    q, k, v = inputs.qkv((4, 16, 8192, 128), dtype=torch.bfloat16, device=DEV, seed=5)
    g = torch.Generator(device=DEV).manual_seed(11)
    do = torch.randn(q.shape, dtype=q.dtype, device=DEV, generator=g)

    def call():
        return la.prefill_backward(q, k, v, do)

    assert _repeat_identical(call, 60) == 0
