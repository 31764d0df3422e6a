"""Host-side argument checks of the tensor helpers: the C entry points take raw
pointers and cannot check sizes, so every helper must reject a tensor of the
wrong shape, dtype or device before anything is launched.  Runs on CPU: the
CUDA-device test is relaxed and the raw C calls are replaced by recorders, so
a check that is missing shows up as a recorded call instead of a ValueError."""
import pytest
import torch

import linear_attention_13_b200 as la

RAW = ("la_prefill_from_state", "la_prefill_varlen_from_state", "la_prefill_backward",
       "la_state_increment", "la_state_prefix", "la_decode_step", "la_decode_step_slots",
       "la_decode_step_q8", "la_state_quantize_q8", "la_state_dequantize_q8")


@pytest.fixture
def calls(monkeypatch):
    made = []

    def relaxed_check(t, name):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")

    monkeypatch.setattr(la, "_check", relaxed_check)
    monkeypatch.setattr(la, "_stream_ptr", lambda stream: None)
    for name in RAW:
        monkeypatch.setattr(la, name, lambda *a, _n=name: made.append(_n) or la.LA_OK)
    return made


def t(*shape, dtype=torch.bfloat16):
    return torch.zeros(shape, dtype=dtype)


def f32(*shape):
    return t(*shape, dtype=torch.float32)


def test_well_formed_calls_reach_the_library(calls):
    q = t(2, 3, 16, 128)
    la.prefill(q, t(2, 3, 16, 128), t(2, 3, 16, 128))
    cu = torch.tensor([0, 5, 16], dtype=torch.int32)
    la.prefill_varlen(t(3, 16, 128), t(3, 16, 128), t(3, 16, 128), cu)
    la.decode_step(t(2, 3, 128), t(2, 3, 128), t(2, 3, 128), f32(2, 3, 128, 128))
    la.state_increment(q, t(2, 3, 16, 128))
    assert calls == ["la_prefill_from_state", "la_prefill_varlen_from_state", "la_decode_step",
                     "la_state_increment"]


@pytest.mark.parametrize("bad", [
    dict(k=t(2, 3, 8, 128)),                       # shorter k
    dict(v=f32(2, 3, 16, 128)),                    # fp32 v with bf16 q (twice the bytes)
    dict(out=t(2, 3, 8, 128)),                     # small output
    dict(out=f32(2, 3, 16, 128)),                  # output of another dtype
    dict(state_out=f32(2, 3, 128, 64)),            # wrong state shape
    dict(state_out=t(2, 3, 128, 128)),             # bf16 state
    dict(state_in=f32(1, 3, 128, 128)),            # state_in for fewer sequences
])
def test_prefill_rejects_mismatched_tensors(calls, bad):
    args = dict(q=t(2, 3, 16, 128), k=t(2, 3, 16, 128), v=t(2, 3, 16, 128))
    kw = {}
    for n, x in bad.items():
        (args if n in args else kw)[n] = x
    with pytest.raises(ValueError):
        la.prefill(args["q"], args["k"], args["v"], **kw)
    assert calls == []


@pytest.mark.parametrize("bad", ["k", "v", "out", "state_out", "cu_device"])
def test_prefill_varlen_rejects_mismatched_tensors(calls, bad):
    q, k, v = t(3, 16, 128), t(3, 16, 128), t(3, 16, 128)
    cu = torch.tensor([0, 5, 16], dtype=torch.int32)
    kw = {}
    if bad == "k":
        k = t(3, 15, 128)
    elif bad == "v":
        v = f32(3, 16, 128)
    elif bad == "out":
        kw["out"] = t(2, 16, 128)
    elif bad == "state_out":
        kw["state_out"] = f32(3, 3, 128, 128)      # three sequences' states for two
    else:
        cu = torch.tensor([0, 5, 16], dtype=torch.int32, device="meta")
    with pytest.raises((ValueError, TypeError)):
        la.prefill_varlen(q, k, v, cu, **kw)
    assert calls == []


@pytest.mark.parametrize("state", [f32(1, 3, 128, 128), f32(2, 3, 64, 64), t(2, 3, 128, 128),
                                   f32(2, 2, 128, 128)])
def test_decode_step_rejects_a_state_that_does_not_cover_the_batch(calls, state):
    # la_decode_step updates B*H states: a smaller array would be overrun
    with pytest.raises(ValueError):
        la.decode_step(t(2, 3, 128), t(2, 3, 128), t(2, 3, 128), state)
    assert calls == []


def test_decode_helpers_reject_mismatched_vectors(calls):
    q = t(2, 3, 128)
    with pytest.raises(ValueError):
        la.decode_step(q, t(2, 3, 64), t(2, 3, 128), f32(2, 3, 128, 128))
    with pytest.raises(ValueError):
        la.decode_step(q, t(2, 3, 128), t(2, 3, 128), f32(2, 3, 128, 128), out=f32(2, 3, 128))
    with pytest.raises(ValueError):
        la.decode_step_slots(q, t(2, 3, 128), f32(2, 3, 128), f32(4, 3, 128, 128), None)
    codes = torch.zeros((1, 3, 128, 128), dtype=torch.int8)
    with pytest.raises(ValueError):   # no slots: row b uses slot b, but only one slot exists
        la.decode_step_q8(q, t(2, 3, 128), t(2, 3, 128), codes, f32(1, 3, 128))
    assert calls == []


def test_state_helpers_reject_mismatched_tensors(calls):
    k = t(2, 3, 16, 128)
    with pytest.raises(ValueError):
        la.state_increment(k, t(2, 3, 16, 64))
    with pytest.raises(ValueError):
        la.state_increment(k, t(2, 3, 16, 128), out=f32(2, 3, 128, 64))
    with pytest.raises(ValueError):
        la.state_prefix(f32(4, 2, 3, 128, 128), 2, out=f32(2, 3, 64, 64))
    S = f32(2, 3, 128, 128)
    with pytest.raises(ValueError):
        la.state_quantize_q8(S, codes=torch.zeros((2, 3, 128, 64), dtype=torch.int8))
    with pytest.raises(ValueError):
        la.state_quantize_q8(S, scales=f32(2, 3, 64))
    codes = torch.zeros((2, 3, 128, 128), dtype=torch.int8)
    with pytest.raises(ValueError):
        la.state_dequantize_q8(codes, f32(2, 3, 64))
    with pytest.raises(ValueError):
        la.state_dequantize_q8(codes, f32(2, 3, 128), out=f32(2, 3, 128, 64))
    assert calls == []


def test_backward_rejects_mismatched_gradients(calls):
    q = t(1, 2, 16, 128)
    with pytest.raises(ValueError):
        la.prefill_backward(q, q, q, t(1, 2, 8, 128))
    with pytest.raises(ValueError):
        la.prefill_backward(q, q, q, q, out=(t(1, 2, 16, 128), f32(1, 2, 16, 128), t(1, 2, 16, 128)))
    assert calls == []
