"""GPU parity of the slot-pool decode and the 8-bit decode state (through the
C ABI) against the oracle.

* Codes and scales are integer decisions taken in fp32 on both sides, so they
  are compared bit for bit, at every step of multi-step trajectories.
* o is an fp32 sum on the GPU and an fp64 sum on the host over the same fp32
  values: compared at the fp32 / bf16 bar.
* Padding rows (negative slot) write zeros and leave every state untouched;
  an out-of-range slot reports LA_ERR_BAD_SLOT and is treated as padding.
"""
import numpy as np
import pytest
import torch

import linear_attention_13_b200 as la
from linear_attention_13_b200 import inputs
from linear_attention_13_b200.decode_batch import PaddedDecoder
import oracle
from _util import TOL_O_BF16, TOL_O_F32, host64, per_head_rel_err, round_like

pytestmark = pytest.mark.gpu
DEV = "cuda"
DTS = [pytest.param(torch.bfloat16, id="bf16"), pytest.param(torch.float32, id="f32")]


def _tol(dt):
    return TOL_O_BF16 if dt == torch.bfloat16 else TOL_O_F32


def _np(t):
    return t.detach().cpu().numpy()


def _states(shape, seed, special_rows=True):
    """fp32 states with the row kinds the rounding rules single out: ordinary
    normal rows, zero rows, negligible rows (< 2^-100), rows of exact ties."""
    g = torch.Generator().manual_seed(seed)
    S = torch.randn(shape, generator=g, dtype=torch.float32) * 3.0
    if special_rows:
        d = shape[-1]
        flat = S.view(-1, d)
        flat[1::97] = 0.0
        flat[2::97] = 1e-31
        ties = torch.arange(d, dtype=torch.float32) - d / 2 + 0.5     # x.5 values
        ties[0] = 127.0                                               # max 127: scale 1
        flat[3::97] = ties
    return S


@pytest.mark.parametrize("d", [64, 128])
def test_quantize_dequantize_bit_exact(d):
    S = _states((5, 7, d, d), seed=d)
    c, a = la.state_quantize_q8(S.to(DEV))
    assert la.la_get_last_error() == la.LA_OK
    c_ref, a_ref = oracle.state_quantize_q8(S.numpy())
    assert np.array_equal(_np(c), c_ref)
    assert np.array_equal(_np(a), a_ref)
    back = la.state_dequantize_q8(c, a)
    assert np.array_equal(_np(back), oracle.state_dequantize_q8(c_ref, a_ref))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dt", DTS)
def test_q8_trajectory_bit_exact_codes(d, dt):
    # 48 steps from a quantised random state: codes and scales equal the
    # oracle's at every step, o within the bar
    B, H, steps = 3, 4, 48
    c, a = la.state_quantize_q8(_states((B, H, d, d), seed=1, special_rows=False).to(DEV))
    c_ref, a_ref = _np(c), _np(a)
    for step in range(steps):
        q, k, v = inputs.decode_step_inputs(B, H, d, step + 1, dtype=dt, device=DEV)
        o = la.decode_step_q8(q, k, v, c, a)
        assert la.la_get_last_error() == la.LA_OK
        o_ref, c_ref, a_ref = oracle.decode_step_q8(host64(q), host64(k), host64(v), c_ref, a_ref)
        assert np.array_equal(_np(c), c_ref), step
        assert np.array_equal(_np(a), a_ref), step
        assert per_head_rel_err(host64(o), o_ref, head_dims=1) <= _tol(dt), step


def test_q8_integer_state_exact():
    # integer rows with max exactly 127 keep scale 1; one-hot keys and small
    # integer values keep every value an integer, so o is exact in bf16
    B, H, d = 2, 6, 128
    g = torch.Generator().manual_seed(3)
    S = torch.randint(-60, 61, (B, H, d, d), generator=g).to(torch.float32)
    S[..., 0] = 127.0
    c, a = la.state_quantize_q8(S.to(DEV))
    assert torch.all(a == 1.0)
    q = torch.randint(-1, 2, (B, H, d), generator=g).to(torch.bfloat16)
    k = torch.zeros((B, H, d), dtype=torch.bfloat16)
    rows = torch.randint(0, d, (B, H), generator=g)
    k.view(-1, d)[torch.arange(B * H), rows.view(-1)] = 1.0
    v = torch.randint(-2, 3, (B, H, d), generator=g).to(torch.bfloat16)
    v[..., 0] = 0.0
    o = la.decode_step_q8(q.to(DEV), k.to(DEV), v.to(DEV), c, a)
    o_ref, c_ref, a_ref = oracle.decode_step_q8(host64(q), host64(k), host64(v), S.numpy().astype(np.int8),
                                                np.ones((B, H, d), np.float32))
    assert np.array_equal(host64(o), round_like(o_ref, torch.bfloat16))
    assert np.array_equal(_np(c), c_ref) and np.array_equal(_np(a), a_ref)
    want = S.numpy() + np.einsum("bhi,bhj->bhij", host64(k), host64(v))
    assert np.array_equal(_np(c).astype(np.float64), want)


@pytest.mark.parametrize("dt", DTS)
def test_q8_rows_becoming_zero(dt):
    # a row the step cancels exactly and a row below 2^-100 become zero rows
    # (codes 0, scale 0), every other row as the oracle says
    d = 128
    g = torch.Generator().manual_seed(17)
    S = torch.randn((1, 2, d, d), generator=g) * 2.0
    c, a = oracle.state_quantize_q8(S.numpy())
    c[0, 0, 0] = 0
    c[0, 0, 0, :4] = [1, 2, 0, -3]
    a[0, 0, 0] = 1.0
    c[0, 1, 5] = 0
    c[0, 1, 5, 0] = 127
    a[0, 1, 5] = np.float32(2.0 ** -108) / np.float32(127)
    q, k, v = inputs.decode_step_inputs(1, 2, d, 3, dtype=dt, device="cpu")
    k[0, 0] = 0
    k[0, 0, 0] = -1.0
    v[0, 0] = 0
    v[0, 0, :4] = torch.tensor([1.0, 2.0, 0.0, -3.0])
    k[0, 1, 5] = 0
    cd, ad = torch.from_numpy(c).to(DEV), torch.from_numpy(a).to(DEV)
    o = la.decode_step_q8(q.to(DEV), k.to(DEV), v.to(DEV), cd, ad)
    assert la.la_get_last_error() == la.LA_OK
    o_ref, c_ref, a_ref = oracle.decode_step_q8(host64(q), host64(k), host64(v), c, a)
    assert a_ref[0, 0, 0] == 0 and a_ref[0, 1, 5] == 0 and not np.any(c_ref[0, 0, 0])
    assert np.array_equal(_np(cd), c_ref) and np.array_equal(_np(ad), a_ref)
    assert per_head_rel_err(host64(o), o_ref, head_dims=1) <= _tol(dt)


def _slot_batch(num_slots, B, n_pad, seed):
    rng = np.random.default_rng(seed)
    live = rng.choice(num_slots, size=B - n_pad, replace=False).tolist()
    slots = live + [-1] * n_pad
    rng.shuffle(slots)
    return slots


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dt", DTS)
def test_slots_fp32_matches_oracle_and_padding_untouched(d, dt):
    num_slots, H, B = 11, 3, 8
    pool = _states((num_slots, H, d, d), seed=5, special_rows=False).to(DEV)
    pool0 = host64(pool)
    slots = _slot_batch(num_slots, B, n_pad=3, seed=d)
    q, k, v = inputs.decode_step_inputs(B, H, d, 1, dtype=dt, device=DEV)
    o = torch.full_like(q, 7.0)
    la.decode_step_slots(q, k, v, pool, torch.tensor(slots, dtype=torch.int32, device=DEV), out=o)
    assert la.la_get_last_error() == la.LA_OK
    o_ref, pool_ref = oracle.decode_step_slots(host64(q), host64(k), host64(v), pool0, slots)
    assert per_head_rel_err(host64(o), o_ref, head_dims=1) <= _tol(dt)
    assert per_head_rel_err(host64(pool), pool_ref) <= 1e-6
    for b, s in enumerate(slots):
        if s < 0:
            assert not torch.any(o[b])
    untouched = sorted(set(range(num_slots)) - {s for s in slots if s >= 0})
    assert np.array_equal(host64(pool)[untouched], pool0[untouched])


@pytest.mark.parametrize("d", [64, 128])
def test_slots_q8_bit_exact_and_padding_untouched(d):
    num_slots, H, B = 9, 5, 6
    c, a = la.state_quantize_q8(_states((num_slots, H, d, d), seed=6).to(DEV))
    c0, a0 = _np(c), _np(a)
    for step in range(4):
        slots = _slot_batch(num_slots, B, n_pad=2, seed=10 * d + step)
        q, k, v = inputs.decode_step_inputs(B, H, d, step + 1, device=DEV)
        o = la.decode_step_q8(q, k, v, c, a, torch.tensor(slots, dtype=torch.int32, device=DEV))
        assert la.la_get_last_error() == la.LA_OK
        o_ref, c0, a0 = oracle.decode_step_q8(host64(q), host64(k), host64(v), c0, a0, slots)
        assert np.array_equal(_np(c), c0) and np.array_equal(_np(a), a0), step
        assert per_head_rel_err(host64(o), o_ref, head_dims=1) <= TOL_O_BF16
        for b, s in enumerate(slots):
            if s < 0:
                assert not torch.any(o[b])


@pytest.mark.parametrize("kind", ["fp32", "q8"])
def test_bad_slot_reports_and_is_skipped(kind):
    num_slots, H, d, B = 4, 2, 128, 3
    q, k, v = inputs.decode_step_inputs(B, H, d, 1, device=DEV)
    slots = torch.tensor([1, 4, 0], dtype=torch.int32, device=DEV)     # 4 is out of range
    assert la.la_get_last_error() == la.LA_OK
    if kind == "fp32":
        pool = torch.randn((num_slots, H, d, d), device=DEV)
        before = pool.clone()
        o = la.decode_step_slots(q, k, v, pool, slots)
        after = pool
    else:
        c, a = la.state_quantize_q8(torch.randn((num_slots, H, d, d), device=DEV))
        before = c.clone()
        o = la.decode_step_q8(q, k, v, c, a, slots)
        after = c
    assert la.la_get_last_error() == la.LA_ERR_BAD_SLOT
    assert la.la_get_last_error() == la.LA_OK          # the status is read and cleared
    assert not torch.any(o[1])
    assert torch.equal(after[2], before[2]) and torch.equal(after[3], before[3])
    assert not torch.equal(after[1], before[1]) and not torch.equal(after[0], before[0])


def test_slots_null_is_dense_step():
    B, H, d = 4, 8, 128
    S = torch.randn((B, H, d, d), device=DEV)
    S2 = S.clone()
    q, k, v = inputs.decode_step_inputs(B, H, d, 2, device=DEV)
    o1 = la.decode_step(q, k, v, S)
    o2 = la.decode_step_slots(q, k, v, S2, None)
    assert torch.equal(o1, o2) and torch.equal(S, S2)


def test_q8_continues_prefill():
    # a prefill's final state, quantised, then 32 steps on the 8-bit state:
    # the oracle's own 8-bit trajectory bit for bit, and the exact fp64
    # recurrence within the rounding bound (half a quantisation step per row
    # per quantisation, plus fp32 rounding)
    B, H, N, d, steps = 2, 4, 1000, 128, 32
    q0, k0, v0 = inputs.qkv((B, H, N, d), dtype=torch.bfloat16, device=DEV, seed=12)
    _, st = la.prefill(q0, k0, v0)
    c, a = la.state_quantize_q8(st)
    c_ref, a_ref = oracle.state_quantize_q8(_np(st))
    assert np.array_equal(_np(c), c_ref) and np.array_equal(_np(a), a_ref)
    exact = host64(st)
    bound = 0.5 * a_ref.astype(np.float64) + 2.0 ** -20 * 127 * a_ref
    for step in range(steps):
        q, k, v = inputs.decode_step_inputs(B, H, d, step + 1, device=DEV)
        o = la.decode_step_q8(q, k, v, c, a)
        o_ref, c_ref, a_ref = oracle.decode_step_q8(host64(q), host64(k), host64(v), c_ref, a_ref)
        assert np.array_equal(_np(c), c_ref) and np.array_equal(_np(a), a_ref), step
        o_exact, exact = oracle.decode_step(host64(q), host64(k), host64(v), exact)
        m = 127.0 * a_ref.astype(np.float64)
        o_bound = np.einsum("bhi,bhi->bh", np.abs(host64(q)), bound + 2.0 ** -20 * m)
        assert np.all(np.abs(o_ref - o_exact) <= o_bound[..., None] + 1e-9), step
        bound = bound + 0.5 * a_ref + 2.0 ** -20 * m
    deq = host64(la.state_dequantize_q8(c, a))
    assert np.all(np.abs(deq - exact) <= bound[..., None] + 1e-9)
    assert np.max(bound) < 0.3 * np.max(np.abs(exact))       # not a vacuous bound


def test_q8_decode_config_all_heads():
    # 128 sequences x 64 heads, d = 128, from quantised prefill-like states:
    # every head's codes and scales bit-exact after one step
    n_seq, H, d = 128, 64, 128
    S = _states((n_seq, H, d, d), seed=9)
    c, a = la.state_quantize_q8(S.to(DEV))
    c_ref, a_ref = oracle.state_quantize_q8(S.numpy())
    assert np.array_equal(_np(c), c_ref) and np.array_equal(_np(a), a_ref)
    q, k, v = inputs.decode_step_inputs(n_seq, H, d, 1, device=DEV)
    o = la.decode_step_q8(q, k, v, c, a)
    assert la.la_get_last_error() == la.LA_OK
    o_ref, c_ref, a_ref = oracle.decode_step_q8(host64(q), host64(k), host64(v), c_ref, a_ref)
    assert np.array_equal(_np(c), c_ref) and np.array_equal(_np(a), a_ref)
    assert per_head_rel_err(host64(o), o_ref, head_dims=1) <= TOL_O_BF16


@pytest.mark.parametrize("kind", ["fp32", "q8"])
@pytest.mark.parametrize("graphs", [True, False], ids=["graphs", "eager"])
def test_padded_decoder_against_oracle(kind, graphs):
    # live batch sizes moving across padding levels; each step's rows compared
    # with the oracle's slot decode; graphs and eager launches give the same
    num_slots, H, d = 40, 4, 128
    dec = PaddedDecoder(num_slots, H, d, state=kind, levels=(1, 4, 16, 32), use_graphs=graphs)
    init = _states((num_slots, H, d, d), seed=13, special_rows=False)
    for s in range(num_slots):
        dec.load_state(s, init[s].to(DEV))
    if kind == "fp32":
        ref_pool = init.numpy().astype(np.float64)
    else:
        ref_c, ref_a = oracle.state_quantize_q8(init.numpy())
    rng = np.random.default_rng(14)
    for step, n in enumerate([1, 3, 16, 5, 17, 32, 2, 4]):
        slots = rng.choice(num_slots, size=n, replace=False).tolist()
        q, k, v = inputs.decode_step_inputs(n, H, d, step + 1, device=DEV)
        o = dec.step(q, k, v, slots)
        torch.cuda.synchronize()
        assert la.la_get_last_error() == la.LA_OK
        if kind == "fp32":
            o_ref, ref_pool = oracle.decode_step_slots(host64(q), host64(k), host64(v), ref_pool, slots)
        else:
            o_ref, ref_c, ref_a = oracle.decode_step_q8(host64(q), host64(k), host64(v), ref_c, ref_a, slots)
        assert per_head_rel_err(host64(o), o_ref, head_dims=1) <= TOL_O_BF16, step
    if kind == "fp32":
        assert per_head_rel_err(host64(dec.pool), ref_pool) <= 1e-5
    else:
        assert np.array_equal(_np(dec.codes), ref_c) and np.array_equal(_np(dec.scales), ref_a)
    if graphs:
        assert dec.captured_levels() == (1, 4, 16, 32)
