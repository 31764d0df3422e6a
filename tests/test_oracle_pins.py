"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Each pin states what fixes the expected value:
  * a hand-worked example from the definition (tests/golden/),
  * the associativity identity (QK^T)V = Q(K^T V) of the nabfollower page
    ("The Core Tech: Lightning Attention") in its masked consequences:
    quadratic == recurrent == block form, final state == K^T V (a numpy GEMM),
    last row == q_{N-1} K^T V,
  * special cases that reduce to textbook routines (d = 1 is a prefix sum,
    numpy.cumsum; N = 1 is (q.k) v),
  * exact brute force in Python integers on small ternary inputs,
  * the running-state semantics of the closing analogy of the same page:
    prefill(N) followed by one decode step equals prefill(N+1),
  * packing (section 4 of the futurefh page): varlen == dense per sequence,
  * the 8-bit state: a hand-worked example of its rounding rules and of one
    step (tests/golden/), integer-exact trajectories, and the fp64 recurrence
    within the error bound the rounding rules give,
  * decode over a slot pool: padding rows touch nothing, live rows equal the
    dense step on their own slot.

``test_pins_catch_planted_mistakes`` compiles altered copies of oracle.c (a
dropped diagonal, a transposed operand, a wrong sign, ...) and checks that every
one of them fails at least one pin, so the pins are strong enough to trust.
"""
from __future__ import annotations

import json
import os
import tempfile

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


# ----------------------------------------------------------------------------
# pins, each a function of one compiled oracle
# ----------------------------------------------------------------------------

def pin_golden(orc):
    g = json.load(open(os.path.join(GOLDEN, "worked_example_n3_d2.json")))
    q = np.array(g["q"], float)[None]
    k = np.array(g["k"], float)[None]
    v = np.array(g["v"], float)[None]
    o_ref = np.array(g["o"], float)
    s_ref = np.array(g["state"], float)
    assert np.array_equal(orc.prefill_quadratic(q, k, v)[0], o_ref)
    o, s = orc.prefill_recurrent(q, k, v)
    assert np.array_equal(o[0], o_ref) and np.array_equal(s[0], s_ref)
    for blk in (1, 2, 3, 4):
        o, s = orc.prefill_blockwise(q, k, v, blk)
        assert np.array_equal(o[0], o_ref) and np.array_equal(s[0], s_ref)


def pin_forms_agree(orc):
    r = _rng(1)
    for (BH, N, d) in ((3, 67, 8), (2, 130, 16)):
        q, k, v = (r.standard_normal((BH, N, d)) for _ in range(3))
        o_quad = orc.prefill_quadratic(q, k, v)
        o_rec, s_rec = orc.prefill_recurrent(q, k, v)
        assert _rel(o_rec, o_quad) < 1e-12
        for blk in (1, 2, 3, 7, 16, 64, N, N + 5):
            o_blk, s_blk = orc.prefill_blockwise(q, k, v, blk)
            assert _rel(o_blk, o_quad) < 1e-12, blk
            assert _rel(s_blk, s_rec) < 1e-12, blk


def pin_state_is_KtV(orc):
    r = _rng(2)
    q, k, v = (r.standard_normal((2, 50, 12)) for _ in range(3))
    ktv = np.einsum("bnd,bne->bde", k, v)            # one GEMM per head (numpy)
    _, s_rec = orc.prefill_recurrent(q, k, v)
    _, s_blk = orc.prefill_blockwise(q, k, v, 8)
    assert _rel(s_rec, ktv) < 1e-12
    assert _rel(s_blk, ktv) < 1e-12


def pin_last_row(orc):
    r = _rng(3)
    q, k, v = (r.standard_normal((2, 41, 10)) for _ in range(3))
    ktv = np.einsum("bnd,bne->bde", k, v)
    want = np.einsum("bd,bde->be", q[:, -1], ktv)     # q_{N-1} (K^T V)
    for o in (orc.prefill_quadratic(q, k, v), orc.prefill_recurrent(q, k, v)[0],
              orc.prefill_blockwise(q, k, v, 16)[0]):
        assert _rel(o[:, -1], want) < 1e-12


def pin_d1_prefix_sum(orc):
    r = _rng(4)
    q, k, v = (r.standard_normal((3, 90, 1)) for _ in range(3))
    want = q[..., 0] * np.cumsum(k[..., 0] * v[..., 0], axis=1)   # textbook prefix sum
    for o in (orc.prefill_quadratic(q, k, v), orc.prefill_recurrent(q, k, v)[0],
              orc.prefill_blockwise(q, k, v, 7)[0]):
        assert _rel(o[..., 0], want) < 1e-12


def pin_N1(orc):
    r = _rng(5)
    q, k, v = (r.standard_normal((4, 1, 9)) for _ in range(3))
    want = np.sum(q * k, axis=-1, keepdims=True) * v      # (q.k) v
    for o in (orc.prefill_quadratic(q, k, v), orc.prefill_recurrent(q, k, v)[0],
              orc.prefill_blockwise(q, k, v, 4)[0]):
        assert _rel(o, want) < 1e-13


def _brute_int(q, k, v):
    """Exact causal linear attention in Python integers (one head)."""
    N, d = len(q), len(q[0])
    o = [[0] * d for _ in range(N)]
    for t in range(N):
        for s in range(t + 1):
            sc = sum(q[t][c] * k[s][c] for c in range(d))
            for j in range(d):
                o[t][j] += sc * v[s][j]
    st = [[sum(k[s][i] * v[s][j] for s in range(N)) for j in range(d)] for i in range(d)]
    return o, st


def pin_ternary_bruteforce(orc):
    r = _rng(6)
    for (N, d) in ((1, 3), (5, 2), (23, 6), (40, 4)):
        q, k, v = (r.integers(-1, 2, (N, d)) for _ in range(3))
        o_ref, s_ref = _brute_int(q.tolist(), k.tolist(), v.tolist())
        o_ref = np.array(o_ref, float)[None]
        s_ref = np.array(s_ref, float)[None]
        qf, kf, vf = (x[None].astype(float) for x in (q, k, v))
        assert np.array_equal(orc.prefill_quadratic(qf, kf, vf), o_ref)
        o, s = orc.prefill_recurrent(qf, kf, vf)
        assert np.array_equal(o, o_ref) and np.array_equal(s, s_ref)
        for blk in (1, 3, 8):
            o, s = orc.prefill_blockwise(qf, kf, vf, blk)
            assert np.array_equal(o, o_ref) and np.array_equal(s, s_ref)


def pin_state_in(orc):
    """Running from the state of a prefix continues the full sequence."""
    r = _rng(7)
    q, k, v = (r.standard_normal((2, 60, 8)) for _ in range(3))
    o_full, s_full = orc.prefill_quadratic(q, k, v), np.einsum("bnd,bne->bde", k, v)
    m = 23
    s_pre = np.einsum("bnd,bne->bde", k[:, :m], v[:, :m])
    o_tail, s_tail = orc.prefill_recurrent(q[:, m:], k[:, m:], v[:, m:], state_in=s_pre)
    assert _rel(o_tail, o_full[:, m:]) < 1e-12
    assert _rel(s_tail, s_full) < 1e-12


def pin_decode(orc):
    r = _rng(8)
    q, k, v = (r.standard_normal((3, 31, 8)) for _ in range(3))
    _, s_prev = orc.prefill_recurrent(q[:, :-1], k[:, :-1], v[:, :-1])
    o1, s1 = orc.decode_step(q[:, -1], k[:, -1], v[:, -1], s_prev)
    o_full = orc.prefill_quadratic(q, k, v)
    assert _rel(o1, o_full[:, -1]) < 1e-12
    assert _rel(s1, np.einsum("bnd,bne->bde", k, v)) < 1e-12
    # closed form of one step: o = q (S + k^T v)
    want = np.einsum("bd,bde->be", q[:, -1], s_prev + np.einsum("bd,be->bde", k[:, -1], v[:, -1]))
    assert _rel(o1, want) < 1e-12


def pin_varlen(orc):
    r = _rng(9)
    lens = [5, 0, 17, 1, 30]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    H, T, d = 3, int(cu[-1]), 6
    q, k, v = (r.integers(-1, 2, (H, T, d)).astype(float) for _ in range(3))
    o, st = orc.prefill_varlen(q, k, v, cu)
    for j, n in enumerate(lens):
        a, b = cu[j], cu[j + 1]
        for h in range(H):
            if n == 0:
                assert not np.any(st[j, h])
                continue
            o_ref, s_ref = _brute_int(q[h, a:b].astype(int).tolist(), k[h, a:b].astype(int).tolist(),
                                     v[h, a:b].astype(int).tolist())
            assert np.array_equal(o[h, a:b], np.array(o_ref, float))
            assert np.array_equal(st[j, h], np.array(s_ref, float))
    o2, st2 = orc.prefill_varlen(q, k, v, cu, heads=[2])
    assert np.array_equal(o2[2], o[2]) and not np.any(o2[:2])
    assert np.array_equal(st2[:, 2], st[:, 2])


def pin_backward_finite_differences(orc):
    """The gradients of L = sum(dO * o) agree with central differences of the
    forward (quadratic) form: a check that does not use the gradient formulas."""
    rng = np.random.default_rng(17)
    BH, N, d = 2, 5, 3
    q, k, v, do = (rng.standard_normal((BH, N, d)) for _ in range(4))
    dq, dk, dv = orc.prefill_backward(q, k, v, do)
    h = 1e-6

    def loss(qq, kk, vv):
        return float(np.sum(do * orc.prefill_quadratic(qq, kk, vv)))

    for x, g, which in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = [q, k, v]
            args_m = [q, k, v]
            args_p[which], args_m[which] = xp, xm
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        assert np.allclose(g, num, rtol=0, atol=1e-6), which


def pin_backward_d1_sums(orc):
    """d = 1: dq_t = k-weighted prefix sum, dk_s and dv_s suffix sums (closed form)."""
    rng = np.random.default_rng(3)
    q, k, v, do = (rng.standard_normal((1, 7, 1)) for _ in range(4))
    dq, dk, dv = orc.prefill_backward(q, k, v, do)
    qf, kf, vf, gf = (x[0, :, 0] for x in (q, k, v, do))
    assert np.allclose(dq[0, :, 0], gf * np.cumsum(vf * kf), atol=1e-12)
    suffix_gq = np.cumsum((gf * qf)[::-1])[::-1]
    assert np.allclose(dk[0, :, 0], vf * suffix_gq, atol=1e-12)
    assert np.allclose(dv[0, :, 0], kf * suffix_gq, atol=1e-12)


def pin_zero_keys_and_unmasked_identity(orc):
    """k = 0 gives o = 0 and a zero state in every form; and the associativity
    the block form rests on, (Q K^T) V = Q (K^T V), holds for plain numpy
    products, while the causal oracle differs from the unmasked product (the
    mask matters)."""
    r = _rng(24)
    q, v = r.standard_normal((2, 9, 5)), r.standard_normal((2, 9, 5))
    k = np.zeros((2, 9, 5))
    assert not np.any(orc.prefill_quadratic(q, k, v))
    o, s = orc.prefill_recurrent(q, k, v)
    assert not np.any(o) and not np.any(s)
    for blk in (1, 4):
        o, s = orc.prefill_blockwise(q, k, v, blk)
        assert not np.any(o) and not np.any(s)
    k = r.standard_normal((2, 9, 5))
    left = np.einsum("bnd,bmd,bme->bne", q, k, v)
    right = np.einsum("bnd,bde->bne", q, np.einsum("bmd,bme->bde", k, v))
    assert _rel(left, right) < 1e-12
    causal = orc.prefill_quadratic(q, k, v)
    assert _rel(causal[:, -1], left[:, -1]) < 1e-12      # the last row sees every key
    assert _rel(causal[:, 0], left[:, 0]) > 1e-3          # the first row sees only itself


def pin_q8_golden(orc):
    g = json.load(open(os.path.join(GOLDEN, "q8_state_worked_example.json")))
    for row in g["quantize"]:
        c, a = orc.state_quantize_q8(np.array([row["x"]], np.float32))
        assert c[0].tolist() == row["codes"], row["why"]
        assert a[0] == np.float32(row["scale"]), row["why"]
        back = orc.state_dequantize_q8(c, a)
        assert np.array_equal(back[0], np.array(row["codes"], np.float32) * np.float32(row["scale"]))
    st = g["step"]
    o, c, a = orc.decode_step_q8(np.array([st["q"]], np.float32), np.array([st["k"]], np.float32),
                                 np.array([st["v"]], np.float32), np.array([st["codes"]], np.int8),
                                 np.array([st["scales"]], np.float32))
    assert o[0].tolist() == st["o"]
    assert c[0].tolist() == st["codes_out"]
    assert a[0].tolist() == [float(np.float32(x)) for x in st["scales_out"]]


def pin_q8_rows_becoming_zero(orc):
    """Worked by hand: a row that a step cancels exactly, and a row whose values
    fall below 2^-100, are both stored as zero rows: codes 0 and scale 0 (not
    the scale they had before)."""
    a1 = np.float32(2.0 ** -108) / np.float32(127)           # row 1 dequantises to ~2^-108
    codes = np.array([[[1, 2, 0, -3], [127, 0, 0, 0], [0, 0, 0, 0], [0, 0, 0, 0]]], np.int8)
    scales = np.array([[1.0, a1, 0.0, 0.0]], np.float32)
    q = np.array([[1.0, 1.0, 1.0, 1.0]], np.float32)
    k = np.array([[-1.0, 0.0, 0.0, 0.0]], np.float32)        # row 0: s = c - v = 0
    v = np.array([[1.0, 2.0, 0.0, -3.0]], np.float32)
    o, c2, a2 = orc.decode_step_q8(q, k, v, codes, scales)
    assert not np.any(c2) and not np.any(a2)
    tiny = float(np.float32(127) * a1)                       # row 1's first value, kept in o
    assert o[0].tolist() == [tiny, 0.0, 0.0, 0.0]


def pin_q8_threshold_and_single_rounding(orc):
    """Worked by hand.  The zero-row cut is strict and sits at 2^-100: rows with
    largest magnitude 2^-100 and 2^-95 quantise normally (code 127, scale
    m / 127), one at 2^-101 is stored as zero.  The step's update is one fused
    multiply-add: with k = v = 1 + 2^-12 and a dequantised -1, k v - 1 =
    2^-11 + 2^-24 exactly, which a separately rounded product would lose
    (fl(k v) = 1 + 2^-11, a tie rounded to even); the row's only non-zero value
    then sets the scale (2^-11 + 2^-24) / 127."""
    for e, zero in ((-100, False), (-95, False), (-101, True)):
        x = np.zeros((1, 8), np.float32)
        x[0, 3] = np.float32(2.0 ** e)
        c, a = orc.state_quantize_q8(x)
        if zero:
            assert not np.any(c) and a[0] == 0
        else:
            assert c[0].tolist() == [0, 0, 0, 127, 0, 0, 0, 0]
            assert a[0] == np.float32(2.0 ** e) / np.float32(127)
    d = 2
    codes = np.array([[[-1, 0], [0, 0]]], np.int8)
    scales = np.array([[1.0, 0.0]], np.float32)
    w = np.float32(1.0 + 2.0 ** -12)
    q = np.array([[1.0, 0.0]], np.float32)
    k = np.array([[w, 0.0]], np.float32)
    v = np.array([[w, 0.0]], np.float32)
    o, c2, a2 = orc.decode_step_q8(q, k, v, codes, scales)
    s00 = 2.0 ** -11 + 2.0 ** -24
    assert o[0].tolist() == [s00, 0.0]
    assert c2[0].tolist() == [[127, 0], [0, 0]]
    assert a2[0, 0] == np.float32(s00) / np.float32(127) and a2[0, 1] == 0
    assert d == codes.shape[-1]


def pin_q8_integer_trajectory(orc):
    """Rows whose largest magnitude stays exactly 127 have scale 1, so codes are
    the state itself: one-hot keys and small integer values keep every step
    exact, and the result is brute force in Python integers."""
    rng = _rng(21)
    BH, d, T = 2, 8, 30
    S = rng.integers(-60, 61, (BH, d, d))
    S[:, :, 0] = 127                       # column 0 holds each row's maximum ...
    codes = S.astype(np.int8)
    scales = np.ones((BH, d), np.float32)
    for t in range(T):
        q = rng.integers(-3, 4, (BH, d))
        k = np.zeros((BH, d), int)
        r = rng.integers(0, d, BH)
        k[np.arange(BH), r] = rng.choice([-1, 1], BH)
        v = rng.integers(-2, 3, (BH, d))
        v[:, 0] = 0                        # ... and no step changes it
        for b in range(BH):                # keep the updated row inside [-127, 127]
            row = S[b, r[b]] + k[b, r[b]] * v[b]
            v[b] = np.where(np.abs(row) > 120, 0, v[b])
        S = S + np.einsum("bi,bj->bij", k, v)
        o_ref = np.einsum("bi,bij->bj", q, S)
        o, codes, scales = orc.decode_step_q8(q.astype(np.float32), k.astype(np.float32),
                                              v.astype(np.float32), codes, scales)
        assert np.array_equal(codes.astype(int), S), t
        assert np.all(scales == 1.0)
        assert np.array_equal(o, o_ref.astype(float)), t


def pin_q8_within_rounding_bound(orc):
    """Against the fp64 recurrence started from the same dequantised state:
    each step adds at most half a quantisation step (a/2) plus fp32 rounding
    (2^-20 of the row's largest magnitude) to every element of a row."""
    rng = _rng(22)
    BH, d, T = 3, 16, 48
    c, a = orc.state_quantize_q8(rng.standard_normal((BH, d, d)).astype(np.float32))
    exact = orc.state_dequantize_q8(c, a).astype(np.float64)
    bound = np.zeros((BH, d))
    for t in range(T):
        q, k, v = (rng.standard_normal((BH, d)).astype(np.float32) for _ in range(3))
        o, c, a_new = orc.decode_step_q8(q, k, v, c, a)
        exact = exact + np.einsum("bi,bj->bij", k.astype(float), v.astype(float))
        m = 127.0 * a_new.astype(float)
        step_bound = bound + 2.0 ** -20 * m   # s before quantisation
        o_ref = np.einsum("bi,bij->bj", q.astype(float), exact)
        o_bound = np.einsum("bi,bi->b", np.abs(q.astype(float)), step_bound)[:, None]
        assert np.all(np.abs(o - o_ref) <= o_bound + 1e-9), t
        bound = bound + 0.5 * a_new.astype(float) + 2.0 ** -20 * m
        got = orc.state_dequantize_q8(c, a_new).astype(np.float64)
        assert np.all(np.abs(got - exact) <= bound[:, :, None] + 1e-12), t
        a = a_new
    assert np.max(bound) < 0.2 * np.max(np.abs(exact))   # and the bound is not vacuous


def pin_decode_slots(orc):
    """Padding rows (negative slot) give zero output and touch no state; every
    live row equals the dense step on its own slot's state."""
    rng = _rng(23)
    H, d, n_slots = 2, 6, 5
    pool = rng.standard_normal((n_slots, H, d, d))
    slots = [3, -1, 0, 4]
    q, k, v = (rng.standard_normal((len(slots), H, d)) for _ in range(3))
    o, pool2 = orc.decode_step_slots(q, k, v, pool, slots)
    assert not np.any(o[1])
    assert np.array_equal(pool2[1], pool[1]) and np.array_equal(pool2[2], pool[2])
    for b, s in enumerate(slots):
        if s < 0:
            continue
        want = np.einsum("hd,hde->he", q[b], pool[s] + np.einsum("hd,he->hde", k[b], v[b]))
        assert _rel(o[b], want) < 1e-12
        assert _rel(pool2[s], pool[s] + np.einsum("hd,he->hde", k[b], v[b])) < 1e-12
    # the 8-bit form over the same slots: padding rows untouched as well
    c, a = orc.state_quantize_q8(pool.astype(np.float32))
    qf, kf, vf = (x.astype(np.float32) for x in (q, k, v))
    o8, c2, a2 = orc.decode_step_q8(qf, kf, vf, c, a, slots)
    assert not np.any(o8[1]) and np.array_equal(c2[1], c[1]) and np.array_equal(a2[2], a[2])
    o_dense, c_dense, a_dense = orc.decode_step_q8(qf[0], kf[0], vf[0], c[3], a[3])
    assert np.array_equal(o8[0], o_dense) and np.array_equal(c2[3], c_dense)


PINS = [pin_golden, pin_forms_agree, pin_state_is_KtV, pin_last_row, pin_d1_prefix_sum, pin_N1,
        pin_ternary_bruteforce, pin_state_in, pin_decode, pin_varlen, pin_backward_finite_differences,
        pin_backward_d1_sums, pin_zero_keys_and_unmasked_identity, pin_q8_golden, pin_q8_rows_becoming_zero, pin_q8_threshold_and_single_rounding, pin_q8_integer_trajectory, pin_q8_within_rounding_bound,
        pin_decode_slots]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(oracle._get())


# ----------------------------------------------------------------------------
# planted mistakes: every altered oracle must fail at least one pin
# ----------------------------------------------------------------------------

MUTANTS = {
    "quadratic_drops_diagonal": ("for (long s = 0; s <= t; ++s)", "for (long s = 0; s < t; ++s)"),
    "quadratic_wrong_v_index": ("O[t * d + j] += score * V[s * d + j]",
                                "O[t * d + j] += score * V[t * d + j]"),
    "recurrent_transposed_update": ("S[i * d + j] += K[t * d + i] * V[t * d + j]",
                                    "S[i * d + j] += K[t * d + j] * V[t * d + i]"),
    "recurrent_transposed_read": ("acc += Q[t * d + i] * S[i * d + j]",
                                  "acc += Q[t * d + i] * S[j * d + i]"),
    "recurrent_ignores_state_in": ("if (state_in)\n", "if (0 && state_in)\n"),
    "blockwise_drops_diagonal": ("if (c <= r)", "if (c < r)"),
    "blockwise_inter_sign": ("= intra + inter;", "= intra - inter;"),
    "blockwise_state_not_accumulated": ("S[x * d + j] += acc;", "S[x * d + j] = acc;"),
    "decode_transposed_update": ("Sb[i * d + j] += kb[i] * vb[j]", "Sb[i * d + j] += kb[j] * vb[i]"),
    "decode_reads_before_update": (
        "        for (long i = 0; i < d; ++i)\n            for (long j = 0; j < d; ++j) Sb[i * d + j] += kb[i] * vb[j];\n",
        ""),
    "varlen_skips_first_token": ("long t0 = cu_seqlens[j], t1", "long t0 = cu_seqlens[j] + 1, t1"),
    "varlen_no_state_reset_shared_offset": ("O[t * d + c] = acc;", "O[t * d + c] = acc + (t == t0);"),
    "backward_dq_uses_q": ("DQ[t * d + c] += gv * K[s * d + c];", "DQ[t * d + c] += gv * Q[s * d + c];"),
    "backward_dk_wrong_token": ("DK[s * d + c] += gv * Q[t * d + c];", "DK[s * d + c] += gv * Q[s * d + c];"),
    "backward_drops_diagonal": ("for (long s = 0; s <= t; s++) {", "for (long s = 0; s < t; s++) {"),
    "q8_truncates": ("rintf(x[j] * inv)", "truncf(x[j] * inv)"),
    "q8_signed_max": ("const float ax = fabsf(x[j]);", "const float ax = x[j];"),
    "q8_no_small_row_cut": ("if (m < 0x1p-100f) {", "if (m <= 0.0f) {"),
    "q8_transposed_update": ("fmaf(kb[i], vb[j], deq)", "fmaf(kb[j], vb[i], deq)"),
    "q8_column_scale": ("(float)cb[i * d + j] * ab[i]", "(float)cb[i * d + j] * ab[j]"),
    "q8_dequantize_column_scale": ("S[r * d + j] = (float)codes[r * d + j] * scales[r];",
                                   "S[r * d + j] = (float)codes[r * d + j] * scales[j % rows];"),
    "q8_zero_row_keeps_old_scale": ("        *a = 0.0f;\n        for (long j = 0; j < d; ++j) c[j] = 0;",
                                    "        for (long j = 0; j < d; ++j) c[j] = 0;"),
    "varlen_state_layout_transposed": ("memcpy(state_out + (j * H + h) * d * d, S,",
                                       "memcpy(state_out + (h * num_seqs + j) * d * d, S,"),
    "varlen_head_list_ignored": ("long h = head_list ? head_list[item / num_seqs] : item / num_seqs;",
                                 "long h = item / num_seqs;"),
    "varlen_reads_other_head_k": ("const double* K = k + h * T * d;",
                                  "const double* K = k + ((h + 1) % H) * T * d;"),
    "blockwise_intra_uses_previous_block_v": (
        "intra += P[r * blk + c] * V[(b0 + c) * d + j];",
        "intra += P[r * blk + c] * V[((b0 >= blk ? b0 - blk : b0) + c) * d + j];"),
    "quadratic_score_uses_q_twice": ("score += Q[t * d + c] * K[s * d + c];",
                                     "score += Q[t * d + c] * Q[s * d + c];"),
    "backward_dv_uses_wrong_score": ("DV[s * d + c] += qk * G[t * d + c];",
                                     "DV[s * d + c] += gv * G[t * d + c];"),
    "q8_threshold_too_high": ("if (m < 0x1p-100f) {", "if (m < 0x1p-90f) {"),
    "q8_update_rounded_twice": ("s[i * d + j] = fmaf(kb[i], vb[j], deq);", "s[i * d + j] = kb[i] * vb[j] + deq;"),
    "q8_reads_before_update": ("acc += (double)qb[i] * (double)s[i * d + j];",
                               "acc += (double)qb[i] * (double)cb[i * d + j] * ab[i];"),
}


def _pins_fail(orc) -> list:
    failed = []
    for p in PINS:
        try:
            p(orc)
        except AssertionError:
            failed.append(p.__name__)
    return failed


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistakes(name):
    src = open(oracle.SOURCE).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, "mutation anchor must occur exactly once"
    if name == "decode_reads_before_update":
        # move the state update after the read: o = q S_old, then S += k^T v
        read_end = ("            for (long i = 0; i < d; ++i) acc += qb[i] * Sb[i * d + j];\n"
                    "            o[bh * d + j] = acc;\n        }\n")
        assert src.count(read_end) == 1
        mutated = src.replace(old, "").replace(read_end, read_end + old)
    else:
        mutated = src.replace(old, new)
    with tempfile.TemporaryDirectory() as td:
        c_path = os.path.join(td, "mut.c")
        open(c_path, "w").write(mutated)
        orc = oracle.Oracle(oracle.compile_source(c_path, os.path.join(td, "libmut.so")))
        failed = _pins_fail(orc)
    assert failed, f"planted mistake {name} passed every pin"
