"""The parity metrics themselves (host only): the packed metric holds every
(sequence, head) to the bar on its own scale, so an error in a short sequence
is not hidden by a long sequence's larger outputs."""
import numpy as np

import oracle
from _util import grads_via_recurrent, per_head_rel_err, per_seq_head_rel_err


def test_packed_metric_normalises_each_sequence_by_its_own_scale():
    rng = np.random.default_rng(0)
    H, d = 2, 4
    lens = [3, 0, 40, 5]
    cu = np.concatenate([[0], np.cumsum(lens)])
    ref = rng.standard_normal((H, cu[-1], d))
    ref[:, cu[2]:cu[3]] *= 10.0          # the long sequence has 10x larger outputs
    got = ref.copy()
    got[1, 0, 0] += 0.05 * np.abs(ref[1, :3]).max()   # 5% error in the first, short sequence
    assert per_head_rel_err(got, ref) < 0.02           # hidden by the whole-head scale
    e = per_seq_head_rel_err(got, ref, cu)
    assert abs(e - 0.05) < 1e-12                       # seen on its own scale


def test_packed_metric_zero_reference_must_match_exactly():
    ref = np.zeros((1, 6, 2))
    got = ref.copy()
    cu = np.array([0, 2, 6])
    assert per_seq_head_rel_err(got, ref, cu) == 0.0
    got[0, 1, 0] = 1e-30
    assert per_seq_head_rel_err(got, ref, cu) == float("inf")


def test_packed_metric_is_the_dense_metric_for_one_sequence():
    rng = np.random.default_rng(1)
    ref = rng.standard_normal((3, 17, 8))
    got = ref + 1e-3 * rng.standard_normal(ref.shape)
    cu = np.array([0, 17])
    assert per_seq_head_rel_err(got, ref, cu) == per_head_rel_err(got, ref)


def test_recurrent_gradient_reference_equals_the_oracle_backward():
    # the long-sequence gradient reference of the GPU tests: three recurrent
    # forms (two on reversed tokens) equal the oracle's backward, which is
    # pinned by finite differences
    rng = np.random.default_rng(8)
    q, k, v, do = (rng.standard_normal((2, 3, 37, 8)) for _ in range(4))
    ref = oracle.prefill_backward(q, k, v, do)
    got = grads_via_recurrent(oracle._get(), q, k, v, do)
    for g, r in zip(got, ref):
        np.testing.assert_allclose(g, r, rtol=0, atol=1e-11)
