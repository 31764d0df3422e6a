"""Helpers shared by the GPU parity tests (comparison metrics, host copies)."""
import numpy as np
import torch

# Tolerances of the parity bar: per head, max |got - ref| / max |ref|.
TOL_O_F32 = 1e-4
TOL_O_BF16 = 2e-2
TOL_STATE = 1e-3


def host64(t: torch.Tensor) -> np.ndarray:
    """Exact fp64 copy of a (bf16 / fp32) tensor's values on the host."""
    return t.detach().to("cpu").to(torch.float64).numpy()


def per_head_rel_err(got, ref, head_dims=2) -> float:
    """max over heads of max|got-ref| / max|ref|; a head is the trailing
    ``head_dims`` axes.  A head whose reference is all zero must match exactly."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    n = int(np.prod(ref.shape[-head_dims:])) if ref.size else 1
    g = got.reshape(-1, n)
    r = ref.reshape(-1, n)
    worst = 0.0
    for i in range(r.shape[0]):
        scale = np.max(np.abs(r[i])) if r.shape[1] else 0.0
        diff = np.max(np.abs(g[i] - r[i])) if r.shape[1] else 0.0
        if scale == 0.0:
            if diff != 0.0:
                return float("inf")
            continue
        worst = max(worst, diff / scale)
    return worst


def per_seq_head_rel_err(got, ref, cu_seqlens) -> float:
    """The parity metric for packed sequences: each (sequence, head) is its own
    attention problem, so its error is normalised by its own largest |ref|.
    got, ref are [H, T, d]; cu_seqlens is [S + 1] (host or device).  Returns
    max over (sequence, head) of max|got - ref| / max|ref| over that
    sequence's rows of that head; a sequence whose reference is all zero must
    match exactly.  Empty sequences contribute nothing."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape and ref.ndim == 3, (got.shape, ref.shape)
    cu = np.asarray(cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens).astype(np.int64)
    assert cu[0] == 0 and cu[-1] == ref.shape[1], (cu[0], cu[-1], ref.shape)
    worst = 0.0
    for a, b in zip(cu[:-1], cu[1:]):
        if b == a:
            continue
        r = ref[:, a:b].reshape(ref.shape[0], -1)
        d = np.abs(got[:, a:b].reshape(ref.shape[0], -1) - r).max(axis=1)
        scale = np.abs(r).max(axis=1)
        if np.any(d[scale == 0.0] != 0.0):
            return float("inf")
        nz = scale > 0.0
        if np.any(nz):
            worst = max(worst, float(np.max(d[nz] / scale[nz])))
    return worst


def round_like(ref: np.ndarray, dtype) -> np.ndarray:
    """Round fp64 values to ``dtype`` with round-to-nearest-even (as the GPU's
    final conversion does) and widen back to fp64."""
    return torch.from_numpy(np.ascontiguousarray(ref)).to(dtype).to(torch.float64).numpy()


def grads_via_recurrent(orc, q, k, v, do):
    """Gradients of sum(dO * o) from the oracle's recurrent (O(N d^2)) form:
    dq is the causal form of (dO, v, k); dk and dv are the anti-causal forms
    of (v, dO, q) and (k, q, dO), i.e. causal forms of the token-reversed
    sequences, reversed back.  For long sequences, where the oracle's own
    (quadratic) backward is too slow; pinned against it on small inputs."""
    def rev(x):
        return np.ascontiguousarray(np.asarray(x)[..., ::-1, :])
    dq, _ = orc.prefill_recurrent(do, v, k)
    dk_r, _ = orc.prefill_recurrent(rev(v), rev(do), rev(q))
    dv_r, _ = orc.prefill_recurrent(rev(k), rev(q), rev(do))
    return dq, rev(dk_r), rev(dv_r)

