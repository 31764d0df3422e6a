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


def round_like(ref: np.ndarray, dtype) -> np.ndarray:
    """Round fp64 values to ``dtype`` with round-to-nearest-even (as the GPU's
    final conversion does) and widen back to fp64."""
    return torch.from_numpy(np.ascontiguousarray(ref)).to(dtype).to(torch.float64).numpy()
