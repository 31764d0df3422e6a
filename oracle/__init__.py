"""fp64 CPU oracle for causal linear attention (Lightning Attention).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this package.  The product
path (``linear_attention_13_b200``) never imports it, and it imports nothing
from the product: the two share only the seeded input generators, which hold
none of the method's arithmetic.

The arithmetic lives in ``oracle.c`` (plain loops, fp64, OpenMP over
independent heads); this module only marshals numpy arrays into it.  Every
function cites the passage it follows in ``oracle.c``:

* ``prefill_quadratic``  -- o_t = sum_{s<=t} (q_t.k_s) v_s, the masked left
  product of section 1 of "MiniMax-01技術報告解讀以及與DeepSeek-V3對比".
* ``prefill_recurrent``  -- S += k_t^T v_t ; o_t = q_t S, the fixed-size state
  of the closing analogy of "MiniMax M2.1 (the 'linear' revolution)".
* ``prefill_blockwise``  -- intra-block left product + inter-block right
  product, section 1 of the futurefh page.
* ``decode_step``        -- one recurrent step (update, then read).
* ``prefill_varlen``     -- recurrent form per packed sequence, state reset.
* ``decode_step_slots``  -- decode over a pool of states addressed by slot id,
  negative ids being padding rows (the multi-level padding of section 3 of
  the futurefh page).
* ``state_quantize_q8`` / ``state_dequantize_q8`` / ``decode_step_q8`` -- the
  8-bit state (int8 codes, one fp32 scale per key row) that the yuliangy.com
  digest's 8-bit quantisation is read as; decisions taken in fp32.

Pins (what checks this oracle against something other than itself) live in
``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")


def compile_source(src_path: str, out_path: str) -> str:
    """Compile a C source of the oracle into a shared library with gcc."""
    tmp = out_path + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", src_path, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out_path)
    return out_path


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (-O2, OpenMP) if missing or stale."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(SOURCE)):
        return _LIB_PATH
    return compile_source(SOURCE, _LIB_PATH)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _f32_exact(a) -> np.ndarray:
    """fp32 copy that must not round (the 8-bit state's inputs are fp32 or bf16)."""
    x = np.asarray(a, dtype=np.float64)
    y = _f32(x)
    if not np.array_equal(y.astype(np.float64), x):
        raise ValueError("inputs of the 8-bit decode step must be exact in fp32")
    return y


def _fptr(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_float))


def _cptr(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_byte))


def _shape_bhnd(q):
    q = np.asarray(q)
    if q.ndim == 4:
        B, H, N, d = q.shape
        return B * H, N, d
    if q.ndim == 3:
        BH, N, d = q.shape
        return BH, N, d
    raise ValueError("q must be [B,H,N,d] or [BH,N,d]")


def _slot_rows(slots, num_slots):
    slots = np.asarray(slots, dtype=np.int64).reshape(-1)
    if np.any(slots >= num_slots):
        raise ValueError("slot id out of range")
    live = slots[slots >= 0]
    if len(np.unique(live)) != len(live):
        raise ValueError("a slot may appear once per batch")
    return slots


class Oracle:
    """ctypes view of one compiled copy of oracle.c (the default one, or a
    deliberately altered copy built by the pin-strength tests)."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int)
        L = ctypes.c_long
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_prefill_quadratic.argtypes = [dp, dp, dp, dp, L, L, L]
        lib.oracle_prefill_recurrent.argtypes = [dp, dp, dp, dp, dp, dp, L, L, L]
        lib.oracle_prefill_blockwise.argtypes = [dp, dp, dp, dp, dp, L, L, L, L]
        lib.oracle_decode_step.argtypes = [dp, dp, dp, dp, dp, L, L]
        lib.oracle_prefill_varlen.argtypes = [dp, dp, dp, ip, L, L, L, L, dp, dp, ip, L]
        lib.oracle_prefill_backward.argtypes = [dp, dp, dp, dp, dp, dp, dp, L, L, L]
        fp = ctypes.POINTER(ctypes.c_float)
        cp = ctypes.POINTER(ctypes.c_byte)
        lib.oracle_state_quantize_q8.argtypes = [fp, cp, fp, L, L]
        lib.oracle_state_dequantize_q8.argtypes = [cp, fp, fp, L, L]
        lib.oracle_decode_step_q8.argtypes = [fp, fp, fp, cp, fp, dp, L, L]
        for f in ("oracle_prefill_quadratic", "oracle_prefill_recurrent",
                  "oracle_prefill_blockwise", "oracle_decode_step", "oracle_prefill_varlen",
                  "oracle_state_quantize_q8", "oracle_state_dequantize_q8", "oracle_decode_step_q8"):
            getattr(lib, f).restype = None
        self.lib = lib

    def num_threads(self) -> int:
        """OpenMP threads the oracle uses (all host cores unless OMP_NUM_THREADS)."""
        return int(self.lib.oracle_num_threads())

    def prefill_quadratic(self, q, k, v) -> np.ndarray:
        """Quadratic masked form o_t = sum_{s<=t}(q_t.k_s)v_s; returns o (fp64)."""
        BH, N, d = _shape_bhnd(q)
        q, k, v = _f64(q), _f64(k), _f64(v)
        o = np.zeros(q.shape, dtype=np.float64)
        self.lib.oracle_prefill_quadratic(_ptr(q), _ptr(k), _ptr(v), _ptr(o), BH, N, d)
        return o

    def prefill_recurrent(self, q, k, v, state_in=None):
        """Recurrent form; returns (o, state_out) in fp64, state [..., d, d]."""
        BH, N, d = _shape_bhnd(q)
        q, k, v = _f64(q), _f64(k), _f64(v)
        s_in = _f64(state_in) if state_in is not None else None
        o = np.zeros(q.shape, dtype=np.float64)
        st = np.zeros(q.shape[:-2] + (d, d), dtype=np.float64)
        self.lib.oracle_prefill_recurrent(_ptr(q), _ptr(k), _ptr(v), _ptr(s_in), _ptr(o),
                                          _ptr(st), BH, N, d)
        return o, st

    def prefill_blockwise(self, q, k, v, blk: int):
        """Block form (intra left product + inter right product); returns (o, state)."""
        BH, N, d = _shape_bhnd(q)
        if blk < 1:
            raise ValueError("blk must be >= 1")
        q, k, v = _f64(q), _f64(k), _f64(v)
        o = np.zeros(q.shape, dtype=np.float64)
        st = np.zeros(q.shape[:-2] + (d, d), dtype=np.float64)
        self.lib.oracle_prefill_blockwise(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(st),
                                          BH, N, d, blk)
        return o, st

    def prefill_backward(self, q, k, v, do):
        """Gradients (dq, dk, dv) of sum(dO * o) for the causal form (fp64)."""
        BH, N, d = _shape_bhnd(q)
        q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
        dq, dk, dv = (np.zeros(q.shape, dtype=np.float64) for _ in range(3))
        self.lib.oracle_prefill_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(dq), _ptr(dk),
                                         _ptr(dv), BH, N, d)
        return dq, dk, dv

    def decode_step(self, q, k, v, state):
        """One decode step; returns (o, new_state), the input state untouched."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        S = _f64(state).copy()
        d = q.shape[-1]
        BH = int(np.prod(q.shape[:-1]))
        o = np.zeros(q.shape, dtype=np.float64)
        self.lib.oracle_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(S), _ptr(o), BH, d)
        return o, S

    def state_quantize_q8(self, state):
        """fp32 states [..., d, d] -> (int8 codes [..., d, d], fp32 scales [..., d])."""
        S = _f32(state)
        d = S.shape[-1]
        rows = S.size // d
        codes = np.zeros(S.shape, dtype=np.int8)
        scales = np.zeros(S.shape[:-1], dtype=np.float32)
        self.lib.oracle_state_quantize_q8(_fptr(S), _cptr(codes), _fptr(scales), rows, d)
        return codes, scales

    def state_dequantize_q8(self, codes, scales):
        """(codes, scales) -> fp32 states, S_ij = c_ij * a_i."""
        c = np.ascontiguousarray(codes, dtype=np.int8)
        a = _f32(scales)
        d = c.shape[-1]
        S = np.zeros(c.shape, dtype=np.float32)
        self.lib.oracle_state_dequantize_q8(_cptr(c), _fptr(a), _fptr(S), c.size // d, d)
        return S

    def decode_step_slots(self, q, k, v, pool, slots):
        """Decode step for a batch whose row b uses state pool[slots[b]].

        q, k, v: [B, H, d]; pool: [num_slots, H, d, d]; a negative slot marks a
        padding row, whose output is zero and which touches no state.  Returns
        (o [B, H, d], pool') in fp64; the input pool is untouched.  Each live row
        is ``decode_step`` applied to its own slot's state."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        pool = _f64(pool).copy()
        slots = _slot_rows(slots, pool.shape[0])
        o = np.zeros(q.shape, dtype=np.float64)
        for b, slot in enumerate(slots):
            if slot < 0:
                continue
            o[b], pool[slot] = self.decode_step(q[b], k[b], v[b], pool[slot])
        return o, pool

    def decode_step_q8(self, q, k, v, codes, scales, slots=None):
        """One step on the 8-bit state; returns (o fp64, codes', scales'), inputs untouched.

        q, k, v must hold values exact in fp32 (fp32 or bf16 inputs).  With
        ``slots`` (one per row of q, negative = padding) row b updates state
        codes[slots[b]], scales[slots[b]] of a [num_slots, H, d, d] pool."""
        if slots is not None:
            q, k, v = np.asarray(q), np.asarray(k), np.asarray(v)
            codes = np.array(codes, dtype=np.int8, copy=True)
            scales = np.array(scales, dtype=np.float32, copy=True)
            slots = _slot_rows(slots, codes.shape[0])
            o = np.zeros(q.shape, dtype=np.float64)
            for b, slot in enumerate(slots):
                if slot < 0:
                    continue
                o[b], codes[slot], scales[slot] = self.decode_step_q8(q[b], k[b], v[b], codes[slot],
                                                                      scales[slot])
            return o, codes, scales
        qf, kf, vf = _f32_exact(q), _f32_exact(k), _f32_exact(v)
        c = np.array(codes, dtype=np.int8, copy=True, order="C")
        a = np.array(scales, dtype=np.float32, copy=True, order="C")
        d = qf.shape[-1]
        BH = qf.size // d
        if c.size != BH * d * d or a.size != BH * d:
            raise ValueError("codes must be [..., d, d] and scales [..., d] for every q row")
        o = np.zeros(qf.shape, dtype=np.float64)
        self.lib.oracle_decode_step_q8(_fptr(qf), _fptr(kf), _fptr(vf), _cptr(c), _fptr(a),
                                       _ptr(o), BH, d)
        return o, c, a

    def prefill_varlen(self, q, k, v, cu_seqlens, heads=None):
        """Packed prefill over [H,T,d] inputs split by cu_seqlens.

        Returns (o [H,T,d], state [num_seqs,H,d,d]) in fp64.  With ``heads`` (a
        list of head indices) only those heads are computed; the rest stay zero.
        """
        q, k, v = _f64(q), _f64(k), _f64(v)
        H, T, d = q.shape
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
        S = cu.shape[0] - 1
        o = np.zeros(q.shape, dtype=np.float64)
        st = np.zeros((S, H, d, d), dtype=np.float64)
        if heads is None:
            hl, nh = None, H
        else:
            hl = np.ascontiguousarray(np.asarray(heads, dtype=np.int32))
            nh = hl.shape[0]
        ip = ctypes.POINTER(ctypes.c_int)
        self.lib.oracle_prefill_varlen(_ptr(q), _ptr(k), _ptr(v), cu.ctypes.data_as(ip), S, H,
                                       T, d, _ptr(o), _ptr(st),
                                       hl.ctypes.data_as(ip) if hl is not None else None, nh)
        return o, st


_default = None


def _get() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def num_threads() -> int:
    return _get().num_threads()


def prefill_quadratic(q, k, v):
    return _get().prefill_quadratic(q, k, v)


def prefill_recurrent(q, k, v, state_in=None):
    return _get().prefill_recurrent(q, k, v, state_in)


def prefill_blockwise(q, k, v, blk: int):
    return _get().prefill_blockwise(q, k, v, blk)


def decode_step(q, k, v, state):
    return _get().decode_step(q, k, v, state)


def prefill_backward(q, k, v, do):
    return _get().prefill_backward(q, k, v, do)


def prefill_varlen(q, k, v, cu_seqlens, heads=None):
    return _get().prefill_varlen(q, k, v, cu_seqlens, heads)


def state_quantize_q8(state):
    return _get().state_quantize_q8(state)


def state_dequantize_q8(codes, scales):
    return _get().state_dequantize_q8(codes, scales)


def decode_step_slots(q, k, v, pool, slots):
    return _get().decode_step_slots(q, k, v, pool, slots)


def decode_step_q8(q, k, v, codes, scales, slots=None):
    return _get().decode_step_q8(q, k, v, codes, scales, slots)
