"""linear_attention_13_b200 -- B200-native causal linear attention (Lightning Attention).

Thin Python binding over the C ABI of ``liblightning.so`` (declared in
``include/lightning.h``).  Every step of the computation runs in the CUDA
kernels of that library; this module only marshals torch tensors (device
pointers, sizes, the current CUDA stream) into the C calls and raises on a
non-OK status.  There is no CPU fallback: if the library is missing or fails
to load, every call raises.

The raw entry points keep the C names (``la_prefill``, ``la_prefill_ex``,
``la_prefill_varlen``, ``la_decode_step``, ``la_status_string``,
``la_get_last_error``, ``la_device_sm_count``).  The tensor-level helpers
``prefill``, ``prefill_varlen`` and ``decode_step`` allocate outputs and call
them.
"""
from __future__ import annotations

import ctypes
import os

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "liblightning.so")

LA_OK = 0
LA_ERR_INVALID_ARG = -1
LA_ERR_UNSUPPORTED = -2
LA_ERR_CUDA = -3
LA_ERR_ALLOC = -4
LA_ERR_TIMEOUT = -5
LA_ERR_BAD_SEQLENS = -6
LA_ERR_BAD_SLOT = -7

LA_F32 = 0
LA_BF16 = 1

LA_FLAG_THREE_PASS = 1
LA_FLAG_FUSED = 2
LA_FLAG_SPLIT_V = 4
LA_FLAG_NO_SPLIT_V = 8

LA_KERNEL_PREFILL_TC = 0
LA_KERNEL_CHUNK_STATE = 1
LA_KERNEL_CHUNK_SCAN = 2
LA_KERNEL_PREFILL_F32 = 3
LA_KERNEL_DECODE = 4
LA_KERNEL_AUX = 5
LA_NUM_KERNEL_IDS = 6

EXPORTED = ("la_prefill", "la_prefill_ex", "la_prefill_varlen", "la_decode_step",
            "la_status_string", "la_get_last_error", "la_device_sm_count",
            "la_timing_enable", "la_timing_read", "la_kernel_name", "la_prefill_noalloc",
            "la_prefill_main_kernel", "la_prefill_from_state", "la_prefill_varlen_from_state",
            "la_state_increment", "la_state_prefix", "la_prefill_backward",
            "la_prefill_varlen_ex", "la_decode_step_slots", "la_decode_step_q8",
            "la_state_quantize_q8", "la_state_dequantize_q8", "la_set_wait_limit_ns",
            "la_debug_fail_allocations", "la_binary_version", "la_debug_skip_lookback_items",
            "la_debug_occupy_sms", "la_debug_stall_split_load")

LA_NOALLOC_SCRATCH_BYTES = 16 << 20

_lib = None


class LightningError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load liblightning.so and declare the C signatures.  Raises if absent."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"CUDA library not built: {path} is missing (run __graft_entry__.build() or "
            "python linear_attention_13_b200/build.py)")
    lib = ctypes.CDLL(path)
    vp, i = ctypes.c_void_p, ctypes.c_int
    lib.la_prefill.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, vp]
    lib.la_prefill_ex.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, vp, i, i]
    lib.la_prefill_varlen.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, vp]
    lib.la_prefill_varlen_ex.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, vp, i, i]
    lib.la_prefill_from_state.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, vp, i, i]
    lib.la_state_increment.argtypes = [vp, vp, vp, i, i, i, i, i, vp]
    lib.la_prefill_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, vp]
    lib.la_state_prefix.argtypes = [vp, i, i, vp, i, i, i, vp]
    lib.la_prefill_varlen_from_state.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, vp, i, i]
    lib.la_decode_step.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, vp]
    lib.la_decode_step_slots.argtypes = [vp, vp, vp, vp, vp, i, vp, i, i, i, i, vp]
    lib.la_decode_step_q8.argtypes = [vp, vp, vp, vp, vp, vp, i, vp, i, i, i, i, vp]
    ll = ctypes.c_longlong
    lib.la_state_quantize_q8.argtypes = [vp, vp, vp, ll, i, vp]
    lib.la_state_dequantize_q8.argtypes = [vp, vp, vp, ll, i, vp]
    lib.la_status_string.argtypes = [i]
    lib.la_status_string.restype = ctypes.c_char_p
    lib.la_get_last_error.argtypes = []
    lib.la_device_sm_count.argtypes = []
    lib.la_timing_enable.argtypes = [i]
    lib.la_timing_read.argtypes = [i, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int)]
    lib.la_prefill_noalloc.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, vp]
    lib.la_kernel_name.argtypes = [i]
    lib.la_kernel_name.restype = ctypes.c_char_p
    lib.la_prefill_main_kernel.argtypes = []
    lib.la_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong, ctypes.POINTER(ctypes.c_ulonglong)]
    lib.la_debug_fail_allocations.argtypes = [i]
    lib.la_binary_version.argtypes = []
    lib.la_debug_skip_lookback_items.argtypes = [i]
    lib.la_debug_occupy_sms.argtypes = [i, ctypes.c_ulonglong, vp]
    lib.la_debug_stall_split_load.argtypes = [i]
    lib.la_prefill_main_kernel.restype = ctypes.c_char_p
    for name in ("la_prefill", "la_prefill_ex", "la_prefill_varlen", "la_prefill_varlen_ex",
                 "la_decode_step",
                 "la_get_last_error", "la_device_sm_count", "la_timing_enable",
                 "la_timing_read", "la_prefill_noalloc", "la_prefill_from_state",
                 "la_prefill_varlen_from_state", "la_state_increment", "la_state_prefix",
                 "la_prefill_backward", "la_decode_step_slots", "la_decode_step_q8",
                 "la_state_quantize_q8", "la_state_dequantize_q8", "la_set_wait_limit_ns",
                 "la_debug_fail_allocations", "la_binary_version", "la_debug_skip_lookback_items",
                 "la_debug_occupy_sms", "la_debug_stall_split_load"):
        getattr(lib, name).restype = ctypes.c_int
    if path == LIB_PATH:
        _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().la_status_string(int(status)).decode()


# ---------------------------------------------------------------- raw C names
def la_prefill(q, k, v, o, state_out, B, H, N, d, blk, dt, stream):
    return load_library().la_prefill(q, k, v, o, state_out, B, H, N, d, blk, dt, stream)


def la_prefill_ex(q, k, v, o, state_out, B, H, N, d, blk, dt, stream, chunk_tokens, flags):
    return load_library().la_prefill_ex(q, k, v, o, state_out, B, H, N, d, blk, dt, stream,
                                        chunk_tokens, flags)


def la_prefill_varlen(q, k, v, o, state_out, cu_seqlens, num_seqs, total_tokens, H, d, blk, dt,
                      stream):
    return load_library().la_prefill_varlen(q, k, v, o, state_out, cu_seqlens, num_seqs,
                                            total_tokens, H, d, blk, dt, stream)


def la_prefill_from_state(q, k, v, o, state_in, state_out, B, H, N, d, blk, dt, stream,
                          chunk_tokens, flags):
    return load_library().la_prefill_from_state(q, k, v, o, state_in, state_out, B, H, N, d, blk,
                                                dt, stream, chunk_tokens, flags)


def la_prefill_varlen_from_state(q, k, v, o, state_in, state_out, cu_seqlens, num_seqs,
                                 total_tokens, H, d, blk, dt, stream, chunk_tokens, flags):
    return load_library().la_prefill_varlen_from_state(q, k, v, o, state_in, state_out, cu_seqlens,
                                                       num_seqs, total_tokens, H, d, blk, dt,
                                                       stream, chunk_tokens, flags)


def la_prefill_backward(q, k, v, do, dq, dk, dv, B, H, N, d, blk, dt, stream):
    return load_library().la_prefill_backward(q, k, v, do, dq, dk, dv, B, H, N, d, blk, dt, stream)


def la_state_increment(k, v, delta_out, B, H, N, d, dt, stream):
    return load_library().la_state_increment(k, v, delta_out, B, H, N, d, dt, stream)


def la_state_prefix(states, R, rank, prefix_out, B, H, d, stream):
    return load_library().la_state_prefix(states, R, rank, prefix_out, B, H, d, stream)


def la_prefill_noalloc(q, k, v, o, state_out, B, H, N, d, blk, dt, stream):
    """la_prefill that allocates no device memory (fixed in-library scratch)."""
    return load_library().la_prefill_noalloc(q, k, v, o, state_out, B, H, N, d, blk, dt, stream)


def la_prefill_varlen_ex(q, k, v, o, state_out, cu_seqlens, num_seqs, total_tokens, H, d, blk,
                         dt, stream, chunk_tokens, flags):
    return load_library().la_prefill_varlen_ex(q, k, v, o, state_out, cu_seqlens, num_seqs,
                                               total_tokens, H, d, blk, dt, stream, chunk_tokens,
                                               flags)


def la_decode_step(q, k, v, state, o, B, H, d, dt, stream):
    return load_library().la_decode_step(q, k, v, state, o, B, H, d, dt, stream)


def la_decode_step_slots(q, k, v, state_pool, slots, num_slots, o, B, H, d, dt, stream):
    return load_library().la_decode_step_slots(q, k, v, state_pool, slots, num_slots, o, B, H, d,
                                               dt, stream)


def la_decode_step_q8(q, k, v, codes, scales, slots, num_slots, o, B, H, d, dt, stream):
    return load_library().la_decode_step_q8(q, k, v, codes, scales, slots, num_slots, o, B, H, d,
                                            dt, stream)


def la_state_quantize_q8(state, codes, scales, n_heads, d, stream):
    return load_library().la_state_quantize_q8(state, codes, scales, n_heads, d, stream)


def la_state_dequantize_q8(codes, scales, state, n_heads, d, stream):
    return load_library().la_state_dequantize_q8(codes, scales, state, n_heads, d, stream)


def la_status_string(status):
    return status_string(status)


def la_get_last_error():
    return load_library().la_get_last_error()


def la_device_sm_count():
    return load_library().la_device_sm_count()


def la_timing_enable(max_launches):
    return load_library().la_timing_enable(max_launches)


def la_timing_read(kernel_id):
    """Returns (status, total_ms, launches) for one kernel id."""
    ms = ctypes.c_double(0.0)
    n = ctypes.c_int(0)
    st = load_library().la_timing_read(kernel_id, ctypes.byref(ms), ctypes.byref(n))
    return st, ms.value, n.value


def la_kernel_name(kernel_id):
    return load_library().la_kernel_name(kernel_id).decode()


def la_set_wait_limit_ns(limit_ns):
    """Bounded-wait limit of the device code on the current device (0 = the
    default of 2 s).  Returns (status, previous limit in ns)."""
    prev = ctypes.c_ulonglong(0)
    st = load_library().la_set_wait_limit_ns(int(limit_ns), ctypes.byref(prev))
    return st, prev.value


def la_debug_fail_allocations(count):
    """Make the library's next ``count`` workspace allocations fail (tests)."""
    return load_library().la_debug_fail_allocations(count)


def la_debug_skip_lookback_items(count):
    """The next look-back launch skips its first ``count`` items (tests)."""
    return load_library().la_debug_skip_lookback_items(count)


def la_debug_stall_split_load(tile):
    """The next split-kernel launch leaves the loads of each CTA's ``tile``-th
    tile unissued (tests); -1 cancels."""
    return load_library().la_debug_stall_split_load(tile)


def la_debug_occupy_sms(ctas, duration_ns, stream=None):
    """Hold ``ctas`` SMs for ``duration_ns`` (<= 1 s) with a waiting kernel (tests)."""
    return load_library().la_debug_occupy_sms(ctas, int(duration_ns), _stream_ptr(stream))


def la_binary_version():
    """Compute capability the loaded kernels were built for (100 = sm_100a)."""
    return load_library().la_binary_version()


def la_prefill_main_kernel():
    """Kernel the most recent bf16 prefill launched for its output pass."""
    return load_library().la_prefill_main_kernel().decode()


# ---------------------------------------------------------------- tensor helpers
def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return LA_BF16
    if t.dtype == torch.float32:
        return LA_F32
    raise TypeError(f"unsupported dtype {t.dtype}; expected bfloat16 or float32")


def _check(t, name):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _like(t, ref, name, ref_name):
    """``t`` must be a contiguous CUDA tensor with ``ref``'s shape, dtype and
    device: the C entry points take raw pointers and cannot check sizes, so a
    mismatch would become an out-of-bounds access on the device."""
    _check(t, name)
    if t.shape != ref.shape or t.dtype != ref.dtype or t.device != ref.device:
        raise ValueError(f"{name} must match {ref_name} in shape, dtype and device "
                         f"(got {tuple(t.shape)} {t.dtype} {t.device}, expected "
                         f"{tuple(ref.shape)} {ref.dtype} {ref.device})")


def _state(t, shape, device, name):
    """``t`` must be a contiguous float32 CUDA tensor of ``shape`` on ``device``."""
    _check(t, name)
    torch = _torch()
    if t.dtype != torch.float32 or tuple(t.shape) != tuple(shape) or t.device != device:
        raise ValueError(f"{name} must be float32 {list(shape)} on {device} "
                         f"(got {t.dtype} {list(t.shape)} on {t.device})")


def _stream_ptr(stream):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _raise(status, where):
    if status != LA_OK:
        raise LightningError(status, where)


def prefill(q, k, v, blk: int = 128, want_state: bool = True, chunk_tokens: int = 0,
            flags: int = 0, out=None, state_out=None, stream=None, state_in=None):
    """Causal linear attention prefill of [B,H,N,d] tensors, from ``state_in``
    ([B,H,d,d] fp32; None = zero).  Returns (o, state)."""
    torch = _torch()
    _check(q, "q")
    if q.dim() != 4:
        raise ValueError("q, k, v must share one [B,H,N,d] shape")
    _like(k, q, "k", "q")
    _like(v, q, "v", "q")
    B, H, N, d = q.shape
    o = out if out is not None else torch.empty_like(q)
    _like(o, q, "out", "q")
    st = state_out
    if st is None and want_state:
        st = torch.empty((B, H, d, d), dtype=torch.float32, device=q.device)
    if st is not None:
        _state(st, (B, H, d, d), q.device, "state_out")
    if state_in is not None:
        _state(state_in, (B, H, d, d), q.device, "state_in")
    status = la_prefill_from_state(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                   state_in.data_ptr() if state_in is not None else None,
                                   st.data_ptr() if st is not None else None, B, H, N, d, blk,
                                   _dtype_code(q), _stream_ptr(stream), chunk_tokens, flags)
    _raise(status, "la_prefill")
    return o, st


def prefill_varlen(q, k, v, cu_seqlens, blk: int = 128, want_state: bool = True, out=None,
                   state_out=None, stream=None, chunk_tokens: int = 0, flags: int = 0,
                   state_in=None):
    """Packed prefill of [H,T,d] tensors split by int32 device cu_seqlens, each
    sequence from its ``state_in`` ([num_seqs,H,d,d] fp32; None = zero).

    Returns (o, state [num_seqs,H,d,d])."""
    torch = _torch()
    _check(q, "q")
    _check(cu_seqlens, "cu_seqlens")
    if q.dim() != 3:
        raise ValueError("q, k, v must share one packed [H,T,d] shape")
    _like(k, q, "k", "q")
    _like(v, q, "v", "q")
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
        raise TypeError("cu_seqlens must be a 1-D int32 tensor of num_seqs + 1 offsets")
    if cu_seqlens.device != q.device:
        raise ValueError("cu_seqlens must be on q's device")
    H, T, d = q.shape
    S = cu_seqlens.numel() - 1
    o = out if out is not None else torch.empty_like(q)
    _like(o, q, "out", "q")
    st = state_out
    if st is None and want_state:
        st = torch.empty((S, H, d, d), dtype=torch.float32, device=q.device)
    if st is not None:
        _state(st, (S, H, d, d), q.device, "state_out")
    if state_in is not None:
        _state(state_in, (S, H, d, d), q.device, "state_in")
    status = la_prefill_varlen_from_state(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                          state_in.data_ptr() if state_in is not None else None,
                                          st.data_ptr() if st is not None else None,
                                          cu_seqlens.data_ptr(), S, T, H, d, blk, _dtype_code(q),
                                          _stream_ptr(stream), chunk_tokens, flags)
    _raise(status, "la_prefill_varlen")
    return o, st


def prefill_backward(q, k, v, do, blk: int = 128, stream=None, out=None):
    """Gradients (dq, dk, dv) of sum(do * prefill(q, k, v)[0]) for [B,H,N,d] tensors
    (written into ``out`` = (dq, dk, dv) when given)."""
    torch = _torch()
    _check(q, "q")
    if q.dim() != 4:
        raise ValueError("q, k, v, do must share one [B,H,N,d] shape")
    for t, n in ((k, "k"), (v, "v"), (do, "do")):
        _like(t, q, n, "q")
    B, H, N, d = q.shape
    if out is not None:
        dq, dk, dv = out
        for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
            _like(t, q, n, "q")
    else:
        dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    status = la_prefill_backward(q.data_ptr(), k.data_ptr(), v.data_ptr(), do.data_ptr(),
                                 dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d, blk,
                                 _dtype_code(q), _stream_ptr(stream))
    _raise(status, "la_prefill_backward")
    return dq, dk, dv


def state_increment(k, v, out=None, stream=None):
    """K^T V over the tokens of [B,H,N,d] bf16 k, v: [B,H,d,d] fp32."""
    torch = _torch()
    _check(k, "k")
    if k.dim() != 4:
        raise ValueError("k, v must share one [B,H,N,d] shape")
    _like(v, k, "v", "k")
    B, H, N, d = k.shape
    o = out if out is not None else torch.empty((B, H, d, d), dtype=torch.float32, device=k.device)
    _state(o, (B, H, d, d), k.device, "out")
    status = la_state_increment(k.data_ptr(), v.data_ptr(), o.data_ptr(), B, H, N, d,
                                _dtype_code(k), _stream_ptr(stream))
    _raise(status, "la_state_increment")
    return o


def state_prefix(states, rank, out=None, stream=None):
    """sum over r < rank of states[r] ([R,B,H,d,d] fp32): [B,H,d,d] fp32."""
    torch = _torch()
    _check(states, "states")
    if states.dtype != torch.float32 or states.dim() != 5:
        raise ValueError("states must be float32 [R,B,H,d,d]")
    R, B, H, d, d2 = states.shape
    if d2 != d:
        raise ValueError("states must be float32 [R,B,H,d,d]")
    o = out if out is not None else torch.empty((B, H, d, d), dtype=torch.float32, device=states.device)
    _state(o, (B, H, d, d), states.device, "out")
    status = la_state_prefix(states.data_ptr(), R, rank, o.data_ptr(), B, H, d, _stream_ptr(stream))
    _raise(status, "la_state_prefix")
    return o


def decode_step(q, k, v, state, out=None, stream=None):
    """One decode step on [B,H,d] inputs; updates ``state`` [B,H,d,d] fp32 in place."""
    torch = _torch()
    _check(q, "q")
    if q.dim() != 3:
        raise ValueError("q, k, v must share one [B,H,d] shape")
    _like(k, q, "k", "q")
    _like(v, q, "v", "q")
    B, H, d = q.shape
    # the C call updates B*H states of d x d: anything smaller would be overrun
    _state(state, (B, H, d, d), q.device, "state")
    o = out if out is not None else torch.empty_like(q)
    _like(o, q, "out", "q")
    status = la_decode_step(q.data_ptr(), k.data_ptr(), v.data_ptr(), state.data_ptr(),
                            o.data_ptr(), B, H, d, _dtype_code(q), _stream_ptr(stream))
    _raise(status, "la_decode_step")
    return o


def _slots_arg(slots, B, torch):
    if slots is None:
        return None
    _check(slots, "slots")
    if slots.dtype != torch.int32 or slots.shape != (B,):
        raise ValueError("slots must be an int32 tensor of shape [B]")
    return slots.data_ptr()


def decode_step_slots(q, k, v, state_pool, slots, out=None, stream=None):
    """Decode step where row b of the [B,H,d] batch updates state_pool[slots[b]]
    ([num_slots,H,d,d] fp32, in place); rows with a negative slot are padding
    (zero output, no state access).  ``slots`` is an int32 CUDA tensor [B]."""
    torch = _torch()
    _check(q, "q")
    if q.dim() != 3:
        raise ValueError("q, k, v must share one [B,H,d] shape")
    _like(k, q, "k", "q")
    _like(v, q, "v", "q")
    _check(state_pool, "state_pool")
    if state_pool.dtype != torch.float32:
        raise TypeError("state_pool must be float32")
    B, H, d = q.shape
    if state_pool.dim() != 4 or state_pool.shape[1:] != (H, d, d) or state_pool.device != q.device:
        raise ValueError("state_pool must be [num_slots, H, d, d] on q's device")
    o = out if out is not None else torch.empty_like(q)
    _like(o, q, "out", "q")
    status = la_decode_step_slots(q.data_ptr(), k.data_ptr(), v.data_ptr(), state_pool.data_ptr(),
                                  _slots_arg(slots, B, torch), state_pool.shape[0], o.data_ptr(),
                                  B, H, d, _dtype_code(q), _stream_ptr(stream))
    _raise(status, "la_decode_step_slots")
    return o


def decode_step_q8(q, k, v, codes, scales, slots=None, out=None, stream=None):
    """Decode step on the 8-bit state: ``codes`` [num_slots,H,d,d] int8 and
    ``scales`` [num_slots,H,d] fp32, updated in place; ``slots`` as for
    ``decode_step_slots`` (None: row b uses slot b)."""
    torch = _torch()
    _check(q, "q")
    if q.dim() != 3:
        raise ValueError("q, k, v must share one [B,H,d] shape")
    _like(k, q, "k", "q")
    _like(v, q, "v", "q")
    for t, n in ((codes, "codes"), (scales, "scales")):
        _check(t, n)
    if codes.dtype != torch.int8 or scales.dtype != torch.float32:
        raise TypeError("codes must be int8 and scales float32")
    B, H, d = q.shape
    if (codes.dim() != 4 or codes.shape[1:] != (H, d, d) or scales.shape != codes.shape[:3]
            or codes.device != q.device or scales.device != q.device):
        raise ValueError("codes must be [num_slots, H, d, d] and scales [num_slots, H, d] on q's device")
    if slots is None and codes.shape[0] < B:
        raise ValueError("without slots, row b uses slot b: codes needs at least B slots")
    o = out if out is not None else torch.empty_like(q)
    _like(o, q, "out", "q")
    status = la_decode_step_q8(q.data_ptr(), k.data_ptr(), v.data_ptr(), codes.data_ptr(),
                               scales.data_ptr(), _slots_arg(slots, B, torch), codes.shape[0],
                               o.data_ptr(), B, H, d, _dtype_code(q), _stream_ptr(stream))
    _raise(status, "la_decode_step_q8")
    return o


def state_quantize_q8(state, codes=None, scales=None, stream=None):
    """fp32 states [..., d, d] -> (int8 codes [..., d, d], fp32 scales [..., d])."""
    torch = _torch()
    _check(state, "state")
    if state.dtype != torch.float32:
        raise TypeError("state must be float32")
    d = state.shape[-1]
    if state.dim() < 2 or state.shape[-2] != d:
        raise ValueError("state must be [..., d, d]")
    c = codes if codes is not None else torch.empty(state.shape, dtype=torch.int8, device=state.device)
    a = scales if scales is not None else torch.empty(state.shape[:-1], dtype=torch.float32,
                                                      device=state.device)
    _check(c, "codes")
    _check(a, "scales")
    if c.dtype != torch.int8 or c.shape != state.shape or c.device != state.device:
        raise ValueError("codes must be int8 with the state's shape and device")
    if a.dtype != torch.float32 or a.shape != state.shape[:-1] or a.device != state.device:
        raise ValueError("scales must be float32 [..., d] on the state's device")
    status = la_state_quantize_q8(state.data_ptr(), c.data_ptr(), a.data_ptr(),
                                  state.numel() // (d * d), d, _stream_ptr(stream))
    _raise(status, "la_state_quantize_q8")
    return c, a


def state_dequantize_q8(codes, scales, out=None, stream=None):
    """(codes, scales) -> fp32 states, S_ij = c_ij * a_i."""
    torch = _torch()
    _check(codes, "codes")
    _check(scales, "scales")
    d = codes.shape[-1]
    if codes.dtype != torch.int8 or codes.dim() < 2 or codes.shape[-2] != d:
        raise ValueError("codes must be int8 [..., d, d]")
    if scales.dtype != torch.float32 or scales.shape != codes.shape[:-1] or scales.device != codes.device:
        raise ValueError("scales must be float32 [..., d] on the codes' device")
    o = out if out is not None else torch.empty(codes.shape, dtype=torch.float32, device=codes.device)
    _state(o, codes.shape, codes.device, "out")
    status = la_state_dequantize_q8(codes.data_ptr(), scales.data_ptr(), o.data_ptr(),
                                    codes.numel() // (d * d), d, _stream_ptr(stream))
    _raise(status, "la_state_dequantize_q8")
    return o
