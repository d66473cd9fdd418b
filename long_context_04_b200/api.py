"""Thin Python binding of ``liblightning.so`` (argument marshalling only).

Each function takes torch tensors, checks that they are contiguous CUDA
tensors of the expected dtype, and passes their data pointers, sizes and the
current CUDA stream to the C entry point of the same name.  Every step of the
computation runs in the library's kernels; there is no Python or CPU path, and
a missing or unloadable library raises ``LightningLibraryError``.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

from . import build as _build

LA_OK, LA_ERR_INVALID_ARG, LA_ERR_UNSUPPORTED, LA_ERR_CUDA = 0, 1, 2, 3
LA_ERR_DEVICE_TIMEOUT, LA_ERR_DEVICE_RANGE = 4, 5
LA_FP32, LA_BF16, LA_OUT_RMSNORM, LA_WRITE_STATE, LA_READ_STATE = 0, 1, 2, 4, 8
LA_MAX_VARLEN_SEQS = 1024


class LightningLibraryError(RuntimeError):
    """The CUDA library is missing or could not be loaded."""


class LightningError(RuntimeError):
    """A library call returned a status other than LA_OK."""

    def __init__(self, fn: str, status: int, text: str):
        super().__init__(f"{fn} failed: {text} ({status})")
        self.status = status


_LIB = None


def lib() -> ctypes.CDLL:
    """The loaded C library with argument types declared (loads it on first use)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = os.environ.get("LA_LIBRARY", _build.LIB)
    if not os.path.exists(path):
        raise LightningLibraryError(
            f"{path} is missing: build it with `python -m long_context_04_b200.build`")
    try:
        L = ctypes.CDLL(path)
    except OSError as e:  # pragma: no cover - depends on the machine
        raise LightningLibraryError(f"cannot load {path}: {e}") from e
    vp, i32, u32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint
    ip = ctypes.POINTER(ctypes.c_int32)
    L.la_prefill.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, ip, i32, u32, vp, vp]
    L.la_prefill.restype = i32
    L.la_decode_step.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, u32, vp]
    L.la_decode_step.restype = i32
    L.la_state_out.argtypes = [vp, vp, i32, i32, i32, vp, i32, vp]
    L.la_state_out.restype = i32
    L.la_chunk_state.argtypes = [vp, vp, i32, i32, i32, i32, ip, i32, u32, vp, vp]
    L.la_chunk_state.restype = i32
    L.la_state_prefix.argtypes = [vp, i32, i32, i32, i32, i32, vp, vp]
    L.la_state_prefix.restype = i32
    L.la_selftest_wait.argtypes = [ctypes.c_ulonglong, vp]
    L.la_selftest_wait.restype = i32
    L.la_status_string.argtypes = [i32]
    L.la_status_string.restype = ctypes.c_char_p
    L.la_get_device_status.argtypes = [vp]
    L.la_get_device_status.restype = i32
    L.la_version.argtypes = []
    L.la_version.restype = i32
    _LIB = L
    return L


def status_string(status: int) -> str:
    return lib().la_status_string(status).decode()


def _check(fn: str, status: int):
    if status != LA_OK:
        raise LightningError(fn, status, status_string(status))


def _stream_ptr(stream) -> int | None:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream or None


def _ptr(t: torch.Tensor | None):
    return None if t is None else t.data_ptr()


def _on_gpu(t: torch.Tensor) -> bool:
    return t.is_cuda


def _need(t: torch.Tensor, name: str, dtype=None, device=None):
    if not isinstance(t, torch.Tensor) or not _on_gpu(t):
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    # the library launches on the current device: every pointer of a call must live there
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, the call's tensors on {device}")


class _on_device:
    """Make ``dev`` the current CUDA device for one library call (the library launches,
    builds tensor maps and reads the status word on the current device), and check
    that an explicit stream belongs to it."""

    def __init__(self, dev, stream=None):
        self.dev = dev
        if stream is not None and getattr(stream, "device", dev) != dev:
            raise ValueError(f"stream is on {stream.device}, the call's tensors on {dev}")

    def __enter__(self):
        self.ctx = torch.cuda.device(self.dev) if self.dev.type == "cuda" else None
        if self.ctx is not None:
            self.ctx.__enter__()
        return self

    def __exit__(self, *exc):
        if self.ctx is not None:
            self.ctx.__exit__(*exc)
        return False


def _overlap(a: torch.Tensor, b: torch.Tensor) -> bool:
    """Whether the byte ranges of two tensors intersect."""
    a0, b0 = a.data_ptr(), b.data_ptr()
    a1, b1 = a0 + a.numel() * a.element_size(), b0 + b.numel() * b.element_size()
    return a0 < b1 and b0 < a1


def _need_shape(t: torch.Tensor, name: str, shape):
    # outputs are written through raw pointers: a wrong shape would be an out-of-bounds write
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _flags_for(dtype) -> int:
    if dtype == torch.bfloat16:
        return LA_BF16
    if dtype == torch.float32:
        return LA_FP32
    raise ValueError(f"unsupported dtype {dtype}: bf16 or fp32")


def prefill(q, k, v, *, beta: int = 128, cu_seqlens=None, rmsnorm: bool = False,
            return_state: bool = False, state_out=None, out=None, initial_state=None,
            stream=None):
    """Causal lightning attention over a batch (length > 1 path).

    ``q, k, v``: ``[B, N, H, D]`` or packed ``[T, H, D]`` (then ``cu_seqlens``,
    a host sequence of S+1 ints, gives the boundaries).  Returns ``o`` of the
    same shape, or ``(o, state)`` with ``return_state`` or ``state_out`` (state
    ``[S, H, D, D]`` fp32, the final KV of each sequence).

    ``initial_state`` (``[S, H, D, D]`` fp32): each sequence continues from it
    (chunked prefill, resume).  The final state then is ``initial + K^T V``; it
    is written over ``initial_state`` itself when ``state_out`` is that tensor,
    otherwise ``initial_state`` is left as it is (``state_out`` must then not
    overlap it).
    """
    _need(q, "q")
    dev = q.device
    for t, n in ((k, "k"), (v, "v")):
        _need(t, n, q.dtype, dev)
        if t.shape != q.shape:
            raise ValueError("q, k, v must have one shape")
    flags = _flags_for(q.dtype)
    if q.dim() == 4:
        B, N, H, D = q.shape
        if cu_seqlens is not None:
            raise ValueError("cu_seqlens needs packed [T, H, D] inputs")
        S = B
    elif q.dim() == 3:
        T, H, D = q.shape
        B, N = 1, T
        S = 1 if cu_seqlens is None else len(cu_seqlens) - 1
    else:
        raise ValueError("q must be [B, N, H, D] or [T, H, D]")
    cu = None
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", q.dtype, dev)
    _need_shape(out, "out", q.shape)
    st = state_out
    if return_state and st is None:
        st = torch.empty((S, H, D, D), dtype=torch.float32, device=dev)
    if st is not None:
        _need(st, "state_out", torch.float32, dev)
        _need_shape(st, "state_out", (S, H, D, D))
        flags |= LA_WRITE_STATE
    ws = st
    copy_in = False
    if initial_state is not None:
        _need(initial_state, "initial_state", torch.float32, dev)
        if tuple(initial_state.shape) != (S, H, D, D):
            raise ValueError("initial_state must be [S, H, D, D]")
        flags |= LA_READ_STATE
        if st is None:
            ws = initial_state                       # read only
        elif st.data_ptr() != initial_state.data_ptr():
            # copied into state_out by the library, then updated there in place; a partial
            # overlap would overwrite initial state values before they are read
            if _overlap(st, initial_state):
                raise ValueError("state_out and initial_state overlap without coinciding")
            copy_in = True
    if rmsnorm:
        flags |= LA_OUT_RMSNORM
    cu_ptr = None if cu is None else cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    with _on_device(dev, stream):
        if copy_in:
            _copy_state(initial_state, st, stream)   # the library's copy kernel
        rc = lib().la_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, N, D, beta, cu_ptr,
                              0 if cu is None else len(cu) - 1, flags, _ptr(ws),
                              _stream_ptr(stream))
    _check("la_prefill", rc)
    return (out, st) if (return_state or state_out is not None) else out


def _copy_state(src, dst, stream):
    if tuple(dst.shape) != tuple(src.shape):
        raise ValueError("state_out must have the shape of initial_state")
    S, H, D, _ = src.shape
    rc = lib().la_state_out(_ptr(src), _ptr(dst), S, H, D, None, S, _stream_ptr(stream))
    _check("la_state_out", rc)


def decode_step(q, k, v, state, *, rmsnorm: bool = False, out=None, stream=None):
    """One token per sequence: ``state += k v^T`` in place, returns ``o = q^T state``.

    ``q, k, v``: ``[B, H, D]``; ``state``: ``[B, H, D, D]`` fp32.
    """
    _need(q, "q")
    dev = q.device
    for t, n in ((k, "k"), (v, "v")):
        _need(t, n, q.dtype, dev)
        if t.shape != q.shape:
            raise ValueError("q, k, v must have one shape")
    _need(state, "state", torch.float32, dev)
    if q.dim() != 3:
        raise ValueError("q must be [B, H, D]")
    B, H, D = q.shape
    if tuple(state.shape) != (B, H, D, D):
        raise ValueError("state must be [B, H, D, D]")
    flags = _flags_for(q.dtype) | (LA_OUT_RMSNORM if rmsnorm else 0)
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", q.dtype, dev)
    _need_shape(out, "out", q.shape)
    with _on_device(dev, stream):
        rc = lib().la_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(state), _ptr(out), B, H, D,
                                  flags, _stream_ptr(stream))
    _check("la_decode_step", rc)
    return out


def state_out(state_ws, state_dst, seq_to_slot=None, *, stream=None):
    """``state_dst[slot(s)] = state_ws[s]`` (slot = ``seq_to_slot[s]``, a CUDA int32 tensor)."""
    _need(state_ws, "state_ws", torch.float32)
    dev = state_ws.device
    _need(state_dst, "state_dst", torch.float32, dev)
    if state_ws.dim() != 4 or state_dst.dim() != 4:
        raise ValueError("state_ws and state_dst must be [*, H, D, D]")
    S, H, D, _ = state_ws.shape
    _need_shape(state_dst, "state_dst", (state_dst.shape[0], H, D, D))
    if _overlap(state_ws, state_dst):
        raise ValueError("state_ws and state_dst must not overlap")
    if seq_to_slot is not None:
        _need(seq_to_slot, "seq_to_slot", torch.int32, dev)
        _need_shape(seq_to_slot, "seq_to_slot", (S,))
    with _on_device(dev, stream):
        rc = lib().la_state_out(_ptr(state_ws), _ptr(state_dst), S, H, D, _ptr(seq_to_slot),
                                state_dst.shape[0], _stream_ptr(stream))
    _check("la_state_out", rc)
    return state_dst


def chunk_state(k, v, *, cu_seqlens=None, state_out=None, stream=None):
    """Each sequence's K^T V alone (no output): ``[S, H, D, D]`` fp32.  The local state
    of a chunk in LASP+ sequence parallelism."""
    _need(k, "k")
    dev = k.device
    _need(v, "v", k.dtype, dev)
    if v.shape != k.shape:
        raise ValueError("k and v must have one shape")
    flags = _flags_for(k.dtype)
    if k.dim() == 4:
        B, N, H, D = k.shape
        if cu_seqlens is not None:
            raise ValueError("cu_seqlens needs packed [T, H, D] inputs")
        S = B
    elif k.dim() == 3:
        T, H, D = k.shape
        B, N = 1, T
        S = 1 if cu_seqlens is None else len(cu_seqlens) - 1
    else:
        raise ValueError("k must be [B, N, H, D] or [T, H, D]")
    cu = None if cu_seqlens is None else np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    if state_out is None:
        state_out = torch.empty((S, H, D, D), dtype=torch.float32, device=dev)
    _need(state_out, "state_out", torch.float32, dev)
    _need_shape(state_out, "state_out", (S, H, D, D))
    cu_ptr = None if cu is None else cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    with _on_device(dev, stream):
        rc = lib().la_chunk_state(_ptr(k), _ptr(v), B, H, N, D, cu_ptr,
                                  0 if cu is None else len(cu) - 1, flags, _ptr(state_out),
                                  _stream_ptr(stream))
    _check("la_chunk_state", rc)
    return state_out


def state_prefix(gathered, rank: int, *, out=None, stream=None):
    """``out = sum_{r < rank} gathered[r]`` for gathered ``[R, S, H, D, D]`` fp32 (the
    chunk states of all ranks): the initial state of chunk ``rank`` in LASP+."""
    _need(gathered, "gathered", torch.float32)
    dev = gathered.device
    if gathered.dim() != 5:
        raise ValueError("gathered must be [R, S, H, D, D]")
    R, S, H, D, _ = gathered.shape
    if out is None:
        out = torch.empty((S, H, D, D), dtype=torch.float32, device=dev)
    _need(out, "out", torch.float32, dev)
    _need_shape(out, "out", (S, H, D, D))
    if _overlap(gathered, out):
        raise ValueError("out must not overlap gathered")
    with _on_device(dev, stream):
        rc = lib().la_state_prefix(_ptr(gathered), R, int(rank), S, H, D, _ptr(out),
                                   _stream_ptr(stream))
    _check("la_state_prefix", rc)
    return out


def selftest_wait(limit_ns: int = 10_000_000, *, stream=None):
    """Launch the self-test kernel whose one wait gives up after ``limit_ns``; the next
    ``device_status`` reports LA_ERR_DEVICE_TIMEOUT."""
    _check("la_selftest_wait", lib().la_selftest_wait(int(limit_ns), _stream_ptr(stream)))


def device_status(stream=None) -> int:
    """Synchronise ``stream`` and return (and clear) the device status word."""
    return lib().la_get_device_status(_stream_ptr(stream))


def version() -> int:
    return lib().la_version()
