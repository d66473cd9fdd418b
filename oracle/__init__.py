"""fp64 CPU oracle for causal lightning attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  It
shares no code with the CUDA path (``long_context_04_b200``) and never imports
it; both sides only receive the same seeded input arrays.

Forms (MiniMax-01, "Scaling Foundation Models with Lightning Attention"; CSDN
digest section 2.1 "right product kernel trick ... intra-block and inter-block
computation avoids the cumsum bottleneck"; mizuki blog appendix "intra-block
left product + inter-block right product, O(N)"):

* ``quadratic``  -- O = [(Q K^T) (.) M] V with the causal 0/1 mask, per
  sequence (the plain definition).
* ``recurrent``  -- KV_i = KV_{i-1} + k_i v_i^T, o_i = q_i^T KV_i (the slow
  causal cumsum the tiling replaces).
* ``blocked``    -- the block-tiled lightning evaluation with block size beta.
* ``decode_step``-- one token per sequence: KV += k v^T, o = q^T KV.
* ``final_state``-- K_s^T V_s per (sequence, head), by a library matmul.

Optional output RMSNorm over the head dimension (NormAttention, CSDN digest
section 2.1): y = x / sqrt(mean(x^2) + eps).

Readings where the pages are silent: no decay, causal diagonal included
(j <= i), no feature map, no 1/sqrt(d) and no denominator; RMSNorm with unit
weight and eps inside the square root, applied after intra + inter.

Every array is float64 ``[T, H, D]``; ``cu_seqlens`` has S+1 entries.
"""
from __future__ import annotations

import ctypes
import math
import os

import numpy as np

from . import build as _build

_LIBS: dict = {}


def _lib(path: str | None = None):
    """Load (once) the compiled oracle; ``path`` selects another build of it."""
    path = path or os.environ.get("LA_ORACLE_LIB") or _build.build()
    if path not in _LIBS:
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        lp = ctypes.POINTER(ctypes.c_int64)
        lib.la_oracle_prefill.argtypes = [ctypes.c_int, dp, dp, dp, dp, dp, dp, ctypes.c_int64,
                                          ctypes.c_int, ctypes.c_int, lp, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int]
        lib.la_oracle_prefill.restype = ctypes.c_int
        lib.la_oracle_decode_step.argtypes = [dp, dp, dp, dp, dp, dp, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                              ctypes.c_int]
        lib.la_oracle_decode_step.restype = ctypes.c_int
        _LIBS[path] = lib
    return _LIBS[path]


_ACTIVE: list = [None]   # library path used by the functions below (None = default build)


class use_library:
    """Context manager: route the functions of this module to another oracle build."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        self.prev = _ACTIVE[0]
        _ACTIVE[0] = self.path
        return self

    def __exit__(self, *exc):
        _ACTIVE[0] = self.prev
        return False


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor: exact upcast of bf16/fp32 values
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _cu(cu_seqlens, T: int) -> np.ndarray:
    if cu_seqlens is None:
        return np.array([0, T], dtype=np.int64)
    return np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


_FORMS = {"quadratic": 0, "recurrent": 1, "blocked": 2}


def _prefill(form: str, q, k, v, cu_seqlens=None, *, beta: int = 0, rmsnorm: bool = False,
             eps: float = 1e-6, want_o: bool = True, want_state: bool = True,
             initial_state=None, nthreads: int | None = None):
    q, k, v = _f64(q), _f64(k), _f64(v)
    if q.ndim != 3 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must share one [T, H, D] shape")
    T, H, D = q.shape
    cu = _cu(cu_seqlens, T)
    S = len(cu) - 1
    x0 = None
    if initial_state is not None:
        x0 = _f64(initial_state)
        if x0.shape != (S, H, D, D):
            raise ValueError("initial_state must be [S, H, D, D]")
    o = np.zeros((T, H, D), np.float64) if want_o or form != "recurrent" else None
    st = np.zeros((S, H, D, D), np.float64) if want_state else None
    rc = _lib(_ACTIVE[0]).la_oracle_prefill(_FORMS[form], _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(st), _ptr(x0), T,
                                  H, D, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), S,
                                  beta, int(rmsnorm), eps, nthreads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (code {rc})")
    return o, st


def quadratic(q, k, v, cu_seqlens=None, *, rmsnorm=False, eps=1e-6, initial_state=None,
              nthreads=None):
    """O = q^T X + [(Q K^T) (.) M] V per sequence (X = initial_state, default 0);
    returns (O, final state X + K^T V)."""
    return _prefill("quadratic", q, k, v, cu_seqlens, rmsnorm=rmsnorm, eps=eps,
                    initial_state=initial_state, nthreads=nthreads)


def recurrent(q, k, v, cu_seqlens=None, *, rmsnorm=False, eps=1e-6, want_o=True,
              initial_state=None, nthreads=None):
    """Token-by-token state recurrence from KV = initial_state (default 0);
    returns (O or None, final state)."""
    return _prefill("recurrent", q, k, v, cu_seqlens, rmsnorm=rmsnorm, eps=eps, want_o=want_o,
                    initial_state=initial_state, nthreads=nthreads)


def blocked(q, k, v, beta: int, cu_seqlens=None, *, rmsnorm=False, eps=1e-6, initial_state=None,
            nthreads=None):
    """Block-tiled lightning evaluation (intra left product + inter right product), the
    state starting at initial_state (default 0)."""
    return _prefill("blocked", q, k, v, cu_seqlens, beta=beta, rmsnorm=rmsnorm, eps=eps,
                    initial_state=initial_state, nthreads=nthreads)


def decode_step(q, k, v, state, *, rmsnorm=False, eps=1e-6, nthreads=None):
    """One decode step: q,k,v [B,H,D], state [B,H,D,D]; returns (o, new state)."""
    q, k, v, st = _f64(q), _f64(k), _f64(v), _f64(state)
    B, H, D = q.shape
    if st.shape != (B, H, D, D):
        raise ValueError("state must be [B, H, D, D]")
    o = np.zeros((B, H, D), np.float64)
    new = np.empty_like(st)
    rc = _lib(_ACTIVE[0]).la_oracle_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(st), _ptr(new), _ptr(o),
                                      B, H, D, int(rmsnorm), eps, nthreads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (code {rc})")
    return o, new


def final_state(k, v, cu_seqlens=None) -> np.ndarray:
    """state[s, h] = K_{s,h}^T V_{s,h} (library fp64 matmul), [S, H, D, D]."""
    k, v = _f64(k), _f64(v)
    T, H, D = k.shape
    cu = _cu(cu_seqlens, T)
    S = len(cu) - 1
    out = np.zeros((S, H, D, D), np.float64)
    for s in range(S):
        a, b = int(cu[s]), int(cu[s + 1])
        for h in range(H):
            out[s, h] = k[a:b, h, :].T @ v[a:b, h, :]
    return out


def rel_l2(x, ref) -> float:
    """||x - ref||_2 / ||ref||_2 in fp64: the error metric of the parity tests.

    Returns 0 when both are zero, and inf when ``x`` holds a NaN or an infinity or
    when ``ref`` is zero and ``x`` is not, so that a non-finite or spurious output
    can never pass a tolerance.  The shapes must agree and ``ref`` must be finite.
    """
    x, ref = _f64(x), _f64(ref)
    if x.shape != ref.shape:
        raise ValueError(f"shapes differ: {x.shape} vs {ref.shape}")
    if not np.isfinite(ref).all():
        raise ValueError("the reference holds a non-finite value")
    if not np.isfinite(x).all():
        return float("inf")
    den = float(np.linalg.norm(ref.ravel()))
    num = float(np.linalg.norm((x - ref).ravel()))
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return num / den


def _worse(worst: float, e: float) -> float:
    # a NaN error counts as infinitely bad (Python's max() would drop it)
    if math.isnan(e):
        return float("inf")
    return e if e > worst else worst


def max_rel_l2_per_head(x, ref, cu_seqlens=None) -> float:
    """Maximum over (sequence, head) of the relative L2 error on ``[T, H, D]`` arrays:
    ``max_{s,h} ||x[a_s:b_s, h] - ref[a_s:b_s, h]|| / ||ref[a_s:b_s, h]||`` with
    ``[a_s, b_s)`` the rows of sequence s (all T rows when ``cu_seqlens`` is None).
    Empty sequences contribute nothing; rows outside every sequence are not allowed
    (``cu_seqlens`` must run from 0 to T)."""
    x, ref = _f64(x), _f64(ref)
    if x.shape != ref.shape or ref.ndim != 3:
        raise ValueError(f"x and ref must share one [T, H, D] shape: {x.shape} vs {ref.shape}")
    T, H, _ = ref.shape
    cu = _cu(cu_seqlens, T)
    if cu.ndim != 1 or len(cu) < 2 or cu[0] != 0 or cu[-1] != T or np.any(np.diff(cu) < 0):
        raise ValueError("cu_seqlens must be non-decreasing from 0 to T")
    worst = 0.0
    for s in range(len(cu) - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        if b == a:
            continue
        for h in range(H):
            worst = _worse(worst, rel_l2(x[a:b, h, :], ref[a:b, h, :]))
    return worst


def max_rel_l2_per_state(x, ref) -> float:
    """Maximum over (sequence, head) of the relative L2 error on ``[S, H, D, D]``
    states.  A zero reference state (an empty sequence) must be matched exactly:
    any non-zero value there gives inf."""
    x, ref = _f64(x), _f64(ref)
    if x.shape != ref.shape or ref.ndim != 4:
        raise ValueError(f"x and ref must share one [S, H, D, D] shape: {x.shape} vs {ref.shape}")
    S, H = ref.shape[:2]
    worst = 0.0
    for s in range(S):
        for h in range(H):
            worst = _worse(worst, rel_l2(x[s, h], ref[s, h]))
    return worst
