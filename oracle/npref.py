"""NumPy twin of the oracle for tiny cases (TEST INFRASTRUCTURE ONLY).

Independent restatement of the same definitions as ``la_oracle.c`` so that
the C oracle has a second, differently written implementation beside it:

* ``quadratic_np``: builds the causal 0/1 mask M of each sequence explicitly
  and evaluates ((Q K^T) * M) V with numpy matmuls (MiniMax-01, CSDN digest
  section 2.1: intra-block masked left product; softmax replaced by an
  element-wise product, emonzhong.com summary, "method").
* ``recurrent_np``: per-token outer-product updates of the D x D state.
* ``brute_force``: pure-Python triple loop over i, j, d (tiny inputs only).
"""
from __future__ import annotations

import math

import numpy as np


def _cu(cu_seqlens, T):
    return [0, T] if cu_seqlens is None else [int(c) for c in cu_seqlens]


def _norm(o, eps):
    ms = np.mean(o * o, axis=-1, keepdims=True)
    return o / np.sqrt(ms + eps)


def quadratic_np(q, k, v, cu_seqlens=None, rmsnorm=False, eps=1e-6):
    q, k, v = (np.asarray(x, np.float64) for x in (q, k, v))
    T, H, D = q.shape
    cu = _cu(cu_seqlens, T)
    o = np.zeros_like(q)
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        n = b - a
        M = np.tril(np.ones((n, n)))
        for h in range(H):
            A = (q[a:b, h] @ k[a:b, h].T) * M
            o[a:b, h] = A @ v[a:b, h]
    return _norm(o, eps) if rmsnorm else o


def recurrent_np(q, k, v, cu_seqlens=None, rmsnorm=False, eps=1e-6):
    q, k, v = (np.asarray(x, np.float64) for x in (q, k, v))
    T, H, D = q.shape
    cu = _cu(cu_seqlens, T)
    o = np.zeros_like(q)
    states = np.zeros((len(cu) - 1, H, D, D))
    for s in range(len(cu) - 1):
        for h in range(H):
            KV = np.zeros((D, D))
            for t in range(cu[s], cu[s + 1]):
                KV = KV + np.outer(k[t, h], v[t, h])
                o[t, h] = q[t, h] @ KV
            states[s, h] = KV
    return (_norm(o, eps) if rmsnorm else o), states


def brute_force(q, k, v, cu_seqlens=None, rmsnorm=False, eps=1e-6):
    """Pure-Python loops; O[i][d] = sum_{j<=i in seq} (sum_e q[i][e] k[j][e]) v[j][d]."""
    T, H, D = len(q), len(q[0]), len(q[0][0])
    cu = _cu(cu_seqlens, T)
    out = [[[0.0] * D for _ in range(H)] for _ in range(T)]
    for s in range(len(cu) - 1):
        for h in range(H):
            for i in range(cu[s], cu[s + 1]):
                for j in range(cu[s], i + 1):
                    w = 0.0
                    for e in range(D):
                        w += float(q[i][h][e]) * float(k[j][h][e])
                    for d in range(D):
                        out[i][h][d] += w * float(v[j][h][d])
                if rmsnorm:
                    ms = sum(x * x for x in out[i][h]) / D
                    r = math.sqrt(ms + eps)
                    out[i][h] = [x / r for x in out[i][h]]
    return np.array(out, dtype=np.float64)
