"""Pins of the fp64 oracle to facts outside itself.

Each ``pin_*`` function raises AssertionError when the oracle (the build that
``oracle.use_library`` currently selects) disagrees with something the pages
or the mathematics fix:

* hand-worked integer examples (``tests/golden/hand_worked.json``);
* brute force: a pure-Python triple loop on tiny inputs;
* special cases with a textbook answer (D = 1 reduces to ``numpy.cumsum``,
  Q = K = e1 gives cumsum(V), orthogonal Q/K give zero, one token gives
  (q.k) v), the final state equal to a library K^T V;
* invariants: linearity, scaling, packed = separate runs, block-size
  independence, decode step = the next prefill row, a sequence run in two
  chunks (the second from the first one's state) = the single run.

``test_oracle.py`` runs them against the oracle; ``test_oracle_mutants.py``
runs them against deliberately broken builds and requires each one to fail.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

import oracle
from oracle import npref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")
TIGHT = 1e-12


def _close(x, ref, tol=TIGHT, what=""):
    err = oracle.rel_l2(x, ref)
    assert err <= tol, f"{what}: rel L2 {err:.3e} > {tol:.0e}"


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def pin_golden_single():
    g = _golden()["single_sequence"]
    q, k, v = (np.array(g[n], np.float64) for n in "qkv")
    o_ref, st_ref = np.array(g["o"], np.float64), np.array(g["state"], np.float64)
    for name, (o, st) in {"quadratic": oracle.quadratic(q, k, v),
                          "recurrent": oracle.recurrent(q, k, v),
                          "blocked1": oracle.blocked(q, k, v, 1),
                          "blocked2": oracle.blocked(q, k, v, 2),
                          "blocked8": oracle.blocked(q, k, v, 8)}.items():
        assert np.array_equal(o, o_ref), f"{name} output {o.tolist()}"
        assert np.array_equal(st, st_ref), f"{name} state {st.tolist()}"


def pin_golden_packed():
    g = _golden()
    q, k, v = (np.array(g["single_sequence"][n], np.float64) for n in "qkv")
    p = g["packed_two_sequences"]
    for fn in (oracle.quadratic, oracle.recurrent, lambda *a: oracle.blocked(*a[:3], 2, a[3])):
        o, st = fn(q, k, v, p["cu_seqlens"])
        assert np.array_equal(o, np.array(p["o"], np.float64)), o.tolist()
        assert np.array_equal(st, np.array(p["state"], np.float64)), st.tolist()


def pin_golden_rmsnorm():
    g = _golden()
    q, k, v = (np.array(g["single_sequence"][n], np.float64) for n in "qkv")
    r = g["rmsnorm_row"]
    for fn in (oracle.quadratic, oracle.recurrent, lambda *a, **kw: oracle.blocked(*a, 2, **kw)):
        o, _ = fn(q, k, v, rmsnorm=True, eps=r["eps"])
        _close(o[1, 0], np.array(r["y"]), 1e-15, "rmsnorm of [4,1]")
        # row 0 is [1,0]: mean square 0.5
        _close(o[0, 0], np.array([1.0, 0.0]) / math.sqrt(0.5 + r["eps"]), 1e-15, "rmsnorm [1,0]")


def pin_golden_decode():
    g = _golden()["decode_step"]
    st, q, k, v = (np.array(g[n], np.float64) for n in ("state", "q", "k", "v"))
    o, new = oracle.decode_step(q, k, v, st)
    assert np.array_equal(new, np.array(g["new_state"], np.float64)), new.tolist()
    assert np.array_equal(o, np.array(g["o"], np.float64)), o.tolist()


def pin_brute_force():
    T, H, D = 11, 2, 3
    q, k, v = _rand((T, H, D), 1), _rand((T, H, D), 2), _rand((T, H, D), 3)
    cu = [0, 4, 4, 11]
    for rms in (False, True):
        ref = npref.brute_force(q.tolist(), k.tolist(), v.tolist(), cu, rmsnorm=rms)
        _close(oracle.quadratic(q, k, v, cu, rmsnorm=rms)[0], ref, what="quadratic")
        _close(oracle.recurrent(q, k, v, cu, rmsnorm=rms)[0], ref, what="recurrent")
        for beta in (1, 2, 3, 5, 16):
            _close(oracle.blocked(q, k, v, beta, cu, rmsnorm=rms)[0], ref, what=f"blocked{beta}")
        _close(npref.quadratic_np(q, k, v, cu, rmsnorm=rms), ref, what="numpy quadratic")
        _close(npref.recurrent_np(q, k, v, cu, rmsnorm=rms)[0], ref, what="numpy recurrent")


def pin_forms_agree():
    """Block-size independence and quadratic = recurrent = blocked (exact algebra)."""
    T, H, D = 300, 3, 16
    q, k, v = _rand((T, H, D), 4), _rand((T, H, D), 5), _rand((T, H, D), 6)
    cu = [0, 1, 1, 97, 300]
    o_q, s_q = oracle.quadratic(q, k, v, cu)
    o_r, s_r = oracle.recurrent(q, k, v, cu)
    _close(o_r, o_q, what="recurrent vs quadratic")
    _close(s_r, s_q, what="state recurrent vs quadratic")
    for beta in (1, 7, 64, 128, 1000):
        o_b, s_b = oracle.blocked(q, k, v, beta, cu)
        _close(o_b, o_q, what=f"blocked beta={beta}")
        _close(s_b, s_q, what=f"state blocked beta={beta}")


def pin_d1_cumsum():
    """D = 1: O_i = q_i * sum_{j<=i} k_j v_j, a numpy cumulative sum."""
    T = 50
    q, k, v = _rand((T, 1, 1), 7), _rand((T, 1, 1), 8), _rand((T, 1, 1), 9)
    ref = q[:, 0, 0] * np.cumsum(k[:, 0, 0] * v[:, 0, 0])
    for fn in (oracle.quadratic, oracle.recurrent, lambda *a: oracle.blocked(*a, 8)):
        _close(fn(q, k, v)[0][:, 0, 0], ref, what="D=1 cumsum")


def pin_e1_cumsum_v():
    """Q = K = rows e1: every score is 1, so O = cumsum(V) along the sequence."""
    T, H, D = 37, 2, 5
    q = np.zeros((T, H, D)); q[:, :, 0] = 1.0
    v = _rand((T, H, D), 10)
    ref = np.cumsum(v, axis=0)
    for fn in (oracle.quadratic, oracle.recurrent, lambda *a: oracle.blocked(*a, 4)):
        _close(fn(q, q.copy(), v)[0], ref, what="Q=K=e1")


def pin_orthogonal_zero():
    """Q rows e_a and K rows e_b with a != b: every score is 0, so O = 0."""
    T, H, D = 29, 1, 4
    q = np.zeros((T, H, D)); q[:, :, 1] = 1.0
    k = np.zeros((T, H, D)); k[:, :, 3] = 1.0
    v = _rand((T, H, D), 11)
    for fn in (oracle.quadratic, oracle.recurrent, lambda *a: oracle.blocked(*a, 4)):
        o, _ = fn(q, k, v)
        assert np.all(o == 0.0)


def pin_single_token():
    """N = 1: o = (q . k) v."""
    H, D = 3, 8
    q, k, v = _rand((1, H, D), 12), _rand((1, H, D), 13), _rand((1, H, D), 14)
    ref = np.einsum("thd,thd->th", q, k)[..., None] * v
    for fn in (oracle.quadratic, oracle.recurrent, lambda *a: oracle.blocked(*a, 64)):
        _close(fn(q, k, v)[0], ref, what="single token")


def pin_state_is_ktv():
    T, H, D = 120, 2, 6
    k, v = _rand((T, H, D), 15), _rand((T, H, D), 16)
    cu = [0, 50, 50, 120]
    ref = np.zeros((3, H, D, D))
    for s in range(3):
        for h in range(H):
            ref[s, h] = np.dot(k[cu[s]:cu[s + 1], h].T, v[cu[s]:cu[s + 1], h])
    for fn in (oracle.quadratic, oracle.recurrent,
               lambda q_, k_, v_, c_: oracle.blocked(q_, k_, v_, 16, c_)):
        _close(fn(k, k, v, cu)[1], ref, what="state = K^T V")


def pin_linearity_and_scaling():
    T, H, D = 70, 2, 6
    q, k = _rand((T, H, D), 17), _rand((T, H, D), 18)
    v1, v2 = _rand((T, H, D), 19), _rand((T, H, D), 20)
    o1 = oracle.blocked(q, k, v1, 16)[0]
    o2 = oracle.blocked(q, k, v2, 16)[0]
    _close(oracle.blocked(q, k, v1 + v2, 16)[0], o1 + o2, 1e-11, "linear in V")
    _close(oracle.blocked(2.5 * q, k, v1, 16)[0], 2.5 * o1, 1e-11, "O(aQ) = a O")
    # RMSNorm output does not change when Q is scaled (eps is negligible here)
    n1 = oracle.recurrent(q, k, v1, rmsnorm=True, eps=0.0)[0]
    n2 = oracle.recurrent(3.0 * q, k, v1, rmsnorm=True, eps=0.0)[0]
    _close(n2, n1, 1e-11, "RMSNorm scale invariance")


def pin_packed_equals_separate():
    T, H, D = 90, 2, 5
    q, k, v = _rand((T, H, D), 21), _rand((T, H, D), 22), _rand((T, H, D), 23)
    cu = [0, 33, 34, 90]
    o_p, s_p = oracle.blocked(q, k, v, 8, cu)
    for s in range(3):
        a, b = cu[s], cu[s + 1]
        o_s, st_s = oracle.blocked(q[a:b], k[a:b], v[a:b], 8)
        _close(o_p[a:b], o_s, what=f"packed seq {s}")
        _close(s_p[s], st_s[0], what=f"packed state {s}")
    # the state after sequence 2 does not depend on sequences 0 and 1
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    k2[:34] = _rand((34, H, D), 24)
    v2[:34] = _rand((34, H, D), 25)
    _close(oracle.blocked(q2, k2, v2, 8, cu)[1][2], s_p[2], what="reset at boundary")


def pin_decode_is_next_row():
    """decode(state of prefill_N, token N+1) = row N+1 of prefill_{N+1}."""
    N, H, D = 40, 2, 6
    q, k, v = _rand((N + 1, H, D), 26), _rand((N + 1, H, D), 27), _rand((N + 1, H, D), 28)
    for rms in (False, True):
        _, st = oracle.recurrent(q[:N], k[:N], v[:N], want_o=False)
        o_full, st_full = oracle.quadratic(q, k, v, rmsnorm=rms)
        o_dec, st_dec = oracle.decode_step(q[N:N + 1], k[N:N + 1], v[N:N + 1], st, rmsnorm=rms)
        _close(o_dec[0], o_full[N], 1e-11, "decode = next prefill row")
        _close(st_dec, st_full, 1e-11, "decode state")


def _forms_with_state():
    return {"quadratic": oracle.quadratic, "recurrent": oracle.recurrent,
            "blocked3": lambda *a, **kw: oracle.blocked(a[0], a[1], a[2], 3, *a[3:], **kw),
            "blocked16": lambda *a, **kw: oracle.blocked(a[0], a[1], a[2], 16, *a[3:], **kw)}


def pin_chunked_equals_whole():
    """Initial state: running each sequence in two chunks, the second one starting
    from the first one's final state, reproduces the single run (rows and states)."""
    T, H, D = 160, 2, 6
    q, k, v = _rand((T, H, D), 40), _rand((T, H, D), 41), _rand((T, H, D), 42)
    cu = [0, 45, 45, 160]                      # lengths 45, 0, 115
    for rms in (False, True):
        ref_o, ref_s = oracle.quadratic(q, k, v, cu, rmsnorm=rms)
        for cut in ((0, 0, 0), (20, 0, 50), (45, 0, 115), (1, 0, 63)):
            # chunk 1 of every sequence packed together, then chunk 2 of every sequence
            c1, c2, rows1, rows2 = [0], [0], [], []
            for s in range(3):
                a, b = cu[s], cu[s + 1]
                m = a + cut[s]
                rows1 += list(range(a, m))
                rows2 += list(range(m, b))
                c1.append(len(rows1))
                c2.append(len(rows2))
            for name, fn in _forms_with_state().items():
                o1, s1 = fn(q[rows1], k[rows1], v[rows1], c1, rmsnorm=rms)
                o2, s2 = fn(q[rows2], k[rows2], v[rows2], c2, rmsnorm=rms, initial_state=s1)
                _close(o1, ref_o[rows1], 1e-11, f"{name} chunk 1 cut {cut}")
                _close(o2, ref_o[rows2], 1e-11, f"{name} chunk 2 cut {cut}")
                _close(s2, ref_s, 1e-11, f"{name} state after chunk 2 cut {cut}")


def pin_d1_cumsum_with_state():
    """D = 1 with initial state x: O_i = q_i (x + sum_{j<=i} k_j v_j), a numpy cumsum."""
    T = 40
    q, k, v = _rand((T, 1, 1), 43), _rand((T, 1, 1), 44), _rand((T, 1, 1), 45)
    x = np.array([[[[1.75]]]])
    ref = q[:, 0, 0] * (1.75 + np.cumsum(k[:, 0, 0] * v[:, 0, 0]))
    for name, fn in _forms_with_state().items():
        o, st = fn(q, k, v, initial_state=x)
        _close(o[:, 0, 0], ref, what=f"{name} D=1 cumsum with state")
        _close(st[0, 0, 0, 0], ref[-1] / q[-1, 0, 0], 1e-11, f"{name} D=1 final state")


def pin_one_token_with_state_is_decode():
    """A one-token sequence continuing from state X is one decode step from X."""
    H, D = 3, 7
    q, k, v = _rand((1, H, D), 46), _rand((1, H, D), 47), _rand((1, H, D), 48)
    X = _rand((1, H, D, D), 49)
    for rms in (False, True):
        o_dec, st_dec = oracle.decode_step(q, k, v, X, rmsnorm=rms)
        for name, fn in _forms_with_state().items():
            o, st = fn(q, k, v, rmsnorm=rms, initial_state=X)
            _close(o, o_dec, 1e-11, f"{name} one token with state")
            _close(st, st_dec, 1e-11, f"{name} state after one token")


def pin_empty_sequence_keeps_state():
    """A zero-length sequence leaves its initial state unchanged (exactly)."""
    H, D = 2, 5
    q = k = v = np.zeros((3, H, D))
    X = _rand((2, H, D, D), 50)
    for name, fn in _forms_with_state().items():
        _, st = fn(q + _rand((3, H, D), 51), k + _rand((3, H, D), 52), v + _rand((3, H, D), 53),
                   [0, 0, 3], initial_state=X)
        assert np.array_equal(st[0], X[0]), f"{name} empty sequence state"


ALL_PINS = [v for n, v in sorted(globals().items()) if n.startswith("pin_")]
