"""Pins of the parity checker itself (CPU only).

Every GPU parity test reduces to ``oracle.max_rel_l2_per_head`` (outputs) or
``oracle.max_rel_l2_per_state`` (states): the relative L2 error per (sequence, head),
maximum reported (the error metric the method's tolerances are stated in: 1e-5 for
the fp32 path, 2e-2 for bf16).  A slip in these functions would make every parity
test pass vacuously, so they are pinned here against values fixed by construction:

* identical arrays give exactly 0;
* scaling one (sequence, head) slice by (1 + eps) gives exactly eps (up to rounding),
  whichever slice it is, including the last head of the last sequence;
* a perturbation that lies in another slice does not leak into the one measured;
* the metric is relative (invariant to a common scale);
* NaN or inf anywhere in the output, even in one head, gives inf;
* a zero reference state must be matched exactly.

``CHECKS`` below runs every pin against a given pair of functions; the real checker
must pass all of them, and each planted mistake (skipping the last sequence, slicing
``x[a:b][h]`` instead of ``x[a:b, h]``, returning before the loop, folding with
Python's ``max`` so that NaN is dropped, ignoring heads) must fail at least one.
"""
import math

import numpy as np
import pytest

import oracle

CU = [0, 5, 5, 12, 20]          # three non-empty sequences and one empty one
T, H, D = 20, 3, 4


def _ref(seed=0):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((T, H, D))


def _scaled(ref, s, h, eps, cu=CU):
    x = ref.copy()
    a, b = cu[s], cu[s + 1]
    x[a:b, h, :] *= 1.0 + eps
    return x


def _pin_identical(fn):
    r = _ref()
    return fn(r.copy(), r, CU) == 0.0


def _pin_each_slice(fn):
    r = _ref(1)
    for s in range(len(CU) - 1):
        if CU[s + 1] == CU[s]:
            continue
        for h in range(H):
            eps = 1e-3 * (1 + s * H + h)
            e = fn(_scaled(r, s, h, eps), r, CU)
            if not (abs(e - eps) <= 1e-12 * (1 + eps)):
                return False
    return True


def _pin_last_slice(fn):
    r = _ref(2)
    e = fn(_scaled(r, len(CU) - 2, H - 1, 3e-2), r, CU)
    return abs(e - 3e-2) <= 1e-12


def _pin_max_of_two(fn):
    r = _ref(3)
    x = _scaled(r, 0, 0, 1e-2)
    x[CU[2]:CU[3], 1, :] *= 1.05      # sequence 2, head 1: the larger one
    return abs(fn(x, r, CU) - 5e-2) <= 1e-12


def _pin_relative(fn):
    r = _ref(4)
    x = _scaled(r, 2, 2, 7e-3)
    return abs(fn(1e6 * x, 1e6 * r, CU) - 7e-3) <= 1e-12


def _pin_no_cu(fn):
    r = _ref(5)
    x = r.copy()
    x[:, 1, :] *= 1.02
    return abs(fn(x, r, None) - 2e-2) <= 1e-12


def _pin_nan_one_head(fn):
    r = _ref(6)
    x = r.copy()
    x[CU[3] + 1, H - 1, 0] = np.nan
    e = fn(x, r, CU)
    return math.isinf(e) and e > 0


def _pin_all_nan(fn):
    r = _ref(7)
    e = fn(np.full_like(r, np.nan), r, CU)
    return math.isinf(e) and e > 0


def _pin_inf(fn):
    r = _ref(8)
    x = r.copy()
    x[0, 0, 0] = np.inf
    e = fn(x, r, CU)
    return math.isinf(e) and e > 0


CHECKS = [_pin_identical, _pin_each_slice, _pin_last_slice, _pin_max_of_two, _pin_relative,
          _pin_no_cu, _pin_nan_one_head, _pin_all_nan, _pin_inf]


@pytest.mark.parametrize("pin", CHECKS, ids=[c.__name__[5:] for c in CHECKS])
def test_checker_pins(pin):
    assert pin(oracle.max_rel_l2_per_head)


# ---------------------------------------------------------------- planted mistakes
def _m_skip_last(x, ref, cu):
    x, ref = np.asarray(x, float), np.asarray(ref, float)
    cu = [0, len(ref)] if cu is None else cu
    worst = 0.0
    for s in range(len(cu) - 2):
        a, b = cu[s], cu[s + 1]
        for h in range(ref.shape[1]):
            if b > a:
                worst = max(worst, oracle.rel_l2(x[a:b, h], ref[a:b, h]))
    return worst


def _m_bad_slice(x, ref, cu):
    x, ref = np.asarray(x, float), np.asarray(ref, float)
    cu = [0, len(ref)] if cu is None else cu
    worst = 0.0
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        for h in range(ref.shape[1]):
            if b > a and h < b - a:
                worst = max(worst, oracle.rel_l2(x[a:b][h], ref[a:b][h]))
    return worst


def _m_early_return(x, ref, cu):
    x, ref = np.asarray(x, float), np.asarray(ref, float)
    cu = [0, len(ref)] if cu is None else cu
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        if b > a:
            return oracle.rel_l2(x[a:b, 0], ref[a:b, 0])
    return 0.0


def _m_python_max_nan(x, ref, cu):
    # the fold that drops NaN, with a rel_l2 that lets NaN through
    x, ref = np.asarray(x, float), np.asarray(ref, float)
    cu = [0, len(ref)] if cu is None else cu
    worst = 0.0
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        for h in range(ref.shape[1]):
            if b > a:
                num = np.linalg.norm((x[a:b, h] - ref[a:b, h]).ravel())
                worst = max(worst, float(num / np.linalg.norm(ref[a:b, h].ravel())))
    return worst


def _m_whole_sequence(x, ref, cu):
    # per sequence over all heads at once: a bad head is diluted by the good ones
    x, ref = np.asarray(x, float), np.asarray(ref, float)
    cu = [0, len(ref)] if cu is None else cu
    worst = 0.0
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        if b > a:
            worst = max(worst, oracle.rel_l2(x[a:b], ref[a:b]))
    return worst


MUTANTS = [_m_skip_last, _m_bad_slice, _m_early_return, _m_python_max_nan, _m_whole_sequence]


@pytest.mark.parametrize("mutant", MUTANTS, ids=[m.__name__[3:] for m in MUTANTS])
def test_checker_mutant_caught(mutant):
    with np.errstate(all="ignore"):
        failed = [c.__name__ for c in CHECKS if not _safe(c, mutant)]
    assert failed, f"{mutant.__name__} passes every pin"


def _safe(check, fn):
    try:
        return bool(check(fn))
    except Exception:
        return False


# ---------------------------------------------------------------- the state checker
def test_state_checker():
    rng = np.random.default_rng(9)
    ref = rng.standard_normal((3, 2, 4, 4))
    ref[1] = 0.0                                  # an empty sequence: zero state
    assert oracle.max_rel_l2_per_state(ref.copy(), ref) == 0.0
    x = ref.copy()
    x[2, 1] *= 1.04
    assert abs(oracle.max_rel_l2_per_state(x, ref) - 4e-2) <= 1e-12
    x = ref.copy()
    x[1, 0, 3, 3] = 1e-30                         # non-zero where the state must be zero
    assert math.isinf(oracle.max_rel_l2_per_state(x, ref))
    x = ref.copy()
    x[0, 1, 0, 0] = np.nan
    assert math.isinf(oracle.max_rel_l2_per_state(x, ref))


def test_checker_rejects_bad_arguments():
    r = _ref()
    with pytest.raises(ValueError):
        oracle.max_rel_l2_per_head(r[:-1], r, None)            # shapes differ
    with pytest.raises(ValueError):
        oracle.max_rel_l2_per_head(r, r, [0, 5, 19])           # does not reach T
    with pytest.raises(ValueError):
        oracle.max_rel_l2_per_head(r, r, [0, 7, 5, 20])        # decreasing
    bad = r.copy()
    bad[0, 0, 0] = np.nan
    with pytest.raises(ValueError):
        oracle.max_rel_l2_per_head(r, bad, None)               # non-finite reference
    with pytest.raises(ValueError):
        oracle.max_rel_l2_per_state(np.zeros((2, 1, 4, 4)), np.zeros((1, 2, 4, 4)))
