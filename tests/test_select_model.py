"""Host model of the kernel's exact top-r selection (bisection on the integer score with the
early exit at exactly r, then the start-position cut of ties), step for step as select_top_r in
alhr_device.cuh does it, checked against a plain sort on random and adversarial inputs.
This tests the selection algorithm the CUDA code follows; the GPU parity tests check the code."""
import numpy as np
import pytest


def model_threshold(scores, starts, r):
    """Returns (T, U): keep score > T, and score == T with start <= U (U = +inf: all ties)."""
    sc = np.asarray(scores, dtype=np.int64)
    lo, hi = int(sc.min()), int(sc.max())
    for _ in range(70):
        if lo >= hi:
            break
        mid = lo + ((hi - lo + 1) >> 1)
        c = int((sc >= mid).sum())
        if c == r:          # early exit: exactly r at or above the midpoint
            return mid, 2**31 - 1
        if c > r:
            lo = mid
        else:
            hi = mid - 1
    T = lo
    gt = int((sc > T).sum())
    eq = int((sc == T).sum())
    need = r - gt
    U = 2**31 - 1
    if need < eq:
        lo2, hi2 = 0, 2**31 - 1
        st = np.asarray(starts)
        for _ in range(34):
            if lo2 >= hi2:
                break
            mid = lo2 + ((hi2 - lo2) >> 1)
            c = int(((sc == T) & (st <= mid)).sum())
            if c >= need:
                hi2 = mid
            else:
                lo2 = mid + 1
        U = lo2
    return T, U


def kept_by_model(scores, starts, r):
    T, U = model_threshold(scores, starts, r)
    sc, st = np.asarray(scores), np.asarray(starts)
    return set(np.nonzero((sc > T) | ((sc == T) & (st <= U)))[0].tolist())


def kept_by_sort(scores, starts, r):
    order = sorted(range(len(scores)), key=lambda k: (-int(scores[k]), int(starts[k])))
    return set(order[:r])


@pytest.mark.parametrize("trial", range(300))
def test_selection_model_matches_sort(trial):
    rng = np.random.default_rng(trial)
    C = int(rng.integers(2, 193))
    r = int(rng.integers(1, C))
    kind = trial % 5
    if kind == 0:
        scores = rng.integers(-2**28, 2**28, size=C)
    elif kind == 1:
        scores = rng.integers(-3, 4, size=C)            # heavy ties
    elif kind == 2:
        scores = np.full(C, 7)                           # all tied
    elif kind == 3:
        scores = rng.integers(-2**33, 2**33, size=C)    # 64-bit range
    else:
        base = rng.integers(-1000, 1000, size=C)
        scores = base * 2**20 + rng.integers(0, 3, size=C)  # clustered with gaps
    starts = rng.choice(1 << 20, size=C, replace=False)
    assert kept_by_model(scores, starts, r) == kept_by_sort(scores, starts, r)
    assert len(kept_by_model(scores, starts, r)) == r
