"""Property tests of the oracle's top-p (hypothesis): generated small rows, ties and zeros
included, checked against brute force over every subset and against the threshold reading of the
bisection ([Notes] "Key designs": the minimal top-p set, and the bisection on m that finds it
without a sort).

Weights are multiples of 2^-20 in [0, 1], so every sum of up to 10 of them is exact in fp64 and
the brute force needs no rounding argument.
"""
import itertools

import numpy as np
from hypothesis import HealthCheck, assume, given, settings
from hypothesis import strategies as st

from oracle import twl_oracle as O
from tests.test_oracle_pins import _bisect_replay_from_threshold

F32, F64 = np.float32, np.float64

_grid = st.one_of(st.sampled_from([0, 1 << 18, 1 << 19, 1 << 20]), st.integers(0, 1 << 20))
rows = st.lists(_grid, min_size=1, max_size=10).map(lambda v: np.array(v, F64) / (1 << 20))
fracs = st.floats(0.02, 1.0, allow_nan=False)
SETTINGS = settings(max_examples=250, deadline=None,
                    suppress_health_check=[HealthCheck.too_slow])


def _min_count_by_subsets(w, p):
    """Smallest subset size whose mass reaches p, over every subset (all n if none does)."""
    n = len(w)
    for k in range(1, n + 1):
        if any(sum(w[i] for i in s) >= p for s in itertools.combinations(range(n), k)):
            return k
    return n


@SETTINGS
@given(rows, fracs)
def test_sort_form_is_the_minimal_set(w, frac):
    assume(w.sum() > 0)
    p = frac * w.sum()
    k_star, m_star, kept = O.top_p_sort(w, p)
    assert k_star == _min_count_by_subsets(w, p)
    assert np.array_equal(kept, np.nonzero(w >= m_star)[0])
    if w.sum() >= p:
        assert w[kept].sum() >= p          # the threshold set reaches p ...
        assert w[w > m_star].sum() < p     # ... and no higher threshold does


@SETTINGS
@given(rows, st.floats(0.02, 0.999, allow_nan=False),
       st.sampled_from([1e-9, 1e-6, 1e-3, 0.05]))
def test_bisection_keeps_enough_within_its_band(w, frac, eps):
    w = (w / max(w.sum(), 1.0)).astype(F32)
    assume(w.astype(F64).sum() > 0)
    p = frac * float(w.astype(F64).sum())
    m, kept = O.top_p_bisect(w, p, eps)
    k_star, m_star, _ = O.top_p_sort(w, p)
    w64 = w.astype(F64)
    assert np.array_equal(kept, np.nonzero(w >= m)[0])
    assert w64[kept].sum() >= p            # the search never drops below p
    assert m <= m_star                     # it keeps the minimal set ...
    band = np.count_nonzero((w64 >= F64(m_star) - eps) & (w64 <= F64(m_star)))
    assert len(kept) <= k_star + band      # ... plus at most the entries in its epsilon band


@SETTINGS
@given(rows, st.floats(0.02, 0.999, allow_nan=False),
       st.sampled_from([1e-9, 1e-6, 1e-3]))
def test_bisection_equals_its_threshold_replay(w, frac, eps):
    w = (w / max(w.sum(), 1.0)).astype(F32)
    assume(w.astype(F64).sum() > 0)
    p = frac * float(w.astype(F64).sum())
    m, _ = O.top_p_bisect(w, p, eps)
    assert F32(m) == _bisect_replay_from_threshold(w, p, eps)
