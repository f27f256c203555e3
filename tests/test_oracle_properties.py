"""Property tests of the oracle (hypothesis).  Top-p: generated small rows, ties and zeros
included, checked against brute force over every subset and against the threshold reading of the
bisection ([Notes] "Key designs": the minimal top-p set, and the bisection on m that finds it
without a sort); fp32 softmax rows of up to 3000 weights against the same readings.  The whole
decode step: generated small layers checked stage by stage against the definitions.

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


softmax_rows = st.fixed_dictionaries({
    "seed": st.integers(0, 10_000),
    "n": st.integers(1, 3000),
    "sigma": st.sampled_from([0.1, 1.0, 3.0, 8.0]),
    "ties": st.booleans(),
    "p": st.sampled_from([0.3, 0.8, 0.85, 0.9, 0.99, 0.999999]),
    "eps": st.sampled_from([1e-9, 1e-6, 1e-3]),
})


@settings(max_examples=80, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(softmax_rows)
def test_bisection_on_softmax_rows(c):
    """fp32 softmax rows of up to 3000 weights (flat to peaked, with or without runs of equal
    logits): the bisection equals its threshold replay, keeps {W >= m} with mass >= p, and keeps
    at most the minimal set plus its epsilon band."""
    rng = np.random.default_rng(c["seed"])
    x = rng.normal(0.0, c["sigma"], c["n"])
    if c["ties"]:
        x = np.round(x * 2) / 2                           # runs of equal logits
    w = O.softmax64(x).astype(F32)
    p, eps = c["p"], c["eps"]
    m, kept = O.top_p_bisect(w, p, eps)
    assert F32(m) == _bisect_replay_from_threshold(w, p, eps)
    w64 = w.astype(F64)
    assert np.array_equal(kept, np.nonzero(w >= m)[0])
    assert w64[kept].sum() >= min(p, w64.sum())
    k_star, m_star, _ = O.top_p_sort(w, p)
    band = np.count_nonzero((w64 >= F64(m_star) - eps) & (w64 <= F64(m_star)))
    assert len(kept) <= k_star + band


# ------------------------------------------------------------------ the whole step, as invariants

layers = st.fixed_dictionaries({
    "seed": st.integers(0, 10_000),
    "hkv": st.sampled_from([1, 2]),
    "g": st.sampled_from([1, 2, 4]),
    "lens": st.lists(st.integers(1, 300), min_size=1, max_size=2),
    "p": st.sampled_from([0.5, 0.85, 0.95, 1.0]),
    "temperature": st.booleans(),
    "budget_pages": st.sampled_from([0, 0, 1, 5]),
})


@settings(max_examples=30, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(layers)
def test_decode_step_invariants(c):
    """Generated small layers (ragged lengths, 1 to 4 heads per group, permuted pages, p up to 1):
    every stage of the oracle's step satisfies what the method defines it to be, checked from the
    definitions rather than by re-running the oracle's routines.
      selection   ceil(P_b / 4) (or the fixed budget, at most P_b) distinct pages, ascending
      candidates  exactly the valid tokens of the selected pages
      estimate    weights >= 0 summing to 1
      top-p       kept = {W >= m*}; its mass reaches p; the weights above m* alone do not
                  (at p = 1 every candidate is kept)
      union       the union of the group's kept tokens, inside the sequence
      attention   o is a convex combination of the union's V rows (channel-wise inside their
                  range) and lse lies in [max logit, max logit + ln |U|]"""
    from workloads import synth
    hkv, g = c["hkv"], c["g"]
    wl = synth.make_decode("prop", len(c["lens"]), g * hkv, hkv, c["lens"], seed=c["seed"],
                           permute_pages=True, temperature=c["temperature"], p=c["p"],
                           budget_pages=c["budget_pages"])
    kb = lambda pb: min(c["budget_pages"], pb) if c["budget_pages"] > 0 else -(-pb // 4)
    r = O.decode_step(wl)
    scale = 1 / np.sqrt(128)
    for b, n in enumerate(wl.seq_lens):
        n = int(n)
        pb = -(-n // 16)
        for kvh in range(hkv):
            union = set()
            for h in range(kvh * g, (kvh + 1) * g):
                hd = r["heads"][(b, h)]
                sel = list(hd["sel"])
                assert len(sel) == kb(pb) and sel == sorted(set(sel))
                assert all(0 <= j < pb for j in sel)
                assert list(hd["cand"]) == [t for t in range(n) if t // 16 in set(sel)]
                w = hd["w"]
                assert np.all(w >= 0) and abs(w.sum() - 1.0) < 1e-12
                m = hd["m_star"]
                assert list(hd["kept"]) == list(np.nonzero(w >= m)[0])
                if wl.p == 1.0:                       # R10: p = 1 keeps every candidate
                    assert len(hd["kept"]) == len(w)
                else:
                    assert w[w >= m].sum() >= wl.p and w[w > m].sum() < wl.p
                union |= set(hd["kept_tok"].tolist())
            grp = r["groups"][(b, kvh)]
            assert list(grp["union"]) == sorted(union) and max(union) < n
            rows = [(int(wl.page_table[b, t // 16]), t % 16) for t in sorted(union)]
            kk = np.stack([wl.k[ph, kvh, i] for ph, i in rows]).astype(F64)
            vv = np.stack([wl.v[ph, kvh, i] for ph, i in rows]).astype(F64)
            for h in range(kvh * g, (kvh + 1) * g):
                o, lse = grp["o"][h], grp["lse"][h]
                assert np.all(o >= vv.min(axis=0) - 1e-12) and np.all(o <= vv.max(axis=0) + 1e-12)
                top = float((kk @ wl.q[b, h].astype(F64)).max()) * scale
                assert top - 1e-12 <= lse <= top + np.log(len(rows)) + 1e-12
