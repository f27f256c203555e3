"""The parity criteria themselves (tests/twl_checks.py), on CPU: a result taken from the oracle
passes every check, and the same result with one planted mistake fails one.  This is what lets a
green GPU parity run mean something.
"""
import numpy as np
import pytest

from oracle import twl_oracle as O
from tests import twl_checks as K
from workloads import synth

F32, F64 = np.float32, np.float64


def _oracle_stats(wl):
    """The stats a correct device step would report, produced by the oracle (fp32 weights, the
    sort-based threshold rounded to fp32) in the layout of twl_step_stats."""
    r = O.decode_step(wl)
    B, hq, hkv = wl.batch, wl.num_q_heads, wl.num_kv_heads
    cs = 16 * wl.max_pages
    st = dict(sel_count=np.zeros((B, hq), np.int32), sel_pages=np.zeros((B, hq, wl.max_pages),
              np.int32), cand_count=np.zeros((B, hq), np.int32),
              cand_tok=np.zeros((B, hq, cs), np.int32), weights=np.zeros((B, hq, cs), F32),
              threshold=np.zeros((B, hq), F32), kept_count=np.zeros((B, hq), np.int32),
              union_count=np.zeros((B, hkv), np.int32), union_tok=np.zeros((B, hkv, cs), np.int32))
    o = np.zeros((B, hq, 128), F32)
    lse = np.zeros((B, hq), F32)
    for (b, h), hd in r["heads"].items():
        st["sel_count"][b, h] = len(hd["sel"])
        st["sel_pages"][b, h, :len(hd["sel"])] = hd["sel"]
        cc = hd["cand"].size
        st["cand_count"][b, h] = cc
        st["cand_tok"][b, h, :cc] = hd["cand"]
        w32 = hd["w"].astype(F32)
        st["weights"][b, h, :cc] = w32
        m = F32(hd["m_star"])
        st["threshold"][b, h] = m
        st["kept_count"][b, h] = int(np.count_nonzero(w32 >= m))
    g = hq // hkv
    for (b, kvh), grp in r["groups"].items():
        # the union of the fp32 kept sets (the checker recomputes kept from the fp32 weights)
        toks = set()
        for h in range(kvh * g, (kvh + 1) * g):
            cc = st["cand_count"][b, h]
            w32 = st["weights"][b, h, :cc]
            toks |= set(st["cand_tok"][b, h, :cc][w32 >= st["threshold"][b, h]].tolist())
        u = np.array(sorted(toks), np.int64)
        st["union_count"][b, kvh] = u.size
        st["union_tok"][b, kvh, :u.size] = u
        att = O.group_attention(wl, {(b, kvh): u})
        for h in range(kvh * g, (kvh + 1) * g):
            o[b, h], lse[b, h] = att[(b, h)]
    return st, o, lse


@pytest.fixture(scope="module")
def case():
    wl = synth.make_decode("chk", 1, 4, 2, [300], seed=12, permute_pages=True)
    st, o, lse = _oracle_stats(wl)
    return wl, st, o, lse


def _copy(st):
    return {k: v.copy() for k, v in st.items()}


def test_oracle_result_passes(case):
    wl, st, o, lse = case
    for kvh in range(wl.num_kv_heads):
        K.check_step_group(wl, 0, kvh, st, o, lse)


def _fails(wl, st, o, lse, kvh):
    with pytest.raises(AssertionError):
        K.check_step_group(wl, 0, kvh, st, o, lse)


def test_planted_selection_mistake_fails(case):
    wl, st, o, lse = case
    bad = _copy(st)
    cnt = bad["sel_count"][0, 1]
    pages = set(bad["sel_pages"][0, 1, :cnt].tolist())
    spare = next(j for j in range(O.num_pages(300)) if j not in pages)
    bad["sel_pages"][0, 1, cnt - 1] = spare          # one page swapped for an unselected one
    bad["sel_pages"][0, 1, :cnt].sort()
    _fails(wl, bad, o, lse, 0)


def test_planted_weight_mistake_fails(case):
    wl, st, o, lse = case
    bad = _copy(st)
    i = int(np.argmax(bad["weights"][0, 2, :bad["cand_count"][0, 2]]))
    bad["weights"][0, 2, i] *= F32(1.002)            # 2e-3 relative, above the 1e-3 criterion
    _fails(wl, bad, o, lse, 1)


def test_planted_threshold_and_count_mistakes_fail(case):
    wl, st, o, lse = case
    bad = _copy(st)
    bad["kept_count"][0, 0] += 1                     # count does not match {W >= m}
    _fails(wl, bad, o, lse, 0)
    # threshold too high (the largest kept weight of a head that keeps several): mass below p
    h = int(np.argmax(st["kept_count"][0]))
    assert st["kept_count"][0, h] >= 2
    bad = _copy(st)
    cc = bad["cand_count"][0, h]
    w = bad["weights"][0, h, :cc]
    bad["threshold"][0, h] = w.max()
    bad["kept_count"][0, h] = int(np.count_nonzero(w >= w.max()))
    _fails(wl, bad, o, lse, h // 2)
    bad = _copy(st)
    bad["threshold"][0, 0] = F32(0.0)                # threshold too low: keeps everything
    bad["kept_count"][0, 0] = bad["cand_count"][0, 0]
    _fails(wl, bad, o, lse, 0)


def test_planted_union_and_attention_mistakes_fail(case):
    wl, st, o, lse = case
    bad = _copy(st)
    uc = bad["union_count"][0, 1]
    bad["union_tok"][0, 1, :uc - 1] = bad["union_tok"][0, 1, 1:uc].copy()   # first token dropped
    bad["union_count"][0, 1] = uc - 1
    _fails(wl, bad, o, lse, 1)
    o2 = o.copy()
    o2[0, 3, 7] += 3e-3
    _fails(wl, st, o2, lse, 1)
    lse2 = lse.copy()
    lse2[0, 2] -= 3e-3
    _fails(wl, st, o, lse2, 1)


def test_prune_row_checks():
    w, _ = synth.config5_rows(4, 4096, seed=7)
    for row in w:
        m, kept = O.top_p_bisect(row, 0.9, 1e-6)
        K.check_prune_row(row, m, kept.size, kept, 0.9, 1e-6)
        assert kept.size > 1
        with pytest.raises(AssertionError):                       # ids out of order
            K.check_prune_row(row, m, kept.size, kept[::-1], 0.9, 1e-6)
        with pytest.raises(AssertionError):                       # count off by one
            K.check_prune_row(row, m, kept.size + 1, None, 0.9, 1e-6)
    # a plainly too-low threshold keeps more than k* plus the epsilon band
    row = w[0]
    k_star, m_star, _ = O.top_p_sort(row, 0.9)
    low = F32(m_star) * F32(0.5)
    with pytest.raises(AssertionError):
        K.check_prune_row(row, low, int(np.count_nonzero(row >= low)), None, 0.9, 1e-6)


def test_prune_check_at_p_one_takes_the_whole_row():
    """At p = 1 a pruner keeps every weight (m = 0).  fp32 weights that sum a little above 1
    (0.5 + 0.3 + 0.2 in fp32 is 1 + 1.5e-8) reach 1.0 after three of five entries, yet keeping
    all five is the reading's result and passes.  Below p = 1 the minimal set still binds:
    keeping all five at p = 0.9 fails."""
    w = np.array([0.5, 0.3, 0.2, 1e-8, 1e-8], np.float32)
    K.check_prune_row(w, 0.0, 5, None, 1.0, 1e-6, "p=1")
    with pytest.raises(AssertionError):
        K.check_prune_row(w, 0.0, 5, None, 0.9, 1e-6, "too many at p=0.9")
