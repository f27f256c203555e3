"""Pins for the CPU oracle: each check ties it to something other than itself.

Sources: [Notes] = "Twilight: Adaptive Attention Sparsity with Hierarchical Top-p Pruning",
Paper-Notes (NeurIPS 2025) page; [Summary] = the paperlayer summary of arXiv 2502.02770v5.

What pins what:
  bounds      invariant mn <= k <= mx with both attained; single-token page; partial page ignores
              rows past the sequence end; a plain scan over ragged, permuted caches salted with
              signed zeros (-0 before +0).
  INT4        hand-worked bytes (tests/golden/int4_rows.json, [Summary] B.1); round-trip error
              <= s/2 (+ fp16 rounding of s); memory identity 1/8 of the KV cache ([Notes] "Key
              designs", 4-bit K cache; [Summary] 4.3).
  scores      unit queries give the bound rows themselves; upper-bound property against every
              token of the page (fp64); equality for a page of identical tokens.
  top-k       brute-force full sort; whole page selection (GQA head map, budget rule, ties) by
              brute force in Python integers on integer-valued q and K (nine draws, four
              budgets).
  order key   every non-NaN fp16 bit pattern: keys rise strictly with the value, -0 before +0.
  softmax     closed forms (uniform; logits 0 and ln 3 give 1/4 and 3/4, also at +1000) and the
              definition term by term with math.fsum.
  estimate    K on the 16-level grid makes the dequantised K exact, so the estimate must equal
              torch's softmax of q.K/sqrt(D) computed from the raw fp16 K.
  top-p       hand examples (tests/golden/top_p_examples.json, [Notes] "Key designs"); p = 1
              keeps the whole distribution even where the fp64 prefix rounds to 1 early;
              brute-force subset search for n <= 14; mass(W >= m*) >= p > mass(W > m*);
              bisection result inside the epsilon band ([Notes] "Key designs", efficient top-p).
  gather      rows that carry their own (token, head, sequence) address, behind a permuted
              page table.
  attention   all tokens kept -> torch scaled_dot_product_attention in fp64; one token kept ->
              o = v_i, lse = q.k_i/sqrt(D); the error bound (1-p)*||V||_F ([Notes] "Key
              designs", oracle top-p guarantee).
  mutation    planted mistakes in copies of oracle functions fail these pins.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import twl_oracle as O
from workloads import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F16, F32, F64 = np.float16, np.float32, np.float64


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ------------------------------------------------------------------------------------- bounds

def check_bounds(bounds_fn, rng):
    k = rng.standard_normal((6, 2, 16, 128)).astype(F16)
    k[5, :, 7:] = F16(1000.0)                         # garbage past the end of sequence 1
    pt = np.array([[0, 1, 2], [3, 4, 5]], dtype=np.int32)
    lens = np.array([48, 39], dtype=np.int32)        # second sequence: last page has 7 rows
    bd = bounds_fn(k, pt, lens)
    ok = True
    for b in range(2):
        for j in range(3):
            phys = pt[b, j]
            r = O.valid_rows(lens[b], j)
            rows = k[phys, :, :r].astype(F64)
            mn = bd[phys, :, 0].astype(F64)
            mx = bd[phys, :, 1].astype(F64)
            ok &= bool(np.all(rows >= mn[:, None, :]) and np.all(rows <= mx[:, None, :]))
            ok &= bool(np.all(rows.min(axis=1) == mn) and np.all(rows.max(axis=1) == mx))
    return ok


def test_bounds_invariants():
    assert check_bounds(O.page_bounds, np.random.default_rng(1))


def check_bounds_brute(bounds_fn):
    """Ragged sequences behind permuted page tables, channels salted with +0 and -0: each bound is
    the smallest / largest valid value found by a plain scan that orders -0 before +0."""
    def tot(x):                                    # value, then -0 before +0
        return (float(x), not np.signbit(x))
    for seed in range(6):
        rng = np.random.default_rng(100 + seed)
        lens = rng.integers(1, 60, size=3)
        pages = [-(-int(n) // 16) for n in lens]
        p_phys = sum(pages) + 2
        perm = rng.permutation(p_phys)
        pt = np.full((3, max(pages)), -1, np.int32)
        o = 0
        for b, m in enumerate(pages):
            pt[b, :m] = perm[o:o + m]
            o += m
        k = rng.standard_normal((p_phys, 2, 16, 8)).astype(F16)
        zero = rng.random(k.shape) < 0.3
        k[zero] = np.where(rng.random(k.shape) < 0.5, F16(0.0), F16(-0.0))[zero]
        bd = bounds_fn(np.pad(k, ((0, 0), (0, 0), (0, 0), (0, 120))), pt, lens)
        for b, n in enumerate(lens):
            for j in range(pages[b]):
                ph, rows = pt[b, j], min(16, int(n) - 16 * j)
                for h in range(2):
                    for c in range(8):
                        col = list(k[ph, h, :rows, c])
                        lo, hi = min(col, key=tot), max(col, key=tot)
                        if u16_1(bd[ph, h, 0, c]) != u16_1(lo) or u16_1(bd[ph, h, 1, c]) != u16_1(hi):
                            return False
    return True


def test_bounds_by_brute_force_with_signed_zeros():
    assert check_bounds_brute(O.page_bounds)

    def numpy_min_max(k, pt, lens):              # np.min / np.max: -0 and +0 compare equal
        out = np.zeros((k.shape[0], k.shape[1], 2, k.shape[3]), F16)
        for b, n in enumerate(lens):
            for j in range(-(-int(n) // 16)):
                rows = k[pt[b, j], :, :min(16, int(n) - 16 * j)]
                out[pt[b, j], :, 0], out[pt[b, j], :, 1] = rows.min(axis=1), rows.max(axis=1)
        return out

    assert not check_bounds_brute(numpy_min_max)


def u16_1(x):
    return int(np.array([x], dtype=F16).view(np.uint16)[0])


def test_bounds_single_token_page():
    rng = np.random.default_rng(2)
    k = rng.standard_normal((1, 1, 16, 128)).astype(F16)
    bd = O.page_bounds(k, np.array([[0]], dtype=np.int32), np.array([1], dtype=np.int32))
    assert np.array_equal(bd[0, 0, 0], k[0, 0, 0]) and np.array_equal(bd[0, 0, 1], k[0, 0, 0])


def test_bounds_signed_zero_total_order():
    k = np.zeros((1, 1, 16, 128), dtype=F16)
    k[0, 0, 1, :] = F16(-0.0)
    bd = O.page_bounds(k, np.array([[0]], dtype=np.int32), np.array([2], dtype=np.int32))
    assert np.all(bd[0, 0, 0].view(np.uint16) == 0x8000)   # min = -0
    assert np.all(bd[0, 0, 1].view(np.uint16) == 0x0000)   # max = +0


# ------------------------------------------------------------------------------------- INT4

def _golden_row(row):
    cyc = np.array(row["cycle"], dtype=F64)
    return np.resize(cyc, 128).astype(F16)


def check_int4_golden(quant_fn):
    ok = True
    for row in _golden("int4_rows.json")["rows"]:
        x = _golden_row(row)
        pk, s, z = quant_fn(x)
        want = np.resize(np.array([int(h, 16) for h in row["bytes_cycle"]], dtype=np.uint8), 64)
        ok &= bool(np.array_equal(np.asarray(pk, dtype=np.uint8), want))
        ok &= float(F16(s)) == row["scale"] and float(F16(z)) == row["zero"]
    return ok


def test_int4_golden_bytes():
    assert check_int4_golden(O.quantize_row)


def test_int4_golden_nibbles():
    for row in _golden("int4_rows.json")["rows"]:
        if "nibbles_cycle" not in row:
            continue
        pk, s, z = O.quantize_row(_golden_row(row))
        assert np.array_equal(O.unpack_row(pk), np.resize(np.array(row["nibbles_cycle"]), 128))


def test_int4_roundtrip_error_bound():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((512, 128)) * rng.uniform(0.01, 30, size=(512, 1))).astype(F16)
    pk, s, z = O.quantize_rows(x)
    for i in range(x.shape[0]):
        kh = O.dequantize_row(pk[i], s[i], z[i])
        err = np.abs(kh - x[i].astype(F64)).max()
        s64 = float(s[i])
        # half a step, plus the clamp at 15 after s was rounded down to fp16 (<= 15 * 2^-11 s)
        assert err <= 0.5 * s64 + 15 * 2.0 ** -11 * s64 + 1e-12


def test_int4_memory_identity():
    # [Notes] "Key designs", 4-bit K cache: the extra memory is 1/8 of the fp16 KV cache
    d, kv_bytes = 128, 2 * 128 * 2
    packed_bytes = d // 2
    assert packed_bytes * 8 == kv_bytes
    pk, s, z = O.quantize_row(np.zeros(d, dtype=F16))
    assert pk.nbytes == packed_bytes and s.nbytes + z.nbytes == 4


def test_quantize_k_partial_page_rows_zero():
    rng = np.random.default_rng(4)
    k = rng.standard_normal((2, 1, 16, 128)).astype(F16)
    q4, sz = O.quantize_k(k, np.array([[1, 0]], dtype=np.int32), np.array([21], dtype=np.int32))
    assert np.all(q4[0, 0, 5:] == 0) and np.all(sz[0, 0, 5:].view(np.uint16) == 0)
    assert np.any(q4[0, 0, :5] != 0)


# ------------------------------------------------------------------------------------- scores

def check_scores(score_fn, rng):
    ok = True
    mn = rng.standard_normal((5, 128)).astype(F16)
    mx = (mn.astype(F32) + np.abs(rng.standard_normal((5, 128)))).astype(F16)
    for j in (0, 17, 127):
        e = np.zeros(128, dtype=F16)
        e[j] = F16(1.0)
        ok &= bool(np.array_equal(score_fn(e, mn, mx), mx[:, j].astype(F32)))
        ok &= bool(np.array_equal(score_fn(-e, mn, mx), -mn[:, j].astype(F32)))
    # upper bound over the actual tokens of random pages
    for _ in range(20):
        toks = rng.standard_normal((16, 128)).astype(F16)
        lo, hi = O.f16_min_max(toks, axis=0)
        q = (rng.standard_normal(128) * 3).astype(F16)
        sc = float(score_fn(q, lo[None], hi[None])[0])
        best = float((toks.astype(F64) @ q.astype(F64)).max())
        exact = float(np.where(q > 0, q.astype(F64) * hi.astype(F64),
                               q.astype(F64) * lo.astype(F64)).sum())
        bound = 128 * 2.0 ** -24 * float(np.abs(q.astype(F64)) @ np.maximum(
            np.abs(lo.astype(F64)), np.abs(hi.astype(F64))))
        ok &= sc >= best - bound and abs(sc - exact) <= bound
    # a page of identical tokens: the bound is the dot product itself
    tok = rng.standard_normal(128).astype(F16)
    q = rng.standard_normal(128).astype(F16)
    sc = float(score_fn(q, tok[None], tok[None])[0])
    ok &= abs(sc - float(tok.astype(F64) @ q.astype(F64))) <= 1e-4
    return ok


def test_scores_pins():
    assert check_scores(O.page_scores, np.random.default_rng(5))


def _score_order_case():
    case = _golden("score_order.json")

    def vec(spec):
        v = np.full(128, spec["default"], dtype=F16)
        for c, x in spec["set"].items():
            v[int(c)] = F16(x)
        return v

    return case, vec(case["q"]), vec(case["min"]), vec(case["max"])


def check_score_order(score_fn):
    """The hand-worked case of tests/golden/score_order.json: only the fixed summation order
    (16 left-to-right partials of 8 channels, then pairs (l, l+8), (l, l+4), (l, l+2), (l, l+1))
    gives its bits."""
    case, q, mn, mx = _score_order_case()
    got = F32(score_fn(q, mn[None], mx[None])[0])
    return int(np.array([got], dtype=F32).view(np.uint32)[0]) == int(case["score_bits"], 16)


def test_scores_summation_order_golden():
    assert check_score_order(O.page_scores)
    case, q, mn, mx = _score_order_case()
    assert float(O.page_scores(q, mn[None], mx[None])[0]) == case["score"]


def test_scores_fixed_order_is_deterministic_fp32():
    rng = np.random.default_rng(6)
    q = rng.standard_normal(128).astype(F16)
    mn = rng.standard_normal((64, 128)).astype(F16)
    mx = (mn.astype(F32) + 1).astype(F16)
    a = O.page_scores(q, mn, mx)
    assert a.dtype == F32 and np.array_equal(a, O.page_scores(q, mn.copy(), mx.copy()))


# ------------------------------------------------------------------------------------- top-k

def test_select_top_k_bruteforce_with_ties():
    rng = np.random.default_rng(7)
    for trial in range(200):
        n = int(rng.integers(1, 40))
        sc = rng.integers(-4, 5, size=n).astype(F32)        # many exact ties
        k = int(rng.integers(1, n + 2))
        got = O.select_top_k(sc, k)
        ranked = sorted(range(n), key=lambda j: (-float(sc[j]), j))
        assert list(got) == sorted(ranked[:min(k, n)])


def test_budget_rule():
    assert O.budget_for(256, 0, 4) == 64          # 4096-token single-head workload: 64 pages
    assert O.budget_for(2048, 0, 4) == 512
    assert O.budget_for(3, 0, 4) == 1 and O.budget_for(5, 0, 4) == 2
    assert O.budget_for(10, 64, 4) == 10 and O.budget_for(100, 64, 4) == 64


def _integer_gqa_case(seed=21):
    """Integer-valued fp16 q and K (|values| <= 3), so every product and every sum of a page
    score is exact in fp32 and in Python integers; ragged lengths, a permuted page table, many
    tied scores."""
    rng = np.random.default_rng(seed)
    hq, hkv, d = 8, 2, 128
    lens = np.array([1, 37, 16 * 9, 16 * 11 + 5])
    pages = [O.num_pages(n) for n in lens]
    p_phys = sum(pages) + 3
    perm = rng.permutation(p_phys)
    pt = np.full((len(lens), max(pages)), -1, dtype=np.int64)
    o = 0
    for b, pb in enumerate(pages):
        pt[b, :pb] = perm[o:o + pb]
        o += pb
    k = rng.integers(-3, 4, size=(p_phys, hkv, 16, d)).astype(F16)
    q = rng.integers(-3, 4, size=(len(lens), hq, d)).astype(F16)
    return q, k, pt, lens, hq, hkv


def check_select_pages(select_fn, budget_pages=0, seed=21):
    """Brute force in Python integers: q-head h reads kv-head h // (Hq / Hkv); score of page j =
    sum over channels of max(q_c mn_jc, q_c mx_jc) over the page's valid tokens; keep
    ceil(P / 4) pages (or the fixed budget), highest score first, ties to the lower page."""
    q, k, pt, lens, hq, hkv = _integer_gqa_case(seed)
    bounds = O.page_bounds(k, pt, lens)
    got = select_fn(q, bounds, pt, lens, hq, hkv, budget_pages, 4)
    for b, n in enumerate(lens):
        n = int(n)
        pb = -(-n // 16)
        kb = min(pb, budget_pages) if budget_pages > 0 else -(-pb // 4)
        for h in range(hq):
            kvh = h // (hq // hkv)
            qi = [int(v) for v in q[b, h]]
            sc = []
            for j in range(pb):
                rows = k[pt[b, j], kvh, : min(16, n - 16 * j)].astype(np.int64)
                mn, mx = rows.min(axis=0), rows.max(axis=0)
                sc.append(sum(max(qc * int(a), qc * int(c)) for qc, a, c in zip(qi, mn, mx)))
            want = sorted(sorted(range(pb), key=lambda j: (-sc[j], j))[:kb])
            g_sc, g_sel = got[(b, h)]
            if list(np.asarray(g_sc, dtype=F64)) != [float(v) for v in sc]:
                return False
            if list(g_sel) != want:
                return False
    return True


def test_select_pages_bruteforce_integer_gqa():
    assert check_select_pages(O.select_pages)
    assert check_select_pages(O.select_pages, budget_pages=3)
    for seed in range(8):                   # other draws: other ties, other page permutations
        for budget in (0, 1, 5, 100):
            assert check_select_pages(O.select_pages, budget_pages=budget, seed=seed), \
                (seed, budget)

    def kv_head_modulo(q, bounds, pt, lens, hq, hkv, budget_pages=0, budget_div=4):
        out = {}
        for b in range(len(lens)):
            pb = O.num_pages(lens[b])
            phys = pt[b, :pb]
            kb = O.budget_for(pb, budget_pages, budget_div)
            for h in range(hq):
                sc = O.page_scores(q[b, h], bounds[phys, h % hkv, 0], bounds[phys, h % hkv, 1])
                out[(b, h)] = (sc, O.select_top_k(sc, kb))
        return out

    def budget_floor(q, bounds, pt, lens, hq, hkv, budget_pages=0, budget_div=4):
        out = O.select_pages(q, bounds, pt, lens, hq, hkv, budget_pages, budget_div)
        res = {}
        for (b, h), (sc, _) in out.items():
            kb = max(1, len(sc) // budget_div) if budget_pages == 0 else min(len(sc), budget_pages)
            res[(b, h)] = (sc, O.select_top_k(sc, kb))
        return res

    def ties_to_higher(q, bounds, pt, lens, hq, hkv, budget_pages=0, budget_div=4):
        out = O.select_pages(q, bounds, pt, lens, hq, hkv, budget_pages, budget_div)
        res = {}
        for (b, h), (sc, sel) in out.items():
            order = sorted(range(len(sc)), key=lambda j: (-float(sc[j]), -j))
            res[(b, h)] = (sc, np.array(sorted(order[:len(sel)])))
        return res

    assert not check_select_pages(kv_head_modulo)
    assert not check_select_pages(budget_floor)
    assert not check_select_pages(ties_to_higher)


# ------------------------------------------------------------------------------------- estimate

def test_estimate_on_grid_matches_textbook_softmax():
    rng = np.random.default_rng(8)
    n, d = 160, 128
    s = rng.choice([0.125, 0.25, 0.5], size=n).astype(F16)
    z = (-rng.integers(0, 16, size=n) * s.astype(F64)).astype(F16)     # on the same grid
    nib = rng.integers(0, 16, size=(n, d))
    nib[:, 0], nib[:, 1] = 0, 15                      # min and max attained on every row
    k = (nib * s[:, None].astype(F64) + z[:, None].astype(F64)).astype(F16)
    assert np.array_equal(k.astype(F64), nib * s[:, None].astype(F64) + z[:, None].astype(F64))
    kk = k.reshape(10, 1, 16, d)
    pt = np.arange(10, dtype=np.int32)[None, :]
    lens = np.array([n], dtype=np.int32)
    q4, sz = O.quantize_k(kk, pt, lens)
    q = (rng.standard_normal(d) * 2).astype(F16)
    sel = np.array([1, 4, 5, 9])
    cand, w = O.estimate_head(q, q4, sz, pt, 0, 0, n, sel)
    ref = torch.softmax(torch.from_numpy(k[cand].astype(F64)) @ torch.from_numpy(
        q.astype(F64)) / math.sqrt(d), dim=0).numpy()
    assert np.array_equal(cand, np.concatenate([np.arange(16 * j, 16 * j + 16) for j in sel]))
    assert np.allclose(w, ref, rtol=1e-12, atol=1e-15)


# ------------------------------------------------------------------------------------- top-p

def _golden_w(case):
    if "w" in case:
        return np.array(case["w"], dtype=F64)
    r = case["w_rule"]
    return np.array([r["A"]] * r["a"] + [r["B"]] * (r["n"] - r["a"]), dtype=F64)


def check_top_p_golden(top_p_fn):
    ok = True
    for case in _golden("top_p_examples.json")["cases"]:
        w = _golden_w(case)
        k_star, m_star, kept = top_p_fn(w, case["p"])
        ok &= k_star == case["k_star"] and abs(float(m_star) - case["m_star"]) < 1e-15
        if "threshold_set" in case:
            ok &= list(kept) == case["threshold_set"]
        else:
            ok &= len(kept) == case["threshold_set_size"]
    return ok


def test_p_one_keeps_the_whole_distribution():
    """Reading R10 by hand: w = (1/2, 1/4, 1/4 - 2^-55, 2^-55) sums to exactly 1, and every
    entry is positive, so mass 1 needs all four.  The fp64 prefix 3/4 + (1/4 - 2^-55) = 1 - 2^-55
    lies within half a unit (2^-54) of 1 and rounds to 1.0, so the sort form stops at three;
    the step's reading keeps all four with m* = 0, as the bisection does."""
    d = 2.0 ** -55
    w = np.array([0.5, 0.25, 0.25 - d, d], dtype=F64)
    assert math.fsum(w) == 1.0 and np.all(w > 0)
    assert O.top_p_sort(w, 1.0)[0] == 3                  # the rounding the reading avoids
    k, m, kept = O.top_p_whole(w, 1.0)
    assert k == 4 and m == 0.0 and list(kept) == [0, 1, 2, 3]
    assert list(O.top_p_bisect(w, 1.0, 1e-6)[1]) == [0, 1, 2, 3]
    for p in (0.5, 0.75, 0.9):                           # below 1 it is the sort form
        a, b = O.top_p_whole(w, p), O.top_p_sort(w, p)
        assert a[0] == b[0] and a[1] == b[1] and list(a[2]) == list(b[2])


def test_top_p_golden():
    assert check_top_p_golden(O.top_p_sort)


def _brute_min_count(w, p):
    n = len(w)
    for size in range(1, n + 1):
        for comb in itertools.combinations(range(n), size):
            if w[list(comb)].sum() >= p:
                return size
    return n


def test_top_p_bruteforce_small():
    rng = np.random.default_rng(9)
    for trial in range(150):
        n = int(rng.integers(1, 15))
        if trial % 3 == 0:
            raw = rng.integers(1, 5, size=n).astype(F64)          # ties
        else:
            raw = rng.exponential(size=n) ** 3
        w = raw / raw.sum()
        p = float(rng.uniform(0.3, 0.97))
        k_star, m_star, kept = O.top_p_sort(w, p)
        assert k_star == _brute_min_count(w, p)
        assert w[kept].sum() >= p and np.all(w[kept] >= m_star)


def test_top_p_threshold_invariant():
    rng = np.random.default_rng(10)
    rows, info = synth.config5_rows(24, 2048, seed=3, tie_frac=0.25)
    for i in range(rows.shape[0]):
        for p in (0.8, 0.9):
            w = rows[i]
            k_star, m_star, kept = O.top_p_sort(w, p)
            w64 = w.astype(F64)
            assert w64[w >= m_star].sum() >= p - 1e-12 or k_star == w.size
            assert w64[w > m_star].sum() < p


def check_bisect_band(bisect_fn, rows, p, eps):
    ok = True
    for w in rows:
        m, kept = bisect_fn(w, p, eps)
        k_star, m_star, _ = O.top_p_sort(w, p)
        ok &= np.array_equal(kept, np.nonzero(w >= m)[0])
        ok &= w[kept].astype(F64).sum() >= p - 1e-6
        band = int(np.count_nonzero((w >= F64(m_star) - eps) & (w <= m_star)))
        ok &= len(kept) <= k_star + band
    return ok


def test_bisect_band_criterion():
    rows, _ = synth.config5_rows(32, 4096, seed=4, tie_frac=0.25)
    for p in (0.8, 0.9):
        assert check_bisect_band(O.top_p_bisect, rows, p, 1e-6)


def _bisect_replay_from_threshold(w, p, eps):
    """The pages' bisection (lo = 0, hi = max W, fp32 midpoints) with its test mass(W >= mid) >= p
    replaced by mid <= T, T = the largest weight v with mass(W >= v) >= p (0 if none), T read off
    the descending cumulative sum.  The standalone pruner computes m this way."""
    w = np.asarray(w, dtype=F32)
    order = np.argsort(-w.astype(F64), kind="stable")
    cs = np.cumsum(w[order].astype(F64))
    hit = np.nonzero(cs >= F64(p))[0]
    T = w[order[hit[0]]] if hit.size else F32(0.0)
    top = F32(w.max())
    if p >= 1.0:
        return F32(0.0)
    if top <= T:
        return top
    lo, hi = F32(0.0), top
    for _ in range(64):
        if F64(hi) - F64(lo) <= eps:
            break
        mid = F32(lo + (hi - lo) / F32(2.0))
        if not (lo < mid < hi):
            break
        if mid <= T:
            lo = mid
        else:
            hi = mid
    return lo


def test_bisect_equals_threshold_replay():
    """mass(W >= t) only changes at weight values, so each test of the bisection is mid <= T; the
    replay gives the oracle's bisection result exactly (normalised rows with ties, an
    unnormalised row, uniform and one-hot rows)."""
    rows, _ = synth.config5_rows(24, 3000, seed=9, tie_frac=0.3)
    extra = [np.full(100, 0.01, dtype=F32), np.eye(1, 64, 5, dtype=F32)[0],
             (np.arange(1, 201, dtype=F32) / 40.0).astype(F32)]
    for w in list(rows) + extra:
        for p in (0.5, 0.8, 0.9, 0.999):
            m, _ = O.top_p_bisect(w, p, 1e-6)
            assert _bisect_replay_from_threshold(w, p, 1e-6) == m


def test_bisect_one_hot_and_keep_all():
    w = np.zeros(64, dtype=F32)
    w[11] = 1.0
    m, kept = O.top_p_bisect(w, 0.85, 1e-6)
    assert m == F32(1.0) and list(kept) == [11]
    w = np.full(50, 0.02, dtype=F32)
    m, kept = O.top_p_bisect(w, 0.999999, 1e-6)
    assert len(kept) == 50


# ------------------------------------------------------------------------------------- attention

def test_attention_all_tokens_matches_torch_sdpa():
    rng = np.random.default_rng(11)
    q = rng.standard_normal(128).astype(F16)
    k = rng.standard_normal((300, 128)).astype(F16)
    v = rng.standard_normal((300, 128)).astype(F16)
    o, lse = O.attention(q, k, v, 1 / math.sqrt(128))
    tq = torch.from_numpy(q.astype(F64)).view(1, 1, 1, 128)
    tk = torch.from_numpy(k.astype(F64)).view(1, 1, 300, 128)
    tv = torch.from_numpy(v.astype(F64)).view(1, 1, 300, 128)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv).view(128).numpy()
    assert np.allclose(o, ref, rtol=1e-12, atol=1e-12)
    s = torch.from_numpy(k.astype(F64)) @ torch.from_numpy(q.astype(F64)) / math.sqrt(128)
    assert abs(lse - torch.logsumexp(s, 0).item()) < 1e-12


def test_attention_single_token():
    rng = np.random.default_rng(12)
    q = rng.standard_normal(128).astype(F16)
    k = rng.standard_normal((1, 128)).astype(F16)
    v = rng.standard_normal((1, 128)).astype(F16)
    o, lse = O.attention(q, k, v, 1 / math.sqrt(128))
    assert np.array_equal(o, v[0].astype(F64))
    assert abs(lse - float(k[0].astype(F64) @ q.astype(F64)) / math.sqrt(128)) < 1e-12


@pytest.mark.parametrize("p", [0.7, 0.85, 0.95])
def test_top_p_error_bound(p):
    # [Notes] "Key designs": the output error of oracle top-p is at most (1 - p) * ||V||_F
    wl = synth.config1(seed=5, n=1024)
    scale = 1 / math.sqrt(128)
    toks = np.arange(1024)
    k = O.gather_tokens(wl.k, wl.page_table, 0, 0, toks)
    v = O.gather_tokens(wl.v, wl.page_table, 0, 0, toks).astype(F64)
    w = O.full_attention_weights(wl.q[0, 0], k, scale)
    k_star, m_star, kept = O.top_p_sort(w, p)
    o_full = w @ v
    o_topp = w[kept] @ v[kept]
    err = np.linalg.norm(o_topp - o_full)
    v_fro = np.linalg.norm(v)
    left_out = 1.0 - w[kept].sum()
    assert err <= left_out * np.linalg.norm(v, axis=1).max() + 1e-12
    assert err <= (1 - p) * v_fro
    # renormalised over the kept set (what sparse attention returns): 2 (1 - S) max|v|
    o_sparse, _ = O.attention(wl.q[0, 0], k[kept], v[kept].astype(F16), scale)
    assert np.linalg.norm(o_sparse - o_full) <= 2 * left_out * np.linalg.norm(v, axis=1).max() \
        + 1e-9
    assert np.linalg.norm(o_sparse - o_full) <= 2 * (1 - p) * v_fro


# ------------------------------------------------------------------------------------- end to end

def test_decode_step_small_consistency():
    wl = synth.config2(seed=1, n=1000, batch=2)
    r = O.decode_step(wl)
    g = wl.num_q_heads // wl.num_kv_heads
    for (b, kvh), grp in r["groups"].items():
        want = set()
        for h in range(kvh * g, (kvh + 1) * g):
            hd = r["heads"][(b, h)]
            assert len(hd["sel"]) == O.budget_for(O.num_pages(wl.seq_lens[b]), 0, 4)
            assert hd["w"].sum() == pytest.approx(1.0, abs=1e-12)
            assert hd["w"][hd["kept"]].sum() >= wl.p
            want |= set(hd["kept_tok"].tolist())
        assert sorted(want) == grp["union"].tolist()
        # p = 1 style check: all kept tokens of the group are inside the sequence
        assert grp["union"].max() < wl.seq_lens[b]


def check_gather(gather_fn):
    """Paged rows that carry their own address: the row of logical token t of sequence b in
    kv-head h holds (t, h, b) in its first three channels, written while walking the sequences'
    pages in logical order (a permuted page table puts them anywhere).  A gather must return
    exactly the rows it was asked for."""
    _, _, pt, lens, _, hkv = _integer_gqa_case(seed=5)
    p_phys = int(pt.max()) + 4
    arr = np.full((p_phys, hkv, 16, 8), -1.0, dtype=F16)
    for b, n in enumerate(lens):
        for t in range(int(n)):
            for h in range(hkv):
                arr[pt[b, t // 16], h, t % 16, :3] = (t, h, b)
    rng = np.random.default_rng(6)
    for b, n in enumerate(lens):
        for h in range(hkv):
            toks = np.sort(rng.choice(int(n), size=min(int(n), 23), replace=False))
            rows = np.asarray(gather_fn(arr, pt, b, h, toks)).astype(F64)
            if rows.shape[0] != toks.size:
                return False
            if not (np.array_equal(rows[:, 0], toks) and np.all(rows[:, 1] == h)
                    and np.all(rows[:, 2] == b)):
                return False
    return True


def test_gather_tokens_returns_the_addressed_rows():
    assert check_gather(O.gather_tokens)

    def gather_no_page_table(arr, pt, b, kvh, toks):     # treats logical pages as physical
        toks = np.asarray(toks, dtype=np.int64)
        return arr[toks // 16, kvh, toks % 16]

    def gather_wrong_row(arr, pt, b, kvh, toks):         # row index from the page, not the token
        toks = np.asarray(toks, dtype=np.int64)
        return arr[pt[b, toks // 16], kvh, (toks // 16) % 16]

    assert not check_gather(gather_no_page_table)
    assert not check_gather(gather_wrong_row)


def check_candidates(cand_fn):
    """The candidates of a page set are the tokens whose page is selected and whose id is below
    the sequence length, ascending; checked against a scan of every token id."""
    rng = np.random.default_rng(9)
    for n in (1, 15, 16, 17, 100, 16 * 9):
        pb = -(-n // 16)
        for _ in range(6):
            sel = np.sort(rng.choice(pb, size=int(rng.integers(0, pb + 1)), replace=False))
            want = [t for t in range(16 * pb) if t < n and (t // 16) in set(sel.tolist())]
            got = np.asarray(cand_fn(sel, n)).tolist()
            if got != want:
                return False
    return True


def test_candidates_by_scan():
    assert check_candidates(O.candidates)

    def cand_full_pages(sel, n):             # keeps the unused rows of a partial last page
        return np.concatenate([np.arange(16 * j, 16 * j + 16) for j in sorted(sel)]) \
            if len(sel) else np.zeros(0, np.int64)

    assert not check_candidates(cand_full_pages)


def test_dense_limit_equals_full_attention():
    # budget = all pages and p = 1: the pipeline reduces to dense attention
    wl = synth.config2(seed=2, n=300, batch=1)
    wl.budget_pages = 10 ** 6
    wl.p = 1.0
    r = O.decode_step(wl)
    toks = np.arange(300)
    for h in range(wl.num_q_heads):
        kvh = h // 4
        k = O.gather_tokens(wl.k, wl.page_table, 0, kvh, toks)
        v = O.gather_tokens(wl.v, wl.page_table, 0, kvh, toks)
        o, lse = O.attention(wl.q[0, h], k, v, 1 / math.sqrt(128))
        grp = r["groups"][(0, kvh)]
        assert len(grp["union"]) == 300          # p = 1 keeps every candidate (R10)
        assert np.allclose(grp["o"][h], o, atol=1e-12)


# ------------------------------------------------------------------------------------- mutations

def test_pins_catch_planted_mistakes():
    """Copies of oracle functions with one plausible mistake each must fail a pin."""
    rng = np.random.default_rng(13)

    def quant_swapped_nibbles(x):
        pk, s, z = O.quantize_row(x)
        return ((pk >> 4) | (pk << 4)).astype(np.uint8), s, z

    def quant_half_away(x):
        x16 = np.asarray(x, dtype=F16)
        mn, mx = O.f16_min_max(x16[None], axis=1)
        s16 = F16((F32(mx[0]) - F32(mn[0])) / F32(15))
        if float(s16) == 0:
            n = np.zeros(128, dtype=np.uint8)
        else:
            r = (x16.astype(F32) - F32(mn[0])) / F32(s16)
            n = np.clip(np.floor(r + F32(0.5)), 0, 15).astype(np.uint8)
        return (n[0::2] | (n[1::2] << 4)).astype(np.uint8), s16, mn[0]

    assert check_int4_golden(O.quantize_row)
    assert not check_int4_golden(quant_swapped_nibbles)
    assert not check_int4_golden(quant_half_away)

    def scores_wrong_sign(q, mn, mx):
        return O.page_scores(q, mx, mn)

    def scores_dropped_term(q, mn, mx):
        q = np.asarray(q, dtype=F16).copy()
        q[-1] = 0
        return O.page_scores(q, mn, mx)

    assert not check_scores(scores_wrong_sign, np.random.default_rng(5))
    assert not check_scores(scores_dropped_term, np.random.default_rng(5))

    # summation orders other than the fixed one (each term is exact, only the order differs)
    def terms(q, mn, mx):
        q = np.asarray(q, dtype=F16).astype(F32)
        return np.where(q > 0, q * np.asarray(mx, F16).astype(F32)[0],
                        q * np.asarray(mn, F16).astype(F32)[0]).astype(F32)

    def seq_sum(vals):
        acc = F32(0)
        for v in vals:
            acc = F32(acc + F32(v))
        return acc

    def tree_sum(vals):                      # adjacent pairs (0,1), (2,3), ...
        v = [F32(x) for x in vals]
        while len(v) > 1:
            v = [F32(v[i] + v[i + 1]) for i in range(0, len(v), 2)]
        return v[0]

    def fixed_tree(part):                    # the pairs (l, l+8), (l, l+4), (l, l+2), (l, l+1)
        part = [F32(x) for x in part]
        while len(part) > 1:
            h = len(part) // 2
            part = [F32(part[l] + part[l + h]) for l in range(h)]
        return part[0]

    wrong_orders = {
        "sequential_128": lambda t: seq_sum(t),
        "adjacent_pairs_over_channels": lambda t: tree_sum(t),
        "partials_paired_adjacent": lambda t: tree_sum([seq_sum(t[8 * l:8 * l + 8])
                                                         for l in range(16)]),
        "strided_lane_partials": lambda t: fixed_tree([seq_sum(t[l::16]) for l in range(16)]),
        "partials_right_to_left": lambda t: fixed_tree([seq_sum(t[8 * l:8 * l + 8][::-1])
                                                         for l in range(16)]),
        "exact_then_rounded": lambda t: F32(math.fsum(float(x) for x in t)),
    }
    want = _golden("score_order.json")["wrong_order_bits"]
    for name, order in wrong_orders.items():
        fn = lambda q, mn, mx, order=order: np.array([order(terms(q, mn, mx))], dtype=F32)
        assert not check_score_order(fn), name
        case, q, mn, mx = _score_order_case()
        got = np.array([fn(q, mn[None], mx[None])[0]], dtype=F32).view(np.uint32)[0]
        assert int(got) == int(want[name], 16), name     # the hand-worked wrong results

    def top_p_strict(w, p):              # '>' instead of '>=' on the mass
        order = np.argsort(-w, kind="stable")
        cs = np.cumsum(w[order])
        hit = np.nonzero(cs > p)[0]
        k = int(hit[0]) + 1 if hit.size else len(w)
        m = w[order[k - 1]]
        return k, m, np.nonzero(w >= m)[0]

    def top_p_off_by_one(w, p):
        k, m, kept = O.top_p_sort(w, p)
        order = np.argsort(-w, kind="stable")
        m2 = w[order[min(k, len(w) - 1)]]
        return k, m2, np.nonzero(w >= m2)[0]

    assert not check_top_p_golden(top_p_strict)
    assert not check_top_p_golden(top_p_off_by_one)

    def bounds_all_rows(k, pt, lens):        # ignores the sequence end
        return O.page_bounds(k, pt, np.full_like(lens, 16 * pt.shape[1]))

    assert not check_bounds(bounds_all_rows, np.random.default_rng(1))

    rows, _ = synth.config5_rows(16, 2048, seed=4, tie_frac=0.25)

    def bisect_returns_hi(w, p, eps):         # returns the upper end of the final interval
        dt = w.dtype.type
        w64 = w.astype(F64)
        top = dt(w.max())
        lo, hi = dt(0.0), top
        if w64[w >= top].sum() < p:
            for _ in range(64):
                if F64(hi) - F64(lo) <= eps:
                    break
                mid = dt(lo + (hi - lo) / dt(2.0))
                if not (lo < mid < hi):
                    break
                if w64[w >= mid].sum() >= p:
                    lo = mid
                else:
                    hi = mid
        return hi, np.nonzero(w >= hi)[0]

    assert check_bisect_band(O.top_p_bisect, rows, 0.9, 1e-6)
    assert not check_bisect_band(bisect_returns_hi, rows, 0.9, 1e-6)



def check_order_key(key_fn):
    """Every non-NaN fp16 bit pattern, ordered by value with -0 before +0: the keys must rise
    strictly along that order (so min/max by key are min/max by value, and -0 < +0)."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = bits.view(F16)
    ok = ~np.isnan(vals)
    bits, vals = bits[ok], vals[ok]
    neg_zero = bits == 0x8000
    order = np.lexsort((~neg_zero, vals.astype(F64)))  # by value, then -0 first
    keys = np.asarray(key_fn(vals[order])).astype(np.int64)
    return bool(np.all(np.diff(keys) > 0))


def check_softmax(fn):
    """Closed forms: uniform logits give 1/n; logits (0, ln 3) give (1/4, 3/4), also shifted by
    1000 (no overflow); a random row against the definition term by term (math.fsum)."""
    try:
        with np.errstate(all="ignore"):
            for n in (1, 2, 7, 1000):
                if not np.allclose(fn(np.zeros(n)), np.full(n, 1.0 / n), rtol=1e-15, atol=0):
                    return False
            for c in (0.0, 1000.0):
                if not np.allclose(fn([c, c + math.log(3.0)]), [0.25, 0.75], rtol=1e-12, atol=0):
                    return False
            x = np.random.default_rng(3).normal(0.0, 4.0, 257)
            w = np.asarray(fn(x), dtype=F64)
    except (FloatingPointError, OverflowError, ValueError):
        return False
    e = [math.exp(v - 10.0) for v in x]
    ref = np.array(e) / math.fsum(e)
    return bool(np.allclose(w, ref, rtol=1e-13, atol=0)) and abs(math.fsum(w) - 1.0) < 1e-15


def test_f16_order_key_orders_every_fp16_value():
    assert check_order_key(O.f16_order_key)
    z = O.f16_order_key(np.array([-0.0, 0.0], F16))
    assert z[0] < z[1]

    def key_magnitude_only(x16):           # drops the sign
        return np.ascontiguousarray(x16, dtype=F16).view(np.uint16).astype(np.int32) & 0x7FFF

    def key_no_minus_one(x16):             # -0 and +0 collide
        b = np.ascontiguousarray(x16, dtype=F16).view(np.uint16).astype(np.int32)
        return np.where(b & 0x8000, -(b & 0x7FFF), b)

    assert not check_order_key(key_magnitude_only)
    assert not check_order_key(key_no_minus_one)


def test_softmax64_closed_forms():
    assert check_softmax(O.softmax64)

    def softmax_unshifted(x):               # no max subtraction: overflows at logits near 1000
        e = np.exp(np.asarray(x, dtype=F64))
        return e / e.sum()

    def softmax_fp32(x):                    # single precision
        x = np.asarray(x, dtype=F32)
        e = np.exp(x - x.max())
        return e / e.sum()

    def softmax_dropped_term(x):            # the normaliser misses the last term
        x = np.asarray(x, dtype=F64)
        e = np.exp(x - x.max())
        return e / (e.sum() - e[-1] if e.size > 1 else e.sum())

    assert not check_softmax(softmax_unshifted)
    assert not check_softmax(softmax_fp32)
    assert not check_softmax(softmax_dropped_term)
