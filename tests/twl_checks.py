"""Comparisons of the CUDA path against the CPU oracle (shared by the GPU tests and smoke()).

Criteria (from the method's statement of correctness):
  bounds, INT4 bytes, scale/zero, page scores, selected pages   bit-exact
  estimated weights      |W_gpu - W_or| <= 1e-3 * W_or + 1e-9 per candidate
  pruning (on the W the device pruner consumed)
      kept = {i : W_i >= m} exactly;  sum_kept W (fp64) >= p - 1e-5;
      |kept| <= k* + #{i : m* - eps <= W_i <= m*}   (k*, m* from the sort-based oracle; at
      p = 1 the whole row, so a row whose fp32 weights sum a little above 1 is not held to a
      prefix that reaches 1.0 early)
  union                  exactly the union of the heads' kept token ids
  attention              |o_gpu - o_or| <= 2e-3, |lse_gpu - lse_or| <= 2e-3 over the device's set
The slack 1e-5 on the kept mass covers fp32 block sums of up to 131072 terms
(~log2(n) * 2^-24 relative, with margin).
"""
from __future__ import annotations

import math

import numpy as np

from oracle import twl_oracle as O
from workloads import synth

W_RTOL, W_ATOL = 1e-3, 1e-9
MASS_SLACK = 1e-5
O_ATOL = 2e-3
LSE_ATOL = 2e-3


def u16(x):
    return np.ascontiguousarray(x).view(np.uint16)


def referenced_pages(wl):
    out = []
    for b in range(wl.batch):
        out.extend(wl.page_table[b, : O.num_pages(wl.seq_lens[b])].tolist())
    return np.array(sorted(set(out)), dtype=np.int64)


def group_workload(wl, b: int, kvh: int):
    """The (b, kv-head) group of a workload as a stand-alone single-group workload."""
    g = wl.num_q_heads // wl.num_kv_heads
    n = int(wl.seq_lens[b])
    pb = O.num_pages(n)
    phys = wl.page_table[b, :pb].astype(np.int64)
    sub = synth.DecodeWorkload(
        name=f"{wl.name}[b{b},kv{kvh}]", q=wl.q[b:b + 1, kvh * g:(kvh + 1) * g].copy(),
        k=wl.k[phys, kvh:kvh + 1].copy(), v=wl.v[phys, kvh:kvh + 1].copy(),
        page_table=np.arange(pb, dtype=np.int32)[None, :], seq_lens=np.array([n], np.int32),
        num_q_heads=g, num_kv_heads=1, p=wl.p, eps=wl.eps, budget_div=wl.budget_div,
        budget_pages=wl.budget_pages)
    return sub


def check_prune_row(w, m, kept_count, kept_idx, p, eps, where=""):
    w = np.asarray(w, dtype=np.float32)
    kept = np.nonzero(w >= np.float32(m))[0]
    assert kept_count == kept.size, f"{where}: kept_count {kept_count} != |W>=m| {kept.size}"
    if kept_idx is not None:
        assert np.array_equal(np.asarray(kept_idx[:kept_count]), kept), f"{where}: kept ids"
    total = float(w.astype(np.float64).sum())
    mass = float(w[kept].astype(np.float64).sum())
    assert mass >= min(p, total) - MASS_SLACK, f"{where}: mass {mass} < p {p}"
    k_star, m_star, _ = O.top_p_whole(w, p)        # p = 1: the whole row (reading R10)
    band = int(np.count_nonzero((w.astype(np.float64) >= float(m_star) - eps) & (w <= m_star)))
    assert kept.size <= k_star + band, f"{where}: |kept| {kept.size} > k* {k_star} + band {band}"
    return kept, mass, k_star


def check_weights(w_gpu, w_or, where=""):
    w_gpu = np.asarray(w_gpu, dtype=np.float64)
    err = np.abs(w_gpu - w_or)
    bad = err > W_RTOL * w_or + W_ATOL
    assert not bad.any(), (f"{where}: {bad.sum()} weights off, worst rel "
                           f"{float((err / np.maximum(w_or, 1e-30)).max()):.3g}")


def check_attention(o_gpu, lse_gpu, o_or, lse_or, where=""):
    if math.isinf(lse_or):
        assert np.all(o_gpu == 0) and math.isinf(lse_gpu) and lse_gpu < 0, where
        return
    d = float(np.abs(np.asarray(o_gpu, np.float64) - o_or).max())
    assert d <= O_ATOL, f"{where}: |o - o_or| = {d}"
    assert abs(float(lse_gpu) - lse_or) <= LSE_ATOL, f"{where}: lse {lse_gpu} vs {lse_or}"


def check_step_group(wl, b, kvh, st, o, lse, check_sel=True):
    """Check one (b, kv-head) group of a decode step against the oracle.

    st: dict of numpy arrays copied from the device stats; o, lse: numpy device outputs.
    Returns a small report dict.
    """
    g = wl.num_q_heads // wl.num_kv_heads
    sub = group_workload(wl, b, kvh)
    bounds = O.page_bounds(sub.k, sub.page_table, sub.seq_lens)
    q4, sz = O.quantize_k(sub.k, sub.page_table, sub.seq_lens)
    sel = O.select_pages(sub.q, bounds, sub.page_table, sub.seq_lens, g, 1, sub.budget_pages,
                         sub.budget_div)
    n = int(wl.seq_lens[b])
    union_expect = set()
    report = dict(kept=[], k_star=[])
    for hl in range(g):
        h = kvh * g + hl
        where = f"{wl.name} b{b} h{h}"
        sc, pages = sel[(0, hl)]
        cnt = int(st["sel_count"][b, h])
        if check_sel:
            assert cnt == len(pages), f"{where}: sel_count {cnt} vs {len(pages)}"
            assert np.array_equal(st["sel_pages"][b, h, :cnt], pages), f"{where}: selection"
        dev_pages = st["sel_pages"][b, h, :cnt]
        cand, w_or = O.estimate_head(sub.q[0, hl], q4, sz, sub.page_table, 0, 0, n, dev_pages)
        cc = int(st["cand_count"][b, h])
        assert cc == cand.size, f"{where}: cand_count {cc} vs {cand.size}"
        assert np.array_equal(st["cand_tok"][b, h, :cc], cand), f"{where}: candidate ids"
        w_dev = st["weights"][b, h, :cc]
        check_weights(w_dev, w_or, where)
        kept, mass, k_star = check_prune_row(w_dev, st["threshold"][b, h],
                                             int(st["kept_count"][b, h]), None, wl.p, wl.eps,
                                             where)
        union_expect |= set(cand[kept].tolist())
        report["kept"].append(kept.size)
        report["k_star"].append(k_star)
    uc = int(st["union_count"][b, kvh])
    union = st["union_tok"][b, kvh, :uc]
    assert np.array_equal(union, np.array(sorted(union_expect))), f"b{b} kv{kvh}: union"
    att = O.group_attention(sub, {(0, 0): union})
    for hl in range(g):
        h = kvh * g + hl
        o_or, lse_or = att[(0, hl)]
        check_attention(o[b, h], lse[b, h], o_or, lse_or, f"{wl.name} b{b} h{h} attention")
    report["union"] = uc
    return report
