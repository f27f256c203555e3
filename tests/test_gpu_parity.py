"""CUDA path vs the CPU oracle, element by element, through the C ABI (libtwl.so).

Small workloads span several tiles and ragged tails (partial last pages, group sizes 1/2/4/8,
permuted page tables); the full-size workloads are checked on sampled (b, kv-head) groups that the
oracle recomputes one by one.  Criteria: see tests/twl_checks.py.
"""

import numpy as np
import pytest
import torch

from oracle import twl_oracle as O
from workloads import synth

from twl_checks import (check_attention, check_prune_row, check_step_group, check_weights,
                        referenced_pages, u16)

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from adaptive_top_sparse_b200 import twl
    from adaptive_top_sparse_b200.layer import DecodeLayer, SM_SCALE


def small_workloads():
    return [
        synth.config1(seed=0),
        synth.make_decode("gqa4_ragged", 2, 8, 2, [2001, 777], seed=3),
        synth.make_decode("gqa8_perm", 3, 16, 2, [1500, 33, 4100], seed=4, permute_pages=True,
                          max_pages=300),
        synth.make_decode("gqa2_short", 2, 4, 2, [1, 16], seed=5),
        synth.make_decode("mha2", 1, 2, 2, [5000], seed=6, tau=1.0),
        synth.config3(seed=7, batch=3, n_lo=700, n_hi=3000),
    ]


@pytest.fixture(scope="module", params=range(6), ids=lambda i: f"wl{i}")
def small(request):
    wl = small_workloads()[request.param]
    layer = DecodeLayer.from_workload(wl)
    layer.build_aux()
    torch.cuda.synchronize()
    return wl, layer


def np_(t):
    return t.detach().cpu().numpy()


# -------------------------------------------------------------------------- cache maintenance

def test_page_bounds_bit_exact(small):
    wl, layer = small
    ref = O.page_bounds(wl.k, wl.page_table, wl.seq_lens)
    pages = referenced_pages(wl)
    got = np_(layer.aux.bounds)
    assert np.array_equal(u16(got[pages]), u16(ref[pages]))


def test_quantize_k_bit_exact(small):
    wl, layer = small
    q4, sz = O.quantize_k(wl.k, wl.page_table, wl.seq_lens)
    pages = referenced_pages(wl)
    assert np.array_equal(np_(layer.aux.k_int4)[pages], q4[pages])
    assert np.array_equal(u16(np_(layer.aux.k_scale_zero)[pages]), u16(sz[pages]))


def test_quantize_golden_rows_on_gpu():
    # the hand-worked rows of tests/golden/int4_rows.json, quantised by the kernel
    import json, os
    rows = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "int4_rows.json")))
    k = np.zeros((1, 1, 16, 128), dtype=np.float16)
    for i, row in enumerate(rows["rows"]):
        k[0, 0, i] = np.resize(np.array(row["cycle"], dtype=np.float64), 128).astype(np.float16)
    nrows = len(rows["rows"])
    layer = DecodeLayer(k, k, np.zeros((1, 1), np.int32), np.array([nrows], np.int32), 1, 1)
    layer.build_aux()
    q4 = np_(layer.aux.k_int4)[0, 0]
    sz = np_(layer.aux.k_scale_zero)[0, 0]
    for i, row in enumerate(rows["rows"]):
        want = np.resize(np.array([int(h, 16) for h in row["bytes_cycle"]], np.uint8), 64)
        assert np.array_equal(q4[i], want), row["name"]
        assert float(sz[i, 0]) == row["scale"] and float(sz[i, 1]) == row["zero"], row["name"]
    assert np.all(q4[nrows:] == 0) and np.all(u16(sz[nrows:]) == 0)


# -------------------------------------------------------------------------- stage by stage

def test_select_pages_bit_exact(small):
    wl, layer = small
    dev = layer.device
    b, hq, mp, mb = wl.batch, wl.num_q_heads, wl.max_pages, layer.max_budget
    q = torch.from_numpy(wl.q).to(dev)
    sel = torch.full((b, hq, mb), -1, dtype=torch.int32, device=dev)
    cnt = torch.zeros((b, hq), dtype=torch.int32, device=dev)
    scores = torch.full((b, hq, mp), float("nan"), dtype=torch.float32, device=dev)
    ws = twl.alloc_workspace(twl.TWL_OP_SELECT, dev, batch=b, num_q_heads=hq,
                             num_kv_heads=wl.num_kv_heads, max_pages=mp)
    twl.twl_select_pages(q, hq, layer.kv, layer.aux.bounds, wl.budget_pages, wl.budget_div, mb,
                         sel, cnt, scores, ws)
    ref = O.select_pages(wl.q, O.page_bounds(wl.k, wl.page_table, wl.seq_lens), wl.page_table,
                         wl.seq_lens, hq, wl.num_kv_heads, wl.budget_pages, wl.budget_div)
    sel, cnt, scores = np_(sel), np_(cnt), np_(scores)
    for (bb, h), (sc, pages) in ref.items():
        pb = O.num_pages(wl.seq_lens[bb])
        assert np.array_equal(scores[bb, h, :pb].view(np.uint32), sc.view(np.uint32)), (bb, h)
        assert cnt[bb, h] == len(pages)
        assert np.array_equal(sel[bb, h, : len(pages)], pages), (bb, h)
    assert twl.twl_device_status(ws)[0] == twl.TWL_OK


def _select_on_device(wl, layer):
    dev = layer.device
    b, hq, mb = wl.batch, wl.num_q_heads, layer.max_budget
    q = torch.from_numpy(wl.q).to(dev)
    sel = torch.full((b, hq, mb), -1, dtype=torch.int32, device=dev)
    cnt = torch.zeros((b, hq), dtype=torch.int32, device=dev)
    ws = twl.alloc_workspace(twl.TWL_OP_SELECT, dev, batch=b, num_q_heads=hq,
                             num_kv_heads=wl.num_kv_heads, max_pages=wl.max_pages)
    twl.twl_select_pages(q, hq, layer.kv, layer.aux.bounds, wl.budget_pages, wl.budget_div, mb,
                         sel, cnt, None, ws)
    return q, sel, cnt


def _estimate_on_device(wl, layer, q, sel, cnt):
    dev = layer.device
    b, hq, mb = wl.batch, wl.num_q_heads, layer.max_budget
    cs = 16 * mb
    w = torch.zeros((b, hq, cs), dtype=torch.float32, device=dev)
    cand = torch.full((b, hq, cs), -1, dtype=torch.int32, device=dev)
    cc = torch.zeros((b, hq), dtype=torch.int32, device=dev)
    ws = twl.alloc_workspace(twl.TWL_OP_ESTIMATE, dev, batch=b, num_q_heads=hq,
                             num_kv_heads=wl.num_kv_heads, max_pages=wl.max_pages)
    twl.twl_estimate(q, hq, layer.kv, layer.aux.k_int4, layer.aux.k_scale_zero, sel, cnt, mb, w,
                     cand, cc, ws)
    return w, cand, cc


def test_estimate_weights(small):
    wl, layer = small
    q, sel, cnt = _select_on_device(wl, layer)
    w, cand, cc = _estimate_on_device(wl, layer, q, sel, cnt)
    q4, sz = O.quantize_k(wl.k, wl.page_table, wl.seq_lens)
    sel, cnt, w, cand, cc = np_(sel), np_(cnt), np_(w), np_(cand), np_(cc)
    g = wl.num_q_heads // wl.num_kv_heads
    for bb in range(wl.batch):
        for h in range(wl.num_q_heads):
            pages = sel[bb, h, : cnt[bb, h]]
            tok, w_or = O.estimate_head(wl.q[bb, h], q4, sz, wl.page_table, bb, h // g,
                                        int(wl.seq_lens[bb]), pages)
            assert cc[bb, h] == tok.size
            assert np.array_equal(cand[bb, h, : tok.size], tok)
            check_weights(w[bb, h, : tok.size], w_or, f"{wl.name} b{bb} h{h}")


def test_prune_decode_rows(small):
    wl, layer = small
    q, sel, cnt = _select_on_device(wl, layer)
    w, cand, cc = _estimate_on_device(wl, layer, q, sel, cnt)
    rows = wl.batch * wl.num_q_heads
    cs = w.shape[2]
    m = torch.zeros(rows, dtype=torch.float32, device=layer.device)
    kc = torch.zeros(rows, dtype=torch.int32, device=layer.device)
    ki = torch.full((rows, cs), -1, dtype=torch.int32, device=layer.device)
    twl.twl_prune_top_p(w, cc, rows, cs, wl.p, wl.eps, m, kc, ki)
    w, cc, m, kc, ki = np_(w).reshape(rows, cs), np_(cc).reshape(-1), np_(m), np_(kc), np_(ki)
    for r in range(rows):
        check_prune_row(w[r, : cc[r]], m[r], int(kc[r]), ki[r], wl.p, wl.eps, f"row {r}")


@pytest.mark.parametrize("n", [1, 7, 1000, 8192, 32768, 50000, 131072])
@pytest.mark.parametrize("p", [0.8, 0.9])
def test_prune_rows(n, p):
    rows = 64 if n <= 32768 else 16
    w_np, info = synth.config5_rows(rows, n, seed=n, tie_frac=0.1)
    w = torch.from_numpy(w_np).cuda()
    m = torch.zeros(rows, dtype=torch.float32, device="cuda")
    kc = torch.zeros(rows, dtype=torch.int32, device="cuda")
    ki = torch.full((rows, n), -1, dtype=torch.int32, device="cuda")
    twl.twl_prune_top_p(w, None, rows, n, p, 1e-6, m, kc, ki)
    m, kc, ki = np_(m), np_(kc), np_(ki)
    for r in range(rows):
        check_prune_row(w_np[r], m[r], int(kc[r]), ki[r], p, 1e-6, f"n{n} row {r}")


def _hard_rows(n, seed):
    """Rows that stress the threshold search: mass carried by many mid-sized weights, unnormalised
    rows (sum far above or below 1, weights above 1), a geometric profile spanning the fp32 range,
    near-uniform rows, a flat power law, and mostly-zero rows."""
    rng = np.random.default_rng(seed)
    rows = []
    r = np.full(n, 1e-9)
    idx = rng.choice(n, size=max(8, n // 16), replace=False)
    r[idx] = rng.uniform(0.9, 1.0, size=idx.size)
    rows.append(r / r.sum())
    rows.append(np.ones(n))                                     # sum n, every weight 1
    rows.append(rng.uniform(0.0, 100.0, size=n))                # weights above 1
    rows.append(0.5 * rng.dirichlet(np.ones(n)))                # sum 0.5 < p
    g = 2.0 ** -np.arange(1, n + 1, dtype=np.float64)
    rows.append(rng.permutation(np.maximum(g, 2.0 ** -140) / g.sum()))
    u = np.exp(0.01 * rng.standard_normal(n))
    rows.append(u / u.sum())                                    # near-uniform
    z = np.arange(1, n + 1, dtype=np.float64) ** -0.3
    rows.append(rng.permutation(z / z.sum()))                   # flat power law
    sp = np.where(rng.random(n) < 0.9, 0.0, np.exp(rng.standard_normal(n)))
    rows.append(sp / sp.sum())                                  # mostly zeros
    return np.stack(rows).astype(np.float32)


@pytest.mark.parametrize("n", [4096, 32768, 131072])
@pytest.mark.parametrize("p", [0.5, 0.9, 0.999])
def test_prune_hard_rows(n, p):
    w_np = _hard_rows(n, seed=n + int(p * 1000))
    rows = w_np.shape[0]
    w = torch.from_numpy(w_np).cuda()
    m = torch.zeros(rows, dtype=torch.float32, device="cuda")
    kc = torch.zeros(rows, dtype=torch.int32, device="cuda")
    ki = torch.full((rows, n), -1, dtype=torch.int32, device="cuda")
    twl.twl_prune_top_p(w, None, rows, n, p, 1e-6, m, kc, ki)
    m, kc, ki = np_(m), np_(kc), np_(ki)
    for r in range(rows):
        check_prune_row(w_np[r], m[r], int(kc[r]), ki[r], p, 1e-6, f"n{n} p{p} hard row {r}")


@pytest.mark.parametrize("n", [8192, 32768, 131072])
def test_prune_rows_mass_below_p(n):
    """Rows whose whole mass is below p: no threshold reaches p, so m = 0 and every weight is
    kept.  Rows whose mass sits just above p (by 1e-6 or 1e-4 relative) must still be searched."""
    rng = np.random.default_rng(n + 5)
    p = 0.9
    base = [rng.dirichlet(np.ones(n)), rng.dirichlet(np.full(n, 0.05))]
    rows = []
    for w in base:
        for scale in (0.5, p * (1 - 1e-4), p * (1 + 1e-6), p * (1 + 1e-4)):
            rows.append(w * scale)
    w_np = np.stack(rows).astype(np.float32)
    nr = w_np.shape[0]
    w = torch.from_numpy(w_np).cuda()
    m = torch.zeros(nr, dtype=torch.float32, device="cuda")
    kc = torch.zeros(nr, dtype=torch.int32, device="cuda")
    ki = torch.full((nr, n), -1, dtype=torch.int32, device="cuda")
    twl.twl_prune_top_p(w, None, nr, n, p, 1e-6, m, kc, ki)
    m, kc, ki = np_(m), np_(kc), np_(ki)
    for r in range(nr):
        total = float(w_np[r].astype(np.float64).sum())
        check_prune_row(w_np[r], m[r], int(kc[r]), ki[r], p, 1e-6, f"n{n} row {r} sum {total}")
        if total < p:
            assert m[r] == 0 and kc[r] == n, (r, total)
        else:   # searched: the bisection's own threshold (fp64 masses in the oracle)
            m_or, _ = O.top_p_bisect(w_np[r], p, 1e-6)
            assert m[r] == m_or, (r, total, float(m[r]), float(m_or))


@pytest.mark.parametrize("n", [8192, 131072])
def test_prune_rows_ragged_lengths(n):
    """Per-row lengths (row_len) shorter than the stride, including 0, 1 and non-multiples of 4."""
    rows = 12
    w_np, _ = synth.config5_rows(rows, n, seed=7)
    lens_np = np.array([0, 1, 3, 5, 17, 1000, n // 2 + 1, n - 3, n - 1, n, 4097, 33], np.int32)
    for r in range(rows):  # renormalise over the valid prefix
        L = int(lens_np[r])
        if L:
            w_np[r, :L] /= w_np[r, :L].astype(np.float64).sum()
    w = torch.from_numpy(w_np).cuda()
    lens = torch.from_numpy(lens_np).cuda()
    m = torch.zeros(rows, dtype=torch.float32, device="cuda")
    kc = torch.zeros(rows, dtype=torch.int32, device="cuda")
    ki = torch.full((rows, n), -1, dtype=torch.int32, device="cuda")
    twl.twl_prune_top_p(w, lens, rows, n, 0.9, 1e-6, m, kc, ki)
    m, kc, ki = np_(m), np_(kc), np_(ki)
    for r in range(rows):
        L = int(lens_np[r])
        if L == 0:
            assert kc[r] == 0
            continue
        check_prune_row(w_np[r, :L], m[r], int(kc[r]), ki[r], 0.9, 1e-6, f"n{n} len {L}")


@pytest.mark.parametrize("n", [8192, 32768, 131072])
def test_prune_rows_full_size(n):
    """The standalone-pruner workload at its full size (4096 rows, the launch the bench times:
    persistent CTAs or clusters that each walk many rows).  Every row: kept = {W >= m} and the
    kept mass reaches p; 48 sampled rows (spread over the launch): the full criteria against the
    oracle, including the ascending index list."""
    rows = 4096
    w_np, _ = synth.config5_rows(rows, n, seed=11)
    w = torch.from_numpy(w_np).cuda()
    m = torch.zeros(rows, dtype=torch.float32, device="cuda")
    kc = torch.zeros(rows, dtype=torch.int32, device="cuda")
    ki = torch.full((rows, n), -1, dtype=torch.int32, device="cuda")
    twl.twl_prune_top_p(w, None, rows, n, 0.9, 1e-6, m, kc, ki)
    m, kc = np_(m), np_(kc)
    keep = w >= torch.from_numpy(m).cuda()[:, None]
    assert np.array_equal(keep.sum(dim=1).cpu().numpy(), kc), "kept counts"
    mass = torch.where(keep, w, torch.zeros_like(w)).sum(dim=1, dtype=torch.float64).cpu().numpy()
    assert np.all(mass >= 0.9 - 1e-5), f"kept mass below p: {mass.min()}"
    sample = np.unique(np.concatenate([np.arange(8), np.linspace(0, rows - 1, 40).astype(int)]))
    ki_s = ki[torch.from_numpy(sample).cuda()].cpu().numpy()
    for j, r in enumerate(sample):
        check_prune_row(w_np[r], m[r], int(kc[r]), ki_s[j], 0.9, 1e-6, f"n{n} row {r}")


@pytest.mark.parametrize("n", [4096, 32768])
def test_prune_rows_nonfinite_and_extreme_parameters(n):
    """Weights outside the method's domain and extreme (p, eps).  NaN weights are never kept and
    carry no mass, negative weights carry none; a row holding +inf keeps exactly its infinite
    entries; a tiny p keeps the largest weight (and its ties); a wide eps stops the bisection
    early, so more is kept, but kept = {W >= m} and the mass condition still hold."""
    rng = np.random.default_rng(n)
    base = rng.dirichlet(np.ones(n)).astype(np.float32)
    rows = np.stack([base.copy() for _ in range(4)])
    rows[0, rng.choice(n, 7, replace=False)] = np.nan
    rows[1, rng.choice(n, 9, replace=False)] = -rng.random(9).astype(np.float32)
    rows[2, [3, 11]] = np.inf
    rows[3, 5] = 0.5
    w = torch.from_numpy(rows).cuda()
    for p, eps in ((0.85, 1e-6), (0.01, 1e-6), (0.85, 0.1)):
        m = torch.zeros(4, dtype=torch.float32, device="cuda")
        kc = torch.zeros(4, dtype=torch.int32, device="cuda")
        ki = torch.full((4, n), -1, dtype=torch.int32, device="cuda")
        twl.twl_prune_top_p(w, None, 4, n, p, eps, m, kc, ki)
        mn, kcn, kin = np_(m), np_(kc), np_(ki)
        for r in range(4):
            with np.errstate(invalid="ignore"):
                keep = np.nonzero(rows[r] >= mn[r])[0]
            assert kcn[r] == keep.size and np.array_equal(kin[r, : keep.size], keep), (p, eps, r)
            if r == 2:
                assert np.isinf(mn[r]) and list(keep) == [3, 11]
                continue
            finite = np.where(np.isfinite(rows[r]) & (rows[r] > 0), rows[r], 0).astype(np.float64)
            assert finite[keep].sum() >= min(p, finite.sum()) - 1e-5, (p, eps, r)
            if eps < 1e-3:
                k_star, m_star, _ = O.top_p_sort(finite, p)
                band = int(np.count_nonzero((finite >= float(m_star) - eps) & (finite <= m_star)))
                assert keep.size <= k_star + band, (p, eps, r)
        if p == 0.01:
            assert kcn[3] == 1 and kin[3, 0] == 5      # the one weight of 0.5


def test_prune_special_rows():
    n = 40
    rows = np.zeros((5, n), dtype=np.float32)
    rows[0, 17] = 1.0                                   # one-hot
    rows[1, :] = 1.0 / n                                # uniform: all ties
    rows[2, :4] = 0.2
    rows[2, 4:24] = 0.01                                # two-level, hand example
    rows[3, :3] = np.float32(0.25)
    rows[3, 3] = np.float32(0.25)                       # dyadic, exact sums
    rows[4, :] = 0.0                                    # all zero
    lens = torch.tensor([n, n, 24, 4, n], dtype=torch.int32, device="cuda")
    w = torch.from_numpy(rows).cuda()
    m = torch.zeros(5, device="cuda")
    kc = torch.zeros(5, dtype=torch.int32, device="cuda")
    ki = torch.full((5, n), -1, dtype=torch.int32, device="cuda")
    twl.twl_prune_top_p(w, lens, 5, n, 0.845, 1e-6, m, kc, ki)
    m, kc, ki = np_(m), np_(kc), np_(ki)
    assert kc[0] == 1 and ki[0, 0] == 17 and m[0] == 1.0
    assert kc[1] == n                                   # ties at the threshold are all kept
    assert kc[2] >= 9                                   # k* = 9; the 0.01 ties come along
    check_prune_row(rows[2, :24], m[2], int(kc[2]), ki[2], 0.845, 1e-6)
    assert kc[3] == 4
    assert kc[4] == n                                   # nothing reaches p: keep all


def test_group_union_exact(small):
    wl, layer = small
    q, sel, cnt = _select_on_device(wl, layer)
    w, cand, cc = _estimate_on_device(wl, layer, q, sel, cnt)
    rows = wl.batch * wl.num_q_heads
    cs = w.shape[2]
    dev = layer.device
    m = torch.zeros(rows, device=dev)
    kc = torch.zeros(rows, dtype=torch.int32, device=dev)
    ki = torch.full((rows, cs), -1, dtype=torch.int32, device=dev)
    twl.twl_prune_top_p(w, cc, rows, cs, wl.p, wl.eps, m, kc, ki)
    us = 16 * wl.max_pages
    ut = torch.full((wl.batch, wl.num_kv_heads, us), -1, dtype=torch.int32, device=dev)
    uc = torch.zeros((wl.batch, wl.num_kv_heads), dtype=torch.int32, device=dev)
    twl.twl_group_union(wl.num_q_heads, layer.kv, cand, ki, kc, cs, ut, uc)
    cand, kc, ki, ut, uc = np_(cand), np_(kc).reshape(wl.batch, -1), np_(ki).reshape(
        wl.batch, wl.num_q_heads, cs), np_(ut), np_(uc)
    g = wl.num_q_heads // wl.num_kv_heads
    for bb in range(wl.batch):
        for kvh in range(wl.num_kv_heads):
            want = set()
            for h in range(kvh * g, (kvh + 1) * g):
                want |= set(cand[bb, h, ki[bb, h, : kc[bb, h]]].tolist())
            assert np.array_equal(ut[bb, kvh, : uc[bb, kvh]], np.array(sorted(want)))


def _token_sets(wl, rng):
    sets = {}
    for bb in range(wl.batch):
        n = int(wl.seq_lens[bb])
        for kvh in range(wl.num_kv_heads):
            kind = (bb + kvh) % 5
            if kind == 0:
                toks = np.arange(n)                                     # dense
            elif kind == 1:
                toks = np.array([int(rng.integers(0, n))])              # one token
            elif kind == 2:
                toks = np.zeros(0, dtype=np.int64)                      # empty
            elif kind == 3:
                toks = np.arange(min(n, 129))                           # one chunk + 1
            else:
                toks = np.sort(rng.choice(n, size=min(n, 300), replace=False))
            sets[(bb, kvh)] = toks.astype(np.int64)
    return sets


def test_sparse_decode_vs_oracle(small):
    wl, layer = small
    rng = np.random.default_rng(11)
    sets = _token_sets(wl, rng)
    stride = 16 * wl.max_pages
    tok = np.full((wl.batch, wl.num_kv_heads, stride), -1, dtype=np.int32)
    cnt = np.zeros((wl.batch, wl.num_kv_heads), dtype=np.int32)
    for (bb, kvh), t in sets.items():
        tok[bb, kvh, : t.size] = t
        cnt[bb, kvh] = t.size
    dev = layer.device
    q = torch.from_numpy(wl.q).to(dev)
    o = torch.zeros((wl.batch, wl.num_q_heads, 128), device=dev)
    lse = torch.zeros((wl.batch, wl.num_q_heads), device=dev)
    ws = twl.alloc_workspace(twl.TWL_OP_SPARSE_DECODE, dev, batch=wl.batch,
                             num_q_heads=wl.num_q_heads, num_kv_heads=wl.num_kv_heads,
                             row_stride=stride)
    twl.twl_sparse_decode(q, wl.num_q_heads, layer.kv, torch.from_numpy(tok).to(dev),
                          torch.from_numpy(cnt).to(dev), stride, SM_SCALE, o, lse, ws)
    ref = O.group_attention(wl, sets)
    o, lse = np_(o), np_(lse)
    for (bb, h), (o_or, lse_or) in ref.items():
        check_attention(o[bb, h], lse[bb, h], o_or, lse_or, f"{wl.name} b{bb} h{h}")


# -------------------------------------------------------------------------- the whole step

def _run_step(wl, layer):
    stats = layer.alloc_stats()
    q = torch.from_numpy(wl.q).to(layer.device)
    o, lse = layer.decode(q, wl.p, wl.eps, stats)
    st = {k: np_(v) for k, v in stats.items()}
    return st, np_(o), np_(lse)


def test_decode_step_vs_oracle(small):
    wl, layer = small
    st, o, lse = _run_step(wl, layer)
    for bb in range(wl.batch):
        for kvh in range(wl.num_kv_heads):
            check_step_group(wl, bb, kvh, st, o, lse)
    assert layer.status()[0] == twl.TWL_OK


def test_decode_step_without_stats_attends_locally(small):
    # without stats each CTA attends over its own kept rows (no ordered union list); the output
    # must match the stats run up to summation order, and the oracle over the same union
    wl, layer = small
    st, o1, lse1 = _run_step(wl, layer)
    q = torch.from_numpy(wl.q).to(layer.device)
    o2, lse2 = layer.decode(q, wl.p, wl.eps, None)
    o2, lse2 = np_(o2), np_(lse2)
    assert np.abs(o2 - o1).max() <= 2e-4 and np.abs(lse2 - lse1).max() <= 2e-4
    for bb in range(wl.batch):
        for kvh in range(wl.num_kv_heads):
            uc = int(st["union_count"][bb, kvh])
            att = O.group_attention(wl, {(bb, kvh): st["union_tok"][bb, kvh, :uc]})
            for (b2, h), (o_or, lse_or) in att.items():
                check_attention(o2[b2, h], lse2[b2, h], o_or, lse_or, f"{wl.name} b{b2} h{h}")


def test_decode_step_deterministic(small):
    wl, layer = small
    a = _run_step(wl, layer)
    b = _run_step(wl, layer)
    for k in a[0]:
        assert np.array_equal(a[0][k], b[0][k]), k
    assert np.array_equal(a[1], b[1]) and np.array_equal(a[2], b[2])


def test_decode_step_equals_staged_calls(small):
    wl, layer = small
    st, o, lse = _run_step(wl, layer)
    q, sel, cnt = _select_on_device(wl, layer)
    w, cand, cc = _estimate_on_device(wl, layer, q, sel, cnt)
    assert np.array_equal(np_(sel), st["sel_pages"]) and np.array_equal(np_(cnt), st["sel_count"])
    assert np.array_equal(np_(cc), st["cand_count"])
    wn, ccn = np_(w), np_(cc)
    for bb in range(wl.batch):
        for h in range(wl.num_q_heads):
            c = ccn[bb, h]
            # two fp32 logit computations that differ in accumulation order (both are checked
            # against the oracle at 1e-3): large logits (~270) move W by ~3e-5 relative
            assert np.allclose(wn[bb, h, :c], st["weights"][bb, h, :c], rtol=5e-4, atol=1e-9)
    dev = layer.device
    stride = 16 * wl.max_pages
    o2 = torch.zeros((wl.batch, wl.num_q_heads, 128), device=dev)
    lse2 = torch.zeros((wl.batch, wl.num_q_heads), device=dev)
    ws = twl.alloc_workspace(twl.TWL_OP_SPARSE_DECODE, dev, batch=wl.batch,
                             num_q_heads=wl.num_q_heads, num_kv_heads=wl.num_kv_heads,
                             row_stride=stride)
    twl.twl_sparse_decode(q, wl.num_q_heads, layer.kv, torch.from_numpy(st["union_tok"]).to(dev),
                          torch.from_numpy(st["union_count"]).to(dev), stride, SM_SCALE, o2,
                          lse2, ws)
    # two fp32 attention kernels that differ only in chunking and summation order
    do, dl = float(np.abs(np_(o2) - o).max()), float(np.abs(np_(lse2) - lse).max())
    assert do <= 2e-4 and dl <= 2e-4, (do, dl)


def test_staged_wrapper_matches_the_oracle(small):
    """The five staged calls through layer.Staged (the bench's staged comparison): every group's
    selection, candidates, weights, kept sets and output against the oracle."""
    wl, layer = small
    stg = layer.staged()
    q = torch.from_numpy(wl.q).to(layer.device)
    o, lse = stg.decode(q, wl.p, wl.eps)
    rows = wl.batch * wl.num_q_heads
    st = {
        "sel_pages": np_(stg.sel), "sel_count": np_(stg.sel_count),
        "weights": np_(stg.weights), "cand_tok": np_(stg.cand_tok),
        "cand_count": np_(stg.cand_count),
        "threshold": np_(stg.m).reshape(wl.batch, wl.num_q_heads),
        "kept_count": np_(stg.kept_count).reshape(wl.batch, wl.num_q_heads),
        "union_tok": np_(stg.union_tok), "union_count": np_(stg.union_count),
    }
    assert rows == st["kept_count"].size
    o, lse = np_(o), np_(lse)
    for bb in range(wl.batch):
        for kvh in range(wl.num_kv_heads):
            check_step_group(wl, bb, kvh, st, o, lse)
    assert twl.twl_device_status(stg.ws_sel)[0] == twl.TWL_OK


def test_decode_step_dense_limit():
    # budget = every page and p = 1: the step is exact dense attention
    wl = synth.make_decode("dense", 1, 8, 2, [700], seed=8)
    wl.budget_pages = 10 ** 4
    wl.p = 1.0
    layer = DecodeLayer.from_workload(wl)
    layer.build_aux()
    st, o, lse = _run_step(wl, layer)
    toks = np.arange(700)
    ref = O.group_attention(wl, {(0, kvh): toks for kvh in range(2)})
    for (bb, h), (o_or, lse_or) in ref.items():
        assert st["union_count"][0, h // 4] == 700
        check_attention(o[bb, h], lse[bb, h], o_or, lse_or, f"dense h{h}")


@pytest.mark.parametrize("shape", [
    (1, 8, 1, [3001]),                      # one group: ~90 one-page score items, 64 slices
    (2, 8, 2, [3001, 515]),                 # 4 groups
    (5, 16, 8, [1999, 17, 4100, 700, 1]),   # 40 groups, ragged, a one-token sequence
    (12, 8, 8, [2500] * 12),                # 96 groups: several items per CTA in every kind
], ids=["1grp", "4grp", "40grp", "96grp"])
def test_decode_step_work_list_shapes(shape):
    """The persistent step cuts each group into score chunks and estimate / attention slices
    sized from the group count; these shapes cover every branch of that plan (one group spread
    over the whole GPU, a few groups, more groups than half the SMs)."""
    batch, hq, hkv, lens = shape
    wl = synth.make_decode("shapes", batch, hq, hkv, lens, seed=9 + batch, permute_pages=True,
                           temperature=True)
    layer = DecodeLayer.from_workload(wl)
    layer.build_aux()
    st, o, lse = _run_step(wl, layer)
    for bb in range(wl.batch):
        for kvh in range(wl.num_kv_heads):
            check_step_group(wl, bb, kvh, st, o, lse)
    assert layer.status()[0] == twl.TWL_OK


def test_decode_step_repeated_launches_on_one_workspace():
    """Back-to-back steps on one workspace (its synchronisation words are cleared by each launch
    for the next), including a different p in between: every launch equals a fresh one."""
    wl = synth.make_decode("repeat", 3, 16, 4, [2000, 900, 3100], seed=41, temperature=True)
    layer = DecodeLayer.from_workload(wl)
    layer.build_aux()
    q = torch.from_numpy(wl.q).cuda()
    first = [t.clone() for t in layer.decode(q, wl.p, wl.eps)]
    for p in (0.9, 0.85, 0.7, 0.85):
        for _ in range(5):
            layer.decode(q, p, wl.eps)
    again = layer.decode(q, wl.p, wl.eps)
    assert torch.equal(first[0], again[0]) and torch.equal(first[1], again[1])
    assert layer.status()[0] == twl.TWL_OK


@pytest.mark.parametrize("shape", [
    (20, 8, 8, 700),     # 160 groups, group size 1
    (40, 16, 8, 500),    # 320 groups, group size 2
    (80, 16, 2, 300),    # 160 groups, group size 8
], ids=["g1", "g2", "g8"])
def test_decode_step_two_ctas_per_sm(shape):
    """More groups than SMs: the 256-thread build (two CTAs per SM) runs; every group size it is
    built for, sampled groups against the oracle."""
    batch, hq, hkv, n = shape
    lens = [n + 29 * i for i in range(batch)]
    wl = synth.make_decode("wide", batch, hq, hkv, lens, seed=51 + hkv, permute_pages=True,
                           temperature=True)
    layer = DecodeLayer.from_workload(wl)
    layer.build_aux()
    st, o, lse = _run_step(wl, layer)
    for bb, kvh in [(0, 0), (batch // 3, hkv - 1), (batch - 1, hkv // 2)]:
        check_step_group(wl, bb, kvh, st, o, lse)
    assert layer.status()[0] == twl.TWL_OK


def test_decode_step_more_groups_than_sms():
    """320 (sequence, kv-head) groups, more than twice the SMs: several items of every kind per
    CTA; sampled groups."""
    lens = [300 + 37 * i for i in range(40)]
    wl = synth.make_decode("many_groups", 40, 32, 8, lens, seed=29, permute_pages=True)
    layer = DecodeLayer.from_workload(wl)
    layer.build_aux()
    st, o, lse = _run_step(wl, layer)
    for bb, kvh in [(0, 0), (7, 3), (21, 5), (39, 7)]:
        check_step_group(wl, bb, kvh, st, o, lse)
    assert layer.status()[0] == twl.TWL_OK


# -------------------------------------------------------------------------- full-size workloads

def _full_check(wl, groups):
    layer = DecodeLayer.from_workload(wl)
    layer.build_aux()
    st, o, lse = _run_step(wl, layer)
    reports = [check_step_group(wl, b, kvh, st, o, lse) for b, kvh in groups]
    assert layer.status()[0] == twl.TWL_OK
    # bounds and INT4 of the sampled groups' pages
    for b, kvh in groups:
        pb = O.num_pages(wl.seq_lens[b])
        phys = wl.page_table[b, :pb].astype(np.int64)
        sub_k = wl.k[phys, kvh:kvh + 1]
        pt = np.arange(pb, dtype=np.int32)[None]
        ref_b = O.page_bounds(sub_k, pt, wl.seq_lens[b:b + 1])
        got_b = np_(layer.aux.bounds)[phys, kvh:kvh + 1]
        assert np.array_equal(u16(got_b), u16(ref_b))
    return reports


def test_full_gqa_32k_all_groups():
    wl = synth.config2()
    _full_check(wl, [(0, kvh) for kvh in range(8)])


def test_full_batch16_sampled():
    wl = synth.config3()
    _full_check(wl, [(0, 0), (5, 3), (15, 7)])


@pytest.fixture(scope="module")
def c4_layer():
    wl = synth.config4()
    layer = DecodeLayer.from_workload(wl)
    layer.build_aux()
    torch.cuda.synchronize()
    return wl, layer


@pytest.mark.parametrize("p", [0.70, 0.85, 0.95])
def test_full_128k_sampled(c4_layer, p):
    """The long-context layer at every p of its sweep (the bench times all three)."""
    wl, layer = c4_layer
    wl.p = p
    try:
        st, o, lse = _run_step(wl, layer)
        for b, kvh in [(0, 1), (1, 4), (3, 6)]:
            check_step_group(wl, b, kvh, st, o, lse)
        assert layer.status()[0] == twl.TWL_OK
    finally:
        wl.p = 0.85


def _live_counts(wl, b, kvh, p):
    """Per head of the group: the oracle's candidate count and the size of the live set
    {W >= (1 - p) / (2 nc)} that a threshold search over live weights would have to rank."""
    from twl_checks import group_workload
    sub = group_workload(wl, b, kvh)
    sub.p = p
    r = O.decode_step(sub, with_attention=False)
    out = []
    for d in r["heads"].values():
        nc = d["cand"].size
        out.append((nc, int(np.count_nonzero(d["w"] >= (1 - p) / (2 * nc)))))
    return out


@pytest.mark.parametrize("n", [8192, 40000])
@pytest.mark.parametrize("p", [0.85, 0.9995])
def test_decode_step_diffuse_heads(n, p):
    """Diffuse heads (no heavy tokens, logit temperature 2-8): most candidates survive top-p, so
    the threshold search runs over thousands of live weights (more than any CTA has threads) and,
    at 40000 tokens, over more candidates than a CTA holds in registers; p within 1e-3 of 1 also
    turns off the live-set bound.  Every group against the oracle."""
    wl = synth.config_diffuse(n=n)
    wl.p = p
    layer = DecodeLayer.from_workload(wl)
    layer.build_aux()
    st, o, lse = _run_step(wl, layer)
    for kvh in range(wl.num_kv_heads):
        check_step_group(wl, 0, kvh, st, o, lse)
    assert layer.status()[0] == twl.TWL_OK
    live = _live_counts(wl, 0, 0, p)
    assert min(l for _, l in live) > 1024, live
    if n == 40000:
        assert min(nc for nc, _ in live) > 16 * 512, live
    kept = st["kept_count"].reshape(-1) / np.maximum(st["cand_count"].reshape(-1), 1)
    assert kept.min() > 0.5, kept
