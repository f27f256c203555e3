"""Planted mistakes in the later stages of the CPU oracle: each check below ties one oracle
function to something other than itself (a closed form, a hand-worked row, brute force or a
library routine of the same definition), and each test shows that the oracle passes the check
while copies of the function with one plausible mistake fail it.

Sources: [Notes] = "Twilight: Adaptive Attention Sparsity with Hierarchical Top-p Pruning",
Paper-Notes (NeurIPS 2025) page; [Summary] = the paperlayer summary of arXiv 2502.02770v5;
[Double-P] = the Double-P summary page.

  estimate     K on the INT4 grid, so the dequantised K is exact: the estimate equals torch's
               softmax of q.K/sqrt(D) over the selected pages' valid tokens ([Summary] 4.2, B.1).
  attention    torch scaled_dot_product_attention and logsumexp in fp64; one kept token gives
               o = v, lse = its logit; no kept token gives o = 0, lse = -inf.
  GQA union    every q-head of a group attends over the union of the group's kept tokens
               ([Summary] B.2): the union is rebuilt by a scan over token ids, the outputs by
               torch over rows gathered with explicit page-table arithmetic.
  centroids    the plain mean where fp32 sums are exact (values on a 1/8 grid), over the valid
               rows only, behind a permuted page table, per kv-head.
  cluster      pages of identical rows: n_j exp(q.c_j/sqrt(D)) is the page's exact attention
  weights      mass, so the weights equal the exact mass shares ([Double-P] "Key designs").
  n-bit codes  hand-worked bytes at 2 bits with round-half-even ties and at 8 bits.
  append       the incremental update equals the full definitions recomputed over the extended
               cache, and a page's first row replaces whatever bounds the page held before.
"""
import math

import numpy as np
import torch

from oracle import twl_oracle as O
from workloads import synth

F16, F32, F64 = np.float16, np.float32, np.float64
D, PAGE = 128, 16


def u16(x):
    return np.ascontiguousarray(x).view(np.uint16)


# ------------------------------------------------------------------------------------- estimate

def _grid_case(seed=8):
    """One kv-head of 150 tokens (the last page holds 6) whose K rows lie on their own INT4 grid:
    k = n*s + z exactly, with the row's minimum and maximum attained, so quantisation loses
    nothing and k_hat = k."""
    rng = np.random.default_rng(seed)
    n_tok, n_pages = 150, 10
    rows = n_pages * PAGE
    s = rng.choice([0.125, 0.25, 0.5], size=rows).astype(F16)
    z = (-rng.integers(1, 16, size=rows) * s.astype(F64)).astype(F16)     # nonzero zero points
    nib = rng.integers(0, 16, size=(rows, D))
    nib[:, 0], nib[:, 1] = 0, 15
    k = (nib * s[:, None].astype(F64) + z[:, None].astype(F64)).astype(F16)
    assert np.array_equal(k.astype(F64), nib * s[:, None].astype(F64) + z[:, None].astype(F64))
    perm = rng.permutation(n_pages)
    kk = np.zeros((n_pages, 1, PAGE, D), F16)
    for j in range(n_pages):                    # logical page j lives in physical page perm[j]
        kk[perm[j], 0] = k[PAGE * j:PAGE * (j + 1)]
    pt = perm.astype(np.int32)[None, :]
    lens = np.array([n_tok], dtype=np.int32)
    q = (rng.standard_normal(D) * 2).astype(F16)
    return k, kk, pt, lens, q


def check_estimate(estimate_fn):
    k, kk, pt, lens, q = _grid_case()
    q4, sz = O.quantize_k(kk, pt, lens)
    n = int(lens[0])
    for sel in ([1, 4, 5, 9], [9], [0, 2, 3, 6, 7, 8]):
        cand, w = estimate_fn(q, q4, sz, pt, 0, 0, n, np.array(sel))
        want_cand = [t for t in range(n) if t // PAGE in sel]
        if list(np.asarray(cand)) != want_cand:
            return False
        logits = torch.from_numpy(k[want_cand].astype(F64)) @ torch.from_numpy(q.astype(F64))
        ref = torch.softmax(logits / math.sqrt(D), dim=0).numpy()
        if not np.allclose(w, ref, rtol=1e-12, atol=1e-15):
            return False
    return True


def _estimate_variant(q16, k_int4, k_sz, page_table, b, kvh, n, sel_pages, *, swap=False,
                      zero=True, scale=None):
    cand = O.candidates(sel_pages, n)
    packed = O.gather_tokens(k_int4, page_table, b, kvh, cand)
    sz = O.gather_tokens(k_sz, page_table, b, kvh, cand)
    nib = np.empty((cand.size, D), dtype=F64)
    lo, hi = packed & 0x0F, packed >> 4
    nib[:, 0::2], nib[:, 1::2] = (hi, lo) if swap else (lo, hi)
    khat = nib * sz[:, 0:1].astype(F64)
    if zero:
        khat = khat + sz[:, 1:2].astype(F64)
    logits = khat @ np.asarray(q16, dtype=F16).astype(F64)
    logits = logits / (math.sqrt(D) if scale is None else scale)
    return cand, O.softmax64(logits)


def test_estimate_mistakes_fail_the_grid_pin():
    assert check_estimate(O.estimate_head)
    assert check_estimate(lambda *a: O.estimate_head_bits(*a, bits=4))
    assert check_estimate(_estimate_variant)                          # the variant as written
    assert not check_estimate(lambda *a: _estimate_variant(*a, swap=True))     # nibble order
    assert not check_estimate(lambda *a: _estimate_variant(*a, zero=False))    # drops z
    assert not check_estimate(lambda *a: _estimate_variant(*a, scale=D))       # 1/D scaling
    assert not check_estimate(lambda *a: _estimate_variant(*a, scale=1.0))     # no scaling

    def full_last_page(q16, k_int4, k_sz, page_table, b, kvh, n, sel_pages):
        return _estimate_variant(q16, k_int4, k_sz, page_table, b, kvh, PAGE * O.num_pages(n),
                                 sel_pages)

    assert not check_estimate(full_last_page)        # keeps the rows past the sequence end


# ------------------------------------------------------------------------------------- attention

def check_attention_fn(attention_fn):
    rng = np.random.default_rng(11)
    scale = 1 / math.sqrt(D)
    for m in (300, 17):
        q = rng.standard_normal(D).astype(F16)
        k = (rng.standard_normal((m, D)) * 2).astype(F16)
        v = rng.standard_normal((m, D)).astype(F16)
        o, lse = attention_fn(q, k, v, scale)
        tq = torch.from_numpy(q.astype(F64)).view(1, 1, 1, D)
        tk = torch.from_numpy(k.astype(F64)).view(1, 1, m, D)
        tv = torch.from_numpy(v.astype(F64)).view(1, 1, m, D)
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv).view(D).numpy()
        if not np.allclose(o, ref, rtol=1e-12, atol=1e-12):
            return False
        s = torch.from_numpy(k.astype(F64)) @ torch.from_numpy(q.astype(F64)) * scale
        if abs(lse - torch.logsumexp(s, 0).item()) > 1e-12:
            return False
    q = rng.standard_normal(D).astype(F16)
    k1 = rng.standard_normal((1, D)).astype(F16)
    v1 = rng.standard_normal((1, D)).astype(F16)
    o, lse = attention_fn(q, k1, v1, scale)
    if not np.array_equal(np.asarray(o), v1[0].astype(F64)):
        return False
    if abs(lse - float(k1[0].astype(F64) @ q.astype(F64)) * scale) > 1e-12:
        return False
    o, lse = attention_fn(q, np.zeros((0, D), F16), np.zeros((0, D), F16), scale)
    return bool(np.all(np.asarray(o) == 0) and lse == -math.inf)


def _attention_variant(q16, k16, v16, scale, *, use_scale=True, normalise=True, log2=False):
    q = np.asarray(q16, dtype=F16).astype(F64)
    k = np.asarray(k16, dtype=F16).astype(F64)
    v = np.asarray(v16, dtype=F16).astype(F64)
    if k.shape[0] == 0:
        return np.zeros(D), -math.inf
    s = k @ q * (F64(scale) if use_scale else 1.0)
    mx = s.max()
    e = np.exp(s - mx)
    l = e.sum()
    o = e @ v / l if normalise else e @ v
    lse = (mx + math.log(l)) / math.log(2.0) if log2 else mx + math.log(l)
    return o, float(lse)


def test_attention_mistakes_fail_the_library_pin():
    assert check_attention_fn(O.attention)
    assert check_attention_fn(_attention_variant)
    assert not check_attention_fn(lambda *a: _attention_variant(*a, use_scale=False))
    assert not check_attention_fn(lambda *a: _attention_variant(*a, normalise=False))
    assert not check_attention_fn(lambda *a: _attention_variant(*a, log2=True))

    def lse_without_max(q16, k16, v16, scale):
        o, lse = _attention_variant(q16, k16, v16, scale)
        s = np.asarray(k16, F16).astype(F64) @ np.asarray(q16, F16).astype(F64) * scale
        return o, float(math.log(np.exp(s - s.max()).sum())) if s.size else lse

    assert not check_attention_fn(lse_without_max)


# ------------------------------------------------------------------------------------- GQA union

def check_group_union(decode_fn):
    """Per (sequence, kv-head) group: the union is every token id some q-head of the group kept
    (q-head h belongs to kv-head h // (Hq / Hkv)), found by a scan over token ids; each head's
    output is torch's attention over the union's rows, gathered by page-table arithmetic."""
    wl = synth.make_decode("union", 2, 8, 2, [400, 233], seed=3, permute_pages=True,
                           temperature=True)
    r = decode_fn(wl)
    g = wl.num_q_heads // wl.num_kv_heads
    for b in range(wl.batch):
        n = int(wl.seq_lens[b])
        for kvh in range(wl.num_kv_heads):
            kept = [set(np.asarray(r["heads"][(b, h)]["kept_tok"]).tolist())
                    for h in range(kvh * g, (kvh + 1) * g)]
            want = [t for t in range(n) if any(t in s for s in kept)]
            grp = r["groups"][(b, kvh)]
            if list(np.asarray(grp["union"])) != want:
                return False
            rows = [(int(wl.page_table[b, t // PAGE]), t % PAGE) for t in want]
            kk = np.stack([wl.k[p, kvh, i] for p, i in rows]).astype(F64)
            vv = np.stack([wl.v[p, kvh, i] for p, i in rows]).astype(F64)
            for h in range(kvh * g, (kvh + 1) * g):
                tq = torch.from_numpy(wl.q[b, h].astype(F64)).view(1, 1, 1, D)
                ref = torch.nn.functional.scaled_dot_product_attention(
                    tq, torch.from_numpy(kk).view(1, 1, -1, D),
                    torch.from_numpy(vv).view(1, 1, -1, D)).view(D).numpy()
                if not np.allclose(grp["o"][h], ref, rtol=1e-11, atol=1e-12):
                    return False
    return True


def _decode_with_union(wl, union_rule):
    """The oracle's per-head stages, then a group stage whose token sets follow `union_rule`
    (a function of (b, kvh, heads) returning {h: tokens})."""
    r = O.decode_step(wl, with_attention=False)
    g = wl.num_q_heads // wl.num_kv_heads
    scale = 1.0 / math.sqrt(wl.head_dim)
    for (b, kvh), grp in r["groups"].items():
        toks = union_rule(b, kvh, r["heads"], g, wl.num_kv_heads)
        grp["o"], grp["lse"] = {}, {}
        grp["union"] = np.unique(np.concatenate(list(toks.values())))
        for h, t in toks.items():
            kk = O.gather_tokens(wl.k, wl.page_table, b, kvh, t)
            vv = O.gather_tokens(wl.v, wl.page_table, b, kvh, t)
            grp["o"][h], grp["lse"][h] = O.attention(wl.q[b, h], kk, vv, scale)
    return r


def test_gqa_union_mistakes_fail_the_scan_pin():
    assert check_group_union(O.decode_step)

    def union(b, kvh, heads, g, hkv):                      # the reading, restated
        t = np.unique(np.concatenate([heads[(b, h)]["kept_tok"]
                                      for h in range(kvh * g, (kvh + 1) * g)]))
        return {h: t for h in range(kvh * g, (kvh + 1) * g)}

    def own_set_only(b, kvh, heads, g, hkv):               # no union: each head its own tokens
        return {h: heads[(b, h)]["kept_tok"] for h in range(kvh * g, (kvh + 1) * g)}

    def head_modulo(b, kvh, heads, g, hkv):                # group = heads h with h % Hkv == kvh
        t = np.unique(np.concatenate([heads[(b, h)]["kept_tok"]
                                      for h in range(kvh, g * hkv, hkv)]))
        return {h: t for h in range(kvh * g, (kvh + 1) * g)}

    def first_head_only(b, kvh, heads, g, hkv):
        t = heads[(b, kvh * g)]["kept_tok"]
        return {h: t for h in range(kvh * g, (kvh + 1) * g)}

    assert check_group_union(lambda wl: _decode_with_union(wl, union))
    for rule in (own_set_only, head_modulo, first_head_only):
        assert not check_group_union(lambda wl, rule=rule: _decode_with_union(wl, rule)), rule


# ------------------------------------------------------------------------------------- centroids

def check_centroids(centroid_fn):
    """Rows on a 1/8 grid make every fp32 partial sum exact, so each centroid is the fp64 mean
    of the page's valid rows rounded to fp16; the rows past the end of sequence 1 hold garbage,
    the page table is permuted and the two kv-heads differ."""
    rng = np.random.default_rng(0)
    k = (rng.integers(-64, 64, (6, 2, PAGE, D)) / 8).astype(F16)
    pt = np.array([[4, 1, 3], [0, 5, 2]], np.int32)
    lens = np.array([48, 16 + 16 + 5])
    k[2, :, 5:] = F16(1000.0)                            # past the end of sequence 1
    cen = centroid_fn(k, pt, lens)
    for b in range(2):
        for j in range(3):
            rows = O.valid_rows(int(lens[b]), j)
            ph = pt[b, j]
            want = k[ph, :, :rows].astype(F64).mean(axis=1).astype(F16)
            if not np.array_equal(u16(cen[ph]), u16(want)):
                return False
    return True


def test_centroid_mistakes_fail_the_exact_mean_pin():
    assert check_centroids(O.page_centroids)

    def over_all_rows(k, pt, lens):                      # ignores the sequence end
        return O.page_centroids(k, pt, np.full_like(lens, PAGE * pt.shape[1]))

    def divides_by_page_size(k, pt, lens):               # sums the valid rows, divides by 16
        cen = O.page_centroids(k, pt, lens).astype(F64)
        for b in range(len(lens)):
            for j in range(O.num_pages(int(lens[b]))):
                rows = O.valid_rows(int(lens[b]), j)
                cen[pt[b, j]] = cen[pt[b, j]] * rows / PAGE
        return cen.astype(F16)

    def logical_pages(k, pt, lens):                      # no page table
        out = np.zeros((k.shape[0], k.shape[1], D), F16)
        ident = np.arange(pt.size, dtype=np.int32).reshape(pt.shape) % k.shape[0]
        got = O.page_centroids(k, ident, lens)
        for b in range(len(lens)):
            for j in range(O.num_pages(int(lens[b]))):
                out[pt[b, j]] = got[ident[b, j]]
        return out

    def kv_heads_swapped(k, pt, lens):
        return O.page_centroids(k, pt, lens)[:, ::-1]

    for fn in (over_all_rows, divides_by_page_size, logical_pages, kv_heads_swapped):
        assert not check_centroids(fn), fn.__name__


# ------------------------------------------------------------------------------------- cluster weights

def check_cluster_weights(weights_fn):
    """Pages of identical rows behind a permuted table, the last page partial: the sum of
    exp(q.k_i/sqrt(D)) over a page's valid rows is exactly n_j exp(q.c_j/sqrt(D)), so the
    weights are the pages' exact shares of the attention mass, summed token by token."""
    rng = np.random.default_rng(1)
    npages, n = 7, 7 * PAGE - 9
    k = np.zeros((npages, 2, PAGE, D), F16)
    for j in range(npages):
        k[j, :, :] = (rng.standard_normal((2, 1, D)) * 0.5).astype(F16)
    pt = rng.permutation(npages).astype(np.int32)[None]
    q = rng.standard_normal(D).astype(F16)
    cen = O.page_centroids(k, pt, np.array([n]))
    for kvh in range(2):
        w = weights_fn(q, cen, pt, 0, kvh, n)
        logits = np.array([k[pt[0, t // PAGE], kvh, t % PAGE].astype(F64) @ q.astype(F64)
                           for t in range(n)]) / math.sqrt(D)
        e = np.exp(logits - logits.max())
        mass = np.array([math.fsum(e[PAGE * j:min(n, PAGE * j + PAGE)]) for j in range(npages)])
        if not np.allclose(w, mass / mass.sum(), rtol=1e-12, atol=0):
            return False
    return True


def _cluster_variant(q16, cen, pt, b, kvh, n, *, size="log", scale=None):
    pb = O.num_pages(n)
    c = cen[np.asarray(pt[b, :pb], np.int64), kvh].astype(F64)
    sizes = np.array([O.valid_rows(n, j) for j in range(pb)], F64)
    logits = c @ np.asarray(q16, F16).astype(F64) / (math.sqrt(D) if scale is None else scale)
    if size == "log":
        logits = logits + np.log(sizes)
    elif size == "linear":
        logits = logits + sizes
    return O.softmax64(logits)


def test_cluster_weight_mistakes_fail_the_exact_mass_pin():
    assert check_cluster_weights(O.cluster_weights)
    assert check_cluster_weights(_cluster_variant)
    assert not check_cluster_weights(lambda *a: _cluster_variant(*a, size=None))     # unweighted
    assert not check_cluster_weights(lambda *a: _cluster_variant(*a, size="linear"))
    assert not check_cluster_weights(lambda *a: _cluster_variant(*a, scale=D))

    def logical_pages(q16, cen, pt, b, kvh, n):
        return _cluster_variant(q16, cen, np.arange(pt.shape[1])[None], b, kvh, n)

    assert not check_cluster_weights(logical_pages)


# ------------------------------------------------------------------------------------- n-bit codes

def check_nbit(quant_fn):
    """Hand-worked rows.  2 bits, channels (0, 1.5, 0.25, 1.25) repeated: min 0, max 1.5,
    s = 0.5; x/s = (0, 3, 0.5, 2.5) rounds half to even to (0, 3, 0, 2), packed from the low
    bits: 0 | 3 << 2 | 0 << 4 | 2 << 6 = 0x8C.  8 bits: x_c = n_c / 64 with n_0 = 0 and
    n_1 = 255, so s = 1/64 exactly and byte c is n_c."""
    x = np.tile(np.array([0.0, 1.5, 0.25, 1.25]), D // 4).astype(F16)[None]
    pk, s, z = quant_fn(x, 2)
    if not (pk.shape == (1, 32) and np.all(pk == 0x8C) and float(s[0]) == 0.5
            and float(z[0]) == 0.0):
        return False
    nn = (37 * np.arange(D) + 11) % 256
    nn[0], nn[1] = 0, 255
    pk, s, z = quant_fn((nn / 64).astype(F16)[None], 8)
    return bool(np.array_equal(pk[0], nn.astype(np.uint8)) and float(s[0]) == 1 / 64)


def _nbit_variant(x16, bits, *, levels=None, half_away=False, high_first=False):
    lv = (1 << bits) - 1 if levels is None else levels
    x16 = np.asarray(x16, F16)
    mn, mx = O.f16_min_max(x16, axis=1)
    s16 = ((mx.astype(F32) - mn.astype(F32)) / F32(lv)).astype(F16)
    r = (x16.astype(F32) - mn.astype(F32)[:, None]) / s16.astype(F32)[:, None]
    r = np.floor(r + F32(0.5)) if half_away else np.rint(r)
    n = np.clip(r, 0, (1 << bits) - 1).astype(np.uint64)
    per = 8 // bits
    packed = np.zeros((n.shape[0], n.shape[1] // per), np.uint64)
    for i in range(per):
        shift = bits * (per - 1 - i) if high_first else bits * i
        packed |= n[:, i::per] << np.uint64(shift)
    return packed.astype(np.uint8), s16, mn


def test_nbit_mistakes_fail_the_hand_worked_rows():
    assert check_nbit(O.quantize_rows_bits)
    assert check_nbit(_nbit_variant)
    assert not check_nbit(lambda x, b: _nbit_variant(x, b, levels=1 << b))     # 2^bits levels
    assert not check_nbit(lambda x, b: _nbit_variant(x, b, half_away=True))    # ties away
    assert not check_nbit(lambda x, b: _nbit_variant(x, b, high_first=True))   # channel order


# ------------------------------------------------------------------------------------- append

def _append_cache(seed=1, lens=(15, 16, 33, 1), extra=21, hkv=2):
    rng = np.random.default_rng(seed)
    need = [-(-(n + extra) // PAGE) + 1 for n in lens]
    pt = np.full((len(lens), max(need) + 1), -1, np.int32)
    perm = rng.permutation(sum(need))
    off = 0
    for b, m in enumerate(need):
        pt[b, :m] = perm[off:off + m]
        off += m
    k = rng.standard_normal((sum(need), hkv, PAGE, D)).astype(F16)
    v = rng.standard_normal((sum(need), hkv, PAGE, D)).astype(F16)
    k[..., 1] = np.where(rng.random(k.shape[:-1]) < 0.5, F16(0.0), F16(-0.0))
    return k, v, pt, np.asarray(lens, np.int64)


def check_append(append_fn):
    """21 appends to four sequences (page crossings, a one-token sequence), with stale bounds
    (9.0) on every page no sequence has reached yet: the incremental state must equal
    page_bounds and quantize_k recomputed over the extended cache, and the new rows must sit at
    the addresses the page table gives."""
    k, v, pt, n = _append_cache()
    bounds = np.full((k.shape[0], k.shape[1], 2, D), F16(9.0))
    ref0 = O.page_bounds(k, pt, n)
    for b in range(len(n)):
        ph = pt[b, :O.num_pages(int(n[b]))]
        bounds[ph] = ref0[ph]
    q4, sz = O.quantize_k(k, pt, n)
    rng = np.random.default_rng(2)
    lens0 = n.copy()
    news = []
    for _ in range(21):
        kn = rng.standard_normal((len(n), k.shape[1], D)).astype(F16)
        vn = rng.standard_normal((len(n), k.shape[1], D)).astype(F16)
        kn[..., 1] = np.where(rng.random(kn.shape[:-1]) < 0.5, F16(-0.0), F16(0.0))
        news.append((kn, vn))
        k, v, bounds, q4, sz, n = append_fn(k, v, bounds, q4, sz, pt, n, kn, vn)
    if n.tolist() != [int(x) + 21 for x in lens0]:
        return False
    for i, (kn, vn) in enumerate(news):
        for b in range(len(n)):
            t = int(lens0[b]) + i
            ph, row = pt[b, t // PAGE], t % PAGE
            if not (np.array_equal(u16(k[ph, :, row]), u16(kn[b]))
                    and np.array_equal(u16(v[ph, :, row]), u16(vn[b]))):
                return False
    live = sorted({int(p) for b in range(len(n)) for p in pt[b, :O.num_pages(int(n[b]))]})
    rb = O.page_bounds(k, pt, n)
    rq, rs = O.quantize_k(k, pt, n)
    return bool(np.array_equal(u16(bounds[live]), u16(rb[live]))
                and np.array_equal(q4[live], rq[live])
                and np.array_equal(u16(sz[live]), u16(rs[live])))


def test_append_mistakes_fail_the_recomputation_pin():
    assert check_append(O.append_token)

    def no_reset(k, v, bounds, q4, sz, pt, lens, kn, vn):   # a fresh page keeps stale bounds
        out = list(O.append_token(k, v, bounds, q4, sz, pt, lens, kn, vn))
        for b in range(len(lens)):
            t = int(lens[b])
            if t % PAGE == 0 and t // PAGE < pt.shape[1] and pt[b, t // PAGE] >= 0:
                ph = pt[b, t // PAGE]
                mn, _ = O.f16_min_max(np.stack([bounds[ph, :, 0], kn[b]]), axis=0)
                _, mx = O.f16_min_max(np.stack([bounds[ph, :, 1], kn[b]]), axis=0)
                out[2][ph, :, 0], out[2][ph, :, 1] = mn, mx
        return tuple(out)

    def logical_page(k, v, bounds, q4, sz, pt, lens, kn, vn):   # writes page j, not pt[b][j]
        ident = np.where(pt >= 0, np.arange(pt.size).reshape(pt.shape) % k.shape[0], -1)
        return O.append_token(k, v, bounds, q4, sz, ident.astype(np.int32), lens, kn, vn)

    def plain_min_max(k, v, bounds, q4, sz, pt, lens, kn, vn):  # numpy min/max: -0 == +0
        out = list(O.append_token(k, v, bounds, q4, sz, pt, lens, kn, vn))
        for b in range(len(lens)):
            t = int(lens[b])
            if t % PAGE and t // PAGE < pt.shape[1] and pt[b, t // PAGE] >= 0:
                ph = pt[b, t // PAGE]
                out[2][ph, :, 0] = np.minimum(kn[b], bounds[ph, :, 0])
                out[2][ph, :, 1] = np.maximum(kn[b], bounds[ph, :, 1])
        return tuple(out)

    def length_not_advanced(k, v, bounds, q4, sz, pt, lens, kn, vn):
        out = O.append_token(k, v, bounds, q4, sz, pt, lens, kn, vn)
        return out[:5] + (np.asarray(lens, np.int64).copy(),)

    for fn in (no_reset, logical_page, plain_min_max, length_not_advanced):
        assert not check_append(fn), fn.__name__
