"""Cluster-level top-p selection (the Double-P selector): page centroids,
size-weighted cluster weights, top-p over pages, then the token-level path on the kept pages.

CPU pins: the centroid is the plain mean where fp32 sums are exact; a page whose rows are
identical has a cluster weight equal to its exact share of the attention mass (the size
weighting is exact there); p = 1 keeps every page; each q-head keeps its own group's dominant
page behind a permuted page table; the entry points reject bad arguments.
GPU: centroids bit-exact, cluster weights and kept pages against the oracle's criteria, and the
whole two-level step against the oracle over the device's sets.
"""
import ctypes as C
import math

import numpy as np
import pytest

from oracle import twl_oracle as O
from tests.twl_checks import check_attention, check_prune_row, check_weights
from workloads import synth

D = 128


def u16(x):
    return np.ascontiguousarray(x).view(np.uint16)


def test_centroid_is_the_mean_when_sums_are_exact():
    rng = np.random.default_rng(0)
    k = (rng.integers(-64, 64, (3, 2, 16, D)) / 8).astype(np.float16)   # multiples of 1/8
    pt = np.array([[0, 1, 2]], np.int32)
    n = np.array([16 + 16 + 5])
    cen = O.page_centroids(k, pt, n)
    for j, rows in ((0, 16), (1, 16), (2, 5)):
        exact = k[j, :, :rows].astype(np.float64).mean(axis=1)           # exact in fp64
        assert np.array_equal(u16(cen[j]), u16(exact.astype(np.float16))), j


def test_single_row_and_constant_pages():
    k = np.zeros((2, 1, 16, D), np.float16)
    k[0, 0, 0] = np.linspace(-3, 3, D).astype(np.float16)
    k[1, 0, :] = np.float16(0.7)
    cen = O.page_centroids(k, np.array([[0], [1]], np.int32), np.array([1, 16]))
    assert np.array_equal(u16(cen[0, 0]), u16(k[0, 0, 0]))
    assert np.all(cen[1, 0] == np.float16(0.7))


def test_cluster_weight_equals_exact_mass_for_uniform_pages():
    """With identical rows inside each page, sum_i exp(q.k_i/sqrt(D)) over the page is exactly
    n_j exp(q.c_j/sqrt(D)): the cluster weights are the pages' exact attention-mass shares."""
    rng = np.random.default_rng(1)
    npages, n = 7, 7 * 16 - 9
    k = np.zeros((npages, 1, 16, D), np.float16)
    for j in range(npages):
        k[j, 0, :] = (rng.standard_normal(D) * 0.5).astype(np.float16)
    pt = np.arange(npages, dtype=np.int32)[None]
    q = (rng.standard_normal(D)).astype(np.float16)
    cen = O.page_centroids(k, pt, np.array([n]))
    w = O.cluster_weights(q, cen, pt, 0, 0, n)
    logits = np.array([k[j, 0, 0].astype(np.float64) @ q.astype(np.float64) / math.sqrt(D)
                       for j in range(npages)])
    sizes = np.array([O.valid_rows(n, j) for j in range(npages)], np.float64)
    mass = sizes * np.exp(logits - logits.max())
    assert np.allclose(w, mass / mass.sum(), rtol=1e-12, atol=0)
    # the planted-mistake check: dropping the size weighting changes the answer
    assert not np.allclose(w, np.exp(logits - logits.max()) / np.exp(logits - logits.max()).sum(),
                           rtol=1e-6, atol=0)


def test_select_clusters_p_one_keeps_every_page():
    wl = synth.make_decode("dp_all", 1, 4, 1, [300], seed=5)
    cen = O.page_centroids(wl.k, wl.page_table, wl.seq_lens)
    sel = O.select_clusters(wl.q, cen, wl.page_table, wl.seq_lens, 4, 1, 1.0)
    for h in range(4):
        assert np.array_equal(sel[(0, h)][1], np.arange(O.num_pages(300)))


def test_select_clusters_follows_each_groups_dominant_page():
    """Four pages behind a permuted page table; kv-head 0 has one page aligned with the query
    (logical page 1), kv-head 1 another (logical page 2), every other row is zero.  That page's
    cluster weight is about 287 / 290, so p = 0.9 keeps it alone, and each q-head keeps the page
    of its own group (q-head h reads kv-head h // 2)."""
    pt = np.array([[2, 0, 3, 1]], np.int32)
    k = np.zeros((4, 2, 16, D), np.float16)
    k[pt[0, 1], 0, :, 0] = 8.0
    k[pt[0, 2], 1, :, 0] = 8.0
    q = np.zeros((1, 4, D), np.float16)
    q[0, :, 0] = 8.0
    lens = np.array([64])
    cen = O.page_centroids(k, pt, lens)

    def kept(select_fn):
        sel = select_fn(q, cen, pt, lens, 4, 2, 0.9)
        return [sel[(0, h)][1].tolist() for h in range(4)]

    assert kept(O.select_clusters) == [[1], [1], [2], [2]]

    def head_modulo(q, cen, pt, lens, hq, hkv, p_cluster):    # q-head h reads kv-head h % hkv
        out = {}
        for h in range(hq):
            w = O.cluster_weights(q[0, h], cen, pt, 0, h % hkv, int(lens[0]))
            out[(0, h)] = (w, np.sort(O.top_p_sort(w, p_cluster)[2]))
        return out

    assert kept(head_modulo) != [[1], [1], [2], [2]]


def test_cluster_calls_reject_bad_arguments():
    from adaptive_top_sparse_b200 import twl
    A = 1 << 20
    kv = twl._PagedKV(A, A + 4096, A + 8192, A + 12288, 2, 8, 128, 16, 64, 128)
    f = twl._lib.twl_select_clusters_top_p
    ok = dict(q=A, hq=32, cen=A, p=0.95, eps=1e-6, sel=A, cnt=A, w=None, ws=A, wsb=1 << 30)

    def call(**over):
        a = dict(ok, **over)
        return f(a["q"], a["hq"], C.byref(kv), a["cen"], a["p"], a["eps"], a["sel"], a["cnt"],
                 a["w"], a["ws"], a["wsb"], None)
    assert call(p=0.0) == twl.TWL_ERR_INVALID_ARG
    assert call(p=1.5) == twl.TWL_ERR_INVALID_ARG
    assert call(eps=0.0) == twl.TWL_ERR_INVALID_ARG
    assert call(cen=0) == twl.TWL_ERR_INVALID_ARG
    assert call(q=A + 8) == twl.TWL_ERR_INVALID_ARG
    assert call(hq=24) == twl.TWL_ERR_UNSUPPORTED
    assert call(wsb=64) == twl.TWL_ERR_WORKSPACE
    assert twl._lib.twl_page_centroids(C.byref(kv), A + 2, None, 0, None) == twl.TWL_ERR_INVALID_ARG
    assert twl.twl_workspace_bytes(twl.TWL_OP_SELECT_CLUSTERS, 2, 32, 8, 64) > 256


# ------------------------------------------------------------------ GPU

@pytest.fixture(scope="module")
def small():
    from adaptive_top_sparse_b200.layer import DecodeLayer
    wl = synth.make_decode("dp_small", 3, 16, 4, [2001, 777, 16], seed=23, permute_pages=True)
    layer = DecodeLayer.from_workload(wl)
    layer.build_aux()
    dp = layer.double_p()
    dp.build_centroids()
    return wl, layer, dp


@pytest.mark.gpu
def test_centroids_bit_exact(small):
    wl, layer, dp = small
    ref = O.page_centroids(wl.k, wl.page_table, wl.seq_lens)
    used = np.array(sorted({int(p) for b in range(wl.batch)
                            for p in wl.page_table[b, :O.num_pages(int(wl.seq_lens[b]))]}))
    assert np.array_equal(u16(dp.centroids.cpu().numpy()[used]), u16(ref[used]))


@pytest.mark.gpu
@pytest.mark.parametrize("p_cluster", [0.5, 0.9, 0.99, 1.0])
def test_cluster_selection_vs_oracle(small, p_cluster):
    import torch
    wl, layer, dp = small
    q = torch.from_numpy(wl.q).cuda()
    from adaptive_top_sparse_b200 import twl
    twl.twl_select_clusters_top_p(q, wl.num_q_heads, layer.kv, dp.centroids, p_cluster, wl.eps,
                                  dp.sel, dp.sel_count, dp.cluster_w, dp.ws_sel)
    cen = O.page_centroids(wl.k, wl.page_table, wl.seq_lens)
    seln, cntn, wn = dp.sel.cpu().numpy(), dp.sel_count.cpu().numpy(), dp.cluster_w.cpu().numpy()
    g = wl.num_q_heads // wl.num_kv_heads
    for b in range(wl.batch):
        n = int(wl.seq_lens[b])
        pb = O.num_pages(n)
        for h in range(wl.num_q_heads):
            w_or = O.cluster_weights(wl.q[b, h], cen, wl.page_table, b, h // g, n)
            w_dev = wn[b, h, :pb]
            check_weights(w_dev, w_or, f"b{b} h{h} clusters")
            kept = np.nonzero(w_dev >= np.float32(0))[0] if p_cluster >= 1 else None
            c = int(cntn[b, h])
            got = seln[b, h, :c]
            assert np.all(np.diff(got) > 0), "ascending"
            m = np.float32(w_dev[got].min()) if c else np.float32(np.inf)
            check_prune_row(w_dev, m, c, got, p_cluster, wl.eps, f"b{b} h{h} clusters")
            if kept is not None:
                assert np.array_equal(got, kept)


@pytest.mark.gpu
def test_two_level_step_vs_oracle(small):
    import torch
    wl, layer, dp = small
    q = torch.from_numpy(wl.q).cuda()
    o, lse = dp.decode(q, 0.95, wl.p, wl.eps)
    torch.cuda.synchronize()
    assert layer.status()[0] == 0
    q4, sz = O.quantize_k(wl.k, wl.page_table, wl.seq_lens)
    g = wl.num_q_heads // wl.num_kv_heads
    seln, cntn = dp.sel.cpu().numpy(), dp.sel_count.cpu().numpy()
    wn, tokn, ccn = (x.cpu().numpy() for x in (dp.weights, dp.cand_tok, dp.cand_count))
    kcn, kin = dp.kept_count.cpu().numpy(), dp.kept_idx.cpu().numpy()
    mn = dp.m.cpu().numpy()
    utok, ucnt = dp.union_tok.cpu().numpy(), dp.union_count.cpu().numpy()
    on, lsen = o.cpu().numpy(), lse.cpu().numpy()
    for b in range(wl.batch):
        n = int(wl.seq_lens[b])
        for kvh in range(wl.num_kv_heads):
            expect = set()
            for hl in range(g):
                h = kvh * g + hl
                r = b * wl.num_q_heads + h
                pages = seln[b, h, :cntn[b, h]]
                cand, w_or = O.estimate_head(wl.q[b, h], q4, sz, wl.page_table, b, kvh, n, pages)
                c = int(ccn[b, h])
                assert c == cand.size and np.array_equal(tokn[b, h, :c], cand)
                check_weights(wn[b, h, :c], w_or, f"b{b} h{h} tokens")
                kept, _, _ = check_prune_row(wn[b, h, :c], mn[r], int(kcn[r]), kin[r], wl.p, wl.eps,
                                             f"b{b} h{h} tokens")
                expect |= set(cand[kept].tolist())
            u = utok[b, kvh, :ucnt[b, kvh]]
            assert np.array_equal(u, np.array(sorted(expect))), (b, kvh)
            att = O.group_attention(wl, {(b, kvh): u})
            for (bb, h), (o_or, lse_or) in att.items():
                check_attention(on[bb, h], lsen[bb, h], o_or, lse_or, f"b{bb} h{h} attention")
