"""The append path: one decode step's cache maintenance fused with the KV append.

CPU: the oracle's incremental restatement (``append_token``) is pinned to the full definitions
(``page_bounds`` and ``quantize_k`` recomputed over the extended cache), which the golden rows
pin in turn; and the C entry point rejects bad arguments before launching anything.
GPU: ``twl_append_token`` against the oracle, bit for bit, over many appended tokens, page
crossings, a full sequence and an unmapped page; then a decode step on the extended cache.
"""
import ctypes as C

import numpy as np
import pytest

from oracle import twl_oracle as O

D, PAGE = 128, 16


def u16(x):
    return np.ascontiguousarray(x).view(np.uint16)


def make_cache(lens, extra_tokens, hkv=2, seed=0, spare_pages=1):
    """Random fp16 K/V with every sequence mapped far enough for ``extra_tokens`` more tokens
    (plus ``spare_pages`` mapped pages beyond), pages dealt from one random permutation.  A few
    channels hold signed zeros and exact ties, the cases the total-order min/max must order."""
    rng = np.random.default_rng(seed)
    need = [-(-(n + extra_tokens) // PAGE) + spare_pages for n in lens]
    max_pages = max(need) + 1
    p_phys = sum(need)
    perm = rng.permutation(p_phys)
    pt = np.full((len(lens), max_pages), -1, np.int32)
    off = 0
    for b, m in enumerate(need):
        pt[b, :m] = perm[off:off + m]
        off += m
    k = rng.standard_normal((p_phys, hkv, PAGE, D)).astype(np.float16)
    v = rng.standard_normal((p_phys, hkv, PAGE, D)).astype(np.float16)
    k[..., 0] = np.float16(-0.0)
    k[..., 1] = np.where(rng.random(k.shape[:-1]) < 0.5, np.float16(0.0), np.float16(-0.0))
    k[..., 2] = np.float16(0.5)
    return k, v, pt, np.asarray(lens, np.int64)


def new_token(rng, batch, hkv):
    kn = rng.standard_normal((batch, hkv, D)).astype(np.float16)
    vn = rng.standard_normal((batch, hkv, D)).astype(np.float16)
    kn[..., 0] = np.float16(0.0)                    # +0 against the cache's -0
    kn[..., 1] = np.where(rng.random((batch, hkv)) < 0.5, np.float16(-0.0), np.float16(0.0))
    kn[..., 3] = np.float16(2.0)                    # a constant channel (ties every row)
    return kn, vn


def referenced(pt, lens):
    out = []
    for b, n in enumerate(lens):
        out.extend(pt[b, :O.num_pages(int(n))].tolist())
    return np.array(sorted(set(out)), np.int64)


def test_oracle_append_equals_recomputation():
    lens = [15, 16, 33, 1]          # row 15 then a new page; a new page; row 1; row 1
    T = 21
    k, v, pt, n = make_cache(lens, T, seed=1)
    bounds = O.page_bounds(k, pt, n)
    q4, sz = O.quantize_k(k, pt, n)
    rng = np.random.default_rng(2)
    for _ in range(T):
        kn, vn = new_token(rng, len(lens), k.shape[1])
        k, v, bounds, q4, sz, n = O.append_token(k, v, bounds, q4, sz, pt, n, kn, vn)
    assert n.tolist() == [x + T for x in lens]
    ref = referenced(pt, n)
    rb = O.page_bounds(k, pt, n)
    rq, rs = O.quantize_k(k, pt, n)
    assert np.array_equal(u16(bounds[ref]), u16(rb[ref]))
    assert np.array_equal(q4[ref], rq[ref])
    assert np.array_equal(u16(sz[ref]), u16(rs[ref]))


def test_oracle_append_writes_the_rows_and_resets_a_fresh_page():
    k, v, pt, n = make_cache([32], 1, hkv=1, seed=3)
    bounds = np.full((k.shape[0], 1, 2, D), np.float16(9.0))   # stale bounds everywhere
    q4 = np.zeros((k.shape[0], 1, PAGE, D // 2), np.uint8)
    sz = np.zeros((k.shape[0], 1, PAGE, 2), np.float16)
    kn, vn = new_token(np.random.default_rng(4), 1, 1)
    k2, v2, b2, q42, sz2, n2 = O.append_token(k, v, bounds, q4, sz, pt, n, kn, vn)
    ph = pt[0, 2]                   # token 32 opens page 2, row 0
    assert n2[0] == 33
    assert np.array_equal(u16(k2[ph, 0, 0]), u16(kn[0, 0]))
    assert np.array_equal(u16(v2[ph, 0, 0]), u16(vn[0, 0]))
    assert np.array_equal(u16(b2[ph, 0, 0]), u16(kn[0, 0]))
    assert np.array_equal(u16(b2[ph, 0, 1]), u16(kn[0, 0]))
    pk, s16, z16 = O.quantize_row(kn[0, 0])
    assert np.array_equal(q42[ph, 0, 0], pk) and u16(sz2[ph, 0, 0, 0]) == u16(s16)


def test_oracle_append_skips_full_and_unmapped_sequences():
    k, v, pt, n = make_cache([16, 20], 0, hkv=1, seed=5, spare_pages=0)
    n = np.array([16 * pt.shape[1], 20])      # sequence 0: table full
    pt[1, 1] = -1                             # sequence 1: position 20 has no page
    bounds = O.page_bounds(k, pt[:, :1], np.array([16, 16]))
    q4, sz = O.quantize_k(k, pt[:, :1], np.array([16, 16]))
    kn, vn = new_token(np.random.default_rng(6), 2, 1)
    out = O.append_token(k, v, bounds, q4, sz, pt, n, kn, vn)
    for before, after in zip((k, v, bounds, q4, sz), out[:5]):
        assert np.array_equal(np.asarray(before).view(np.uint8), np.asarray(after).view(np.uint8))
    assert out[5].tolist() == n.tolist()


# ------------------------------------------------------------------ boundary (no GPU needed)

def test_append_rejects_bad_arguments():
    from adaptive_top_sparse_b200 import twl
    A = 1 << 20
    kv = twl._PagedKV(A, A + 4096, A + 8192, A + 12288, 2, 8, 128, 16, 64, 128)
    aux = twl._KAux(A, A, A)
    f = twl._lib.twl_append_token
    assert f(C.byref(kv), C.byref(aux), A, 0, 1, None, 0, None) == twl.TWL_ERR_INVALID_ARG
    assert f(C.byref(kv), C.byref(aux), A + 8, A, 1, None, 0, None) == twl.TWL_ERR_INVALID_ARG
    assert f(C.byref(kv), C.byref(twl._KAux(A, 0, A)), A, A, 1, None, 0,
             None) == twl.TWL_ERR_INVALID_ARG
    assert f(C.byref(kv), None, A, A, 1, None, 0, None) == twl.TWL_ERR_INVALID_ARG
    bad_v = twl._PagedKV(A, 0, A + 8192, A + 12288, 2, 8, 128, 16, 64, 128)
    assert f(C.byref(bad_v), C.byref(aux), A, A, 1, None, 0, None) == twl.TWL_ERR_INVALID_ARG
    bad_d = twl._PagedKV(A, A, A + 8192, A + 12288, 2, 8, 64, 16, 64, 128)
    assert f(C.byref(bad_d), C.byref(aux), A, A, 1, None, 0, None) == twl.TWL_ERR_UNSUPPORTED
    assert f(C.byref(kv), C.byref(aux), A, A, 1, A, 16, None) == twl.TWL_ERR_WORKSPACE


# ------------------------------------------------------------------ GPU parity

def _device_cache(k, v, pt, n, hkv):
    import torch
    from adaptive_top_sparse_b200 import twl
    dev = torch.device("cuda")
    t = lambda x, dt: torch.as_tensor(np.ascontiguousarray(x)).to(device=dev, dtype=dt)
    kk, vv = t(k, torch.float16), t(v, torch.float16)
    ptt, nn = t(pt, torch.int32), t(n, torch.int32)
    kv = twl.PagedKV(kk, vv, ptt, nn, hkv, k.shape[0])
    p_phys = k.shape[0]
    aux = twl.KAux(torch.zeros((p_phys, hkv, 16, 64), dtype=torch.uint8, device=dev),
                   torch.zeros((p_phys, hkv, 16, 2), dtype=torch.float16, device=dev),
                   torch.zeros((p_phys, hkv, 2, 128), dtype=torch.float16, device=dev))
    ws = twl.alloc_workspace(twl.TWL_OP_CACHE, dev)
    twl.twl_quantize_k(kv, aux.k_int4, aux.k_scale_zero, ws)
    twl.twl_page_bounds(kv, aux.bounds, ws)
    return kv, aux, ws, (kk, vv, ptt, nn)


@pytest.mark.gpu
@pytest.mark.parametrize("hkv", [1, 8, 12])
def test_append_matches_oracle(hkv):
    import torch
    from adaptive_top_sparse_b200 import twl
    lens = [15, 16, 33, 1, 47]
    T = 37
    k, v, pt, n = make_cache(lens, T, hkv=hkv, seed=7 + hkv)
    kv, aux, ws, (kk, vv, ptt, nn) = _device_cache(k, v, pt, n, hkv)
    bounds, q4, sz = O.page_bounds(k, pt, n), *O.quantize_k(k, pt, n)
    rng = np.random.default_rng(8)
    for _ in range(T):
        kn, vn = new_token(rng, len(lens), hkv)
        twl.twl_append_token(kv, aux, torch.from_numpy(kn).cuda(), torch.from_numpy(vn).cuda(),
                             True, ws)
        k, v, bounds, q4, sz, n = O.append_token(k, v, bounds, q4, sz, pt, n, kn, vn)
    torch.cuda.synchronize()
    assert twl.twl_device_status(ws)[0] == twl.TWL_OK
    assert nn.cpu().numpy().tolist() == n.tolist()
    ref = referenced(pt, n)
    g = lambda x: x.cpu().numpy()
    assert np.array_equal(u16(g(kk)[ref]), u16(k[ref]))
    assert np.array_equal(u16(g(vv)[ref]), u16(v[ref]))
    assert np.array_equal(u16(g(aux.bounds)[ref]), u16(bounds[ref]))
    assert np.array_equal(g(aux.k_int4)[ref], q4[ref])
    assert np.array_equal(u16(g(aux.k_scale_zero)[ref]), u16(sz[ref]))
    # and the full definitions over the extended cache
    rb = O.page_bounds(k, pt, n)
    rq, rs = O.quantize_k(k, pt, n)
    assert np.array_equal(u16(g(aux.bounds)[ref]), u16(rb[ref]))
    assert np.array_equal(g(aux.k_int4)[ref], rq[ref])
    assert np.array_equal(u16(g(aux.k_scale_zero)[ref]), u16(rs[ref]))


@pytest.mark.gpu
def test_append_flags_full_and_unmapped_sequences():
    import torch
    from adaptive_top_sparse_b200 import twl
    k, v, pt, n = make_cache([16, 20, 5], 0, hkv=2, seed=9, spare_pages=0)
    n = np.array([16 * pt.shape[1], 20, 5])   # 0: table full; 1: position 20 unmapped; 2: fine
    pt[1, 1] = -1
    kv, aux, ws, (kk, vv, ptt, nn) = _device_cache(k, v, pt, np.array([16, 16, 5]), 2)
    nn.copy_(torch.from_numpy(n.astype(np.int32)))
    before = [x.clone() for x in (kk, vv, aux.bounds, aux.k_int4, aux.k_scale_zero)]
    kn, vn = new_token(np.random.default_rng(10), 3, 2)
    twl.twl_append_token(kv, aux, torch.from_numpy(kn).cuda(), torch.from_numpy(vn).cuda(),
                         True, ws)
    st = twl.twl_device_status(ws, clear=True)[0]
    assert st == twl.TWL_ERR_BAD_INDEX
    assert nn.cpu().numpy().tolist() == [16 * pt.shape[1], 20, 6]
    # only sequence 2's page changed
    ph2 = int(pt[2, 0])
    for a, b in zip(before, (kk, vv, aux.bounds, aux.k_int4, aux.k_scale_zero)):
        a, b = a.cpu().numpy(), b.cpu().numpy()
        keep = np.ones(a.shape[0], bool)
        keep[ph2] = False
        assert np.array_equal(a[keep].view(np.uint8), b[keep].view(np.uint8))


@pytest.mark.gpu
def test_decode_step_after_appends_matches_oracle():
    import torch
    from adaptive_top_sparse_b200.layer import DecodeLayer
    from workloads import synth
    from tests.twl_checks import check_step_group
    wl = synth.make_decode("append_gqa", 2, 8, 2, [1000, 333], seed=11, max_pages=90)
    # map spare pages so the sequences can grow by T tokens
    T = 24
    p_phys = wl.k.shape[0]
    extra = 0
    for b in range(wl.batch):
        have = O.num_pages(int(wl.seq_lens[b]))
        want = O.num_pages(int(wl.seq_lens[b]) + T)
        for j in range(have, want):
            wl.page_table[b, j] = p_phys + extra
            extra += 1
    rng = np.random.default_rng(12)
    wl.k = np.concatenate([wl.k, rng.standard_normal((extra,) + wl.k.shape[1:]).astype(np.float16)])
    wl.v = np.concatenate([wl.v, rng.standard_normal((extra,) + wl.v.shape[1:]).astype(np.float16)])
    layer = DecodeLayer.from_workload(wl)
    layer.build_aux()
    for _ in range(T):
        kn, vn = new_token(rng, wl.batch, wl.num_kv_heads)
        layer.append(torch.from_numpy(kn).cuda(), torch.from_numpy(vn).cuda())
        for b in range(wl.batch):
            nb = int(wl.seq_lens[b])
            ph = int(wl.page_table[b, nb // 16])
            wl.k[ph, :, nb % 16] = kn[b]
            wl.v[ph, :, nb % 16] = vn[b]
        wl.seq_lens = wl.seq_lens + 1
    torch.cuda.synchronize()
    assert layer.seq_lens.cpu().numpy().tolist() == wl.seq_lens.tolist()
    stats = layer.alloc_stats()
    q = torch.from_numpy(wl.q).cuda()
    o, lse = layer.decode(q, wl.p, wl.eps, stats)
    st = {k_: v_.cpu().numpy() for k_, v_ in stats.items()}
    for b in range(wl.batch):
        for kvh in range(wl.num_kv_heads):
            check_step_group(wl, b, kvh, st, o.cpu().numpy(), lse.cpu().numpy())


def test_oracle_append_equals_recomputation_generated():
    """Generated caches (1 to 3 sequences of 1 to 40 tokens, 1 or 3 kv-heads, 1 to 20 appends):
    the incremental state equals page_bounds and quantize_k over the extended cache."""
    from hypothesis import HealthCheck, given, settings
    from hypothesis import strategies as st

    @settings(max_examples=40, deadline=None, suppress_health_check=[HealthCheck.too_slow])
    @given(st.lists(st.integers(1, 40), min_size=1, max_size=3), st.sampled_from([1, 3]),
           st.integers(1, 20), st.integers(0, 1000))
    def run(lens, hkv, appends, seed):
        k, v, pt, n = make_cache(lens, appends, hkv=hkv, seed=seed)
        bounds = O.page_bounds(k, pt, n)
        q4, sz = O.quantize_k(k, pt, n)
        rng = np.random.default_rng(seed + 1)
        for _ in range(appends):
            kn, vn = new_token(rng, len(lens), hkv)
            k, v, bounds, q4, sz, n = O.append_token(k, v, bounds, q4, sz, pt, n, kn, vn)
        assert n.tolist() == [x + appends for x in lens]
        ref = referenced(pt, n)
        assert np.array_equal(u16(bounds[ref]), u16(O.page_bounds(k, pt, n)[ref]))
        rq, rs = O.quantize_k(k, pt, n)
        assert np.array_equal(q4[ref], rq[ref]) and np.array_equal(u16(sz[ref]), u16(rs[ref]))

    run()
