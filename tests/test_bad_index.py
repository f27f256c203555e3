"""Device-side index checks on the decode path (GPU).

Page-table entries inside a sequence's range that point outside the physical pool (-1, the pool
size, 2^30) and sequence lengths outside [1, 16 * max_pages] are caller errors only the device
can see.  Every call on the path must skip the bad page or sequence (no read through the entry),
raise TWL_FLAG_BAD_INDEX in the workspace header and leave the other sequences' results exact.
The corruption is planted on the host side of the test (the page table and lengths are caller
inputs); nothing here faults the GPU: the library range-checks every entry before using it.
"""
import numpy as np
import pytest
import torch

from oracle import twl_oracle as O
from workloads import synth

from twl_checks import check_attention, check_step_group

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from adaptive_top_sparse_b200 import twl
    from adaptive_top_sparse_b200.layer import DecodeLayer, SM_SCALE

BAD_PAGES = (3, 17, 30)          # logical pages of sequence 0 that get bad entries


def _corrupted_layer():
    wl = synth.make_decode("badidx", 2, 8, 2, [700, 300], seed=31, permute_pages=True)
    layer = DecodeLayer.from_workload(wl)
    layer.build_aux()
    assert layer.status(clear=True)[0] == twl.TWL_OK
    bad_vals = (-1, wl.num_phys_pages, 1 << 30)
    for j, v in zip(BAD_PAGES, bad_vals):
        layer.page_table[0, j] = v
    torch.cuda.synchronize()
    return wl, layer


def test_decode_step_skips_bad_page_table_entries():
    wl, layer = _corrupted_layer()
    stats = layer.alloc_stats()
    q = torch.from_numpy(wl.q).cuda()
    o, lse = layer.decode(q, wl.p, wl.eps, stats)
    st = {k: v.cpu().numpy() for k, v in stats.items()}
    o, lse = o.cpu().numpy(), lse.cpu().numpy()
    status, flags = layer.status(clear=True)
    assert status == twl.TWL_ERR_BAD_INDEX and flags & twl.TWL_FLAG_BAD_INDEX
    # sequence 0: the bad pages score -inf, so none of them is selected, attended or kept
    assert np.all(np.isfinite(o[0])) and np.all(np.isfinite(lse[0]))
    for h in range(wl.num_q_heads):
        sel = st["sel_pages"][0, h, : st["sel_count"][0, h]]
        assert not set(BAD_PAGES) & set(sel.tolist()), h
    for kvh in range(wl.num_kv_heads):
        toks = st["union_tok"][0, kvh, : st["union_count"][0, kvh]]
        assert not set(BAD_PAGES) & set((toks // 16).tolist())
    # sequence 1 is untouched: exact against the oracle
    for kvh in range(wl.num_kv_heads):
        check_step_group(wl, 1, kvh, st, o, lse)


def test_select_and_estimate_skip_bad_page_table_entries():
    wl, layer = _corrupted_layer()
    dev = layer.device
    b, hq, mp = wl.batch, wl.num_q_heads, wl.max_pages
    q = torch.from_numpy(wl.q).to(dev)
    # every page selected (budget = all pages), so the estimate meets the bad entries too
    sel = torch.full((b, hq, mp), -1, dtype=torch.int32, device=dev)
    cnt = torch.zeros((b, hq), dtype=torch.int32, device=dev)
    scores = torch.zeros((b, hq, mp), dtype=torch.float32, device=dev)
    ws = twl.alloc_workspace(twl.TWL_OP_SELECT, dev, batch=b, num_q_heads=hq,
                             num_kv_heads=wl.num_kv_heads, max_pages=mp)
    twl.twl_select_pages(q, hq, layer.kv, layer.aux.bounds, mp, 4, mp, sel, cnt, scores, ws)
    assert twl.twl_device_status(ws)[0] == twl.TWL_ERR_BAD_INDEX
    sc = scores.cpu().numpy()
    for j in BAD_PAGES:
        assert np.all(np.isneginf(sc[0, :, j]))
    cs = 16 * mp
    w = torch.zeros((b, hq, cs), dtype=torch.float32, device=dev)
    cand = torch.full((b, hq, cs), -1, dtype=torch.int32, device=dev)
    cc = torch.zeros((b, hq), dtype=torch.int32, device=dev)
    ws2 = twl.alloc_workspace(twl.TWL_OP_ESTIMATE, dev, batch=b, num_q_heads=hq,
                              num_kv_heads=wl.num_kv_heads, max_pages=mp)
    twl.twl_estimate(q, hq, layer.kv, layer.aux.k_int4, layer.aux.k_scale_zero, sel, cnt, mp, w,
                     cand, cc, ws2)
    assert twl.twl_device_status(ws2)[0] == twl.TWL_ERR_BAD_INDEX
    w, cand, cc = w.cpu().numpy(), cand.cpu().numpy(), cc.cpu().numpy()
    for h in range(hq):
        tok = cand[0, h, : cc[0, h]]
        on_bad = np.isin(tok // 16, BAD_PAGES)
        assert on_bad.sum() == 16 * len(BAD_PAGES)
        assert np.all(w[0, h, : cc[0, h]][on_bad] == 0)         # skipped: weight exactly 0
        assert abs(float(w[0, h, : cc[0, h]].astype(np.float64).sum()) - 1.0) < 1e-4
    # sequence 1's weights are the oracle's
    q4, sz = O.quantize_k(wl.k, wl.page_table, wl.seq_lens)
    g = hq // wl.num_kv_heads
    sel_np, cnt_np = sel.cpu().numpy(), cnt.cpu().numpy()
    for h in range(hq):
        pages = sel_np[1, h, : cnt_np[1, h]]
        tok, w_or = O.estimate_head(wl.q[1, h], q4, sz, wl.page_table, 1, h // g,
                                    int(wl.seq_lens[1]), pages)
        assert np.allclose(w[1, h, : tok.size], w_or, rtol=1e-3, atol=1e-9)


def test_sparse_decode_skips_tokens_on_bad_pages():
    wl, layer = _corrupted_layer()
    dev = layer.device
    stride = 16 * wl.max_pages
    tok = np.full((wl.batch, wl.num_kv_heads, stride), -1, dtype=np.int32)
    cnt = np.zeros((wl.batch, wl.num_kv_heads), dtype=np.int32)
    good = {}
    for b in range(wl.batch):
        n = int(wl.seq_lens[b])
        for kvh in range(wl.num_kv_heads):
            t = np.arange(0, n, 3)
            tok[b, kvh, : t.size] = t
            cnt[b, kvh] = t.size
            good[(b, kvh)] = t[~np.isin(t // 16, BAD_PAGES)] if b == 0 else t
    q = torch.from_numpy(wl.q).to(dev)
    o = torch.zeros((wl.batch, wl.num_q_heads, 128), device=dev)
    lse = torch.zeros((wl.batch, wl.num_q_heads), device=dev)
    ws = twl.alloc_workspace(twl.TWL_OP_SPARSE_DECODE, dev, batch=wl.batch,
                             num_q_heads=wl.num_q_heads, num_kv_heads=wl.num_kv_heads,
                             row_stride=stride)
    twl.twl_sparse_decode(q, wl.num_q_heads, layer.kv, torch.from_numpy(tok).to(dev),
                          torch.from_numpy(cnt).to(dev), stride, SM_SCALE, o, lse, ws)
    assert twl.twl_device_status(ws)[0] == twl.TWL_ERR_BAD_INDEX
    ref = O.group_attention(wl, good)
    o, lse = o.cpu().numpy(), lse.cpu().numpy()
    for (b, h), (o_or, lse_or) in ref.items():
        check_attention(o[b, h], lse[b, h], o_or, lse_or, f"b{b} h{h}")


@pytest.mark.parametrize("bad_len", [0, -5, 16 * 45 + 1])
def test_decode_step_skips_bad_sequence_lengths(bad_len):
    wl = synth.make_decode("badlen", 2, 8, 2, [700, 300], seed=32)
    layer = DecodeLayer.from_workload(wl)
    layer.build_aux()
    assert layer.status(clear=True)[0] == twl.TWL_OK
    layer.seq_lens[0] = bad_len                  # max_pages is 44: 16 * 45 + 1 is too long
    stats = layer.alloc_stats()
    q = torch.from_numpy(wl.q).cuda()
    o, lse = layer.decode(q, wl.p, wl.eps, stats)
    st = {k: v.cpu().numpy() for k, v in stats.items()}
    o, lse = o.cpu().numpy(), lse.cpu().numpy()
    assert layer.status(clear=True)[0] == twl.TWL_ERR_BAD_INDEX
    assert np.all(o[0] == 0) and np.all(np.isneginf(lse[0]))
    assert np.all(st["sel_count"][0] == 0) and np.all(st["kept_count"][0] == 0)
    for kvh in range(wl.num_kv_heads):
        check_step_group(wl, 1, kvh, st, o, lse)
