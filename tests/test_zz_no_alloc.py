"""twl_sparse_decode_noalloc: the attention call for callers that cannot allocate device memory
(plug-ins inside a framework that owns all device memory, real-time code that may not call
cudaMalloc, fixed memory plans).  Its scratch is a fixed-size array inside libtwl.so instead of a
caller workspace.  It must give the results of twl_sparse_decode on consecutive calls (the shared
scratch keeps the previous call's contents) and must refuse requests larger than its scratch.

This file is named to be collected last, so that a run stopping at its first failure has already
run every other test.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from adaptive_top_sparse_b200 import twl
from workloads import synth

from twl_checks import LSE_ATOL, O_ATOL

A = 1 << 20  # a fake aligned address: the size check below fails before anything is touched


def test_noalloc_rejects_requests_beyond_its_scratch():
    kv = twl._PagedKV(A, A, A, A, 64, 8, 128, 16, 32768, 1 << 16)
    need = twl.twl_workspace_bytes(twl.TWL_OP_SPARSE_DECODE, 64, 32, 8, 0, 0, 0, 16 * 32768)
    assert need > twl.twl_noalloc_scratch_bytes()
    st = twl._lib.twl_sparse_decode_noalloc(A, 32, C.byref(kv), A, A, 16 * 32768, 0.088, A, A,
                                            None)
    assert st == twl.TWL_ERR_SCRATCH_LIMIT
    assert twl.twl_status_string(st) != "unknown status"
    assert twl._lib.twl_sparse_decode_noalloc(A, 32, None, A, A, 64, 0.088, A, A, None) == \
        twl.TWL_ERR_INVALID_ARG


def _token_sets(wl, seed):
    rng = np.random.default_rng(seed)
    sets = {}
    for b in range(wl.batch):
        n = int(wl.seq_lens[b])
        for kvh in range(wl.num_kv_heads):
            size = int(rng.integers(1, min(n, 700) + 1))
            sets[(b, kvh)] = np.sort(rng.choice(n, size=size, replace=False))
    return sets


@pytest.mark.gpu
def test_noalloc_matches_workspace_call_on_consecutive_calls():
    from adaptive_top_sparse_b200.layer import SM_SCALE
    wl = synth.make_decode("noalloc", 2, 16, 4, [3000, 1234], seed=21)
    dev = torch.device("cuda")
    k = torch.from_numpy(wl.k).to(dev)
    v = torch.from_numpy(wl.v).to(dev)
    kv = twl.PagedKV(k, v, torch.from_numpy(wl.page_table).to(dev),
                     torch.from_numpy(wl.seq_lens).to(dev), wl.num_kv_heads, wl.k.shape[0])
    q = torch.from_numpy(wl.q).to(dev)
    stride = 16 * wl.max_pages
    ws = twl.alloc_workspace(twl.TWL_OP_SPARSE_DECODE, dev, batch=wl.batch,
                             num_q_heads=wl.num_q_heads, num_kv_heads=wl.num_kv_heads,
                             row_stride=stride)
    for call, seed in enumerate((1, 2)):       # two calls in a row, different token sets
        sets = _token_sets(wl, seed)
        tok = np.full((wl.batch, wl.num_kv_heads, stride), -1, dtype=np.int32)
        cnt = np.zeros((wl.batch, wl.num_kv_heads), dtype=np.int32)
        for (b, kvh), t in sets.items():
            tok[b, kvh, : t.size] = t
            cnt[b, kvh] = t.size
        tok_d, cnt_d = torch.from_numpy(tok).to(dev), torch.from_numpy(cnt).to(dev)
        shape = (wl.batch, wl.num_q_heads)
        o_ref = torch.zeros(shape + (128,), device=dev)
        lse_ref = torch.zeros(shape, device=dev)
        o_na = torch.full(shape + (128,), float("nan"), device=dev)
        lse_na = torch.full(shape, float("nan"), device=dev)
        twl.twl_sparse_decode(q, wl.num_q_heads, kv, tok_d, cnt_d, stride, SM_SCALE, o_ref,
                              lse_ref, ws)
        twl.twl_sparse_decode_noalloc(q, wl.num_q_heads, kv, tok_d, cnt_d, stride, SM_SCALE,
                                      o_na, lse_na)
        torch.cuda.synchronize()
        o_ref, lse_ref, o_na, lse_na = (t.cpu().numpy() for t in (o_ref, lse_ref, o_na, lse_na))
        assert np.all(np.isfinite(o_na)) and np.all(np.isfinite(lse_na)), f"call {call}"
        assert np.abs(o_na - o_ref).max() <= O_ATOL, f"call {call}: o"
        assert np.abs(lse_na - lse_ref).max() <= LSE_ATOL, f"call {call}: lse"
