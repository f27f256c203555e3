"""Device-side state of one decode-attention layer and the calls a user makes on it.

``DecodeLayer`` owns device tensors (PyTorch is only the allocator here): the paged fp16 K/V, the
page table, the derived INT4 K and page bounds, a workspace, and the outputs.  Every computation
is a call into libtwl.so.
"""
from __future__ import annotations

import math

import torch

from . import twl


def budget_bound(max_pages: int, budget_pages: int, budget_div: int) -> int:
    """Largest page budget any sequence can get (the sel_pages row stride)."""
    if budget_pages > 0:
        return min(budget_pages, max_pages)
    return -(-max_pages // budget_div)


def expect_tensor(name: str, t, shape, dtype, device) -> None:
    """Raises unless `t` is a contiguous tensor of `shape` and `dtype` on `device`.  The library
    takes raw pointers: it cannot tell a host buffer, a tensor on another GPU or a mis-shaped one
    from a good one, and a kernel would read or write the wrong memory."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if t.device != device:
        raise ValueError(f"{name}: tensor on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: tensor is not contiguous")


class DecodeLayer:
    """One layer's paged KV cache on a GPU and its decode step.

    k, v: fp16 [num_phys_pages][num_kv_heads][16][128]; page_table: int32 [B][max_pages] (logical
    page -> physical page, -1 unmapped); seq_lens: int32 [B].  Arrays on the host are copied to
    `device`.  budget_pages > 0 fixes the pages each head selects, else ceil(P_b / budget_div).
    Every call on a layer uses the layer's one workspace: issue them in order on one stream (the
    current stream when `stream` is None)."""

    def __init__(self, k, v, page_table, seq_lens, num_q_heads: int, num_kv_heads: int,
                 budget_pages: int = 0, budget_div: int = 4, device="cuda"):
        dev = torch.device(device)
        t = lambda x, dt: torch.as_tensor(x).to(device=dev, dtype=dt).contiguous()
        self.k = t(k, torch.float16)
        self.v = t(v, torch.float16)
        self.page_table = t(page_table, torch.int32)
        self.seq_lens = t(seq_lens, torch.int32)
        self.num_q_heads = num_q_heads
        self.num_kv_heads = num_kv_heads
        self.budget_pages = budget_pages
        self.budget_div = budget_div
        self.device = dev
        p_phys = self.k.shape[0]
        self.kv = twl.PagedKV(self.k, self.v, self.page_table, self.seq_lens, num_kv_heads,
                              p_phys)
        self.batch = self.kv.batch
        self.max_pages = self.kv.max_pages
        self.max_budget = budget_bound(self.max_pages, budget_pages, budget_div)
        self.aux = twl.KAux(
            torch.zeros((p_phys, num_kv_heads, 16, 64), dtype=torch.uint8, device=dev),
            torch.zeros((p_phys, num_kv_heads, 16, 2), dtype=torch.float16, device=dev),
            torch.zeros((p_phys, num_kv_heads, 2, 128), dtype=torch.float16, device=dev))
        self.ws = twl.alloc_workspace(twl.TWL_OP_DECODE_STEP, dev, batch=self.batch,
                                      num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
                                      max_pages=self.max_pages, max_budget=self.max_budget)
        self.o = torch.zeros((self.batch, num_q_heads, 128), dtype=torch.float32, device=dev)
        self.lse = torch.zeros((self.batch, num_q_heads), dtype=torch.float32, device=dev)

    @classmethod
    def from_workload(cls, wl, device="cuda"):
        return cls(wl.k, wl.v, wl.page_table, wl.seq_lens, wl.num_q_heads, wl.num_kv_heads,
                   wl.budget_pages, wl.budget_div, device)

    # ------------------------------------------------------------------ cache maintenance
    def build_aux(self, stream=None) -> None:
        """INT4 K and page bounds for every referenced page."""
        twl.twl_quantize_k(self.kv, self.aux.k_int4, self.aux.k_scale_zero, self.ws, stream)
        twl.twl_page_bounds(self.kv, self.aux.bounds, self.ws, stream)

    def append(self, k_new, v_new, stream=None) -> None:
        """Append one token per sequence at position seq_lens[b] (K, V, INT4 K and page bounds
        in one launch) and advance seq_lens.  The page for the position must be mapped."""
        for name, t in (("k_new", k_new), ("v_new", v_new)):
            expect_tensor(name, t, (self.batch, self.num_kv_heads, 128), torch.float16,
                          self.k.device)
        twl.twl_append_token(self.kv, self.aux, k_new, v_new, True, self.ws, stream)

    # ------------------------------------------------------------------ stats buffers
    def alloc_stats(self) -> dict:
        b, hq, hkv, mb = self.batch, self.num_q_heads, self.num_kv_heads, self.max_budget
        dev, i32, f32 = self.device, torch.int32, torch.float32
        cs, us = 16 * mb, 16 * self.max_pages
        return dict(
            sel_pages=torch.full((b, hq, mb), -1, dtype=i32, device=dev),
            sel_count=torch.zeros((b, hq), dtype=i32, device=dev),
            weights=torch.zeros((b, hq, cs), dtype=f32, device=dev),
            cand_tok=torch.full((b, hq, cs), -1, dtype=i32, device=dev),
            cand_count=torch.zeros((b, hq), dtype=i32, device=dev),
            threshold=torch.zeros((b, hq), dtype=f32, device=dev),
            kept_count=torch.zeros((b, hq), dtype=i32, device=dev),
            union_tok=torch.full((b, hkv, us), -1, dtype=i32, device=dev),
            union_count=torch.zeros((b, hkv), dtype=i32, device=dev))

    # ------------------------------------------------------------------ the decode step
    def decode(self, q, p: float = 0.85, eps: float = 1e-6, stats: dict | None = None,
               stream=None):
        """One select -> estimate -> prune -> union -> attend step for query q [B][Hq][128] fp16
        (device tensor), one launch of the library's persistent step kernel.  Returns the
        layer's (o, lse) device tensors (o and lse are attributes a caller may point at slices
        of its own buffers)."""
        self.expect_query(q)
        st = twl.make_stats(**stats) if stats is not None else None
        twl.twl_decode_step(q, self.num_q_heads, self.kv, self.aux, self.budget_pages,
                            self.budget_div, self.max_budget, p, eps, self.o, self.lse, st,
                            self.ws, stream)
        return self.o, self.lse

    def expect_query(self, q) -> None:
        """q must be fp16 [B][Hq][128], contiguous, on the layer's GPU."""
        expect_tensor("q", q, (self.batch, self.num_q_heads, 128), torch.float16, self.k.device)

    # ------------------------------------------------------------------ other paths
    def staged(self) -> "Staged":
        """The same step as five separate library calls (see Staged)."""
        return Staged(self)

    def double_p(self) -> "DoubleP":
        """The two-level top-p path on this layer's cache (built on first use)."""
        if getattr(self, "_double_p", None) is None:
            self._double_p = DoubleP(self)
        return self._double_p

    def status(self, clear: bool = False):
        return twl.twl_device_status(self.ws, clear)


SM_SCALE = 1.0 / math.sqrt(128.0)


class DoubleP:
    """The two-level top-p step: top-p over page clusters scored by size-weighted centroids
    (twl_select_clusters_top_p), then the token-level path on the kept pages: INT4 estimate,
    top-p prune, group union, sparse attention.  Five library calls; this class only owns the
    buffers between them."""

    def __init__(self, layer: DecodeLayer):
        self.layer = layer
        L, dev = layer, layer.device
        b, hq, hkv, mp = L.batch, L.num_q_heads, L.num_kv_heads, L.max_pages
        i32, f32 = torch.int32, torch.float32
        self.centroids = torch.zeros((L.k.shape[0], hkv, 128), dtype=torch.float16, device=dev)
        self.sel = torch.full((b, hq, mp), -1, dtype=i32, device=dev)
        self.sel_count = torch.zeros((b, hq), dtype=i32, device=dev)
        self.cluster_w = torch.zeros((b, hq, mp), dtype=f32, device=dev)
        cs = 16 * mp
        self.weights = torch.zeros((b, hq, cs), dtype=f32, device=dev)
        self.cand_tok = torch.full((b, hq, cs), -1, dtype=i32, device=dev)
        self.cand_count = torch.zeros((b, hq), dtype=i32, device=dev)
        self.m = torch.zeros(b * hq, dtype=f32, device=dev)
        self.kept_count = torch.zeros(b * hq, dtype=i32, device=dev)
        self.kept_idx = torch.zeros((b * hq, cs), dtype=i32, device=dev)
        self.union_tok = torch.full((b, hkv, cs), -1, dtype=i32, device=dev)
        self.union_count = torch.zeros((b, hkv), dtype=i32, device=dev)
        dims = dict(batch=b, num_q_heads=hq, num_kv_heads=hkv, max_pages=mp, max_budget=mp)
        self.ws_sel = twl.alloc_workspace(twl.TWL_OP_SELECT_CLUSTERS, dev, **dims)
        self.ws_est = twl.alloc_workspace(twl.TWL_OP_ESTIMATE, dev, **dims)
        self.ws_att = twl.alloc_workspace(twl.TWL_OP_SPARSE_DECODE, dev, batch=b, num_q_heads=hq,
                                          num_kv_heads=hkv, row_stride=cs)
        self.ws_cache = twl.alloc_workspace(twl.TWL_OP_CACHE, dev)

    def build_centroids(self, stream=None) -> None:
        twl.twl_page_centroids(self.layer.kv, self.centroids, self.ws_cache, stream)

    def decode(self, q, p_cluster: float = 0.95, p: float = 0.85, eps: float = 1e-6,
               stream=None):
        L = self.layer
        L.expect_query(q)
        hq, mp = L.num_q_heads, L.max_pages
        cs = 16 * mp
        twl.twl_select_clusters_top_p(q, hq, L.kv, self.centroids, p_cluster, eps, self.sel,
                                      self.sel_count, self.cluster_w, self.ws_sel, stream)
        twl.twl_estimate(q, hq, L.kv, L.aux.k_int4, L.aux.k_scale_zero, self.sel,
                         self.sel_count, mp, self.weights, self.cand_tok, self.cand_count,
                         self.ws_est, stream)
        rows = L.batch * hq
        twl.twl_prune_top_p(self.weights.view(rows, cs), self.cand_count.view(rows), rows, cs,
                            p, eps, self.m, self.kept_count, self.kept_idx, None, stream)
        twl.twl_group_union(hq, L.kv, self.cand_tok, self.kept_idx, self.kept_count, cs,
                            self.union_tok, self.union_count, None, stream)
        twl.twl_sparse_decode(q, hq, L.kv, self.union_tok, self.union_count, cs, SM_SCALE, L.o,
                              L.lse, self.ws_att, stream)
        return L.o, L.lse


class Staged:
    """The decode step as its five staged library calls (twl_select_pages, twl_estimate,
    twl_prune_top_p, twl_group_union, twl_sparse_decode) instead of the one fused launch: the
    comparison the flattened per-stage work lists give.  Only owns the buffers between calls."""

    def __init__(self, layer: DecodeLayer):
        self.layer = layer
        L, dev = layer, layer.device
        b, hq, hkv, mb = L.batch, L.num_q_heads, L.num_kv_heads, L.max_budget
        i32, f32 = torch.int32, torch.float32
        cs = 16 * mb
        self.sel = torch.full((b, hq, mb), -1, dtype=i32, device=dev)
        self.sel_count = torch.zeros((b, hq), dtype=i32, device=dev)
        self.weights = torch.zeros((b, hq, cs), dtype=f32, device=dev)
        self.cand_tok = torch.full((b, hq, cs), -1, dtype=i32, device=dev)
        self.cand_count = torch.zeros((b, hq), dtype=i32, device=dev)
        self.m = torch.zeros(b * hq, dtype=f32, device=dev)
        self.kept_count = torch.zeros(b * hq, dtype=i32, device=dev)
        self.kept_idx = torch.zeros((b * hq, cs), dtype=i32, device=dev)
        us = 16 * L.max_pages  # union rows: up to every token of the sequence
        self.union_tok = torch.full((b, hkv, us), -1, dtype=i32, device=dev)
        self.union_count = torch.zeros((b, hkv), dtype=i32, device=dev)
        dims = dict(batch=b, num_q_heads=hq, num_kv_heads=hkv, max_pages=L.max_pages,
                    max_budget=mb)
        self.ws_sel = twl.alloc_workspace(twl.TWL_OP_SELECT, dev, **dims)
        self.ws_est = twl.alloc_workspace(twl.TWL_OP_ESTIMATE, dev, **dims)
        self.ws_att = twl.alloc_workspace(twl.TWL_OP_SPARSE_DECODE, dev, batch=b, num_q_heads=hq,
                                          num_kv_heads=hkv, row_stride=us)

    def decode(self, q, p: float = 0.85, eps: float = 1e-6, stream=None):
        L = self.layer
        L.expect_query(q)
        hq, mb = L.num_q_heads, L.max_budget
        cs = 16 * mb
        twl.twl_select_pages(q, hq, L.kv, L.aux.bounds, L.budget_pages, L.budget_div, mb,
                             self.sel, self.sel_count, None, self.ws_sel, stream)
        twl.twl_estimate(q, hq, L.kv, L.aux.k_int4, L.aux.k_scale_zero, self.sel,
                         self.sel_count, mb, self.weights, self.cand_tok, self.cand_count,
                         self.ws_est, stream)
        rows = L.batch * hq
        twl.twl_prune_top_p(self.weights.view(rows, cs), self.cand_count.view(rows), rows, cs,
                            p, eps, self.m, self.kept_count, self.kept_idx, None, stream)
        twl.twl_group_union(hq, L.kv, self.cand_tok, self.kept_idx, self.kept_count, cs,
                            self.union_tok, self.union_count, None, stream)
        twl.twl_sparse_decode(q, hq, L.kv, self.union_tok, self.union_count, 16 * L.max_pages,
                              SM_SCALE, L.o, L.lse, self.ws_att, stream)
        return L.o, L.lse
