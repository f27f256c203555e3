"""Python binding of libtwl.so (ctypes).  Argument marshalling only: every step runs in the
library's CUDA kernels.  Device tensors come from PyTorch (memory and streams only).

Each function has the name of the C entry point it wraps (see include/twl.h for the meaning,
layout, ownership and error behaviour of every argument) and raises TwlError when the library
returns a status other than TWL_OK.  Importing this module fails loudly when libtwl.so has not
been built: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtwl.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m adaptive_top_sparse_b200.build`")
_lib = C.CDLL(LIB_PATH)

TWL_OK = 0
TWL_ERR_INVALID_ARG = -1
TWL_ERR_UNSUPPORTED = -2
TWL_ERR_CUDA = -3
TWL_ERR_TIMEOUT = -4
TWL_ERR_WORKSPACE = -5
TWL_ERR_BAD_INDEX = -6
TWL_ERR_SCRATCH_LIMIT = -7
TWL_FLAG_BAD_INDEX = 1
TWL_FLAG_TIMEOUT = 2

TWL_OP_CACHE = 1
TWL_OP_SELECT = 2
TWL_OP_ESTIMATE = 3
TWL_OP_PRUNE = 4
TWL_OP_UNION = 5
TWL_OP_SPARSE_DECODE = 6
TWL_OP_DECODE_STEP = 7
TWL_OP_SELECT_CLUSTERS = 8

EXPORTED = [
    "twl_workspace_bytes", "twl_workspace_init", "twl_device_status", "twl_status_string",
    "twl_page_bounds", "twl_quantize_k", "twl_append_token", "twl_quantize_k_nbit",
    "twl_estimate_nbit", "twl_page_centroids", "twl_select_clusters_top_p", "twl_select_pages", "twl_estimate", "twl_prune_top_p",
    "twl_group_union", "twl_sparse_decode", "twl_decode_step", "twl_noalloc_scratch_bytes",
    "twl_sparse_decode_noalloc", "twl_test_set_waits",
]


class TwlError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {twl_status_string(status)} ({status})")


class _PagedKV(C.Structure):
    _fields_ = [("k", C.c_void_p), ("v", C.c_void_p), ("page_table", C.c_void_p),
                ("seq_lens", C.c_void_p), ("batch", C.c_int32), ("num_kv_heads", C.c_int32),
                ("head_dim", C.c_int32), ("page_size", C.c_int32), ("max_pages", C.c_int32),
                ("num_phys_pages", C.c_int32)]


class _KAux(C.Structure):
    _fields_ = [("k_int4", C.c_void_p), ("k_scale_zero", C.c_void_p), ("bounds", C.c_void_p)]


class _StepStats(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("sel_pages", "sel_count", "weights", "cand_tok",
                                          "cand_count", "threshold", "kept_count", "union_tok",
                                          "union_count")]


_vp, _i32, _f32, _sz = C.c_void_p, C.c_int32, C.c_float, C.c_size_t
_sigs = {
    "twl_workspace_bytes": (_sz, [_i32] * 8),
    "twl_workspace_init": (_i32, [_vp, _sz, _vp]),
    "twl_device_status": (_i32, [_vp, C.POINTER(C.c_uint32), _i32, _vp]),
    "twl_status_string": (C.c_char_p, [_i32]),
    "twl_page_bounds": (_i32, [C.POINTER(_PagedKV), _vp, _vp, _sz, _vp]),
    "twl_quantize_k": (_i32, [C.POINTER(_PagedKV), _vp, _vp, _vp, _sz, _vp]),
    "twl_append_token": (_i32, [C.POINTER(_PagedKV), C.POINTER(_KAux), _vp, _vp, _i32, _vp,
                                _sz, _vp]),
    "twl_select_pages": (_i32, [_vp, _i32, C.POINTER(_PagedKV), _vp, _i32, _i32, _i32, _vp, _vp,
                                _vp, _vp, _sz, _vp]),
    "twl_estimate": (_i32, [_vp, _i32, C.POINTER(_PagedKV), _vp, _vp, _vp, _vp, _i32, _vp, _vp,
                            _vp, _vp, _sz, _vp]),
    "twl_page_centroids": (_i32, [C.POINTER(_PagedKV), _vp, _vp, _sz, _vp]),
    "twl_select_clusters_top_p": (_i32, [_vp, _i32, C.POINTER(_PagedKV), _vp, _f32, _f32, _vp,
                                         _vp, _vp, _vp, _sz, _vp]),
    "twl_quantize_k_nbit": (_i32, [C.POINTER(_PagedKV), _i32, _vp, _vp, _vp, _sz, _vp]),
    "twl_estimate_nbit": (_i32, [_vp, _i32, C.POINTER(_PagedKV), _i32, _vp, _vp, _vp, _vp, _i32,
                                 _vp, _vp, _vp, _vp, _sz, _vp]),
    "twl_prune_top_p": (_i32, [_vp, _vp, _i32, _i32, _f32, _f32, _vp, _vp, _vp, _vp, _sz, _vp]),
    "twl_group_union": (_i32, [_i32, C.POINTER(_PagedKV), _vp, _vp, _vp, _i32, _vp, _vp, _vp,
                               _sz, _vp]),
    "twl_sparse_decode": (_i32, [_vp, _i32, C.POINTER(_PagedKV), _vp, _vp, _i32, _f32, _vp, _vp,
                                 _vp, _sz, _vp]),
    "twl_noalloc_scratch_bytes": (_sz, []),
    "twl_test_set_waits": (None, [C.c_uint32, _i32]),
    "twl_sparse_decode_noalloc": (_i32, [_vp, _i32, C.POINTER(_PagedKV), _vp, _vp, _i32, _f32,
                                         _vp, _vp, _vp]),
    "twl_decode_step": (_i32, [_vp, _i32, C.POINTER(_PagedKV), C.POINTER(_KAux), _i32, _i32,
                               _i32, _f32, _f32, _vp, _vp, C.POINTER(_StepStats), _vp, _sz,
                               _vp]),
}
for _name, (_res, _args) in _sigs.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        if torch.cuda.is_available():
            return torch.cuda.current_stream().cuda_stream
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(st: int, where: str) -> None:
    if st != TWL_OK:
        raise TwlError(st, where)


def _nbytes(t) -> int:
    return 0 if t is None else t.numel() * t.element_size()


@dataclass
class PagedKV:
    """Tensors of a paged KV cache (see include/twl.h for the layout)."""
    k: torch.Tensor | None
    v: torch.Tensor | None
    page_table: torch.Tensor
    seq_lens: torch.Tensor
    num_kv_heads: int
    num_phys_pages: int
    head_dim: int = 128
    page_size: int = 16

    @property
    def batch(self) -> int:
        return int(self.page_table.shape[0])

    @property
    def max_pages(self) -> int:
        return int(self.page_table.shape[1])

    def c(self) -> _PagedKV:
        return _PagedKV(_ptr(self.k), _ptr(self.v), _ptr(self.page_table), _ptr(self.seq_lens),
                        self.batch, self.num_kv_heads, self.head_dim, self.page_size,
                        self.max_pages, self.num_phys_pages)


def twl_status_string(status: int) -> str:
    return _lib.twl_status_string(int(status)).decode()


def twl_workspace_bytes(op: int, batch: int = 0, num_q_heads: int = 0, num_kv_heads: int = 0,
                        max_pages: int = 0, max_budget: int = 0, rows: int = 0,
                        row_stride: int = 0) -> int:
    return int(_lib.twl_workspace_bytes(op, batch, num_q_heads, num_kv_heads, max_pages,
                                        max_budget, rows, row_stride))


def twl_workspace_init(ws, stream=None) -> None:
    _check(_lib.twl_workspace_init(_ptr(ws), _nbytes(ws), _stream(stream)), "twl_workspace_init")


def twl_device_status(ws, clear: bool = False, stream=None) -> tuple[int, int]:
    """Returns (status, flags) of the workspace's sticky device flags (waits on the stream)."""
    fl = C.c_uint32(0)
    st = _lib.twl_device_status(_ptr(ws), C.byref(fl), int(clear), _stream(stream))
    return int(st), int(fl.value)


def alloc_workspace(op: int, device, **dims) -> torch.Tensor:
    """A zero-initialised workspace tensor of twl_workspace_bytes(op, **dims) bytes."""
    n = twl_workspace_bytes(op, **dims)
    if n == 0:
        raise TwlError(TWL_ERR_INVALID_ARG, "twl_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def twl_page_bounds(kv: PagedKV, bounds, ws=None, stream=None) -> None:
    ckv = kv.c()
    _check(_lib.twl_page_bounds(C.byref(ckv), _ptr(bounds), _ptr(ws), _nbytes(ws),
                                _stream(stream)), "twl_page_bounds")


def twl_quantize_k(kv: PagedKV, k_int4, k_scale_zero, ws=None, stream=None) -> None:
    ckv = kv.c()
    _check(_lib.twl_quantize_k(C.byref(ckv), _ptr(k_int4), _ptr(k_scale_zero), _ptr(ws),
                               _nbytes(ws), _stream(stream)), "twl_quantize_k")


def twl_append_token(kv: PagedKV, aux: "KAux", k_new, v_new, advance: bool = True, ws=None,
                     stream=None) -> None:
    ckv, caux = kv.c(), aux.c()
    _check(_lib.twl_append_token(C.byref(ckv), C.byref(caux), _ptr(k_new), _ptr(v_new),
                                 1 if advance else 0, _ptr(ws), _nbytes(ws), _stream(stream)),
           "twl_append_token")


def twl_select_pages(q, num_q_heads: int, kv: PagedKV, bounds, budget_pages: int,
                     budget_div: int, max_budget: int, sel_pages, sel_count, scores=None,
                     ws=None, stream=None) -> None:
    ckv = kv.c()
    _check(_lib.twl_select_pages(_ptr(q), num_q_heads, C.byref(ckv), _ptr(bounds), budget_pages,
                                 budget_div, max_budget, _ptr(sel_pages), _ptr(sel_count),
                                 _ptr(scores), _ptr(ws), _nbytes(ws), _stream(stream)),
           "twl_select_pages")


def twl_estimate(q, num_q_heads: int, kv: PagedKV, k_int4, k_scale_zero, sel_pages, sel_count,
                 max_budget: int, weights, cand_tok, cand_count, ws=None, stream=None) -> None:
    ckv = kv.c()
    _check(_lib.twl_estimate(_ptr(q), num_q_heads, C.byref(ckv), _ptr(k_int4),
                             _ptr(k_scale_zero), _ptr(sel_pages), _ptr(sel_count), max_budget,
                             _ptr(weights), _ptr(cand_tok), _ptr(cand_count), _ptr(ws),
                             _nbytes(ws), _stream(stream)), "twl_estimate")


def twl_page_centroids(kv: PagedKV, centroids, ws=None, stream=None) -> None:
    ckv = kv.c()
    _check(_lib.twl_page_centroids(C.byref(ckv), _ptr(centroids), _ptr(ws), _nbytes(ws),
                                   _stream(stream)), "twl_page_centroids")


def twl_select_clusters_top_p(q, num_q_heads: int, kv: PagedKV, centroids, p_cluster: float,
                              eps: float, sel_pages, sel_count, cluster_weights=None, ws=None,
                              stream=None) -> None:
    ckv = kv.c()
    _check(_lib.twl_select_clusters_top_p(_ptr(q), num_q_heads, C.byref(ckv), _ptr(centroids),
                                          p_cluster, eps, _ptr(sel_pages), _ptr(sel_count),
                                          _ptr(cluster_weights), _ptr(ws), _nbytes(ws),
                                          _stream(stream)), "twl_select_clusters_top_p")


def twl_quantize_k_nbit(kv: PagedKV, bits: int, k_codes, k_scale_zero, ws=None,
                        stream=None) -> None:
    ckv = kv.c()
    _check(_lib.twl_quantize_k_nbit(C.byref(ckv), bits, _ptr(k_codes), _ptr(k_scale_zero),
                                    _ptr(ws), _nbytes(ws), _stream(stream)),
           "twl_quantize_k_nbit")


def twl_estimate_nbit(q, num_q_heads: int, kv: PagedKV, bits: int, k_codes, k_scale_zero,
                      sel_pages, sel_count, max_budget: int, weights, cand_tok, cand_count,
                      ws=None, stream=None) -> None:
    ckv = kv.c()
    _check(_lib.twl_estimate_nbit(_ptr(q), num_q_heads, C.byref(ckv), bits, _ptr(k_codes),
                                  _ptr(k_scale_zero), _ptr(sel_pages), _ptr(sel_count),
                                  max_budget, _ptr(weights), _ptr(cand_tok), _ptr(cand_count),
                                  _ptr(ws), _nbytes(ws), _stream(stream)), "twl_estimate_nbit")


def twl_prune_top_p(w, row_len, rows: int, row_stride: int, p: float, eps: float, m_out,
                    kept_count, kept_idx=None, ws=None, stream=None) -> None:
    _check(_lib.twl_prune_top_p(_ptr(w), _ptr(row_len), rows, row_stride, p, eps, _ptr(m_out),
                                _ptr(kept_count), _ptr(kept_idx), _ptr(ws), _nbytes(ws),
                                _stream(stream)), "twl_prune_top_p")


def twl_group_union(num_q_heads: int, kv: PagedKV, cand_tok, kept_idx, kept_count,
                    cand_stride: int, union_tok, union_count, ws=None, stream=None) -> None:
    ckv = kv.c()
    _check(_lib.twl_group_union(num_q_heads, C.byref(ckv), _ptr(cand_tok), _ptr(kept_idx),
                                _ptr(kept_count), cand_stride, _ptr(union_tok),
                                _ptr(union_count), _ptr(ws), _nbytes(ws), _stream(stream)),
           "twl_group_union")


def twl_sparse_decode(q, num_q_heads: int, kv: PagedKV, tok, tok_count, tok_stride: int,
                      sm_scale: float, o, lse, ws=None, stream=None) -> None:
    ckv = kv.c()
    _check(_lib.twl_sparse_decode(_ptr(q), num_q_heads, C.byref(ckv), _ptr(tok), _ptr(tok_count),
                                  tok_stride, sm_scale, _ptr(o), _ptr(lse), _ptr(ws),
                                  _nbytes(ws), _stream(stream)), "twl_sparse_decode")


@dataclass
class KAux:
    k_int4: torch.Tensor
    k_scale_zero: torch.Tensor
    bounds: torch.Tensor

    def c(self) -> _KAux:
        return _KAux(_ptr(self.k_int4), _ptr(self.k_scale_zero), _ptr(self.bounds))


def make_stats(**tensors) -> _StepStats:
    s = _StepStats()
    for name, t in tensors.items():
        setattr(s, name, _ptr(t))
    return s


def twl_decode_step(q, num_q_heads: int, kv: PagedKV, aux: KAux, budget_pages: int,
                    budget_div: int, max_budget: int, p: float, eps: float, o, lse, stats=None,
                    ws=None, stream=None) -> None:
    ckv = kv.c()
    caux = aux.c()
    cst = C.byref(stats) if stats is not None else None
    _check(_lib.twl_decode_step(_ptr(q), num_q_heads, C.byref(ckv), C.byref(caux), budget_pages,
                                budget_div, max_budget, p, eps, _ptr(o), _ptr(lse), cst,
                                _ptr(ws), _nbytes(ws), _stream(stream)), "twl_decode_step")


def twl_noalloc_scratch_bytes() -> int:
    return int(_lib.twl_noalloc_scratch_bytes())


def twl_test_set_waits(max_polls: int = 0, stall_estimate: bool = False) -> None:
    """Test hook of the decode step's bounded waits (see include/twl.h)."""
    _lib.twl_test_set_waits(int(max_polls), 1 if stall_estimate else 0)


def twl_sparse_decode_noalloc(q, num_q_heads: int, kv: PagedKV, tok, tok_count, tok_stride: int,
                              sm_scale: float, o, lse, stream=None) -> None:
    """twl_sparse_decode without a workspace, for callers that cannot allocate device memory;
    the scratch is a fixed-size array inside the library (see include/twl.h)."""
    ckv = kv.c()
    _check(_lib.twl_sparse_decode_noalloc(_ptr(q), num_q_heads, C.byref(ckv), _ptr(tok),
                                          _ptr(tok_count), tok_stride, sm_scale, _ptr(o),
                                          _ptr(lse), _stream(stream)),
           "twl_sparse_decode_noalloc")
