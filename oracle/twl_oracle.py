"""CPU oracle for hierarchical top-p sparse decode attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` may import this module.  The CUDA library never calls it, and it shares no code,
table or constant generator with the CUDA sources: it is a plain, slow restatement of what the
method computes, in numpy, fp64 wherever the method leaves the precision open.

Sources (cited by page title and section):
  [Notes]   "Twilight: Adaptive Attention Sparsity with Hierarchical Top-p Pruning", Paper-Notes
            (NeurIPS 2025) page: sections "Overall framework", "Key designs" (oracle top-p
            formulation, binary-search top-p, 4-bit K cache, load balancing), "Limitations".
  [Summary] "Twilight: Adaptive Attention Sparsity with Hierarchical Top-p Pruning", paperlayer
            summary of arXiv 2502.02770v5: sections 3.2, 4.1, 4.2, 4.3, B.1, B.2.

Readings where the pages are silent (each also listed in the design notes):
  * Page score (Quest selector; the pages only name it): score_j = sum_c t_c with
    t_c = q_c*mx_c if q_c > 0 else q_c*mn_c, the tight upper bound of q.k over the page's
    channel-wise bounding box.  Every t_c is exact in fp32 (fp16 x fp16), so the only rounding
    is the summation, done in one fixed order: 16 partial sums of 8 consecutive channels,
    each accumulated left to right from +0, then a pairwise tree (l, l+8), (l, l+4), (l, l+2),
    (l, l+1).
  * Budget: k_b = budget_pages if > 0, else ceil(P_b / budget_div); all pages if P_b <= k_b.
    Ties in score go to the lower logical page index; the selection is reported ascending.
  * INT4 K ([Summary] B.1: per-head dynamic asymmetric quantisation, fp16 scale and zero point,
    two values per byte): one group = the 128 channels of one token row of one head;
    s = fp16(fp32(mx - mn) / 15), z = mn, n_c = clamp(rint_even(fp32(x_c - z) / s), 0, 15)
    (n_c = 0 when s = 0); channel 2j in the low nibble of byte j.  Rows past the sequence end
    of a referenced page are written as zeros.  fp16 min/max use the total order in which
    -0 < +0.
  * Estimated weights: logit_i = q . khat_i / sqrt(D), khat = n*s + z, softmax over the head's
    own candidates (valid tokens of its selected pages) in fp64.
  * Top-p: the minimal set by sort + cumulative sum ([Notes] "Key designs", formal statement),
    and the pages' threshold bisection ([Notes] "Key designs", efficient top-p;
    [Summary] 4.2) with lo = 0, hi = max W, mid = lo + (hi - lo) / 2.  p = 1 keeps every
    candidate (m = 0) in both forms.
  * GQA: each group attends over the union of its heads' kept tokens ([Summary] B.2).
"""
from __future__ import annotations

import math

import numpy as np

F16 = np.float16
F32 = np.float32
F64 = np.float64
PAGE = 16


# ----------------------------------------------------------------------------------------------
# fp16 total order (used for bit-exact min / max)
# ----------------------------------------------------------------------------------------------

def f16_order_key(x16: np.ndarray) -> np.ndarray:
    """Integer key that orders fp16 values with -0 < +0 (finite inputs)."""
    b = np.ascontiguousarray(x16, dtype=F16).view(np.uint16).astype(np.int32)
    return np.where(b & 0x8000, -1 - (b & 0x7FFF), b)


def f16_min_max(x16: np.ndarray, axis: int):
    key = f16_order_key(x16)
    imn = np.expand_dims(key.argmin(axis=axis), axis)
    imx = np.expand_dims(key.argmax(axis=axis), axis)
    mn = np.take_along_axis(x16, imn, axis=axis).squeeze(axis)
    mx = np.take_along_axis(x16, imx, axis=axis).squeeze(axis)
    return mn, mx


def num_pages(n: int) -> int:
    return (int(n) + PAGE - 1) // PAGE


def valid_rows(n: int, j: int) -> int:
    """Tokens of logical page j that lie inside a sequence of n tokens."""
    return max(0, min(PAGE, int(n) - PAGE * j))


# ----------------------------------------------------------------------------------------------
# Cache maintenance: page bounds and INT4 K
# ----------------------------------------------------------------------------------------------

def page_bounds(k, page_table, seq_lens, out=None):
    """Channel-wise min and max of K over each referenced page's valid tokens.

    Returns fp16 [P_phys][Hkv][2][D] (row 0 = min, row 1 = max); pages that no sequence
    references keep the content of ``out`` (zeros by default).
    """
    p_phys, hkv, page, d = k.shape
    bounds = np.zeros((p_phys, hkv, 2, d), dtype=F16) if out is None else out.copy()
    for b in range(len(seq_lens)):
        n = int(seq_lens[b])
        pb = num_pages(n)
        phys = np.asarray(page_table[b, :pb], dtype=np.int64)
        full = phys[:-1]
        if full.size:
            mn, mx = f16_min_max(k[full], axis=2)                      # [pb-1][Hkv][D]
            bounds[full, :, 0, :] = mn
            bounds[full, :, 1, :] = mx
        last = int(phys[-1])
        mn, mx = f16_min_max(k[last, :, : valid_rows(n, pb - 1), :], axis=1)
        bounds[last, :, 0, :] = mn
        bounds[last, :, 1, :] = mx
    return bounds


def quantize_rows(x16: np.ndarray):
    """Token rows (fp16 [R][D]) -> (packed uint8 [R][D/2], scale fp16 [R], zero fp16 [R])."""
    x16 = np.asarray(x16, dtype=F16)
    mn, mx = f16_min_max(x16, axis=1)
    s16 = ((mx.astype(F32) - mn.astype(F32)) / F32(15.0)).astype(F16)
    z16 = mn
    s32 = s16.astype(F32)[:, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.rint((x16.astype(F32) - z16.astype(F32)[:, None]) / s32)
    r = np.where(s32 == F32(0.0), F32(0.0), r)
    n = np.clip(r, 0, 15).astype(np.uint8)
    packed = (n[:, 0::2] | (n[:, 1::2] << 4)).astype(np.uint8)
    return packed, s16, z16


def quantize_row(x16: np.ndarray):
    """One token row (fp16[D]) -> (packed uint8[D/2], scale fp16, zero fp16)."""
    pk, s, z = quantize_rows(np.asarray(x16, dtype=F16)[None, :])
    return pk[0], s[0], z[0]


def unpack_row(packed: np.ndarray) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8)
    n = np.empty(packed.size * 2, dtype=np.int64)
    n[0::2] = packed & 0x0F
    n[1::2] = packed >> 4
    return n


def dequantize_row(packed, s16, z16) -> np.ndarray:
    """khat = n * s + z, exact in fp64."""
    return unpack_row(packed).astype(F64) * F64(F16(s16)) + F64(F16(z16))


def quantize_k(k, page_table, seq_lens, out_int4=None, out_sz=None):
    """INT4 K for every referenced page: (uint8 [P][Hkv][16][D/2], fp16 [P][Hkv][16][2])."""
    p_phys, hkv, page, d = k.shape
    q4 = np.zeros((p_phys, hkv, page, d // 2), dtype=np.uint8) if out_int4 is None \
        else out_int4.copy()
    sz = np.zeros((p_phys, hkv, page, 2), dtype=F16) if out_sz is None else out_sz.copy()
    for b in range(len(seq_lens)):
        n = int(seq_lens[b])
        pb = num_pages(n)
        phys = np.asarray(page_table[b, :pb], dtype=np.int64)
        rows = k[phys].reshape(-1, d)                                   # [pb*Hkv*16][D]
        pk, s16, z16 = quantize_rows(rows)
        pk = pk.reshape(pb, hkv, page, d // 2)
        s16 = s16.reshape(pb, hkv, page)
        z16 = z16.reshape(pb, hkv, page)
        r_valid = n - PAGE * (pb - 1)                                   # rows of the last page
        pk[pb - 1, :, r_valid:] = 0
        s16[pb - 1, :, r_valid:] = F16(0.0)
        z16[pb - 1, :, r_valid:] = F16(0.0)
        q4[phys] = pk
        sz[phys, :, :, 0] = s16
        sz[phys, :, :, 1] = z16
    return q4, sz


def append_token(k, v, bounds, q4, sz, page_table, seq_lens, k_new, v_new):
    """One decode step of cache maintenance: sequence b's new token goes to logical position
    n_b = seq_lens[b], i.e. row n_b % 16 of physical page page_table[b][n_b // 16].

    Per kv-head: the K and V rows are written; the page's bounds become the new row itself when
    it is the page's first row, else the channel-wise (total-order) min and max of the old bounds
    and the row; the INT4 row and its scale / zero are ``quantize_rows`` of the row.  Then
    seq_lens[b] = n_b + 1.  A sequence whose position has no mapped page (the table is full or
    the entry is negative) is left unchanged.  The result equals ``page_bounds`` and
    ``quantize_k`` recomputed over the extended cache (min and max are associative, and the
    INT4 scheme is per row).  Returns new arrays (k, v, bounds, q4, sz, seq_lens).
    """
    k, v, bounds, q4, sz = (np.array(x, copy=True) for x in (k, v, bounds, q4, sz))
    seq_lens = np.array(seq_lens, dtype=np.int64, copy=True)
    max_pages = page_table.shape[1]
    for b in range(len(seq_lens)):
        n = int(seq_lens[b])
        j, row = n // PAGE, n % PAGE
        if j >= max_pages or int(page_table[b, j]) < 0:
            continue
        ph = int(page_table[b, j])
        x = np.asarray(k_new[b], dtype=F16)                               # [Hkv][D]
        k[ph, :, row, :] = x
        v[ph, :, row, :] = np.asarray(v_new[b], dtype=F16)
        if row == 0:
            bounds[ph, :, 0, :] = x
            bounds[ph, :, 1, :] = x
        else:
            mn, _ = f16_min_max(np.stack([bounds[ph, :, 0, :], x]), axis=0)
            _, mx = f16_min_max(np.stack([bounds[ph, :, 1, :], x]), axis=0)
            bounds[ph, :, 0, :] = mn
            bounds[ph, :, 1, :] = mx
        pk, s16, z16 = quantize_rows(x)
        q4[ph, :, row, :] = pk
        sz[ph, :, row, 0] = s16
        sz[ph, :, row, 1] = z16
        seq_lens[b] = n + 1
    return k, v, bounds, q4, sz, seq_lens


# ----------------------------------------------------------------------------------------------
# Quest-style page scoring and top-k selection
# ----------------------------------------------------------------------------------------------

def page_scores(q16: np.ndarray, mn16: np.ndarray, mx16: np.ndarray) -> np.ndarray:
    """Upper bound of q.k over each page's bounding box, fp32 in the fixed order above.

    q16: fp16 [D]; mn16, mx16: fp16 [P][D].  Returns fp32 [P].
    """
    q = np.asarray(q16, dtype=F16).astype(F32)
    mn = np.asarray(mn16, dtype=F16).astype(F32)
    mx = np.asarray(mx16, dtype=F16).astype(F32)
    t = np.where(q[None, :] > 0, q[None, :] * mx, q[None, :] * mn)      # exact products
    p, d = t.shape
    t = t.reshape(p, d // 8, 8)
    part = np.zeros((p, d // 8), dtype=F32)
    for i in range(8):
        part = part + t[:, :, i]
    while part.shape[1] > 1:
        half = part.shape[1] // 2
        part = part[:, :half] + part[:, half:]
    return part[:, 0]


def budget_for(n_pages: int, budget_pages: int, budget_div: int) -> int:
    """Pages the selector keeps: budget_pages if > 0, else ceil(P / budget_div), at most P
    ([Notes] "Overall framework": a conservative base budget such as 1/4; [Summary] 4.3)."""
    if budget_pages > 0:
        return min(int(budget_pages), int(n_pages))
    return min(int(n_pages), -(-int(n_pages) // int(budget_div)))


def select_top_k(scores: np.ndarray, k: int) -> np.ndarray:
    """k highest scores, ties to the lower index; returned ascending."""
    n = len(scores)
    if k >= n:
        return np.arange(n, dtype=np.int64)
    order = np.lexsort((np.arange(n), -scores.astype(F64)))
    return np.sort(order[:k]).astype(np.int64)


# ----------------------------------------------------------------------------------------------
# Weight estimation from INT4 K, top-p
# ----------------------------------------------------------------------------------------------

def softmax64(x: np.ndarray) -> np.ndarray:
    x = np.asarray(x, dtype=F64)
    e = np.exp(x - x.max())
    return e / e.sum()


def top_p_sort(w: np.ndarray, p: float):
    """Minimal top-p set by sort + cumulative sum ([Notes] "Key designs", oracle top-p).

    Returns (k_star, m_star, threshold_set) where k_star is the smallest count whose largest
    weights sum (fp64) to >= p (all n if none does), m_star the k_star-th largest weight and
    threshold_set = {i : w_i >= m_star} (ties at m_star included), ascending.
    """
    w = np.asarray(w)
    n = w.size
    order = np.argsort(-w.astype(F64), kind="stable")
    cs = np.cumsum(w[order].astype(F64))
    hit = np.nonzero(cs >= F64(p))[0]
    k_star = int(hit[0]) + 1 if hit.size else n
    m_star = w[order[k_star - 1]]
    kept = np.nonzero(w >= m_star)[0]
    return k_star, m_star, kept


def top_p_whole(w: np.ndarray, p: float):
    """``top_p_sort`` for a normalised distribution (softmax weights summing to 1), with p = 1
    read as the whole distribution ([Notes] "Key designs": the kept mass must reach p, which at
    p = 1 is all of it): every entry is kept and m* = 0.  The sort form cannot decide
    p = 1 by itself: the fp64 sum of the largest weights can round to exactly 1.0 while positive
    weights remain, and an exact sum of the rounded weights can land on either side of 1."""
    w = np.asarray(w)
    if p >= 1.0:
        return w.size, w.dtype.type(0.0), np.arange(w.size, dtype=np.int64)
    return top_p_sort(w, p)


def top_p_bisect(w: np.ndarray, p: float, eps: float, max_iter: int = 64):
    """Threshold bisection of [Notes] "Key designs" (efficient top-p) / [Summary] 4.2.

    Searches m with mass(w >= m) >= p: lo = 0, hi = max w; mid = lo + (hi - lo) / 2 in the
    dtype of ``w``; mass(>= mid) >= p moves lo up, else hi down; stops once hi - lo <= eps or
    mid no longer splits the interval; p >= 1 keeps every entry.  Masses are fp64 sums.
    Returns (m, kept).
    """
    w = np.asarray(w)
    dt = w.dtype.type
    w64 = w.astype(F64)

    def mass(t):
        return float(w64[w >= t].sum())

    top = dt(w.max())
    if p >= 1.0:
        m = dt(0.0)           # p = 1: the whole distribution, every candidate is kept
    elif mass(top) >= p:
        m = top
    else:
        lo, hi = dt(0.0), top
        for _ in range(max_iter):
            if F64(hi) - F64(lo) <= eps:
                break
            mid = dt(lo + (hi - lo) / dt(2.0))
            if not (lo < mid < hi):
                break
            if mass(mid) >= p:
                lo = mid
            else:
                hi = mid
        m = lo
    return m, np.nonzero(w >= m)[0]


# ----------------------------------------------------------------------------------------------
# Attention
# ----------------------------------------------------------------------------------------------

def attention(q16, k16, v16, scale: float):
    """Exact softmax(q K^T * scale) V in fp64 over the given rows; lse in natural log ([Notes]
    "Overall framework": the final attention runs over the kept tokens only, renormalised)."""
    q = np.asarray(q16, dtype=F16).astype(F64)
    k = np.asarray(k16, dtype=F16).astype(F64)
    v = np.asarray(v16, dtype=F16).astype(F64)
    if k.shape[0] == 0:
        return np.zeros(q.shape[-1]), -math.inf
    s = (k @ q) * F64(scale)
    mx = s.max()
    e = np.exp(s - mx)
    l = e.sum()
    return (e @ v) / l, float(mx + math.log(l))


def gather_tokens(arr, page_table, b: int, kvh: int, tokens):
    """Rows of a paged [P][Hkv][16][D] array for logical token ids of sequence b."""
    tokens = np.asarray(tokens, dtype=np.int64)
    phys = page_table[b, tokens // PAGE]
    return arr[phys, kvh, tokens % PAGE]


# ----------------------------------------------------------------------------------------------
# The decode path, stage by stage
# ----------------------------------------------------------------------------------------------

def select_pages(q, bounds, page_table, seq_lens, num_q_heads, num_kv_heads,
                 budget_pages=0, budget_div=4):
    """Per (b, q-head): (scores fp32 [P_b], selected logical pages ascending)."""
    g = num_q_heads // num_kv_heads
    out = {}
    for b in range(len(seq_lens)):
        pb = num_pages(seq_lens[b])
        phys = page_table[b, :pb]
        kb = budget_for(pb, budget_pages, budget_div)
        for h in range(num_q_heads):
            kvh = h // g
            sc = page_scores(q[b, h], bounds[phys, kvh, 0], bounds[phys, kvh, 1])
            out[(b, h)] = (sc, select_top_k(sc, kb))
    return out


def candidates(sel_pages, n: int) -> np.ndarray:
    """Valid logical token ids of the selected pages, ascending (the candidates the selector
    hands to top-p: [Notes] "Overall framework"; [Summary] 4.1)."""
    toks = [np.arange(PAGE * j, PAGE * j + valid_rows(n, j)) for j in sorted(sel_pages)]
    return np.concatenate(toks).astype(np.int64) if toks else np.zeros(0, dtype=np.int64)


def estimate_head(q16, k_int4, k_sz, page_table, b, kvh, n, sel_pages, head_dim=128):
    """Estimated weights of one head over its candidates (fp64), with the token ids: softmax of
    q . khat / sqrt(D) with khat = n*s + z from the INT4 copy ([Notes] "Key designs": top-p needs
    weight values, estimated from the 4-bit K cache; [Summary] 4.2, B.1)."""
    cand = candidates(sel_pages, n)
    if cand.size == 0:
        return cand, np.zeros(0)
    packed = gather_tokens(k_int4, page_table, b, kvh, cand)            # [C][D/2]
    sz = gather_tokens(k_sz, page_table, b, kvh, cand)                  # [C][2]
    nib = np.empty((cand.size, head_dim), dtype=F64)
    nib[:, 0::2] = packed & 0x0F
    nib[:, 1::2] = packed >> 4
    khat = nib * sz[:, 0:1].astype(F64) + sz[:, 1:2].astype(F64)
    logits = (khat @ np.asarray(q16, dtype=F16).astype(F64)) / math.sqrt(head_dim)
    return cand, softmax64(logits)


# ----------------------------------------------------------------------------------------------
# Estimator bit widths ([Notes] "Key designs": the 4-bit K cache, and lower / higher precisions
# compared in the ablation; [Summary] 4.3 and the bit-width figures): the same per-row
# asymmetric scheme with L = 2^bits - 1 levels.
# ----------------------------------------------------------------------------------------------

def quantize_rows_bits(x16: np.ndarray, bits: int):
    """Token rows (fp16 [R][D]) -> (packed uint8 [R][D*bits/8], scale fp16 [R], zero fp16 [R]).

    s = fp16(fp32(max - min) / L), z = min, n_c = clamp(rint_even(fp32(x_c - z) / s), 0, L)
    (n_c = 0 when s = 0), L = 2^bits - 1.  Channel c occupies bits [c*bits, (c+1)*bits) of the
    row, counted from the low bit of byte 0 (for bits = 4: channel 2j in the low nibble of
    byte j, as ``quantize_rows``)."""
    assert bits in (2, 4, 8)
    levels = (1 << bits) - 1
    x16 = np.asarray(x16, dtype=F16)
    mn, mx = f16_min_max(x16, axis=1)
    s16 = ((mx.astype(F32) - mn.astype(F32)) / F32(levels)).astype(F16)
    s32 = s16.astype(F32)[:, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.rint((x16.astype(F32) - mn.astype(F32)[:, None]) / s32)
    r = np.where(s32 == F32(0.0), F32(0.0), r)
    n = np.clip(r, 0, levels).astype(np.uint64)
    per = 8 // bits                                    # values per byte
    rows, d = n.shape
    packed = np.zeros((rows, d // per), dtype=np.uint64)
    for i in range(per):
        packed |= n[:, i::per] << np.uint64(bits * i)
    return packed.astype(np.uint8), s16, mn


def unpack_rows_bits(packed: np.ndarray, bits: int) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8).astype(np.int64)
    per = 8 // bits
    mask = (1 << bits) - 1
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * per,), dtype=np.int64)
    for i in range(per):
        out[..., i::per] = (packed >> (bits * i)) & mask
    return out


def quantize_k_bits(k, page_table, seq_lens, bits: int):
    """``quantize_k`` at another bit width: (uint8 [P][Hkv][16][D*bits/8], fp16 [P][Hkv][16][2])."""
    p_phys, hkv, page, d = k.shape
    q = np.zeros((p_phys, hkv, page, d * bits // 8), dtype=np.uint8)
    sz = np.zeros((p_phys, hkv, page, 2), dtype=F16)
    for b in range(len(seq_lens)):
        n = int(seq_lens[b])
        pb = num_pages(n)
        phys = np.asarray(page_table[b, :pb], dtype=np.int64)
        pk, s16, z16 = quantize_rows_bits(k[phys].reshape(-1, d), bits)
        pk = pk.reshape(pb, hkv, page, -1)
        s16 = s16.reshape(pb, hkv, page)
        z16 = z16.reshape(pb, hkv, page)
        r_valid = n - PAGE * (pb - 1)
        pk[pb - 1, :, r_valid:] = 0
        s16[pb - 1, :, r_valid:] = F16(0.0)
        z16[pb - 1, :, r_valid:] = F16(0.0)
        q[phys] = pk
        sz[phys, :, :, 0] = s16
        sz[phys, :, :, 1] = z16
    return q, sz


def estimate_head_bits(q16, k_q, k_sz, page_table, b, kvh, n, sel_pages, bits, head_dim=128):
    """``estimate_head`` from the ``bits``-wide copy of K: khat = n*s + z, fp64 logits (the
    bit-width ablation of [Summary] 4.3)."""
    cand = candidates(sel_pages, n)
    if cand.size == 0:
        return cand, np.zeros(0)
    packed = gather_tokens(k_q, page_table, b, kvh, cand)
    sz = gather_tokens(k_sz, page_table, b, kvh, cand)
    khat = unpack_rows_bits(packed, bits).astype(F64) * sz[:, 0:1].astype(F64) \
        + sz[:, 1:2].astype(F64)
    logits = (khat @ np.asarray(q16, dtype=F16).astype(F64)) / math.sqrt(head_dim)
    return cand, softmax64(logits)


def exact_weights(q16, k, page_table, b, kvh, cand, head_dim=128):
    """Softmax of the exact q.k / sqrt(D) (fp16 K, fp64 arithmetic) over the candidates: the
    weights the estimate stands in for."""
    kk = gather_tokens(k, page_table, b, kvh, cand).astype(F64)
    logits = (kk @ np.asarray(q16, dtype=F16).astype(F64)) / math.sqrt(head_dim)
    return softmax64(logits)


# ----------------------------------------------------------------------------------------------
# Cluster-level top-p selection (the Double-P summary page, "Technical framework" and "Key
# designs": a first top-p over clusters scored with size-weighted centroids, then token-level
# top-p inside the kept clusters).  The page gives no clustering method; the reading here takes
# the page (16 consecutive tokens) as the cluster, its centroid as the mean of its valid K rows,
# and its size as the number of those rows.
# ----------------------------------------------------------------------------------------------

def page_centroids(k, page_table, seq_lens, out=None):
    """fp16 [P][Hkv][D]: per referenced page and kv-head, the mean of the valid K rows, summed
    in fp32 from row 0 upwards, divided by the row count in fp32, rounded to fp16."""
    p_phys, hkv, page, d = k.shape
    cen = np.zeros((p_phys, hkv, d), dtype=F16) if out is None else out.copy()
    for b in range(len(seq_lens)):
        n = int(seq_lens[b])
        for j in range(num_pages(n)):
            ph = int(page_table[b, j])
            rows = valid_rows(n, j)
            acc = np.zeros((hkv, d), dtype=F32)
            for r in range(rows):                   # left to right, fp32
                acc = (acc + k[ph, :, r, :].astype(F32)).astype(F32)
            cen[ph] = (acc / F32(rows)).astype(F16)
    return cen


def cluster_weights(q16, cen, page_table, b, kvh, n, head_dim=128):
    """Size-weighted centroid estimate of each page's share of the attention mass:
    A_j = n_j exp(q . c_j / sqrt(D)), normalised over the sequence's pages (fp64) (the Double-P
    summary page, "Key designs": clusters scored by size-weighted centroids)."""
    pb = num_pages(n)
    phys = np.asarray(page_table[b, :pb], dtype=np.int64)
    c = cen[phys, kvh].astype(F64)                                      # [pb][D]
    sizes = np.array([valid_rows(n, j) for j in range(pb)], dtype=F64)
    logits = np.log(sizes) + (c @ np.asarray(q16, dtype=F16).astype(F64)) / math.sqrt(head_dim)
    return softmax64(logits)


def select_clusters(q, cen, page_table, seq_lens, num_q_heads, num_kv_heads, p_cluster):
    """Per (b, head): the pages kept by top-p (sort form) over the cluster weights, ascending.
    Returns {(b, h): (weights, pages)}."""
    g = num_q_heads // num_kv_heads
    out = {}
    for b in range(len(seq_lens)):
        n = int(seq_lens[b])
        for h in range(num_q_heads):
            w = cluster_weights(q[b, h], cen, page_table, b, h // g, n)
            _, _, kept = top_p_whole(w, p_cluster)
            out[(b, h)] = (w, np.sort(np.asarray(kept, dtype=np.int64)))
    return out


def decode_step(wl, bounds=None, k_int4=None, k_sz=None, with_attention=True):
    """Full oracle pass of select -> estimate -> top-p -> group union -> attention.

    ``wl`` is a workloads.synth.DecodeWorkload.  Returns a dict keyed by stage.
    """
    hq, hkv = wl.num_q_heads, wl.num_kv_heads
    g = hq // hkv
    if bounds is None:
        bounds = page_bounds(wl.k, wl.page_table, wl.seq_lens)
    if k_int4 is None or k_sz is None:
        k_int4, k_sz = quantize_k(wl.k, wl.page_table, wl.seq_lens)
    sel = select_pages(wl.q, bounds, wl.page_table, wl.seq_lens, hq, hkv,
                       wl.budget_pages, wl.budget_div)
    heads = {}
    for (b, h), (sc, pages) in sel.items():
        cand, w = estimate_head(wl.q[b, h], k_int4, k_sz, wl.page_table, b, h // g,
                                int(wl.seq_lens[b]), pages, wl.head_dim)
        k_star, m_star, kept = top_p_whole(w, wl.p)
        heads[(b, h)] = dict(scores=sc, sel=pages, cand=cand, w=w, k_star=k_star,
                             m_star=m_star, kept=kept, kept_tok=cand[kept])
    groups = {}
    scale = 1.0 / math.sqrt(wl.head_dim)
    for b in range(wl.batch):
        for kvh in range(hkv):
            toks = np.unique(np.concatenate(
                [heads[(b, h)]["kept_tok"] for h in range(kvh * g, (kvh + 1) * g)]))
            grp = dict(union=toks)
            if with_attention:
                kk = gather_tokens(wl.k, wl.page_table, b, kvh, toks)
                vv = gather_tokens(wl.v, wl.page_table, b, kvh, toks)
                grp["o"] = {}
                grp["lse"] = {}
                for h in range(kvh * g, (kvh + 1) * g):
                    o, lse = attention(wl.q[b, h], kk, vv, scale)
                    grp["o"][h] = o
                    grp["lse"][h] = lse
            groups[(b, kvh)] = grp
    return dict(bounds=bounds, k_int4=k_int4, k_sz=k_sz, heads=heads, groups=groups)


def group_attention(wl, tok_lists):
    """Attention of every q-head over its group's given token set: {(b,h): (o, lse)} (GQA
    groups attend over one token set: [Summary] B.2)."""
    g = wl.num_q_heads // wl.num_kv_heads
    scale = 1.0 / math.sqrt(wl.head_dim)
    out = {}
    for (b, kvh), toks in tok_lists.items():
        kk = gather_tokens(wl.k, wl.page_table, b, kvh, toks)
        vv = gather_tokens(wl.v, wl.page_table, b, kvh, toks)
        for h in range(kvh * g, (kvh + 1) * g):
            out[(b, h)] = attention(wl.q[b, h], kk, vv, scale)
    return out


def full_attention_weights(q16, k16, scale):
    """Exact softmax weights over every token (for the top-p error bound of [Notes] "Key
    designs", oracle top-p)."""
    s = (np.asarray(k16, dtype=F16).astype(F64) @ np.asarray(q16, dtype=F16).astype(F64))
    return softmax64(s * F64(scale))
