/*
 * twl.h - C ABI of a B200 (sm_100a) library for hierarchical top-p sparse decode attention.
 *
 * The method is the select-then-prune decode path of "Twilight: Adaptive Attention Sparsity with
 * Hierarchical Top-p Pruning".  Two pages describe it and are cited below:
 *   [Notes]   Paper-Notes (NeurIPS 2025) page: "Overall framework", "Key designs" (oracle top-p,
 *             binary-search top-p, 4-bit K cache, load balancing), "Limitations".
 *   [Summary] paperlayer summary of arXiv 2502.02770v5: sections 3.2, 4.1, 4.2, 4.3, B.1, B.2.
 *
 * Per query head the path is:
 *   select   a Quest-style selector scores 16-token pages by their channel-wise K bounds and
 *            keeps a conservative top-k page budget (1/4 of the pages by default)
 *   estimate attention weights over the selected tokens from an INT4 copy of K
 *   prune    the smallest set whose estimated weight reaches p, found by bisection on a
 *            weight threshold m (no sort)
 *   attend   exact fp16 attention over the kept tokens; for GQA each group attends over the
 *            union of its heads' kept tokens, split into chunks over a flattened work list.
 *
 * Conventions for every call
 *   - All array pointers are DEVICE memory owned by the caller.  The library never allocates,
 *     frees or synchronises, except twl_device_status (which waits on the stream).
 *   - fp16 arrays are passed as raw IEEE binary16 bits (uint16_t / void*).
 *   - Calls are asynchronous and ordered on `stream` (a cudaStream_t; NULL = legacy stream).
 *   - Errors the host can see (NULL pointers, unsupported sizes, p outside (0,1], eps <= 0,
 *     misaligned pointers, a workspace that is too small) are returned immediately and nothing
 *     is launched.  TWL_ERR_CUDA reports a failed launch (cudaGetLastError).
 *   - Errors only the device can see (a page-table entry outside [0, num_phys_pages), a sequence
 *     length < 1 or longer than max_pages * page_size, an index list entry out of range) never
 *     trap: the offending page / token / sequence is skipped, its outputs are left empty or
 *     zero, and a sticky flag is set in the workspace header; read it with twl_device_status.
 *   - A workspace is caller-owned device memory of at least twl_workspace_bytes(...) bytes,
 *     256-byte aligned.  Its first 256 bytes are a header that must be zero before first use
 *     (twl_workspace_init).  Workspaces may be reused across calls on the same stream; calls
 *     that run concurrently must not share one.
 *   - Supported shapes: head_dim = 128, page_size = 16, num_q_heads / num_kv_heads in
 *     {1, 2, 4, 8}, max_pages <= 32768 (512K tokens per sequence).
 *
 * Paged KV cache layout (PagedAttention-style, [Summary] 4.3):
 *   k, v          fp16  [num_phys_pages][num_kv_heads][page_size][head_dim]
 *   page_table    int32 [batch][max_pages]   logical page j of sequence b -> physical page;
 *                                            entries j >= ceil(seq_lens[b] / 16) are ignored
 *   seq_lens      int32 [batch]              tokens of each sequence (>= 1)
 * Derived K data, same physical paging ([Summary] B.1, 4.3):
 *   k_int4        uint8 [num_phys_pages][num_kv_heads][16][64]   channel 2j in the low nibble of
 *                                                                byte j of its token row
 *   k_scale_zero  fp16  [num_phys_pages][num_kv_heads][16][2]    (scale, zero) per token row
 *   bounds        fp16  [num_phys_pages][num_kv_heads][2][128]   channel min row, then max row
 * Token ids are logical positions 0 .. seq_lens[b]-1 of their sequence.
 */
#ifndef TWL_H_
#define TWL_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t twl_status;
#define TWL_OK 0
#define TWL_ERR_INVALID_ARG (-1) /* bad pointer, size, p, eps or alignment (host-detected) */
#define TWL_ERR_UNSUPPORTED (-2) /* valid but not supported: head_dim, page_size, group size */
#define TWL_ERR_CUDA (-3)        /* a CUDA launch or copy failed */
#define TWL_ERR_TIMEOUT (-4)     /* device flag: a bounded wait inside a kernel gave up */
#define TWL_ERR_WORKSPACE (-5)   /* workspace NULL, misaligned or smaller than required */
#define TWL_ERR_BAD_INDEX (-6)   /* device flag: page table / seq_lens / index list out of range */
#define TWL_ERR_SCRATCH_LIMIT (-7) /* request larger than twl_sparse_decode_noalloc's scratch */

/* Device flag bits reported by twl_device_status (sticky until cleared). */
#define TWL_FLAG_BAD_INDEX 1u
#define TWL_FLAG_TIMEOUT 2u

typedef void* twl_stream_t; /* a cudaStream_t */

typedef struct twl_paged_kv {
  const void* k;              /* fp16 [P][Hkv][16][128]                              */
  const void* v;              /* fp16 [P][Hkv][16][128]; may be NULL where V unused  */
  const int32_t* page_table;  /* int32 [batch][max_pages]                            */
  const int32_t* seq_lens;    /* int32 [batch]                                       */
  int32_t batch;
  int32_t num_kv_heads;
  int32_t head_dim;           /* must be 128 */
  int32_t page_size;          /* must be 16  */
  int32_t max_pages;          /* page_table row stride; >= ceil(max seq_len / 16) */
  int32_t num_phys_pages;     /* P */
} twl_paged_kv;

/* Derived K data (see layouts above).  Written by twl_quantize_k / twl_page_bounds. */
typedef struct twl_k_aux {
  void* k_int4;
  void* k_scale_zero;
  void* bounds;
} twl_k_aux;

/* Optional outputs of twl_decode_step (any member may be NULL; NULL struct = none).
 * Strides: max_budget as given to twl_decode_step, cs = 16 * max_budget candidate slots,
 * us = 16 * max_pages union slots. */
typedef struct twl_step_stats {
  int32_t* sel_pages;    /* [B][Hq][max_budget] selected logical pages, ascending   */
  int32_t* sel_count;    /* [B][Hq]                                                  */
  float* weights;        /* [B][Hq][cs] estimated weights W of the candidates        */
  int32_t* cand_tok;     /* [B][Hq][cs] logical token id of each candidate           */
  int32_t* cand_count;   /* [B][Hq]                                                  */
  float* threshold;      /* [B][Hq] the top-p threshold m                            */
  int32_t* kept_count;   /* [B][Hq] |{i : W_i >= m}|                                 */
  int32_t* union_tok;    /* [B][Hkv][us] union of the group's kept tokens, ascending */
  int32_t* union_count;  /* [B][Hkv]                                                 */
} twl_step_stats;

/* Workspace sizing.  op is one of the TWL_OP_* values; unused dimensions may be 0. */
#define TWL_OP_CACHE 1         /* twl_page_bounds, twl_quantize_k: header only */
#define TWL_OP_SELECT 2        /* twl_select_pages                          */
#define TWL_OP_ESTIMATE 3      /* twl_estimate                              */
#define TWL_OP_PRUNE 4         /* twl_prune_top_p                           */
#define TWL_OP_UNION 5         /* twl_group_union                           */
#define TWL_OP_SPARSE_DECODE 6 /* twl_sparse_decode (row_stride = tok_stride) */
#define TWL_OP_DECODE_STEP 7   /* twl_decode_step                           */
#define TWL_OP_SELECT_CLUSTERS 8 /* twl_select_clusters_top_p                 */
size_t twl_workspace_bytes(int32_t op, int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                           int32_t max_pages, int32_t max_budget, int32_t rows,
                           int32_t row_stride);

/* Zero the whole workspace: a stream-ordered memset of ws_bytes, which clears the header's device
 * flags and, for twl_decode_step, the synchronisation words and page masks that must start at
 * zero (each step launch leaves them zero again for the next). */
twl_status twl_workspace_init(void* ws, size_t ws_bytes, twl_stream_t stream);

/* Wait for `stream`, then report the sticky device flags of `ws` in *flags (may be NULL).
 * Returns TWL_OK if no flag is set, else TWL_ERR_BAD_INDEX or TWL_ERR_TIMEOUT.  If clear != 0
 * the flags are reset to zero afterwards. */
twl_status twl_device_status(void* ws, uint32_t* flags, int32_t clear, twl_stream_t stream);

const char* twl_status_string(twl_status s);

/* ---------------------------------------------------------------- cache maintenance (a0)
 * twl_page_bounds: channel-wise min and max of K over the valid tokens of every referenced
 *   page, per kv-head (the page metadata a Quest selector scores; the selector is named in
 *   [Notes] "Background" and [Summary] 5.1).  fp16 min/max use the total order -0 < +0.
 *   Writes bounds[p][h][0][:] = min, bounds[p][h][1][:] = max for each physical page p that
 *   some sequence references; other pages are untouched.
 * twl_quantize_k: INT4 copy of K ([Summary] B.1, per-head dynamic asymmetric quantisation with
 *   fp16 scale and zero point, two values per byte; [Notes] "Key designs", 4-bit K cache).  Per
 *   token row of one head: s = fp16_rn(fp32(max - min) / 15), z = min,
 *   n_c = min(15, rint_even(fp32(x_c - z) / s)) in IEEE fp32 (n_c = 0 when s = 0).  Rows past
 *   the end of a sequence in its last page are written as zeros.
 * Workspace (TWL_OP_CACHE) may be NULL; it only carries the device flags. */
twl_status twl_page_bounds(const twl_paged_kv* kv, void* bounds, void* ws, size_t ws_bytes,
                           twl_stream_t stream);
twl_status twl_quantize_k(const twl_paged_kv* kv, void* k_int4, void* k_scale_zero, void* ws,
                          size_t ws_bytes, twl_stream_t stream);

/* twl_append_token: the cache maintenance of one decode step, fused with the KV append (the 4-bit
 *   K cache and the page metadata are kept current as tokens arrive: [Summary] B.1, 4.3; [Notes]
 *   "Key designs", 4-bit K cache).  For every sequence b with n_b = seq_lens[b], the new token
 *   goes to logical position n_b: row n_b % 16 of physical page page_table[b][n_b / 16], which
 *   the caller has mapped.  Per kv-head h:
 *     K row = k_new[b][h][:], V row = v_new[b][h][:];
 *     the INT4 row and its (scale, zero) are written exactly as twl_quantize_k writes them;
 *     the page bounds become the K row itself when it is the page's first row (n_b % 16 == 0),
 *     else the channel-wise min / max (total order, -0 < +0) of the old bounds and the row.
 *   The result equals twl_page_bounds + twl_quantize_k over the extended cache, bit for bit.
 *   If advance != 0, seq_lens[b] becomes n_b + 1 afterwards (device side, same launch).
 *   k_new, v_new: device fp16 [batch][num_kv_heads][128], 16-byte aligned.  kv->k, kv->v and
 *   (with advance) kv->seq_lens are written through: the caller's buffers must be writable.
 *   A sequence whose position has no mapped page (n_b >= 16 * max_pages, or a negative or
 *   out-of-range table entry) is left unchanged and not advanced; TWL_FLAG_BAD_INDEX is raised.
 *   Workspace (TWL_OP_CACHE) may be NULL; it only carries the device flags.
 *   Returns TWL_ERR_INVALID_ARG for NULL or misaligned pointers, TWL_ERR_UNSUPPORTED for shapes
 *   the library does not support (head_dim != 128, page_size != 16). */
twl_status twl_append_token(const twl_paged_kv* kv, const twl_k_aux* aux, const void* k_new,
                            const void* v_new, int32_t advance, void* ws, size_t ws_bytes,
                            twl_stream_t stream);

/* ---------------------------------------------------------------- select (a1, a2)
 * Per (b, q-head h): score every page j < P_b = ceil(seq_lens[b]/16) by
 *   score_j = sum_c t_c,  t_c = q_c * max_c if q_c > 0 else q_c * min_c
 * (the bounding-box upper bound of q.k; the pages name the Quest selector without its formula).
 * t_c is exact in fp32; the sum is taken in one fixed order (16 partial sums of 8 consecutive
 * channels, each from +0 left to right, then pairs (l,l+8), (l,l+4), (l,l+2), (l,l+1)) so scores
 * are bit-reproducible.  Keep k_b = budget_pages if > 0 else ceil(P_b / budget_div) pages (all
 * if P_b <= k_b) with the highest scores, ties to the lower logical page ([Notes] "Overall
 * framework": a conservative base budget such as 1/4; [Summary] 4.1, 4.3).
 *   q          fp16 [B][Hq][128]
 *   bounds     from twl_page_bounds
 *   max_budget sel_pages row stride; must be >= every k_b
 *   sel_pages  int32 [B][Hq][max_budget] out, ascending; sel_count int32 [B][Hq] out
 *   scores     float [B][Hq][max_pages] out, or NULL; entries j >= P_b are not written */
twl_status twl_select_pages(const void* q, int32_t num_q_heads, const twl_paged_kv* kv,
                            const void* bounds, int32_t budget_pages, int32_t budget_div,
                            int32_t max_budget, int32_t* sel_pages, int32_t* sel_count,
                            float* scores, void* ws, size_t ws_bytes, twl_stream_t stream);

/* ---------------------------------------------------------------- estimate (a3, a4)
 * Candidates of head h = the valid tokens of its selected pages in ascending order; candidate
 * slot i = 16 * (rank of the page in sel_pages) + row.  logit = q . khat / sqrt(128) with
 * khat = n * s + z from the INT4 copy; weights = softmax over the head's candidates in fp32
 * ([Notes] "Key designs": top-p needs weight values, estimated from the 4-bit K cache;
 * [Summary] 4.2, B.1).  INT4 K is read once per GQA group over the union of its heads'
 * selected pages ([Summary] B.2).
 *   weights   float [B][Hq][16*max_budget] out; cand_tok int32 same shape out (token ids);
 *   cand_count int32 [B][Hq] out.  Slots >= cand_count are not written. */
twl_status twl_estimate(const void* q, int32_t num_q_heads, const twl_paged_kv* kv,
                        const void* k_int4, const void* k_scale_zero, const int32_t* sel_pages,
                        const int32_t* sel_count, int32_t max_budget, float* weights,
                        int32_t* cand_tok, int32_t* cand_count, void* ws, size_t ws_bytes,
                        twl_stream_t stream);

/* ---------------------------------------------------------------- cluster-level top-p (f4)
 * The Double-P selector (Double-P summary page, "Technical framework" and "Key designs": a
 * top-p over clusters scored by size-weighted centroids, then token-level top-p inside the
 * kept clusters, which twl_estimate / twl_prune_top_p / twl_group_union / twl_sparse_decode
 * do with the pages kept here).  The page gives no clustering method: a cluster is one page.
 *   twl_page_centroids: centroids fp16 [P][Hkv][128]; per referenced page and kv-head the mean
 *     of the valid K rows (fp32 sum from row 0 upwards, IEEE fp32 division by the row count,
 *     fp16 round to nearest even).  Workspace (TWL_OP_CACHE) may be NULL.
 *   twl_select_clusters_top_p: per (b, q-head) A_j = n_j exp(q . c_j / sqrt(128)) over the
 *     sequence's pages j (n_j valid rows), W_j = A_j / sum A; then the bisection of
 *     twl_prune_top_p at p_cluster, eps.  sel_pages int32 [B][Hq][max_pages] out (kept pages,
 *     ascending; pass max_budget = max_pages to twl_estimate), sel_count int32 [B][Hq] out,
 *     cluster_weights float [B][Hq][max_pages] out (W; slots past P_b unwritten) or NULL.
 *     Workspace TWL_OP_SELECT_CLUSTERS.  p_cluster outside (0, 1], eps <= 0 or not finite:
 *     TWL_ERR_INVALID_ARG. */
twl_status twl_page_centroids(const twl_paged_kv* kv, void* centroids, void* ws, size_t ws_bytes,
                              twl_stream_t stream);
twl_status twl_select_clusters_top_p(const void* q, int32_t num_q_heads, const twl_paged_kv* kv,
                                     const void* centroids, float p_cluster, float eps,
                                     int32_t* sel_pages, int32_t* sel_count,
                                     float* cluster_weights, void* ws, size_t ws_bytes,
                                     twl_stream_t stream);

/* ---------------------------------------------------------------- estimator bit widths (f2)
 * The estimator ablation ([Notes] "Key designs": a 4-bit K cache suffices for the weight
 * estimate; [Summary] 4.3 and its bit-width figures): the INT4 scheme of twl_quantize_k at
 * bits = 2 or 8 (bits = 4 is exactly twl_quantize_k / twl_estimate).  Per token row:
 * L = 2^bits - 1, s = fp16_rn(fp32(max - min) / L), z = min,
 * n_c = min(L, rint_even(fp32(x_c - z) / s)) (n_c = 0 when s = 0); channel c occupies bits
 * [c*bits, (c+1)*bits) of the row, from the low bit of byte 0.
 *   twl_quantize_k_nbit: k_codes uint8 [P][Hkv][16][128*bits/8], k_scale_zero as twl_quantize_k.
 *   twl_estimate_nbit: twl_estimate reading that copy (workspace TWL_OP_ESTIMATE).
 * bits outside {2, 4, 8} returns TWL_ERR_UNSUPPORTED; other errors as the INT4 calls. */
twl_status twl_quantize_k_nbit(const twl_paged_kv* kv, int32_t bits, void* k_codes,
                               void* k_scale_zero, void* ws, size_t ws_bytes,
                               twl_stream_t stream);
twl_status twl_estimate_nbit(const void* q, int32_t num_q_heads, const twl_paged_kv* kv,
                             int32_t bits, const void* k_codes, const void* k_scale_zero,
                             const int32_t* sel_pages, const int32_t* sel_count,
                             int32_t max_budget, float* weights, int32_t* cand_tok,
                             int32_t* cand_count, void* ws, size_t ws_bytes,
                             twl_stream_t stream);

/* ---------------------------------------------------------------- prune (a5)
 * Per row r of w (float [rows][row_stride], row length row_len[r] or row_stride if row_len is
 * NULL, weights >= 0 summing to ~1): bisection on the threshold m ([Notes] "Key designs",
 * efficient top-p: find m with sum_{W[i] >= m} W[i] >= p in O(log(max W / eps)) rounds of O(n)
 * parallel work, no sort; [Summary] 4.2).  If mass(W >= max W) >= p then m = max W; else
 * lo = 0, hi = max W, mid = lo + (hi - lo)/2 (fp32); mass(W >= mid) >= p sets lo = mid, else
 * hi = mid; stop when hi - lo <= eps or mid no longer splits; m = lo.  p = 1 keeps every entry
 * (m = 0).
 * Rows whose stride is a multiple of 4 (at most 262144) on a 16-byte aligned base are read once:
 * the test at mid equals "mid <= T" for T = the largest weight v with mass(W >= v) >= p, so T is
 * found from bit-pattern histograms with exact per-bin masses and the bisection is replayed on
 * it; the mass of the weights above the final histogram's range is an fp32-pairwise / fp64 sum
 * (redone in fp64 when the decision falls within its error bound).  Other rows run the direct
 * bisection with fp32 block sums.  Negative weights carry no mass; NaN weights are never kept.
 *   m_out      float [rows] out
 *   kept_count int32 [rows] out = |{i : W_i >= m}|
 *   kept_idx   int32 [rows][row_stride] out (ascending indices) or NULL
 *   ws, ws_bytes  unused (NULL and 0 are fine; twl_workspace_bytes(TWL_OP_PRUNE, ...) gives
 *                 the 256-byte header size, which this call does not need)
 * TWL_ERR_INVALID_ARG for NULL w / m_out / kept_count, rows < 0, row_stride < 1, p outside
 * (0, 1], eps not positive and finite, or w not 4-byte aligned; rows == 0 launches nothing. */
twl_status twl_prune_top_p(const float* w, const int32_t* row_len, int32_t rows,
                           int32_t row_stride, float p, float eps, float* m_out,
                           int32_t* kept_count, int32_t* kept_idx, void* ws, size_t ws_bytes,
                           twl_stream_t stream);

/* ---------------------------------------------------------------- union (a6)
 * Per (b, kv-head): the union of the kept tokens of the group's q-heads ([Summary] B.2: GQA
 * groups select the union so each K/V row is read once).  Kept token of head h, entry i:
 * cand_tok[b][h][kept_idx[b][h][i]], i < kept_count[b][h], row stride cand_stride.
 *   union_tok int32 [B][Hkv][16*max_pages] out, ascending; union_count int32 [B][Hkv] out. */
twl_status twl_group_union(int32_t num_q_heads, const twl_paged_kv* kv, const int32_t* cand_tok,
                           const int32_t* kept_idx, const int32_t* kept_count,
                           int32_t cand_stride, int32_t* union_tok, int32_t* union_count,
                           void* ws, size_t ws_bytes, twl_stream_t stream);

/* ---------------------------------------------------------------- attend (a7, a8)
 * For every q-head h of group (b, kvh): o = softmax(q_h K_U^T * sm_scale) V_U over the tokens
 * tok[b][kvh][0 .. tok_count-1] (fp16 K/V, fp32 math), lse = natural-log sum of exp of the
 * scaled scores ([Notes] "Overall framework": attention runs only on the kept tokens; "Key
 * designs", load balancing: heads are flattened and the work redistributed).  The token lists
 * of all groups are cut into fixed-size chunks that form one flattened work list; partial
 * (o, lse) per chunk are merged by log-sum-exp.  An empty list gives o = 0, lse = -inf.
 *   tok    int32 [B][Hkv][tok_stride]; tok_count int32 [B][Hkv]
 *   o      float [B][Hq][128] out;   lse float [B][Hq] out */
twl_status twl_sparse_decode(const void* q, int32_t num_q_heads, const twl_paged_kv* kv,
                             const int32_t* tok, const int32_t* tok_count, int32_t tok_stride,
                             float sm_scale, float* o, float* lse, void* ws, size_t ws_bytes,
                             twl_stream_t stream);

/* ---------------------------------------------------------------- attend, no allocation
 * The paper has no counterpart to this call; it serves callers that cannot allocate device
 * memory for a workspace: plug-ins inside a framework that owns all device memory, real-time
 * code that may not call cudaMalloc (it can synchronise the device), and deployments whose memory
 * plan is fixed up front.  Same arguments and results as twl_sparse_decode, minus the workspace:
 * the split-KV scratch comes from one statically sized device array inside the library
 * (twl_noalloc_scratch_bytes() bytes, 8 MiB), held by every GPU that loads the library until the
 * process exits.  A request whose scratch (twl_workspace_bytes(TWL_OP_SPARSE_DECODE, ...)) exceeds
 * it returns TWL_ERR_SCRATCH_LIMIT and launches nothing.  The first call on a device looks up the
 * array's device address (once per device, that device current); make it before any stream
 * capture.  That address is kept for the life of the process: it does not survive cudaDeviceReset
 * or serve another context made current on the same device, so do not call this entry point after
 * either.  Every call shares the array: calls that overlap on the GPU race.  Device flags are not
 * reported by this call.  Arguments are checked as by twl_sparse_decode before the scratch size.
 * It allocates nothing. */
size_t twl_noalloc_scratch_bytes(void);
twl_status twl_sparse_decode_noalloc(const void* q, int32_t num_q_heads, const twl_paged_kv* kv,
                                     const int32_t* tok, const int32_t* tok_count,
                                     int32_t tok_stride, float sm_scale, float* o, float* lse,
                                     twl_stream_t stream);

/* ---------------------------------------------------------------- the whole step
 * select -> estimate -> prune (p, eps) -> group union -> attend, with sm_scale = 1/sqrt(128)
 * ([Notes] "Overall framework"; [Summary] 4.1 and Figure 5), as one persistent launch over every
 * SM.  The selections, candidates and weights equal those of the five calls above in sequence;
 * the threshold m is the bisection's result computed from exact fixed-point masses (units of
 * 2^-48, each weight rounded to that unit), so it can differ from twl_prune_top_p's only when p
 * is within that rounding (n * 2^-49 for n candidates) of a prefix mass.
 * max_budget: as for twl_select_pages (>= every k_b).
 *   o float [B][Hq][128] out; lse float [B][Hq] out; stats optional (see twl_step_stats).
 * The workspace (TWL_OP_DECODE_STEP bytes, zeroed once by twl_workspace_init) carries the
 * launch's synchronisation words, which every launch leaves cleared for the next; launches on
 * one workspace must be stream-ordered.  Device-side errors are reported through the workspace
 * flags (twl_device_status): page-table entries outside the pool and bad sequence lengths are
 * skipped (TWL_FLAG_BAD_INDEX); a wait between work items that gives up after its bounded number
 * of polls aborts the launch (TWL_FLAG_TIMEOUT, outputs undefined).
 * Shapes: every work item keeps one head's page-score keys (4 bytes per page of the page-table
 * stride) in its CTA's shared memory.  With more (sequence, kv-head) groups than SMs the step runs
 * two 256-thread CTAs per SM, each with half of the SM's shared memory; there max_pages above
 * 23296 (on a 148-SM B200: 228 KB per SM) returns TWL_ERR_UNSUPPORTED and launches nothing.
 * Split such a batch into calls of at most SM-count groups, which take the one-CTA-per-SM build
 * and accept max_pages up to 32768.
 * Residency: the grid is one (or two) CTAs per SM and each CTA's first work item is fixed by its
 * index, so the launch counts on all of its CTAs running at once.  Do not run two
 * twl_decode_step launches concurrently (on different streams or processes sharing the GPU),
 * nor next to a kernel that keeps SMs busy for the whole step: CTAs that cannot start hold up
 * the items waiting on theirs, and those waits give up after their bound (2^22 polls, each at
 * least a 64 ns sleep) with TWL_FLAG_TIMEOUT and undefined outputs rather than hang. */
twl_status twl_decode_step(const void* q, int32_t num_q_heads, const twl_paged_kv* kv,
                           const twl_k_aux* aux, int32_t budget_pages, int32_t budget_div,
                           int32_t max_budget, float p, float eps, float* o, float* lse,
                           const twl_step_stats* stats, void* ws, size_t ws_bytes,
                           twl_stream_t stream);

/* ---------------------------------------------------------------- test hook of the bounded waits
 * twl_decode_step's work items wait for one another by polling counters in the workspace; each
 * wait gives up after a bounded number of polls, raises TWL_FLAG_TIMEOUT and aborts the launch
 * (the kernel returns; the context stays usable; the next launch on the workspace is valid).
 * This hook exists so that a test can make that happen without a device fault: max_polls sets
 * the polls before a wait gives up for later launches (0 = the default, 2^22), and
 * stall_estimate != 0 makes the INT4-estimate items wait for a count that is never reached.
 * Process-wide, read at each twl_decode_step call; not for production use. */
void twl_test_set_waits(uint32_t max_polls, int32_t stall_estimate);

#ifdef __cplusplus
}
#endif
#endif /* TWL_H_ */
