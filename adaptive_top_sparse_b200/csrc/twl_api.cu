// C ABI of the twl library: argument validation, workspace layout, launches.
// Each entry point validates everything it can on the host before launching anything.
#include <math.h>

#include <atomic>
#include <mutex>
#include <stdlib.h>

#include "twl_common.cuh"
#include "twl_kernels.h"
#include "twl_step.h"

namespace twl {

int num_sms() {
  static std::atomic<int> cache[128];  // zero-initialised: not yet queried
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return 148;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

// Bump allocator over a workspace; with base == nullptr it only measures.
struct Carve {
  char* base;
  size_t off = kHeaderBytes;
  template <typename T>
  T* take(size_t count) {
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off = align_up(off + count * sizeof(T));
    return p;
  }
};

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

twl_status check_kv(const twl_paged_kv* kv, bool need_k, bool need_v, KV* out) {
  if (!kv) return TWL_ERR_INVALID_ARG;
  if ((need_k && !kv->k) || (need_v && !kv->v) || !kv->page_table || !kv->seq_lens)
    return TWL_ERR_INVALID_ARG;
  if (kv->batch < 1 || kv->num_kv_heads < 1 || kv->max_pages < 1 || kv->num_phys_pages < 1)
    return TWL_ERR_INVALID_ARG;
  if (kv->head_dim != kHeadDim || kv->page_size != kPage) return TWL_ERR_UNSUPPORTED;
  if (kv->max_pages > kMaxPages) return TWL_ERR_UNSUPPORTED;
  // K/V row index (phys * Hkv + h) * 16 + r must fit 32 bits
  if ((uint64_t)kv->num_phys_pages * (uint64_t)kv->num_kv_heads * kPage >= 0xFFFFFFFFull)
    return TWL_ERR_UNSUPPORTED;
  if ((kv->k && !aligned(kv->k, 16)) || (kv->v && !aligned(kv->v, 16)) ||
      !aligned(kv->page_table, 4) || !aligned(kv->seq_lens, 4))
    return TWL_ERR_INVALID_ARG;
  if (out) {
    out->k = static_cast<const uint16_t*>(kv->k);
    out->v = static_cast<const uint16_t*>(kv->v);
    out->page_table = kv->page_table;
    out->seq_lens = kv->seq_lens;
    out->batch = kv->batch;
    out->hkv = kv->num_kv_heads;
    out->max_pages = kv->max_pages;
    out->num_phys = kv->num_phys_pages;
  }
  return TWL_OK;
}

twl_status check_heads(int hq, int hkv) {
  if (hq < 1 || hkv < 1 || hq % hkv != 0) return TWL_ERR_INVALID_ARG;
  const int g = hq / hkv;
  if (g != 1 && g != 2 && g != 4 && g != 8) return TWL_ERR_UNSUPPORTED;
  return TWL_OK;
}

twl_status check_budget(int budget_pages, int budget_div, int max_budget, int max_pages) {
  if (budget_pages < 0 || max_budget < 1) return TWL_ERR_INVALID_ARG;
  if (budget_pages == 0 && budget_div < 1) return TWL_ERR_INVALID_ARG;
  const long long bound = budget_pages > 0
                              ? (budget_pages < max_pages ? budget_pages : max_pages)
                              : ((long long)max_pages + budget_div - 1) / budget_div;
  if (max_budget < bound || max_budget > max_pages) return TWL_ERR_INVALID_ARG;
  return TWL_OK;
}

twl_status check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (!ws || !aligned(ws, kAlign) || ws_bytes < need) return TWL_ERR_WORKSPACE;
  return TWL_OK;
}

twl_status cuda_status(cudaError_t e) { return e == cudaSuccess ? TWL_OK : TWL_ERR_CUDA; }

uint32_t* flags_of(void* ws) { return ws ? &reinterpret_cast<WsHeader*>(ws)->flags : nullptr; }

size_t decode_step_ws_bytes(int batch, int hq, int hkv, int max_pages, int max_budget) {
  return step_wide(batch * hkv, num_sms())
             ? step256::workspace_bytes(batch, hq, hkv, max_pages, max_budget)
             : step::workspace_bytes(batch, hq, hkv, max_pages, max_budget);
}

// ---------------------------------------------------------------- workspace layouts
struct SelectWs {
  float* scores;
};
SelectWs carve_select(Carve& c, int batch, int hq, int max_pages) {
  SelectWs w;
  w.scores = c.take<float>((size_t)batch * hq * max_pages);
  return w;
}

struct ClusterWs {
  float* w;
  int* row_len;
  float* m;
};
ClusterWs carve_clusters(Carve& c, int batch, int hq, int max_pages) {
  ClusterWs w;
  w.w = c.take<float>((size_t)batch * hq * max_pages);
  w.row_len = c.take<int>((size_t)batch * hq);
  w.m = c.take<float>((size_t)batch * hq);
  return w;
}

struct EstimateWs {
  int* rank;
  int* union_pages;
  uint32_t* union_mask;
  int* union_npages;
};
EstimateWs carve_estimate(Carve& c, int batch, int hq, int hkv, int max_pages) {
  EstimateWs w;
  w.rank = c.take<int>((size_t)batch * hq * max_pages);
  w.union_pages = c.take<int>((size_t)batch * hkv * max_pages);
  w.union_mask = c.take<uint32_t>((size_t)batch * hkv * max_pages);
  w.union_npages = c.take<int>((size_t)batch * hkv);
  return w;
}

}  // namespace

twl_status check_sparse_decode_args(const void* q, int num_q_heads, const twl_paged_kv* kv,
                                    const int32_t* tok, const int32_t* tok_count, int tok_stride,
                                    float sm_scale, const float* o, const float* lse, KV* out) {
  twl_status st = check_kv(kv, true, true, out);
  if (st != TWL_OK) return st;
  if ((st = check_heads(num_q_heads, out->hkv)) != TWL_OK) return st;
  if (!q || !tok || !tok_count || !o || !lse || tok_stride < 1 || !aligned(q, 16) ||
      !aligned(o, 16) || !(sm_scale > 0.f) || isinf(sm_scale))
    return TWL_ERR_INVALID_ARG;
  if ((long long)out->batch * out->hkv > 4096) return TWL_ERR_UNSUPPORTED;
  return TWL_OK;
}

}  // namespace twl

using namespace twl;

extern "C" {

size_t twl_workspace_bytes(int32_t op, int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                           int32_t max_pages, int32_t max_budget, int32_t rows,
                           int32_t row_stride) {
  (void)rows;
  if (batch < 0 || num_q_heads < 0 || num_kv_heads < 0 || max_pages < 0 || max_budget < 0 ||
      row_stride < 0)
    return 0;
  Carve c{nullptr};
  switch (op) {
    case TWL_OP_CACHE:
    case TWL_OP_PRUNE:
    case TWL_OP_UNION:
      break;
    case TWL_OP_SELECT:
      carve_select(c, batch, num_q_heads, max_pages);
      break;
    case TWL_OP_ESTIMATE:
      carve_estimate(c, batch, num_q_heads, num_kv_heads, max_pages);
      break;
    case TWL_OP_SELECT_CLUSTERS:
      carve_clusters(c, batch, num_q_heads, max_pages);
      break;
    case TWL_OP_SPARSE_DECODE:
      if (num_kv_heads < 1) return 0;
      c.take<char>(attend_partial_bytes(batch, num_q_heads, num_kv_heads, row_stride));
      break;
    case TWL_OP_DECODE_STEP:
      if (num_kv_heads < 1 || num_q_heads < num_kv_heads || max_pages < 1 || max_budget < 1)
        return 0;
      c.take<char>(decode_step_ws_bytes(batch, num_q_heads, num_kv_heads, max_pages,
                                         max_budget));
      break;
    default:
      return 0;
  }
  return c.off;
}

twl_status twl_workspace_init(void* ws, size_t ws_bytes, twl_stream_t stream) {
  if (!ws || ws_bytes < (size_t)kHeaderBytes || !aligned(ws, kAlign)) return TWL_ERR_WORKSPACE;
  return cuda_status(cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream));
}

twl_status twl_device_status(void* ws, uint32_t* flags, int32_t clear, twl_stream_t stream) {
  if (!ws || !aligned(ws, kAlign)) return TWL_ERR_WORKSPACE;
  uint32_t h = 0;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemcpyAsync(&h, ws, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return TWL_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return TWL_ERR_CUDA;
  if (flags) *flags = h;
  if (clear && cudaMemsetAsync(ws, 0, sizeof(uint32_t), s) != cudaSuccess) return TWL_ERR_CUDA;
  if (h & TWL_FLAG_BAD_INDEX) return TWL_ERR_BAD_INDEX;
  if (h & TWL_FLAG_TIMEOUT) return TWL_ERR_TIMEOUT;
  return TWL_OK;
}

const char* twl_status_string(twl_status s) {
  switch (s) {
    case TWL_OK: return "ok";
    case TWL_ERR_INVALID_ARG: return "invalid argument";
    case TWL_ERR_UNSUPPORTED: return "unsupported shape or group size";
    case TWL_ERR_CUDA: return "CUDA launch or copy failed";
    case TWL_ERR_TIMEOUT: return "a bounded device wait gave up";
    case TWL_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case TWL_ERR_BAD_INDEX: return "page table, sequence length or index list out of range";
    case TWL_ERR_SCRATCH_LIMIT: return "request exceeds the built-in scratch of the no-allocation call";
    default: return "unknown status";
  }
}

twl_status twl_page_bounds(const twl_paged_kv* kv, void* bounds, void* ws, size_t ws_bytes,
                           twl_stream_t stream) {
  KV k;
  twl_status st = check_kv(kv, true, false, &k);
  if (st != TWL_OK) return st;
  if (!bounds || !aligned(bounds, 16)) return TWL_ERR_INVALID_ARG;
  if (ws && (st = check_ws(ws, ws_bytes, kHeaderBytes)) != TWL_OK) return st;
  return cuda_status(launch_page_bounds(k, static_cast<uint16_t*>(bounds), flags_of(ws),
                                        (cudaStream_t)stream));
}

twl_status twl_quantize_k(const twl_paged_kv* kv, void* k_int4, void* k_scale_zero, void* ws,
                          size_t ws_bytes, twl_stream_t stream) {
  KV k;
  twl_status st = check_kv(kv, true, false, &k);
  if (st != TWL_OK) return st;
  if (!k_int4 || !k_scale_zero || !aligned(k_int4, 16) || !aligned(k_scale_zero, 16))
    return TWL_ERR_INVALID_ARG;
  if (ws && (st = check_ws(ws, ws_bytes, kHeaderBytes)) != TWL_OK) return st;
  return cuda_status(launch_quantize_k(k, static_cast<uint8_t*>(k_int4),
                                       static_cast<uint16_t*>(k_scale_zero), flags_of(ws),
                                       (cudaStream_t)stream));
}

twl_status twl_append_token(const twl_paged_kv* kv, const twl_k_aux* aux, const void* k_new,
                            const void* v_new, int32_t advance, void* ws, size_t ws_bytes,
                            twl_stream_t stream) {
  KV k;
  twl_status st = check_kv(kv, true, true, &k);
  if (st != TWL_OK) return st;
  if (!aux || !aux->k_int4 || !aux->k_scale_zero || !aux->bounds || !aligned(aux->k_int4, 16) ||
      !aligned(aux->k_scale_zero, 16) || !aligned(aux->bounds, 16))
    return TWL_ERR_INVALID_ARG;
  if (!k_new || !v_new || !aligned(k_new, 16) || !aligned(v_new, 16)) return TWL_ERR_INVALID_ARG;
  if (ws && (st = check_ws(ws, ws_bytes, kHeaderBytes)) != TWL_OK) return st;
  // the caller's cache buffers are written through (see the declaration)
  return cuda_status(launch_append_token(
      k, const_cast<uint16_t*>(k.k), const_cast<uint16_t*>(k.v),
      static_cast<const uint16_t*>(k_new), static_cast<const uint16_t*>(v_new),
      static_cast<uint8_t*>(aux->k_int4), static_cast<uint16_t*>(aux->k_scale_zero),
      static_cast<uint16_t*>(aux->bounds), advance ? const_cast<int32_t*>(kv->seq_lens) : nullptr,
      flags_of(ws), (cudaStream_t)stream));
}

twl_status twl_page_centroids(const twl_paged_kv* kv, void* centroids, void* ws, size_t ws_bytes,
                              twl_stream_t stream) {
  KV k;
  twl_status st = check_kv(kv, true, false, &k);
  if (st != TWL_OK) return st;
  if (!centroids || !aligned(centroids, 16)) return TWL_ERR_INVALID_ARG;
  if (ws && (st = check_ws(ws, ws_bytes, kHeaderBytes)) != TWL_OK) return st;
  return cuda_status(launch_page_centroids(k, static_cast<uint16_t*>(centroids), flags_of(ws),
                                           (cudaStream_t)stream));
}

twl_status twl_select_clusters_top_p(const void* q, int32_t num_q_heads, const twl_paged_kv* kv,
                                     const void* centroids, float p_cluster, float eps,
                                     int32_t* sel_pages, int32_t* sel_count,
                                     float* cluster_weights, void* ws, size_t ws_bytes,
                                     twl_stream_t stream) {
  KV k;
  twl_status st = check_kv(kv, false, false, &k);
  if (st != TWL_OK) return st;
  if ((st = check_heads(num_q_heads, k.hkv)) != TWL_OK) return st;
  if (!q || !centroids || !sel_pages || !sel_count || !aligned(q, 16) || !aligned(centroids, 16))
    return TWL_ERR_INVALID_ARG;
  if (cluster_weights && !aligned(cluster_weights, 4)) return TWL_ERR_INVALID_ARG;
  if (!(p_cluster > 0.f && p_cluster <= 1.f) || !(eps > 0.f) || isinf(eps))
    return TWL_ERR_INVALID_ARG;
  if ((long long)k.batch * num_q_heads > 0x7FFFFFFFll) return TWL_ERR_UNSUPPORTED;  // rows
  Carve c{static_cast<char*>(ws)};
  ClusterWs w = carve_clusters(c, k.batch, num_q_heads, k.max_pages);
  if ((st = check_ws(ws, ws_bytes, c.off)) != TWL_OK) return st;
  float* rows = cluster_weights ? cluster_weights : w.w;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = launch_cluster_weights(static_cast<const uint16_t*>(q), num_q_heads, k,
                                         static_cast<const uint16_t*>(centroids), rows,
                                         w.row_len, flags_of(ws), s);
  if (e == cudaSuccess)
    e = launch_prune(rows, w.row_len, nullptr, k.batch * num_q_heads, k.max_pages, p_cluster, eps,
                     w.m, sel_count, sel_pages, s);
  return cuda_status(e);
}

twl_status twl_select_pages(const void* q, int32_t num_q_heads, const twl_paged_kv* kv,
                            const void* bounds, int32_t budget_pages, int32_t budget_div,
                            int32_t max_budget, int32_t* sel_pages, int32_t* sel_count,
                            float* scores, void* ws, size_t ws_bytes, twl_stream_t stream) {
  KV k;
  twl_status st = check_kv(kv, false, false, &k);
  if (st != TWL_OK) return st;
  if ((st = check_heads(num_q_heads, k.hkv)) != TWL_OK) return st;
  if (!q || !bounds || !sel_pages || !sel_count || !aligned(q, 16) || !aligned(bounds, 16))
    return TWL_ERR_INVALID_ARG;
  if ((st = check_budget(budget_pages, budget_div, max_budget, k.max_pages)) != TWL_OK) return st;
  Carve c{static_cast<char*>(ws)};
  SelectWs w = carve_select(c, k.batch, num_q_heads, k.max_pages);
  if ((st = check_ws(ws, ws_bytes, c.off)) != TWL_OK) return st;
  float* sc = scores ? scores : w.scores;
  cudaStream_t s = (cudaStream_t)stream;
  uint32_t* fl = flags_of(ws);
  cudaError_t e = launch_page_scores(static_cast<const uint16_t*>(q), num_q_heads, k,
                                     static_cast<const uint16_t*>(bounds), sc, fl, s);
  if (e == cudaSuccess)
    e = launch_topk_pages(sc, num_q_heads, k, budget_pages, budget_div, max_budget, sel_pages,
                          sel_count, fl, s);
  return cuda_status(e);
}

static twl_status estimate_impl(const void* q, int32_t num_q_heads, const twl_paged_kv* kv,
                                int bits, const void* k_int4, const void* k_scale_zero,
                                const int32_t* sel_pages, const int32_t* sel_count,
                                int32_t max_budget, float* weights, int32_t* cand_tok,
                                int32_t* cand_count, void* ws, size_t ws_bytes,
                                twl_stream_t stream) {
  KV k;
  twl_status st = check_kv(kv, false, false, &k);
  if (st != TWL_OK) return st;
  if ((st = check_heads(num_q_heads, k.hkv)) != TWL_OK) return st;
  if (!q || !k_int4 || !k_scale_zero || !sel_pages || !sel_count || !weights || !cand_tok ||
      !cand_count || !aligned(q, 16) || !aligned(k_int4, 16) || !aligned(k_scale_zero, 16))
    return TWL_ERR_INVALID_ARG;
  if (max_budget < 1 || max_budget > k.max_pages) return TWL_ERR_INVALID_ARG;
  Carve c{static_cast<char*>(ws)};
  EstimateWs w = carve_estimate(c, k.batch, num_q_heads, k.hkv, k.max_pages);
  if ((st = check_ws(ws, ws_bytes, c.off)) != TWL_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  uint32_t* fl = flags_of(ws);
  cudaError_t e = launch_union_pages(num_q_heads, k, sel_pages, sel_count, max_budget, w.rank,
                                     w.union_pages, w.union_mask, w.union_npages, fl, s);
  if (e == cudaSuccess)
    e = launch_estimate_logits(static_cast<const uint16_t*>(q), num_q_heads, k, bits,
                               static_cast<const uint8_t*>(k_int4),
                               static_cast<const uint16_t*>(k_scale_zero), w.rank, w.union_pages,
                               w.union_mask, w.union_npages, kPage * max_budget, weights,
                               cand_tok, fl, s);
  if (e == cudaSuccess)
    e = launch_softmax_rows(num_q_heads, k, sel_pages, sel_count, max_budget, weights,
                            cand_count, s);
  return cuda_status(e);
}

twl_status twl_estimate(const void* q, int32_t num_q_heads, const twl_paged_kv* kv,
                        const void* k_int4, const void* k_scale_zero, const int32_t* sel_pages,
                        const int32_t* sel_count, int32_t max_budget, float* weights,
                        int32_t* cand_tok, int32_t* cand_count, void* ws, size_t ws_bytes,
                        twl_stream_t stream) {
  return estimate_impl(q, num_q_heads, kv, 4, k_int4, k_scale_zero, sel_pages, sel_count,
                       max_budget, weights, cand_tok, cand_count, ws, ws_bytes, stream);
}

twl_status twl_estimate_nbit(const void* q, int32_t num_q_heads, const twl_paged_kv* kv,
                             int32_t bits, const void* k_codes, const void* k_scale_zero,
                             const int32_t* sel_pages, const int32_t* sel_count,
                             int32_t max_budget, float* weights, int32_t* cand_tok,
                             int32_t* cand_count, void* ws, size_t ws_bytes,
                             twl_stream_t stream) {
  if (bits != 2 && bits != 4 && bits != 8) return TWL_ERR_UNSUPPORTED;
  return estimate_impl(q, num_q_heads, kv, bits, k_codes, k_scale_zero, sel_pages, sel_count,
                       max_budget, weights, cand_tok, cand_count, ws, ws_bytes, stream);
}

twl_status twl_quantize_k_nbit(const twl_paged_kv* kv, int32_t bits, void* k_codes,
                               void* k_scale_zero, void* ws, size_t ws_bytes,
                               twl_stream_t stream) {
  if (bits != 2 && bits != 4 && bits != 8) return TWL_ERR_UNSUPPORTED;
  KV k;
  twl_status st = check_kv(kv, true, false, &k);
  if (st != TWL_OK) return st;
  if (!k_codes || !k_scale_zero || !aligned(k_codes, 16) || !aligned(k_scale_zero, 16))
    return TWL_ERR_INVALID_ARG;
  if (ws && (st = check_ws(ws, ws_bytes, kHeaderBytes)) != TWL_OK) return st;
  return cuda_status(launch_quantize_k_bits(k, bits, static_cast<uint8_t*>(k_codes),
                                            static_cast<uint16_t*>(k_scale_zero), flags_of(ws),
                                            (cudaStream_t)stream));
}

twl_status twl_prune_top_p(const float* w, const int32_t* row_len, int32_t rows,
                           int32_t row_stride, float p, float eps, float* m_out,
                           int32_t* kept_count, int32_t* kept_idx, void* ws, size_t ws_bytes,
                           twl_stream_t stream) {
  (void)ws;
  (void)ws_bytes;
  if (!w || !m_out || !kept_count || rows < 0 || row_stride < 1) return TWL_ERR_INVALID_ARG;
  if (!(p > 0.f && p <= 1.f) || !(eps > 0.f) || isinf(eps)) return TWL_ERR_INVALID_ARG;
  if (!aligned(w, 4)) return TWL_ERR_INVALID_ARG;
  if (rows == 0) return TWL_OK;
  return cuda_status(launch_prune(w, row_len, nullptr, rows, row_stride, p, eps, m_out,
                                  kept_count, kept_idx, (cudaStream_t)stream));
}

twl_status twl_group_union(int32_t num_q_heads, const twl_paged_kv* kv, const int32_t* cand_tok,
                           const int32_t* kept_idx, const int32_t* kept_count,
                           int32_t cand_stride, int32_t* union_tok, int32_t* union_count,
                           void* ws, size_t ws_bytes, twl_stream_t stream) {
  KV k;
  twl_status st = check_kv(kv, false, false, &k);
  if (st != TWL_OK) return st;
  if ((st = check_heads(num_q_heads, k.hkv)) != TWL_OK) return st;
  if (!cand_tok || !kept_idx || !kept_count || !union_tok || !union_count || cand_stride < 1)
    return TWL_ERR_INVALID_ARG;
  if (ws && (st = check_ws(ws, ws_bytes, kHeaderBytes)) != TWL_OK) return st;
  return cuda_status(launch_group_union(num_q_heads, k, cand_tok, kept_idx, kept_count, nullptr,
                                        cand_stride, union_tok, union_count, flags_of(ws),
                                        (cudaStream_t)stream));
}

twl_status twl_sparse_decode(const void* q, int32_t num_q_heads, const twl_paged_kv* kv,
                             const int32_t* tok, const int32_t* tok_count, int32_t tok_stride,
                             float sm_scale, float* o, float* lse, void* ws, size_t ws_bytes,
                             twl_stream_t stream) {
  KV k;
  twl_status st = check_sparse_decode_args(q, num_q_heads, kv, tok, tok_count, tok_stride,
                                           sm_scale, o, lse, &k);
  if (st != TWL_OK) return st;
  Carve c{static_cast<char*>(ws)};
  void* partials = c.take<char>(attend_partial_bytes(k.batch, num_q_heads, k.hkv, tok_stride));
  if ((st = check_ws(ws, ws_bytes, c.off)) != TWL_OK) return st;
  return cuda_status(launch_sparse_decode(static_cast<const uint16_t*>(q), num_q_heads, k, tok,
                                          tok_count, tok_stride, sm_scale, o, lse, partials,
                                          flags_of(ws), (cudaStream_t)stream));
}

twl_status twl_decode_step(const void* q, int32_t num_q_heads, const twl_paged_kv* kv,
                           const twl_k_aux* aux, int32_t budget_pages, int32_t budget_div,
                           int32_t max_budget, float p, float eps, float* o, float* lse,
                           const twl_step_stats* stats, void* ws, size_t ws_bytes,
                           twl_stream_t stream) {
  KV k;
  twl_status st = check_kv(kv, true, true, &k);
  if (st != TWL_OK) return st;
  if ((st = check_heads(num_q_heads, k.hkv)) != TWL_OK) return st;
  if (!q || !aux || !aux->k_int4 || !aux->k_scale_zero || !aux->bounds || !o || !lse ||
      !aligned(q, 16) || !aligned(o, 16) || !aligned(aux->k_int4, 16) ||
      !aligned(aux->k_scale_zero, 16) || !aligned(aux->bounds, 16))
    return TWL_ERR_INVALID_ARG;
  if (!(p > 0.f && p <= 1.f) || !(eps > 0.f) || isinf(eps)) return TWL_ERR_INVALID_ARG;
  if ((st = check_budget(budget_pages, budget_div, max_budget, k.max_pages)) != TWL_OK) return st;
  const bool wide = step_wide(k.batch * k.hkv, num_sms());
  const step::Plan pl =
      wide ? step256::plan(k.batch, num_q_heads, k.hkv, k.max_pages, max_budget)
           : step::plan(k.batch, num_q_heads, k.hkv, k.max_pages, max_budget);
  if (!pl.ok) return TWL_ERR_UNSUPPORTED;
  Carve c{static_cast<char*>(ws)};
  char* sws = c.take<char>(decode_step_ws_bytes(k.batch, num_q_heads, k.hkv, k.max_pages,
                                                max_budget));
  if ((st = check_ws(ws, ws_bytes, c.off)) != TWL_OK) return st;
  const twl_step_stats none = {};
  const twl_step_stats& so = stats ? *stats : none;
  step::Args a = {};
  a.q = static_cast<const uint16_t*>(q);
  a.hq = num_q_heads;
  a.kv = k;
  a.k_int4 = static_cast<const uint8_t*>(aux->k_int4);
  a.k_sz = static_cast<const uint16_t*>(aux->k_scale_zero);
  a.bounds = static_cast<const uint16_t*>(aux->bounds);
  a.budget_pages = budget_pages;
  a.budget_div = budget_div;
  a.max_budget = max_budget;
  a.p = p;
  a.eps = eps;
  a.sm_scale = 0.08838834764831845f;
  a.o = o;
  a.lse = lse;
  a.sel_pages = so.sel_pages;
  a.sel_count = so.sel_count;
  a.weights_out = so.weights;
  a.cand_tok = so.cand_tok;
  a.cand_count = so.cand_count;
  a.threshold = so.threshold;
  a.kept_count = so.kept_count;
  a.union_tok = so.union_tok;
  a.union_count = so.union_count;
  a.flags = flags_of(ws);
  if (wide) {
    step256::carve(a, sws, pl, k.batch, num_q_heads, k.hkv, k.max_pages);
    return cuda_status(step256::launch(a, pl, (cudaStream_t)stream));
  }
  step::carve(a, sws, pl, k.batch, num_q_heads, k.hkv, k.max_pages);
  return cuda_status(step::launch(a, pl, (cudaStream_t)stream));
}

void twl_test_set_waits(uint32_t max_polls, int32_t stall_estimate) {
  step::set_test_waits(max_polls, stall_estimate);
  step256::set_test_waits(max_polls, stall_estimate);
}

}  // extern "C"
