// Internal launchers of the twl kernels (host side).  Arguments are validated by twl_api.cu
// before any of these is called; each returns cudaGetLastError() of its launches.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "twl.h"

namespace twl {

struct KV {
  const uint16_t* k;
  const uint16_t* v;
  const int* page_table;
  const int* seq_lens;
  int batch, hkv, max_pages, num_phys;
};

// twl_cache.cu
cudaError_t launch_page_bounds(const KV& kv, uint16_t* bounds, uint32_t* flags, cudaStream_t s);
cudaError_t launch_append_token(const KV& kv, uint16_t* k_cache, uint16_t* v_cache,
                                const uint16_t* k_new, const uint16_t* v_new, uint8_t* k_int4,
                                uint16_t* k_sz, uint16_t* bounds, int32_t* seq_lens_out,
                                uint32_t* flags, cudaStream_t s);
cudaError_t launch_quantize_k(const KV& kv, uint8_t* k_int4, uint16_t* k_sz, uint32_t* flags,
                              cudaStream_t s);
cudaError_t launch_quantize_k_bits(const KV& kv, int bits, uint8_t* k_codes, uint16_t* k_sz,
                                   uint32_t* flags, cudaStream_t s);

cudaError_t launch_page_centroids(const KV& kv, uint16_t* centroids, uint32_t* flags,
                                  cudaStream_t s);

// twl_select.cu
cudaError_t launch_cluster_weights(const uint16_t* q, int hq, const KV& kv, const uint16_t* cen,
                                   float* w, int* row_len, uint32_t* flags, cudaStream_t s);
cudaError_t launch_page_scores(const uint16_t* q, int hq, const KV& kv, const uint16_t* bounds,
                               float* scores, uint32_t* flags, cudaStream_t s);
cudaError_t launch_topk_pages(const float* scores, int hq, const KV& kv, int budget_pages,
                              int budget_div, int max_budget, int* sel_pages, int* sel_count,
                              uint32_t* flags, cudaStream_t s);

// twl_estimate.cu
cudaError_t launch_union_pages(int hq, const KV& kv, const int* sel_pages, const int* sel_count,
                               int max_budget, int* rank, int* union_pages,
                               uint32_t* union_mask, int* union_npages, uint32_t* flags,
                               cudaStream_t s);
cudaError_t launch_estimate_logits(const uint16_t* q, int hq, const KV& kv, int bits,
                                   const uint8_t* k_codes, const uint16_t* k_sz, const int* rank,
                                   const int* union_pages, const uint32_t* union_mask,
                                   const int* union_npages, int cand_stride, float* logits,
                                   int* cand_tok, uint32_t* flags, cudaStream_t s);
cudaError_t launch_softmax_rows(int hq, const KV& kv, const int* sel_pages, const int* sel_count,
                                int max_budget, float* weights, int* cand_count,
                                cudaStream_t s);

// twl_prune_rows.cu (32 weights per thread) and twl_prune_rows64.cu (64): the read-once pruner;
// cudaErrorNotSupported (nothing launched) when the rows do not fit it
namespace rows32 {
cudaError_t launch_prune_rows(const float* w, const int* row_len, const int* row_len_cap,
                              int rows, int row_stride, float p, float eps, float* m_out,
                              int* kept_count, int* kept_idx, cudaStream_t s);
}
namespace rows64 {
cudaError_t launch_prune_rows(const float* w, const int* row_len, const int* row_len_cap,
                              int rows, int row_stride, float p, float eps, float* m_out,
                              int* kept_count, int* kept_idx, cudaStream_t s);
}

// twl_prune.cu
cudaError_t launch_prune(const float* w, const int* row_len, const int* row_len_cap, int rows,
                         int row_stride, float p, float eps, float* m_out, int* kept_count,
                         int* kept_idx, cudaStream_t s);

// twl_attend.cu
cudaError_t launch_group_union(int hq, const KV& kv, const int* cand_tok, const int* kept_idx,
                               const int* kept_count, const int* cand_count, int cand_stride,
                               int* union_tok, int* union_count, uint32_t* flags,
                               cudaStream_t s);
constexpr int kChunk = 128;  // tokens per attention work item
size_t attend_partial_bytes(int batch, int hq, int hkv, int tok_stride);
cudaError_t launch_sparse_decode(const uint16_t* q, int hq, const KV& kv, const int* tok,
                                 const int* tok_count, int tok_stride, float sm_scale, float* o,
                                 float* lse, void* partials, uint32_t* flags, cudaStream_t s);

int num_sms();

// twl_api.cu: the argument checks of twl_sparse_decode (also run by its no-allocation variant
// before it sizes the request); fills *out on success.
twl_status check_sparse_decode_args(const void* q, int num_q_heads, const twl_paged_kv* kv,
                                    const int32_t* tok, const int32_t* tok_count, int tok_stride,
                                    float sm_scale, const float* o, const float* lse, KV* out);

}  // namespace twl
