// The fused decode-step kernel (twl_fused.cu): arguments, launch plan, workspace carving.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "twl_kernels.h"

namespace twl {

struct FusedArgs {
  // inputs
  const uint16_t* q;
  int hq;
  KV kv;
  const uint8_t* k_int4;
  const uint16_t* k_sz;
  const uint16_t* bounds;
  int budget_pages, budget_div, max_budget;
  float p, eps, sm_scale;
  // outputs
  float* o;
  float* lse;
  // optional outputs (NULL = not written)
  int* sel_pages;
  int* sel_count;
  float* weights_out;
  int* cand_tok;
  int* cand_count;
  float* threshold;
  int* kept_count;
  int* union_count;
  int* union_tok;  // the workspace's list when the caller does not ask for it
  int want_union;  // build the group's ordered union list (the caller asked for it)
  int pt_smem;        // stage the sequence's page table in shared memory
  // workspace
  float* scores;
  uint32_t* selbits;
  float* logits;
  uint32_t* keptbits;  // [B * Hq][kept_words]: bit i = candidate row i passes top-p
  int* union_part;
  float* part_att;
  uint32_t* flags;
  // strides and launch shape
  int sel_words, cand_stride, union_stride, kept_words;
  int cluster;
  int smem_bytes;
};

struct FusedPlan {
  int cluster;
  int smem_bytes;
  int sel_words, cand_stride, union_stride;
  bool pt_smem;
  bool ok;
};

// Two builds of twl_fused.cu: 512-thread CTAs (one per SM), and 256-thread CTAs with half the
// shared memory (two per SM) for batches with more groups than SMs.
#define TWL_FUSED_DECLS                                                                     \
  FusedPlan plan_fused(int batch, int hq, int hkv, int max_pages, int max_budget);           \
  size_t fused_workspace_bytes(int batch, int hq, int hkv, int max_pages, int max_budget);   \
  void carve_fused(FusedArgs& a, char* ws, const FusedPlan& pl, int batch, int hq, int hkv, \
                   int max_pages);                                                           \
  int fit_cluster(int g, int want, int groups, int smem_bytes);                              \
  cudaError_t launch_fused(const FusedArgs& a, const FusedPlan& pl, cudaStream_t s);
namespace fused512 {
TWL_FUSED_DECLS
}
namespace fused256 {
TWL_FUSED_DECLS
}
#undef TWL_FUSED_DECLS

}  // namespace twl
