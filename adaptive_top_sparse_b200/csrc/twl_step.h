// The decode step as one persistent grid over every SM (twl_step.cu): arguments, work list, launch.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "twl_kernels.h"

namespace twl {
namespace step {

// Work-item kinds, in dependency order: an item only waits on items of earlier kinds of its own
// (sequence, kv-head) group.
enum Phase : int {
  kScore = 0,   // page scores of a chunk of the group's pages (all G heads)
  kTopK = 1,    // top-k pages of one q-head
  kEst = 2,     // INT4 estimate over the union pages in a range of the group's logical pages
  kPrune = 3,   // softmax + top-p threshold of one q-head; the last builds the kept-page list
  kAttend = 4,  // a worker of the attention queue: takes chunks of kept pages from every group
};

// A run of consecutive item indices: groups [g0, g1), `per` items per group, group-major.
struct Segment {
  int phase, g0, g1, per, first;
};
constexpr int kMaxSegments = 40;

// Synchronisation words (uint32, in the workspace): globals, then per group one counter per
// dependency.  All are zero between launches: the last CTA of a launch clears them.
//   kNext    next work item           kExit    CTAs that left        kAbort   a wait gave up
//   kQAlloc  attention chunks published (allocated)    kQNext  chunks taken by workers
//   kQGroups groups whose chunks are published
enum { kNext = 0, kExit = 1, kAbort = 2, kQAlloc = 3, kQNext = 4, kQGroups = 5, kSyncHead = 8 };
// Kept tokens per attention chunk of the flattened work list: chunks are cut at page bounds, to
// at least kAttChunkTok and at most kAttChunkMax tokens (+15 at a page edge).
constexpr int kAttChunkTok = 128;
constexpr int kAttChunkMax = 1024;
enum { kCntScore = 0, kCntTopK, kCntEst, kCntPrune, kCntAttend, kCounters };

struct Args {
  // inputs
  const uint16_t* q;
  int hq, g;
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
  int* union_tok;
  int* union_count;
  // workspace
  uint32_t* flags;     // header word 0 (sticky device flags)
  uint32_t* sync;      // synchronisation words
  uint32_t* keys;      // [B*Hq][max_pages]   order keys of the page scores
  uint32_t* selbits;   // [B*Hq][sel_words]   selected-page bitmaps
  int* ncand;          // [B*Hq]              candidate rows of each head
  int* hpre;           // [B*Hq][sel_words]   exclusive prefix counts of the selected-page bitmaps
  float* logits;       // [B*Hq][cand_stride] estimated logits, then weights
  uint32_t* pmask;     // [groups][pm_words]  kept rows of two logical pages per word (OR over
                       //                     the group's heads); zero between launches
  int4* kpages;        // [groups][max_pages] kept pages, ascending: (K/V row index of row 0, row
                       //                     mask, logical page, kept tokens before the page)
  int* qtab;           // [q_cap][4] attention chunks: (group, first kept page, end page, -)
  uint32_t* qvalid;    // [q_cap] 1 once the chunk is published
  int* cbase;          // [groups][2] first chunk and chunk count of each group
  float* part;         // [q_cap][G][2 + 128] attention partials per chunk (max, sum, o)
  unsigned long long* trace;  // trace builds only (-DTWL_STEP_TRACE): 17 words per item
  // strides and the work list
  int groups, sel_words, cand_stride, kept_words, pm_words;
  int s_per, s_chunk, e_per, e_chunk, q_cap;
  int att_chunks;  // chunks a group's kept tokens are cut into, before the size limits
  uint32_t spin_limit;  // polls before a wait between items gives up (TWL_FLAG_TIMEOUT)
  int stall_estimate;   // test of the timeout path: the estimate items wait for a count never reached
  int n_items;
  int smem_bytes;  // dynamic shared memory of each CTA
  int nseg;
  Segment seg[kMaxSegments];
};

struct Plan {
  int grid;        // CTAs (all resident at once)
  int smem_bytes;  // dynamic shared memory per CTA
  int s_per, s_chunk, e_per, e_chunk, q_cap, att_chunks;
  int sel_words, cand_stride, kept_words;
  bool ok;
};

Plan plan(int batch, int hq, int hkv, int max_pages, int max_budget);
size_t workspace_bytes(int batch, int hq, int hkv, int max_pages, int max_budget);
// Points the workspace arrays of `a` into `ws` (which starts after the 256-byte header) and fills
// the strides and the work list from the plan.
void carve(Args& a, char* ws, const Plan& pl, int batch, int hq, int hkv, int max_pages);
cudaError_t launch(const Args& a, const Plan& pl, cudaStream_t s);
// Test knobs for the bounded waits (twl_test_set_waits): the polls before a wait gives up (0 =
// the default) and whether the estimate items wait for a count that is never reached.
void set_test_waits(uint32_t spin_limit, int stall_estimate);

}  // namespace step

// The same kernel built with 256-thread CTAs, two per SM (twl_step_256.cu), for batches with
// more (sequence, kv-head) groups than SMs.  Same arguments and workspace contents.
namespace step256 {
step::Plan plan(int batch, int hq, int hkv, int max_pages, int max_budget);
size_t workspace_bytes(int batch, int hq, int hkv, int max_pages, int max_budget);
void carve(step::Args& a, char* ws, const step::Plan& pl, int batch, int hq, int hkv,
           int max_pages);
cudaError_t launch(const step::Args& a, const step::Plan& pl, cudaStream_t s);
void set_test_waits(uint32_t spin_limit, int stall_estimate);
}  // namespace step256

// Whether the decode step of `groups` (sequence, kv-head) groups runs the 256-thread build
// (measured: 306 vs 424 us per layer-step at 512 groups; no gain at 128 groups on 148 SMs).
inline bool step_wide(int groups, int sms) { return groups > sms; }
}  // namespace twl
