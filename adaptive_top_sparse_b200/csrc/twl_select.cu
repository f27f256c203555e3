// Page selection: Quest-style bounding-box scores and the top-k page budget.
//
// "Twilight: Adaptive Attention Sparsity with Hierarchical Top-p Pruning", notes page, "Overall
// framework": a base selector keeps a conservative budget (e.g. 1/4 of the pages) before top-p
// pruning; summary, sections 4.1 and 4.3 (B0 = N/4).  The score of page j for query q is the
// upper bound of q.k over the page's channel-wise [min, max] box:
//   score_j = sum_c t_c,  t_c = q_c * max_c if q_c > 0 else q_c * min_c.
// Each t_c is a product of two fp16 numbers and therefore exact in fp32.  The sum is taken in one
// fixed order so a score is bit-reproducible: lane l of a half-warp accumulates channels
// 8l .. 8l+7 from +0 with fused multiply-adds (one rounding per term, as an add of the exact
// term), then the 16 partials combine by xor butterflies over offsets 8, 4, 2, 1.
#include "twl_common.cuh"
#include "twl_kernels.h"

namespace twl {
namespace {

constexpr int kScoreThreads = 256;
constexpr int kScoreIters = 4;                                      // page pairs per warp
constexpr int kScorePagesPerBlock = (kScoreThreads / 32) * 2 * kScoreIters;  // 64

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// grid (page tiles of 64, Hkv, B).  A half-warp scores one page for all G heads of the group.
template <int G>
__global__ void __launch_bounds__(kScoreThreads)
    k_page_scores(const uint16_t* __restrict__ q, int hq, KV kv,
                  const uint16_t* __restrict__ bounds, float* __restrict__ scores,
                  uint32_t* flags) {
  const int b = blockIdx.z, kvh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int half = lane >> 4, l = lane & 15;
  Seq sq = load_seq(kv.seq_lens, b, kv.max_pages, flags,
                    blockIdx.x == 0 && kvh == 0 && threadIdx.x == 0);
  const int tile0 = blockIdx.x * kScorePagesPerBlock;
  if (tile0 >= sq.pages) return;

  float qv[G][8];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const uint4 raw = *reinterpret_cast<const uint4*>(
        q + ((size_t)b * hq + kvh * G + h) * kHeadDim + 8 * l);
    unpack8(raw, qv[h]);
  }

  // Issue all bound loads of this warp first (memory-level parallelism), then compute.
  uint4 bmn[kScoreIters], bmx[kScoreIters];
  int pg[kScoreIters];
  bool ok[kScoreIters];
#pragma unroll
  for (int it = 0; it < kScoreIters; ++it) {
    const int j = tile0 + it * (kScoreThreads / 32) * 2 + 2 * warp + half;
    pg[it] = j;
    ok[it] = false;
    bmn[it] = make_uint4(0, 0, 0, 0);
    bmx[it] = bmn[it];
    if (j < sq.pages) {
      const int ph = load_phys(kv.page_table, b, j, kv.max_pages, kv.num_phys, flags);
      if (ph >= 0) {
        const uint16_t* base = bounds + (((size_t)ph * kv.hkv + kvh) * 2) * kHeadDim + 8 * l;
        bmn[it] = __ldg(reinterpret_cast<const uint4*>(base));
        bmx[it] = __ldg(reinterpret_cast<const uint4*>(base + kHeadDim));
        ok[it] = true;
      }
    }
  }
#pragma unroll
  for (int it = 0; it < kScoreIters; ++it) {
    float mn[8], mx[8];
    unpack8(bmn[it], mn);
    unpack8(bmx[it], mx);
    float acc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float a = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) a = __fmaf_rn(qv[h][c], qv[h][c] > 0.f ? mx[c] : mn[c], a);
      acc[h] = a;
    }
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) {
#pragma unroll
      for (int h = 0; h < G; ++h) acc[h] = __fadd_rn(acc[h], __shfl_xor_sync(0xffffffffu, acc[h], off));
    }
    const int j = pg[it];
    if (j < sq.pages && l < G) {
      float v = acc[0];
#pragma unroll
      for (int h = 1; h < G; ++h) v = (l == h) ? acc[h] : v;
      if (!ok[it]) v = -INFINITY;
      scores[((size_t)b * hq + kvh * G + l) * kv.max_pages + j] = v;
    }
  }
}

// ---------------------------------------------------------------------------- top-k pages
constexpr int kTopkThreads = 512;

// Radix select of the k largest keys among keys[0..n) (uint32, larger = better), ties to the
// lower index.  Writes the selected indices ascending to out[]; returns the count (k).
__device__ void block_select_topk(const uint32_t* keys, int n, int k, int* out, uint32_t* hist,
                                  int* scan_sh, uint32_t* sh_state) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t prefix = 0, mask = 0;
  int remaining = k;
  const int n_iter = (n + blockDim.x - 1) / blockDim.x;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int it = 0; it < n_iter; ++it) {
      const int i = it * blockDim.x + tid;
      bool take = false;
      uint32_t digit = 0;
      if (i < n) {
        const uint32_t key = keys[i];
        take = (key & mask) == prefix;
        digit = (key >> shift) & 0xFFu;
      }
      // warp-aggregated histogram update: one atomic per distinct digit in the warp
      const uint32_t tag = take ? digit : 256u + lane;
      const uint32_t peers = __match_any_sync(0xffffffffu, tag);
      if (take && (__ffs(peers) - 1) == lane) atomicAdd(&hist[digit], (uint32_t)__popc(peers));
    }
    __syncthreads();
    if (warp == 0) {
      // lane i covers digits 255-8i .. 248-8i, scanned from the top
      uint32_t c[8];
      uint32_t tot = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        c[e] = hist[255 - 8 * lane - e];
        tot += c[e];
      }
      uint32_t incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const uint32_t excl = incl - tot;
      const bool hit = excl < (uint32_t)remaining && incl >= (uint32_t)remaining;
      if (hit) {
        uint32_t run = excl;
        for (int e = 0; e < 8; ++e) {
          if (run + c[e] >= (uint32_t)remaining) {
            sh_state[0] = prefix | ((uint32_t)(255 - 8 * lane - e) << shift);
            sh_state[1] = (uint32_t)remaining - run;
            break;
          }
          run += c[e];
        }
      }
    }
    __syncthreads();
    prefix = sh_state[0];
    remaining = (int)sh_state[1];
    mask |= 0xFFu << shift;
    __syncthreads();
  }
  // prefix = the k-th largest key; take all keys above it and the first `remaining` equal ones.
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int beg = min(n, tid * per), end = min(n, beg + per);
  int n_eq = 0;
  for (int i = beg; i < end; ++i) n_eq += keys[i] == prefix;
  int eq_before = block_exclusive_scan(n_eq, scan_sh, nullptr);
  int n_sel = 0;
  {
    int e = eq_before;
    for (int i = beg; i < end; ++i) {
      const uint32_t key = keys[i];
      if (key > prefix) ++n_sel;
      else if (key == prefix) { n_sel += e < remaining; ++e; }
    }
  }
  int pos = block_exclusive_scan(n_sel, scan_sh, nullptr);
  {
    int e = eq_before;
    for (int i = beg; i < end; ++i) {
      const uint32_t key = keys[i];
      bool s = false;
      if (key > prefix) s = true;
      else if (key == prefix) { s = e < remaining; ++e; }
      if (s) out[pos++] = i;
    }
  }
}

// One block per (b, q-head).  Dynamic shared memory: max_pages keys.
__global__ void __launch_bounds__(kTopkThreads)
    k_topk_pages(const float* __restrict__ scores, int hq, KV kv, int budget_pages,
                 int budget_div, int max_budget, int* __restrict__ sel_pages,
                 int* __restrict__ sel_count, uint32_t* flags) {
  extern __shared__ uint32_t keys[];
  __shared__ uint32_t hist[256];
  __shared__ int scan_sh[33];
  __shared__ uint32_t state[2];
  const int bh = blockIdx.x, b = bh / hq;
  Seq sq = load_seq(kv.seq_lens, b, kv.max_pages, flags, false);
  const int n = sq.pages;
  int kb = budget_pages > 0 ? budget_pages : (n + budget_div - 1) / budget_div;
  kb = min(min(kb, n), max_budget);
  int* out = sel_pages + (size_t)bh * max_budget;
  if (n <= kb) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) out[i] = i;
    if (threadIdx.x == 0) sel_count[bh] = n;
    return;
  }
  const float* row = scores + (size_t)bh * kv.max_pages;
  for (int i = threadIdx.x; i < n; i += blockDim.x) keys[i] = f32_key(row[i]);
  __syncthreads();
  block_select_topk(keys, n, kb, out, hist, scan_sh, state);
  if (threadIdx.x == 0) sel_count[bh] = kb;
}

// Cluster-level weights (size-weighted centroids): one block per (b, q-head).  A warp scores a
// page at a time: logit_j = ln(n_j) + (q . c_j) / sqrt(128), n_j the page's valid rows; then the
// row is normalised in place (softmax over the sequence's pages) and its length recorded.
__global__ void __launch_bounds__(512) k_cluster_weights(const uint16_t* __restrict__ q, int hq,
                                                         KV kv, const uint16_t* __restrict__ cen,
                                                         float* __restrict__ w,
                                                         int* __restrict__ row_len,
                                                         uint32_t* flags) {
  __shared__ float red[33];
  const int bh = blockIdx.x, b = bh / hq, h = bh % hq;
  const int kvh = h / (hq / kv.hkv);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  Seq sq = load_seq(kv.seq_lens, b, kv.max_pages, flags, h == 0 && threadIdx.x == 0);
  const int np = sq.pages;
  float* row = w + (size_t)bh * kv.max_pages;
  float qv[4];
  {
    const uint2 raw = *reinterpret_cast<const uint2*>(q + (size_t)bh * kHeadDim + lane * 4);
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
    const float2 c = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
    qv[0] = a.x; qv[1] = a.y; qv[2] = c.x; qv[3] = c.y;
  }
  const float inv_sqrt_d = 0.08838834764831845f;
  float mx = -INFINITY;
  for (int j = warp; j < np; j += nwarps) {
    const int ph = load_phys(kv.page_table, b, j, kv.max_pages, kv.num_phys, flags);
    float dot = 0.f;
    if (ph >= 0) {
      const uint2 raw =
          *reinterpret_cast<const uint2*>(cen + ((size_t)ph * kv.hkv + kvh) * kHeadDim + lane * 4);
      const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
      const float2 c = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
      dot = qv[0] * a.x + qv[1] * a.y + qv[2] * c.x + qv[3] * c.y;
    }
    dot = warp_sum(dot);
    const float l = ph >= 0 ? logf((float)page_rows(sq.n, j)) + dot * inv_sqrt_d : -INFINITY;
    if (lane == 0) row[j] = l;
    mx = fmaxf(mx, l);
  }
  mx = block_max(mx, red);  // every warp's lane 0 wrote its pages before the barriers inside
  float sum = 0.f;
  for (int j = threadIdx.x; j < np; j += blockDim.x) {
    const float e = mx > -INFINITY ? __expf(row[j] - mx) : 0.f;
    row[j] = e;
    sum += e;
  }
  sum = block_sum(sum, red);
  const float inv = sum > 0.f ? 1.f / sum : 0.f;
  for (int j = threadIdx.x; j < np; j += blockDim.x) row[j] *= inv;
  if (threadIdx.x == 0) row_len[bh] = np;
}

}  // namespace

cudaError_t launch_cluster_weights(const uint16_t* q, int hq, const KV& kv, const uint16_t* cen,
                                   float* w, int* row_len, uint32_t* flags, cudaStream_t s) {
  k_cluster_weights<<<kv.batch * hq, 512, 0, s>>>(q, hq, kv, cen, w, row_len, flags);
  return cudaGetLastError();
}

cudaError_t launch_page_scores(const uint16_t* q, int hq, const KV& kv, const uint16_t* bounds,
                               float* scores, uint32_t* flags, cudaStream_t s) {
  const int g = hq / kv.hkv;
  dim3 grid((kv.max_pages + kScorePagesPerBlock - 1) / kScorePagesPerBlock, kv.hkv, kv.batch);
  switch (g) {
    case 1: k_page_scores<1><<<grid, kScoreThreads, 0, s>>>(q, hq, kv, bounds, scores, flags); break;
    case 2: k_page_scores<2><<<grid, kScoreThreads, 0, s>>>(q, hq, kv, bounds, scores, flags); break;
    case 4: k_page_scores<4><<<grid, kScoreThreads, 0, s>>>(q, hq, kv, bounds, scores, flags); break;
    case 8: k_page_scores<8><<<grid, kScoreThreads, 0, s>>>(q, hq, kv, bounds, scores, flags); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_topk_pages(const float* scores, int hq, const KV& kv, int budget_pages,
                              int budget_div, int max_budget, int* sel_pages, int* sel_count,
                              uint32_t* flags, cudaStream_t s) {
  const size_t smem = (size_t)kv.max_pages * sizeof(uint32_t);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k_topk_pages, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  k_topk_pages<<<kv.batch * hq, kTopkThreads, smem, s>>>(scores, hq, kv, budget_pages, budget_div,
                                                         max_budget, sel_pages, sel_count, flags);
  return cudaGetLastError();
}

}  // namespace twl
