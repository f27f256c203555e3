// Group union of kept tokens, split-KV sparse attention over a flattened work list, LSE merge.
//
// "Twilight: Adaptive Attention Sparsity with Hierarchical Top-p Pruning":
//   notes page, "Overall framework": the final sparse attention runs only on the kept tokens;
//   notes page, "Key designs" (load balancing): per-head budgets differ (2% vs 50%), so the head
//   dimension is flattened and the work redistributed;
//   summary, appendix B.2: a GQA group attends over the union of its heads' kept tokens so each
//   K/V row is read once (group-wise variable-length attention).
//
// Work list: the token list of every (b, kv-head) group is cut into chunks of kChunk tokens; all
// chunks of all groups form one flat list that a persistent grid walks with a fixed stride, so a
// group with 50x more kept tokens simply owns 50x more chunks.  A chunk gathers its K and V rows
// (256 B each) into shared memory with cp.async, computes the scores of the group's heads and a
// partial (o, lse); a second kernel merges the partials by log-sum-exp.
#include "twl_common.cuh"
#include "twl_kernels.h"

namespace twl {
namespace {

constexpr int kAttThreads = kChunk;  // one thread per token for scores, per channel for P.V
constexpr int kMaxGroups = 4096;
constexpr uint32_t kBadRow = 0xFFFFFFFFu;

// ------------------------------------------------------------------ union of kept tokens
__global__ void __launch_bounds__(512)
    k_group_union(int hq, KV kv, const int* __restrict__ cand_tok,
                  const int* __restrict__ kept_idx, const int* __restrict__ kept_count,
                  const int* __restrict__ cand_count, int cand_stride, int* __restrict__ union_tok,
                  int* __restrict__ union_count, uint32_t* flags) {
  extern __shared__ uint32_t bits[];  // [ceil(16 * max_pages / 32)]
  __shared__ int scan_sh[33];
  const int gi = blockIdx.x, b = gi / kv.hkv, kvh = gi % kv.hkv;
  const int g = hq / kv.hkv;
  Seq sq = load_seq(kv.seq_lens, b, kv.max_pages, flags, false);
  const int nwords = (sq.n + 31) >> 5;
  for (int i = threadIdx.x; i < nwords; i += blockDim.x) bits[i] = 0u;
  __syncthreads();
  for (int hl = 0; hl < g; ++hl) {
    const int bh = b * hq + kvh * g + hl;
    const int cc = cand_count ? min(max(cand_count[bh], 0), cand_stride) : cand_stride;
    const int kc = min(max(kept_count[bh], 0), cc);
    const int* ki = kept_idx + (size_t)bh * cand_stride;
    const int* ct = cand_tok + (size_t)bh * cand_stride;
    for (int i = threadIdx.x; i < kc; i += blockDim.x) {
      const int c = ki[i];
      const int tok = (c >= 0 && c < cc) ? ct[c] : -1;
      if (tok < 0 || tok >= sq.n) {
        raise_flag(flags, TWL_FLAG_BAD_INDEX);
        continue;
      }
      atomicOr(&bits[tok >> 5], 1u << (tok & 31));
    }
  }
  __syncthreads();
  const int per = (nwords + blockDim.x - 1) / blockDim.x;
  const int beg = min(nwords, (int)threadIdx.x * per), end = min(nwords, beg + per);
  int cnt = 0;
  for (int i = beg; i < end; ++i) cnt += __popc(bits[i]);
  int total;
  int pos = block_exclusive_scan(cnt, scan_sh, &total);
  int* out = union_tok + (size_t)gi * kPage * kv.max_pages;
  for (int i = beg; i < end; ++i) {
    uint32_t w = bits[i];
    while (w) {
      const int bit = __ffs(w) - 1;
      out[pos++] = 32 * i + bit;
      w &= w - 1;
    }
  }
  if (threadIdx.x == 0) union_count[gi] = total;
}

// ------------------------------------------------------------------ split-KV attention
struct AttSmem {
  // K rows: chunk c (8 channels) of token t is stored at position (c + t) % 16 so that threads
  // reading the same chunk of consecutive tokens hit different banks.
  uint4 k[kChunk][16];
  uint4 v[kChunk][16];
};

__device__ __forceinline__ int find_group(const int* prefix, int ngroups, int item) {
  int lo = 0, hi = ngroups;  // prefix[lo] <= item < prefix[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= item) lo = mid;
    else hi = mid;
  }
  return lo;
}

// Items prefix over groups: prefix[gi] = sum_{g' < gi} ceil(count / kChunk).
__device__ void build_item_prefix(const int* tok_count, int tok_stride, int ngroups, int* prefix,
                                  int* scan_sh) {
  int carry = 0;
  for (int base = 0; base < ngroups; base += blockDim.x) {
    const int gi = base + threadIdx.x;
    int c = 0;
    if (gi < ngroups) {
      const int cnt = min(max(tok_count[gi], 0), tok_stride);
      c = (cnt + kChunk - 1) / kChunk;
    }
    int total;
    const int ex = block_exclusive_scan(c, scan_sh, &total);
    if (gi < ngroups) prefix[gi] = carry + ex;
    carry += total;
  }
  if (threadIdx.x == 0) prefix[ngroups] = carry;
  __syncthreads();
}

template <int G>
__global__ void __launch_bounds__(kAttThreads)
    k_sparse_attend(const uint16_t* __restrict__ q, int hq, KV kv, const int* __restrict__ tok,
                    const int* __restrict__ tok_count, int tok_stride, float sm_scale,
                    float* __restrict__ part_o, float* __restrict__ part_lse,
                    int* __restrict__ item_prefix_out, uint32_t* flags) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  AttSmem& S = *reinterpret_cast<AttSmem*>(smem_raw);
  int* prefix = reinterpret_cast<int*>(smem_raw + sizeof(AttSmem));  // [ngroups + 1]
  __shared__ float qs[G][kHeadDim];
  __shared__ float ps[G][kChunk];
  __shared__ float red[G][kAttThreads / 32];
  __shared__ uint32_t rowidx[kChunk];
  __shared__ int scan_sh[33];

  const int ngroups = kv.batch * kv.hkv;
  build_item_prefix(tok_count, tok_stride, ngroups, prefix, scan_sh);
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i <= ngroups; i += blockDim.x) item_prefix_out[i] = prefix[i];
  const int n_items = prefix[ngroups];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int gi = find_group(prefix, ngroups, item);
    const int chunk = item - prefix[gi];
    const int b = gi / kv.hkv, kvh = gi % kv.hkv;
    const int count = min(max(tok_count[gi], 0), tok_stride);
    const int t0 = chunk * kChunk;
    const int nt = min(kChunk, count - t0);
    Seq sq = load_seq(kv.seq_lens, b, kv.max_pages, flags, false);

    // queries of the group, fp32
    for (int i = tid; i < G * kHeadDim; i += blockDim.x) {
      const int h = i / kHeadDim, c = i % kHeadDim;
      qs[h][c] = __half2float(__ushort_as_half(q[((size_t)b * hq + kvh * G + h) * kHeadDim + c]));
    }
    // token -> K/V row index
    {
      uint32_t ri = kBadRow;
      if (tid < nt) {
        const int tk = tok[(size_t)gi * tok_stride + t0 + tid];
        if (tk >= 0 && tk < sq.n) {
          const int ph = load_phys(kv.page_table, b, tk >> 4, kv.max_pages, kv.num_phys, flags);
          if (ph >= 0) ri = (uint32_t)(((size_t)ph * kv.hkv + kvh) * kPage + (tk & 15));
        } else {
          raise_flag(flags, TWL_FLAG_BAD_INDEX);
        }
      }
      rowidx[tid] = ri;
    }
    __syncthreads();
    // gather: thread copies 16-byte chunk (tid & 15) of tokens (tid >> 4) + 8 * it
#pragma unroll 4
    for (int it = 0; it < kChunk / 8; ++it) {
      const int t = (tid >> 4) + 8 * it;
      const int c = tid & 15;
      const uint32_t ri = rowidx[t];
      const bool ok = ri != kBadRow;
      const size_t off = ok ? (size_t)ri * kHeadDim + 8 * c : 0;
      cp_async16(&S.k[t][(c + t) & 15], kv.k + off, ok);
      cp_async16(&S.v[t][c], kv.v + off, ok);
    }
    cp_async_commit();
    cp_async_wait_all();
    __syncthreads();

    // scores: thread = token
    float s[G];
    const bool tok_ok = tid < nt && rowidx[tid] != kBadRow;
#pragma unroll
    for (int h = 0; h < G; ++h) s[h] = 0.f;
    if (tok_ok) {
#pragma unroll 4
      for (int c = 0; c < 16; ++c) {
        const uint4 raw = S.k[tid][(c + tid) & 15];
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
        float kf[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
          kf[2 * i] = f.x;
          kf[2 * i + 1] = f.y;
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float4 qa = *reinterpret_cast<const float4*>(&qs[h][8 * c]);
          const float4 qb = *reinterpret_cast<const float4*>(&qs[h][8 * c + 4]);
          s[h] += qa.x * kf[0] + qa.y * kf[1] + qa.z * kf[2] + qa.w * kf[3] + qb.x * kf[4] +
                  qb.y * kf[5] + qb.z * kf[6] + qb.w * kf[7];
        }
      }
    }
#pragma unroll
    for (int h = 0; h < G; ++h) s[h] = tok_ok ? s[h] * sm_scale : -INFINITY;
    // block max and sum per head
    float mh[G], lh[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float m = warp_max(s[h]);
      if (lane == 0) red[h][warp] = m;
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float m = red[h][0];
#pragma unroll
      for (int w = 1; w < kAttThreads / 32; ++w) m = fmaxf(m, red[h][w]);
      mh[h] = m;
      const float pv = (tok_ok && m > -INFINITY) ? __expf(s[h] - m) : 0.f;
      ps[h][tid] = pv;
      s[h] = pv;
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float l = warp_sum(s[h]);
      if (lane == 0) red[h][warp] = l;
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float l = 0.f;
#pragma unroll
      for (int w = 0; w < kAttThreads / 32; ++w) l += red[h][w];
      lh[h] = l;
    }
    // P.V: thread = channel
    float o[G];
#pragma unroll
    for (int h = 0; h < G; ++h) o[h] = 0.f;
    const __half* vrow = reinterpret_cast<const __half*>(&S.v[0][0]);
    for (int t = 0; t < nt; ++t) {
      const float vv = __half2float(vrow[t * kHeadDim + tid]);
#pragma unroll
      for (int h = 0; h < G; ++h) o[h] = fmaf(ps[h][t], vv, o[h]);
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const bool any = lh[h] > 0.f;
      part_o[((size_t)item * G + h) * kHeadDim + tid] = any ? o[h] / lh[h] : 0.f;
      if (tid == 0) part_lse[(size_t)item * G + h] = any ? mh[h] + __logf(lh[h]) : -INFINITY;
    }
    __syncthreads();
  }
}

// One warp per (b, q-head): log-sum-exp merge of the group's chunk partials.
template <int G>
__global__ void __launch_bounds__(256)
    k_merge_partials(int hq, int hkv, int batch, const float* __restrict__ part_o,
                     const float* __restrict__ part_lse, const int* __restrict__ item_prefix,
                     float* __restrict__ o, float* __restrict__ lse) {
  const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (wid >= batch * hq) return;
  const int b = wid / hq, h = wid % hq, kvh = h / G, hl = h % G;
  const int gi = b * hkv + kvh;
  const int i0 = item_prefix[gi], i1 = item_prefix[gi + 1];
  float M = -INFINITY;
  for (int i = i0; i < i1; ++i) M = fmaxf(M, part_lse[(size_t)i * G + hl]);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float wsum = 0.f;
  if (M > -INFINITY) {
    for (int i = i0; i < i1; ++i) {
      const float l = part_lse[(size_t)i * G + hl];
      const float wt = __expf(l - M);
      const float4 po =
          *reinterpret_cast<const float4*>(part_o + ((size_t)i * G + hl) * kHeadDim + 4 * lane);
      acc.x = fmaf(wt, po.x, acc.x);
      acc.y = fmaf(wt, po.y, acc.y);
      acc.z = fmaf(wt, po.z, acc.z);
      acc.w = fmaf(wt, po.w, acc.w);
      wsum += wt;
    }
    const float inv = 1.f / wsum;
    acc.x *= inv; acc.y *= inv; acc.z *= inv; acc.w *= inv;
  }
  *reinterpret_cast<float4*>(o + (size_t)wid * kHeadDim + 4 * lane) = acc;
  if (lane == 0) lse[wid] = M > -INFINITY ? M + __logf(wsum) : -INFINITY;
}

}  // namespace

size_t attend_partial_bytes(int batch, int hq, int hkv, int tok_stride) {
  const int g = hq / hkv;
  const size_t items = (size_t)batch * hkv * (((size_t)tok_stride + kChunk - 1) / kChunk);
  size_t bytes = items * g * (kHeadDim + 1) * sizeof(float);
  bytes += ((size_t)batch * hkv + 1) * sizeof(int);
  return (bytes + 255) & ~(size_t)255;
}

cudaError_t launch_group_union(int hq, const KV& kv, const int* cand_tok, const int* kept_idx,
                               const int* kept_count, const int* cand_count, int cand_stride,
                               int* union_tok, int* union_count, uint32_t* flags,
                               cudaStream_t s) {
  const size_t smem = (size_t)((kv.max_pages * kPage + 31) / 32) * sizeof(uint32_t);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k_group_union,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  k_group_union<<<kv.batch * kv.hkv, 512, smem, s>>>(hq, kv, cand_tok, kept_idx, kept_count,
                                                     cand_count, cand_stride, union_tok,
                                                     union_count, flags);
  return cudaGetLastError();
}

cudaError_t launch_sparse_decode(const uint16_t* q, int hq, const KV& kv, const int* tok,
                                 const int* tok_count, int tok_stride, float sm_scale, float* o,
                                 float* lse, void* partials, uint32_t* flags, cudaStream_t s) {
  const int g = hq / kv.hkv;
  const int ngroups = kv.batch * kv.hkv;
  if (ngroups > kMaxGroups) return cudaErrorInvalidValue;
  const size_t items = (size_t)ngroups * ((tok_stride + kChunk - 1) / kChunk);
  float* part_o = reinterpret_cast<float*>(partials);
  float* part_lse = part_o + items * g * kHeadDim;
  int* prefix = reinterpret_cast<int*>(part_lse + items * g);
  const size_t smem = sizeof(AttSmem) + (size_t)(ngroups + 1) * sizeof(int);
  const size_t cap = (size_t)num_sms() * 3;
  const int grid = (int)(items == 0 ? 1 : (items < cap ? items : cap));
  const int merge_blocks = (kv.batch * hq * 32 + 255) / 256;
#define TWL_ATT(G)                                                                           \
  do {                                                                                       \
    cudaError_t e = cudaFuncSetAttribute(k_sparse_attend<G>,                                 \
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,        \
                                         (int)smem);                                         \
    if (e != cudaSuccess) return e;                                                          \
    k_sparse_attend<G><<<grid, kAttThreads, smem, s>>>(q, hq, kv, tok, tok_count, tok_stride, \
                                                       sm_scale, part_o, part_lse, prefix,   \
                                                       flags);                               \
    k_merge_partials<G><<<merge_blocks, 256, 0, s>>>(hq, kv.hkv, kv.batch, part_o, part_lse, \
                                                     prefix, o, lse);                        \
  } while (0)
  switch (g) {
    case 1: TWL_ATT(1); break;
    case 2: TWL_ATT(2); break;
    case 4: TWL_ATT(4); break;
    case 8: TWL_ATT(8); break;
    default: return cudaErrorInvalidValue;
  }
#undef TWL_ATT
  return cudaGetLastError();
}

}  // namespace twl
