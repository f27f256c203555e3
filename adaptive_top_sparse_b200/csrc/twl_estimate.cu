// Weight estimation from the INT4 K copy.
//
// "Twilight: Adaptive Attention Sparsity with Hierarchical Top-p Pruning":
//   notes page, "Key designs": top-p needs attention-weight values, estimated with a 4-bit K cache;
//   summary, section 4.2 and appendix B.1: fp16 query x INT4 key SpGEMV, keys dequantised on the
//   fly (fp16 scale and zero point, two values per byte), memory-bound;
//   summary, appendix B.2: for GQA the INT4 rows are loaded once per group over the union of the
//   group's selected pages.
//
// With khat = n * s + z per token row:  q . khat = s * (q . n) + z * sum(q).  The q . n products are
// computed on the tensor cores: one 16-token page is exactly the M = 16 tile of
// mma.m16n8k16, the 128 channels are 8 K-steps and the N = 8 columns hold the group's query heads
// (zero-padded when the group is smaller).  Codes become exact fp16 integers with bit
// arithmetic: the binary16 pattern 0x6400 | n (exponent 10, mantissa n) is the number 1024 + n, so
// one half2 subtraction of 1024 yields n exactly (any n < 1024, so 2-, 4- and 8-bit codes alike).
// The mma's K index is mapped to channels so that each lane's codes unpack with a mask and a
// shift; the query fragment uses the same map.
#include "twl_common.cuh"
#include "twl_kernels.h"

namespace twl {
namespace {

// ------------------------------------------------------------------ union of selected pages
// One block per (b, kv-head): marks the pages selected by each head of the group, records each
// head's rank of the page in its ascending selection, and compacts the union (ascending).
__global__ void __launch_bounds__(512)
    k_union_pages(int hq, KV kv, const int* __restrict__ sel_pages,
                  const int* __restrict__ sel_count, int max_budget, int* __restrict__ rank,
                  int* __restrict__ union_pages, uint32_t* __restrict__ union_mask,
                  int* __restrict__ union_npages, uint32_t* flags) {
  extern __shared__ uint32_t mask[];  // [max_pages]
  __shared__ int scan_sh[33];
  const int b = blockIdx.x / kv.hkv, kvh = blockIdx.x % kv.hkv;
  const int g = hq / kv.hkv;
  Seq sq = load_seq(kv.seq_lens, b, kv.max_pages, flags, false);
  const int n = sq.pages;
  for (int i = threadIdx.x; i < n; i += blockDim.x) mask[i] = 0u;
  __syncthreads();
  for (int hl = 0; hl < g; ++hl) {
    const int bh = b * hq + kvh * g + hl;
    const int cnt = min(max(sel_count[bh], 0), min(n, max_budget));
    const int* sel = sel_pages + (size_t)bh * max_budget;
    for (int i = threadIdx.x; i < cnt; i += blockDim.x) {
      const int j = sel[i];
      if (j < 0 || j >= n) {
        raise_flag(flags, TWL_FLAG_BAD_INDEX);
        continue;
      }
      atomicOr(&mask[j], 1u << hl);
      rank[(size_t)bh * kv.max_pages + j] = i;
    }
  }
  __syncthreads();
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int beg = min(n, (int)threadIdx.x * per), end = min(n, beg + per);
  int cnt = 0;
  for (int i = beg; i < end; ++i) cnt += mask[i] != 0u;
  int total;
  int pos = block_exclusive_scan(cnt, scan_sh, &total);
  const size_t base = (size_t)blockIdx.x * kv.max_pages;
  for (int i = beg; i < end; ++i) {
    const uint32_t m = mask[i];
    if (m) {
      union_pages[base + pos] = i;
      union_mask[base + pos] = m;
      ++pos;
    }
  }
  if (threadIdx.x == 0) union_npages[blockIdx.x] = total;
}

// ------------------------------------------------------------------ INT4 dot products
constexpr int kEstThreads = 256;
constexpr int kEstPagesPerWarp = 4;
constexpr int kEstPagesPerBlock = (kEstThreads / 32) * kEstPagesPerWarp;  // 32

// Lane (g = lane/4, t = lane%4) holds, for K-step ks (w = ks/2, e = ks%2), the query values of
// channels 32t + 8w + {2e, 2e+4} (fragment b0) and {2e+1, 2e+5} (fragment b1) for head g.
__device__ __forceinline__ void load_q_fragments(const uint16_t* qh, bool valid,
                                                 uint32_t (&bf)[8][2]) {
  const int t = threadIdx.x & 3;
  uint32_t w[16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 v = valid ? *reinterpret_cast<const uint4*>(qh + 32 * t + 8 * i) : make_uint4(0, 0, 0, 0);
    w[4 * i + 0] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
  }
  // word 4*w8 + k holds channels 32t + 8*w8 + 2k, +2k+1 (low, high half)
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const int w8 = ks >> 1, e = ks & 1;
    const uint32_t a = w[4 * w8 + e];      // channels 2e, 2e+1
    const uint32_t c = w[4 * w8 + e + 2];  // channels 2e+4, 2e+5
    bf[ks][0] = __byte_perm(a, c, 0x5410);  // (2e, 2e+4)
    bf[ks][1] = __byte_perm(a, c, 0x7632);  // (2e+1, 2e+5)
  }
}

// The values of channels ca and cb (within the lane's block of 32 channels, BITS bits each,
// channel c at bit c * BITS) as an exact fp16 pair: 0x6400 | v is 1024 + v for v < 1024.
template <int BITS>
__device__ __forceinline__ uint32_t code_pair(const uint32_t (&w)[BITS], int ca, int cb) {
  constexpr uint32_t kMask = (1u << BITS) - 1u;
  const uint32_t va = (w[(ca * BITS) >> 5] >> ((ca * BITS) & 31)) & kMask;
  const uint32_t vb = (w[(cb * BITS) >> 5] >> ((cb * BITS) & 31)) & kMask;
  uint32_t v = (va | (vb << 16)) | 0x64006400u;
  const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&v), __float2half2_rn(1024.f));
  return *reinterpret_cast<const uint32_t*>(&r);
}

// The lane's 32 channels of one row: 4 * BITS bytes at byte 4 * BITS * t of the row.
template <int BITS>
__device__ __forceinline__ void load_codes(const uint8_t* row, int t, uint32_t (&w)[BITS]) {
  const uint32_t* p = reinterpret_cast<const uint32_t*>(row + 4 * BITS * t);
  if constexpr (BITS == 2) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
    w[0] = v.x;
    w[1] = v.y;
  } else {
#pragma unroll
    for (int i = 0; i < BITS; i += 4) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(p + i));
      w[i] = v.x;
      w[i + 1] = v.y;
      w[i + 2] = v.z;
      w[i + 3] = v.w;
    }
  }
}

// grid (ceil(max_pages / 32), Hkv, B).  Each warp handles union pages of group (b, kvh).
// BITS = 4 is the INT4 copy; 2 and 8 are the estimator bit-width variants (same scheme).
template <int G, int BITS>
__global__ void __launch_bounds__(kEstThreads)
    k_estimate_logits(const uint16_t* __restrict__ q, int hq, KV kv,
                      const uint8_t* __restrict__ k_codes, const uint16_t* __restrict__ k_sz,
                      const int* __restrict__ rank, const int* __restrict__ union_pages,
                      const uint32_t* __restrict__ union_mask,
                      const int* __restrict__ union_npages, int cand_stride,
                      float* __restrict__ logits, int* __restrict__ cand_tok, uint32_t* flags) {
  static_assert(G <= 8, "one mma covers up to 8 heads");
  const int b = blockIdx.z, kvh = blockIdx.y;
  const int gi = b * kv.hkv + kvh;
  const int npages = union_npages[gi];
  const int tile0 = blockIdx.x * kEstPagesPerBlock;
  if (tile0 >= npages) return;
  Seq sq = load_seq(kv.seq_lens, b, kv.max_pages, flags, false);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gr = lane >> 2, t = lane & 3;
  const float inv_sqrt_d = 0.08838834764831845f;  // 1/sqrt(128)

  // query fragments (column gr = head gr of the group) and the sums of q per head
  uint32_t bf[8][2];
  const bool head_ok = gr < G;
  const uint16_t* qh = q + ((size_t)b * hq + kvh * G + (head_ok ? gr : 0)) * kHeadDim;
  load_q_fragments(qh, head_ok, bf);
  float qs_part = 0.f;
  if (head_ok) {
#pragma unroll
    for (int i = 0; i < 32; ++i) qs_part += __half2float(__ushort_as_half(qh[32 * t + i]));
  }
  qs_part += __shfl_xor_sync(0xffffffffu, qs_part, 1);
  qs_part += __shfl_xor_sync(0xffffffffu, qs_part, 2);
  // after this every lane of quad gr holds sum(q) of head gr; fetch heads 2t, 2t+1
  const float qsum0 = __shfl_sync(0xffffffffu, qs_part, (2 * t) * 4);
  const float qsum1 = __shfl_sync(0xffffffffu, qs_part, (2 * t + 1) * 4);

  const size_t ubase = (size_t)gi * kv.max_pages;
  for (int it = 0; it < kEstPagesPerWarp; ++it) {
    const int u = tile0 + warp * kEstPagesPerWarp + it;
    if (u >= npages) break;  // warp-uniform
    const int j = union_pages[ubase + u];
    const uint32_t hm = union_mask[ubase + u];
    const int ph = load_phys(kv.page_table, b, j, kv.max_pages, kv.num_phys, flags);
    const bool bad = ph < 0;  // warp-uniform: its candidates get logit -inf
    uint32_t r0[BITS], r1[BITS];
#pragma unroll
    for (int i = 0; i < BITS; ++i) r0[i] = r1[i] = 0u;
    uint32_t sz0 = 0, sz1 = 0;
    if (!bad) {
      const size_t tile = ((size_t)ph * kv.hkv + kvh) * kPage;
      const uint8_t* src = k_codes + tile * (kHeadDim * BITS / 8);
      load_codes<BITS>(src + gr * (kHeadDim * BITS / 8), t, r0);        // row gr
      load_codes<BITS>(src + (gr + 8) * (kHeadDim * BITS / 8), t, r1);  // row gr + 8
      sz0 = __ldg(reinterpret_cast<const uint32_t*>(k_sz + tile * 2) + gr);
      sz1 = __ldg(reinterpret_cast<const uint32_t*>(k_sz + tile * 2) + gr + 8);
    }
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int c0 = 8 * (ks >> 1) + 2 * (ks & 1);
      uint32_t a[4];
      a[0] = code_pair<BITS>(r0, c0, c0 + 4);      // row gr,   K cols 2t, 2t+1
      a[1] = code_pair<BITS>(r1, c0, c0 + 4);      // row gr+8
      a[2] = code_pair<BITS>(r0, c0 + 1, c0 + 5);  // row gr,   K cols 2t+8, 2t+9
      a[3] = code_pair<BITS>(r1, c0 + 1, c0 + 5);  // row gr+8
      mma_16816(acc, a, bf[ks][0], bf[ks][1]);
    }
    const int rows = page_rows(sq.n, j);
    const float s0 = __half2float(__ushort_as_half((unsigned short)(sz0 & 0xFFFFu)));
    const float z0 = __half2float(__ushort_as_half((unsigned short)(sz0 >> 16)));
    const float s1 = __half2float(__ushort_as_half((unsigned short)(sz1 & 0xFFFFu)));
    const float z1 = __half2float(__ushort_as_half((unsigned short)(sz1 >> 16)));
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int hl = 2 * t + e;
      if (hl >= G || !((hm >> hl) & 1u)) continue;
      const int bh = b * hq + kvh * G + hl;
      const int rk = rank[(size_t)bh * kv.max_pages + j];
      const float qsum = e ? qsum1 : qsum0;
      const size_t obase = (size_t)bh * cand_stride + (size_t)rk * kPage;
      if (gr < rows) {
        logits[obase + gr] = bad ? -INFINITY : (s0 * acc[e] + z0 * qsum) * inv_sqrt_d;
        cand_tok[obase + gr] = kPage * j + gr;
      }
      if (gr + 8 < rows) {
        logits[obase + gr + 8] = bad ? -INFINITY : (s1 * acc[2 + e] + z1 * qsum) * inv_sqrt_d;
        cand_tok[obase + gr + 8] = kPage * j + gr + 8;
      }
    }
  }
}

// ------------------------------------------------------------------ softmax over candidates
// One block per (b, q-head): weights[0 .. C) = softmax(logits) in place, C from the selection.
__global__ void __launch_bounds__(512)
    k_softmax_rows(int hq, KV kv, const int* __restrict__ sel_pages,
                   const int* __restrict__ sel_count, int max_budget, float* __restrict__ w,
                   int* __restrict__ cand_count) {
  __shared__ float red[33];
  const int bh = blockIdx.x, b = bh / hq;
  Seq sq = load_seq(kv.seq_lens, b, kv.max_pages, nullptr, false);
  const int cnt = min(max(sel_count[bh], 0), min(sq.pages, max_budget));
  int c = 0;
  if (cnt > 0) {
    const int jl = sel_pages[(size_t)bh * max_budget + cnt - 1];
    const int rl = (jl >= 0 && jl < sq.pages) ? page_rows(sq.n, jl) : 0;
    c = kPage * (cnt - 1) + rl;
  }
  float* row = w + (size_t)bh * kPage * max_budget;
  float m = -INFINITY;
  for (int i = threadIdx.x; i < c; i += blockDim.x) m = fmaxf(m, row[i]);
  m = block_max(m, red);
  float s = 0.f;
  for (int i = threadIdx.x; i < c; i += blockDim.x) s += m > -INFINITY ? __expf(row[i] - m) : 0.f;
  s = block_sum(s, red);
  const float inv = 1.f / s;
  const bool empty = !(m > -INFINITY);  // every candidate invalid: all weights zero
  for (int i = threadIdx.x; i < c; i += blockDim.x)
    row[i] = empty ? 0.f : __expf(row[i] - m) * inv;
  if (threadIdx.x == 0) cand_count[bh] = c;
}

}  // namespace

cudaError_t launch_union_pages(int hq, const KV& kv, const int* sel_pages, const int* sel_count,
                               int max_budget, int* rank, int* union_pages,
                               uint32_t* union_mask, int* union_npages, uint32_t* flags,
                               cudaStream_t s) {
  const size_t smem = (size_t)kv.max_pages * sizeof(uint32_t);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k_union_pages,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  k_union_pages<<<kv.batch * kv.hkv, 512, smem, s>>>(hq, kv, sel_pages, sel_count, max_budget,
                                                     rank, union_pages, union_mask, union_npages,
                                                     flags);
  return cudaGetLastError();
}

cudaError_t launch_estimate_logits(const uint16_t* q, int hq, const KV& kv, int bits,
                                   const uint8_t* k_codes, const uint16_t* k_sz, const int* rank,
                                   const int* union_pages, const uint32_t* union_mask,
                                   const int* union_npages, int cand_stride, float* logits,
                                   int* cand_tok, uint32_t* flags, cudaStream_t s) {
  const int g = hq / kv.hkv;
  dim3 grid((kv.max_pages + kEstPagesPerBlock - 1) / kEstPagesPerBlock, kv.hkv, kv.batch);
#define TWL_EST(G, B)                                                                         \
  k_estimate_logits<G, B><<<grid, kEstThreads, 0, s>>>(q, hq, kv, k_codes, k_sz, rank,        \
                                                       union_pages, union_mask, union_npages, \
                                                       cand_stride, logits, cand_tok, flags)
#define TWL_EST_G(B)               \
  switch (g) {                     \
    case 1: TWL_EST(1, B); break;  \
    case 2: TWL_EST(2, B); break;  \
    case 4: TWL_EST(4, B); break;  \
    case 8: TWL_EST(8, B); break;  \
    default: return cudaErrorInvalidValue; \
  }
  switch (bits) {
    case 2: TWL_EST_G(2); break;
    case 8: TWL_EST_G(8); break;
    default: TWL_EST_G(4); break;
  }
#undef TWL_EST_G
#undef TWL_EST
  return cudaGetLastError();
}

cudaError_t launch_softmax_rows(int hq, const KV& kv, const int* sel_pages, const int* sel_count,
                                int max_budget, float* weights, int* cand_count,
                                cudaStream_t s) {
  k_softmax_rows<<<kv.batch * hq, 512, 0, s>>>(hq, kv, sel_pages, sel_count, max_budget, weights,
                                               cand_count);
  return cudaGetLastError();
}

}  // namespace twl
