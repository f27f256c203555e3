// Cache maintenance kernels: page bounds for the page selector and the INT4 copy of K.
//
// "Twilight: Adaptive Attention Sparsity with Hierarchical Top-p Pruning":
//   - page bounds: per-page channel min/max of K, the metadata a Quest-style selector scores
//     (the selector is named in the notes page, "Background", and the summary, section 5.1).
//   - INT4 K: summary, appendix B.1 (per-head dynamic quantisation, fp16 scale and zero point,
//     two 4-bit values per byte); notes page, "Key designs" (4-bit K cache, 1/8 extra memory).
//
// The full kernels give one warp to one (sequence, logical page, kv-head): the page-head tile is
// 16 rows x 256 B, contiguous; lane l owns channels 4l .. 4l+3 (8 bytes of every row).  The
// append kernel gives one warp to one (sequence, kv-head) of the new token, same lane layout.
#include "twl_common.cuh"
#include "twl_kernels.h"

namespace twl {
namespace {

struct Half4 {
  uint32_t lo, hi;  // channels (4l, 4l+1) and (4l+2, 4l+3)
};

__device__ __forceinline__ Half4 load_half4(const uint16_t* p) {
  uint2 v = *reinterpret_cast<const uint2*>(p);
  return Half4{v.x, v.y};
}

__device__ __forceinline__ bool decode_warp(long warp, const KV& kv, int* b, int* j, int* h) {
  long total = (long)kv.batch * kv.max_pages * kv.hkv;
  if (warp >= total) return false;
  *h = int(warp % kv.hkv);
  long t = warp / kv.hkv;
  *j = int(t % kv.max_pages);
  *b = int(t / kv.max_pages);
  return true;
}

__global__ void __launch_bounds__(256) k_page_bounds(KV kv, uint16_t* __restrict__ bounds,
                                                     uint32_t* flags) {
  const long warp = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  int b, j, h;
  if (!decode_warp(warp, kv, &b, &j, &h)) return;
  Seq sq = load_seq(kv.seq_lens, b, kv.max_pages, flags, j == 0 && h == 0 && lane == 0);
  if (j >= sq.pages) return;
  int ph = kv.page_table[(size_t)b * kv.max_pages + j];
  if (ph < 0 || ph >= kv.num_phys) {
    if (lane == 0 && h == 0) raise_flag(flags, TWL_FLAG_BAD_INDEX);
    return;
  }
  const int rows = page_rows(sq.n, j);
  const uint16_t* src = kv.k + (((size_t)ph * kv.hkv + h) * kPage) * kHeadDim + lane * 4;
  int mn[4], mx[4];
  {
    Half4 v = load_half4(src);
    mn[0] = mx[0] = f16_key(v.lo);
    mn[1] = mx[1] = f16_key(v.lo >> 16);
    mn[2] = mx[2] = f16_key(v.hi);
    mn[3] = mx[3] = f16_key(v.hi >> 16);
  }
  for (int r = 1; r < rows; ++r) {
    Half4 v = load_half4(src + r * kHeadDim);
    int k0 = f16_key(v.lo), k1 = f16_key(v.lo >> 16), k2 = f16_key(v.hi), k3 = f16_key(v.hi >> 16);
    mn[0] = min(mn[0], k0); mx[0] = max(mx[0], k0);
    mn[1] = min(mn[1], k1); mx[1] = max(mx[1], k1);
    mn[2] = min(mn[2], k2); mx[2] = max(mx[2], k2);
    mn[3] = min(mn[3], k3); mx[3] = max(mx[3], k3);
  }
  uint16_t* dst = bounds + (((size_t)ph * kv.hkv + h) * 2) * kHeadDim + lane * 4;
  uint2 lo, hi;
  lo.x = f16_from_key(mn[0]) | (f16_from_key(mn[1]) << 16);
  lo.y = f16_from_key(mn[2]) | (f16_from_key(mn[3]) << 16);
  hi.x = f16_from_key(mx[0]) | (f16_from_key(mx[1]) << 16);
  hi.y = f16_from_key(mx[2]) | (f16_from_key(mx[3]) << 16);
  *reinterpret_cast<uint2*>(dst) = lo;
  *reinterpret_cast<uint2*>(dst + kHeadDim) = hi;
}

// One code: n = min(L, rint_even(fp32(x - z) / s)); x - z >= 0 because z is the row minimum.
__device__ __forceinline__ uint32_t code_of(uint32_t xbits, float z, float s, float levels) {
  float x = __half2float(__ushort_as_half((unsigned short)(xbits & 0xFFFFu)));
  float r = rintf(__fdiv_rn(__fsub_rn(x, z), s));
  r = fminf(fmaxf(r, 0.f), levels);
  return (uint32_t)r;
}
__device__ __forceinline__ uint32_t nibble(uint32_t xbits, float z, float s) {
  return code_of(xbits, z, s, 15.f);
}

// The same scheme at BITS bits (L = 2^BITS - 1 levels): the lane's 4 codes (channel c at bit
// c * BITS of the row) and, in *sz, fp16 scale | fp16 zero << 16.
template <int BITS>
__device__ __forceinline__ uint32_t quantize_row_warp_bits(const uint32_t lo, const uint32_t hi,
                                                           uint32_t* sz) {
  constexpr float kLevels = (float)((1 << BITS) - 1);
  int k0 = f16_key(lo), k1 = f16_key(lo >> 16), k2 = f16_key(hi), k3 = f16_key(hi >> 16);
  int kmn = __reduce_min_sync(0xffffffffu, min(min(k0, k1), min(k2, k3)));
  int kmx = __reduce_max_sync(0xffffffffu, max(max(k0, k1), max(k2, k3)));
  const uint32_t mn_bits = f16_from_key(kmn), mx_bits = f16_from_key(kmx);
  const float mn = __half2float(__ushort_as_half((unsigned short)mn_bits));
  const float mx = __half2float(__ushort_as_half((unsigned short)mx_bits));
  const __half s16 = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), kLevels));
  const float s = __half2float(s16);
  uint32_t packed = 0;
  if (s != 0.f) {
    packed = code_of(lo, mn, s, kLevels) | (code_of(lo >> 16, mn, s, kLevels) << BITS) |
             (code_of(hi, mn, s, kLevels) << (2 * BITS)) |
             (code_of(hi >> 16, mn, s, kLevels) << (3 * BITS));
  }
  *sz = uint32_t(__half_as_ushort(s16)) | (mn_bits << 16);
  return packed;
}

// 2- and 8-bit copies of K for the estimator bit-width variants: a warp per (sequence, page,
// kv-head), lane l writes the 4 * BITS bits of channels 4l .. 4l+3 of every row.
template <int BITS>
__global__ void __launch_bounds__(256) k_quantize_k_bits(KV kv, uint8_t* __restrict__ k_codes,
                                                         uint16_t* __restrict__ k_sz,
                                                         uint32_t* flags) {
  const long warp = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  int b, j, h;
  if (!decode_warp(warp, kv, &b, &j, &h)) return;
  Seq sq = load_seq(kv.seq_lens, b, kv.max_pages, flags, j == 0 && h == 0 && lane == 0);
  if (j >= sq.pages) return;
  int ph = kv.page_table[(size_t)b * kv.max_pages + j];
  if (ph < 0 || ph >= kv.num_phys) {
    if (lane == 0 && h == 0) raise_flag(flags, TWL_FLAG_BAD_INDEX);
    return;
  }
  const int rows = page_rows(sq.n, j);
  const size_t tile = ((size_t)ph * kv.hkv + h) * kPage;
  const uint16_t* src = kv.k + tile * kHeadDim + lane * 4;
  uint8_t* dst = k_codes + tile * (kHeadDim * BITS / 8) + lane * (BITS / 2);
  uint32_t* dst_sz = reinterpret_cast<uint32_t*>(k_sz + tile * 2);
  for (int r = 0; r < kPage; ++r) {
    uint32_t packed = 0, sz = 0;
    if (r < rows) {
      const Half4 v = load_half4(src + r * kHeadDim);
      packed = quantize_row_warp_bits<BITS>(v.lo, v.hi, &sz);
    }
    uint8_t* d = dst + r * (kHeadDim * BITS / 8);
    if constexpr (BITS == 2) *d = (uint8_t)packed;
    else *reinterpret_cast<uint32_t*>(d) = packed;
    if (lane == 0) dst_sz[r] = sz;
  }
}

// INT4 of one token row held by a warp (lane l: channels 4l .. 4l+3): returns the lane's 4
// nibbles (channel 2j in the low nibble of byte j) and, in *sz, fp16 scale | fp16 zero << 16.
__device__ __forceinline__ uint16_t quantize_row_warp(const Half4& v, uint32_t* sz) {
  int k0 = f16_key(v.lo), k1 = f16_key(v.lo >> 16), k2 = f16_key(v.hi), k3 = f16_key(v.hi >> 16);
  int kmn = min(min(k0, k1), min(k2, k3));
  int kmx = max(max(k0, k1), max(k2, k3));
  kmn = __reduce_min_sync(0xffffffffu, kmn);
  kmx = __reduce_max_sync(0xffffffffu, kmx);
  const uint32_t mn_bits = f16_from_key(kmn), mx_bits = f16_from_key(kmx);
  const float mn = __half2float(__ushort_as_half((unsigned short)mn_bits));
  const float mx = __half2float(__ushort_as_half((unsigned short)mx_bits));
  const __half s16 = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), 15.f));
  const float s = __half2float(s16);
  uint32_t packed = 0;
  if (s != 0.f) {
    uint32_t n0 = nibble(v.lo, mn, s), n1 = nibble(v.lo >> 16, mn, s);
    uint32_t n2 = nibble(v.hi, mn, s), n3 = nibble(v.hi >> 16, mn, s);
    packed = n0 | (n1 << 4) | (n2 << 8) | (n3 << 12);
  }
  *sz = uint32_t(__half_as_ushort(s16)) | (mn_bits << 16);
  return (uint16_t)packed;
}

__global__ void __launch_bounds__(256) k_quantize_k(KV kv, uint8_t* __restrict__ k_int4,
                                                    uint16_t* __restrict__ k_sz,
                                                    uint32_t* flags) {
  const long warp = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  int b, j, h;
  if (!decode_warp(warp, kv, &b, &j, &h)) return;
  Seq sq = load_seq(kv.seq_lens, b, kv.max_pages, flags, j == 0 && h == 0 && lane == 0);
  if (j >= sq.pages) return;
  int ph = kv.page_table[(size_t)b * kv.max_pages + j];
  if (ph < 0 || ph >= kv.num_phys) {
    if (lane == 0 && h == 0) raise_flag(flags, TWL_FLAG_BAD_INDEX);
    return;
  }
  const int rows = page_rows(sq.n, j);
  const size_t tile = ((size_t)ph * kv.hkv + h) * kPage;
  const uint16_t* src = kv.k + tile * kHeadDim + lane * 4;
  uint16_t* dst_q = reinterpret_cast<uint16_t*>(k_int4 + tile * (kHeadDim / 2)) + lane;
  uint32_t* dst_sz = reinterpret_cast<uint32_t*>(k_sz + tile * 2);
  for (int r = 0; r < kPage; ++r) {
    if (r >= rows) {  // past the end of the sequence: zeros
      dst_q[r * (kHeadDim / 4)] = 0;
      if (lane == 0) dst_sz[r] = 0u;
      continue;
    }
    uint32_t sz;
    const uint16_t packed = quantize_row_warp(load_half4(src + r * kHeadDim), &sz);
    dst_q[r * (kHeadDim / 4)] = packed;
    if (lane == 0) dst_sz[r] = sz;
  }
}

// Page centroids for cluster-level selection: per (sequence, page, kv-head) warp, lane l sums
// channels 4l .. 4l+3 over the valid rows in fp32 from row 0 upwards, divides by the row count
// (IEEE fp32) and rounds to fp16.
__global__ void __launch_bounds__(256) k_page_centroids(KV kv, uint16_t* __restrict__ centroids,
                                                        uint32_t* flags) {
  const long warp = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  int b, j, h;
  if (!decode_warp(warp, kv, &b, &j, &h)) return;
  Seq sq = load_seq(kv.seq_lens, b, kv.max_pages, flags, j == 0 && h == 0 && lane == 0);
  if (j >= sq.pages) return;
  int ph = kv.page_table[(size_t)b * kv.max_pages + j];
  if (ph < 0 || ph >= kv.num_phys) {
    if (lane == 0 && h == 0) raise_flag(flags, TWL_FLAG_BAD_INDEX);
    return;
  }
  const int rows = page_rows(sq.n, j);
  const uint16_t* src = kv.k + (((size_t)ph * kv.hkv + h) * kPage) * kHeadDim + lane * 4;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int r = 0; r < rows; ++r) {
    const Half4 v = load_half4(src + r * kHeadDim);
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&v.lo));
    const float2 c = __half22float2(*reinterpret_cast<const __half2*>(&v.hi));
    acc[0] = __fadd_rn(acc[0], a.x);
    acc[1] = __fadd_rn(acc[1], a.y);
    acc[2] = __fadd_rn(acc[2], c.x);
    acc[3] = __fadd_rn(acc[3], c.y);
  }
  const float fr = (float)rows;
  const __half2 lo = __floats2half2_rn(__fdiv_rn(acc[0], fr), __fdiv_rn(acc[1], fr));
  const __half2 hi = __floats2half2_rn(__fdiv_rn(acc[2], fr), __fdiv_rn(acc[3], fr));
  uint2 out;
  out.x = *reinterpret_cast<const uint32_t*>(&lo);
  out.y = *reinterpret_cast<const uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(centroids + ((size_t)ph * kv.hkv + h) * kHeadDim + lane * 4) = out;
}

// One decode step's append: CTA b writes the new token of sequence b (one warp per kv-head,
// looping when there are more heads than warps), then advances seq_lens[b].
__global__ void __launch_bounds__(256) k_append_token(KV kv, uint16_t* __restrict__ k_cache,
                                                      uint16_t* __restrict__ v_cache,
                                                      const uint16_t* __restrict__ k_new,
                                                      const uint16_t* __restrict__ v_new,
                                                      uint8_t* __restrict__ k_int4,
                                                      uint16_t* __restrict__ k_sz,
                                                      uint16_t* __restrict__ bounds,
                                                      int32_t* seq_lens_out, uint32_t* flags) {
  __shared__ int s_n, s_ph;
  const int b = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  if (threadIdx.x == 0) {
    const int n = kv.seq_lens[b];
    const int j = n >> 4;
    int ph = -1;
    if (n >= 0 && j < kv.max_pages) ph = kv.page_table[(size_t)b * kv.max_pages + j];
    if (ph < 0 || ph >= kv.num_phys) {
      raise_flag(flags, TWL_FLAG_BAD_INDEX);
      ph = -1;
    }
    s_n = n;
    s_ph = ph;
  }
  __syncthreads();
  const int n = s_n, ph = s_ph;
  if (ph < 0) return;  // uniform over the CTA
  const int row = n & (kPage - 1);
  for (int h = warp; h < kv.hkv; h += nwarps) {
    const size_t tile = ((size_t)ph * kv.hkv + h) * kPage;
    const size_t in_off = ((size_t)b * kv.hkv + h) * kHeadDim + lane * 4;
    const Half4 x = load_half4(k_new + in_off);
    *reinterpret_cast<uint2*>(k_cache + (tile + row) * kHeadDim + lane * 4) = make_uint2(x.lo, x.hi);
    *reinterpret_cast<uint2*>(v_cache + (tile + row) * kHeadDim + lane * 4) =
        *reinterpret_cast<const uint2*>(v_new + in_off);
    // INT4 row, as k_quantize_k writes it
    uint32_t sz;
    const uint16_t packed = quantize_row_warp(x, &sz);
    reinterpret_cast<uint16_t*>(k_int4 + tile * (kHeadDim / 2))[row * (kHeadDim / 4) + lane] = packed;
    if (lane == 0) reinterpret_cast<uint32_t*>(k_sz + tile * 2)[row] = sz;
    // page bounds: the row itself on a fresh page, else min / max with the old bounds
    int key[4] = {f16_key(x.lo), f16_key(x.lo >> 16), f16_key(x.hi), f16_key(x.hi >> 16)};
    int mn[4], mx[4];
    uint16_t* dst = bounds + (((size_t)ph * kv.hkv + h) * 2) * kHeadDim + lane * 4;
    if (row == 0) {
#pragma unroll
      for (int c = 0; c < 4; ++c) mn[c] = mx[c] = key[c];
    } else {
      const Half4 omn = load_half4(dst), omx = load_half4(dst + kHeadDim);
      const int okn[4] = {f16_key(omn.lo), f16_key(omn.lo >> 16), f16_key(omn.hi), f16_key(omn.hi >> 16)};
      const int okx[4] = {f16_key(omx.lo), f16_key(omx.lo >> 16), f16_key(omx.hi), f16_key(omx.hi >> 16)};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        mn[c] = min(okn[c], key[c]);
        mx[c] = max(okx[c], key[c]);
      }
    }
    uint2 lo, hi;
    lo.x = f16_from_key(mn[0]) | (f16_from_key(mn[1]) << 16);
    lo.y = f16_from_key(mn[2]) | (f16_from_key(mn[3]) << 16);
    hi.x = f16_from_key(mx[0]) | (f16_from_key(mx[1]) << 16);
    hi.y = f16_from_key(mx[2]) | (f16_from_key(mx[3]) << 16);
    *reinterpret_cast<uint2*>(dst) = lo;
    *reinterpret_cast<uint2*>(dst + kHeadDim) = hi;
  }
  if (seq_lens_out) {
    __syncthreads();  // every head of the token is written before the length moves
    if (threadIdx.x == 0) seq_lens_out[b] = n + 1;
  }
}

}  // namespace

cudaError_t launch_append_token(const KV& kv, uint16_t* k_cache, uint16_t* v_cache,
                                const uint16_t* k_new, const uint16_t* v_new, uint8_t* k_int4,
                                uint16_t* k_sz, uint16_t* bounds, int32_t* seq_lens_out,
                                uint32_t* flags, cudaStream_t s) {
  const int threads = kv.hkv >= 8 ? 256 : 32 * kv.hkv;
  k_append_token<<<kv.batch, threads, 0, s>>>(kv, k_cache, v_cache, k_new, v_new, k_int4, k_sz,
                                              bounds, seq_lens_out, flags);
  return cudaGetLastError();
}

cudaError_t launch_quantize_k_bits(const KV& kv, int bits, uint8_t* k_codes, uint16_t* k_sz,
                                   uint32_t* flags, cudaStream_t s) {
  long warps = (long)kv.batch * kv.max_pages * kv.hkv;
  long blocks = (warps * 32 + 255) / 256;
  if (bits == 2) k_quantize_k_bits<2><<<(unsigned)blocks, 256, 0, s>>>(kv, k_codes, k_sz, flags);
  else if (bits == 8) k_quantize_k_bits<8><<<(unsigned)blocks, 256, 0, s>>>(kv, k_codes, k_sz, flags);
  else return launch_quantize_k(kv, k_codes, k_sz, flags, s);
  return cudaGetLastError();
}

cudaError_t launch_page_centroids(const KV& kv, uint16_t* centroids, uint32_t* flags,
                                  cudaStream_t s) {
  long warps = (long)kv.batch * kv.max_pages * kv.hkv;
  long blocks = (warps * 32 + 255) / 256;
  k_page_centroids<<<(unsigned)blocks, 256, 0, s>>>(kv, centroids, flags);
  return cudaGetLastError();
}

cudaError_t launch_page_bounds(const KV& kv, uint16_t* bounds, uint32_t* flags, cudaStream_t s) {
  long warps = (long)kv.batch * kv.max_pages * kv.hkv;
  long blocks = (warps * 32 + 255) / 256;
  k_page_bounds<<<(unsigned)blocks, 256, 0, s>>>(kv, bounds, flags);
  return cudaGetLastError();
}

cudaError_t launch_quantize_k(const KV& kv, uint8_t* k_int4, uint16_t* k_sz, uint32_t* flags,
                              cudaStream_t s) {
  long warps = (long)kv.batch * kv.max_pages * kv.hkv;
  long blocks = (warps * 32 + 255) / 256;
  k_quantize_k<<<(unsigned)blocks, 256, 0, s>>>(kv, k_int4, k_sz, flags);
  return cudaGetLastError();
}

}  // namespace twl
