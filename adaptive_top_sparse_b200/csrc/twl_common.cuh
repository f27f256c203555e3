// Device helpers shared by the twl kernels (sm_100a).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "twl.h"

namespace twl {

constexpr int kHeadDim = 128;
constexpr int kPage = 16;
constexpr int kHeaderBytes = 256;
constexpr int kMaxPages = 32768;

// Workspace header: word 0 = sticky device flags (TWL_FLAG_*); the rest is reserved.
struct WsHeader {
  uint32_t flags;
  uint32_t reserved[kHeaderBytes / 4 - 1];
};

__device__ __forceinline__ void raise_flag(uint32_t* flags, uint32_t f) {
  if (flags != nullptr) atomicOr(flags, f);
}

// ------------------------------------------------------------------ sequence / page lookups
struct Seq {
  int n;      // tokens
  int pages;  // ceil(n / 16)
};

// Length of sequence b, or pages = 0 (and a flag) when it is out of range.
__device__ __forceinline__ Seq load_seq(const int* seq_lens, int b, int max_pages,
                                        uint32_t* flags, bool report) {
  int n = seq_lens[b];
  int pages = (n + kPage - 1) / kPage;
  if (n < 1 || pages > max_pages) {
    if (report) raise_flag(flags, TWL_FLAG_BAD_INDEX);
    return Seq{0, 0};
  }
  return Seq{n, pages};
}

// Physical page of logical page j of sequence b, or -1 (and a flag) when out of range.
__device__ __forceinline__ int load_phys(const int* page_table, int b, int j, int max_pages,
                                         int num_phys, uint32_t* flags) {
  int ph = page_table[(size_t)b * max_pages + j];
  if (ph < 0 || ph >= num_phys) {
    raise_flag(flags, TWL_FLAG_BAD_INDEX);
    return -1;
  }
  return ph;
}

__device__ __forceinline__ int page_rows(int n, int j) {
  int r = n - kPage * j;
  return r < kPage ? r : kPage;
}

// ------------------------------------------------------------------ order keys
// fp16 bits -> integer with the same order as the values and -0 < +0.
__device__ __forceinline__ int f16_key(uint32_t bits) {
  bits &= 0xFFFFu;
  return (bits & 0x8000u) ? -1 - int(bits & 0x7FFFu) : int(bits);
}
__device__ __forceinline__ uint32_t f16_from_key(int key) {
  return key < 0 ? (0x8000u | uint32_t(-1 - key)) : uint32_t(key);
}

// fp32 -> uint32 whose unsigned order is the value order (larger value = larger key).
// -0 is mapped to the key of +0 so equal values get equal keys.
__device__ __forceinline__ uint32_t f32_key(float x) {
  uint32_t u = __float_as_uint(x);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ------------------------------------------------------------------ warp / block reductions
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Sum over the block in a fixed order (warp butterflies, then warp 0 over the warp sums).
// `red` needs blockDim.x / 32 + 1 floats.  Every thread gets the same value.
__device__ __forceinline__ float block_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    float t = lane < nw ? red[lane] : 0.f;
    t = warp_sum(t);
    if (lane == 0) red[32] = t;
  }
  __syncthreads();
  return red[32];
}
__device__ __forceinline__ float block_max(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    float t = lane < nw ? red[lane] : -INFINITY;
    t = warp_max(t);
    if (lane == 0) red[32] = t;
  }
  __syncthreads();
  return red[32];
}

// Exclusive prefix sum over the block (int).  `sh` needs blockDim.x / 32 + 1 ints.
// Returns the exclusive prefix of this thread; *total gets the block total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* sh, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int t = lane < nw ? sh[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < nw) sh[lane] = t;  // inclusive warp totals
    if (lane == nw - 1) sh[32] = t;
  }
  __syncthreads();
  int base = warp > 0 ? sh[warp - 1] : 0;
  if (total) *total = sh[32];
  int r = base + x - v;
  __syncthreads();
  return r;
}

// ------------------------------------------------------------------ top-p bisection
// The midpoint of the bisection on the threshold ([Notes] "Key designs", efficient top-p):
// mid = lo + (hi - lo) * 0.5 in fp32.
__device__ __forceinline__ float mid_of(float lo, float hi) {
  return __fadd_rn(lo, __fmul_rn(__fsub_rn(hi, lo), 0.5f));
}

// The search on (0, top] when its test "mass(W >= mid) >= p" is known to equal "mid <= T": with
// exact masses, mass(W >= t) is a non-increasing step function of t that changes only at values
// of W, so the test passes exactly for t <= T = the largest weight v with mass(W >= v) >= p
// (T = 0 when no weight qualifies).  lo = 0, hi = top; stop when hi - lo <= eps, when the
// midpoint no longer splits, or after 64 steps; the threshold is lo (top when the test passes at
// top itself).
// Four steps per trip, predicated (the same steps and stops as one step per trip).  While
// hi - lo >= 2^-100, (hi - lo) * 0.5 is exact, so fma(hi - lo, 0.5, lo) rounds the same sum as
// lo + (hi - lo) * 0.5; eps >= 2^-100 keeps every tested width there.
__device__ __forceinline__ float bisect_scalar(float top, float T, float eps) {
  if (top <= T) return top;
  float lo = 0.f, hi = top;
  if (!(eps >= 0x1p-100f)) {
#pragma unroll 1
    for (int steps = 0; steps < 64; ++steps) {
      if (__fsub_rn(hi, lo) <= eps) break;
      const float mid = mid_of(lo, hi);
      if (!(lo < mid && mid < hi)) break;
      if (mid <= T) lo = mid;
      else hi = mid;
    }
    return lo;
  }
  bool done = false;
#pragma unroll 1
  for (int steps = 0; steps < 64 && !done; steps += 4) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float d = __fsub_rn(hi, lo);
      const float mid = __fmaf_rn(d, 0.5f, lo);
      done = done || d <= eps || !(lo < mid && mid < hi);
      const bool down = mid <= T;
      lo = !done && down ? mid : lo;
      hi = !done && !down ? mid : hi;
    }
  }
  return lo;
}

// ------------------------------------------------------------------ tensor-core helper
// D = A(16x16 fp16, row) * B(16x8 fp16, col) + C, fp32 accumulate (register operands).
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_half2(__half lo, __half hi) {
  return uint32_t(__half_as_ushort(lo)) | (uint32_t(__half_as_ushort(hi)) << 16);
}

// ------------------------------------------------------------------ async copies
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid) {
  uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
  int src_bytes = valid ? 16 : 0;  // 0 -> the 16 destination bytes are zero-filled
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem),
               "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n"); }
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;\n" ::: "memory");
}

}  // namespace twl
