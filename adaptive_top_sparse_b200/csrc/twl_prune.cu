// Top-p pruning by bisection on the weight threshold.
//
// "Twilight: Adaptive Attention Sparsity with Hierarchical Top-p Pruning", notes page, "Key
// designs" (efficient top-p): instead of sorting, search the threshold m with
// sum_{W[i] >= m} W[i] >= p; each round is one O(n) parallel pass, and O(log(max W / eps)) rounds
// suffice.  Summary, section 4.2: the search is fused with the other top-p operations.
//
// This is the direct form of the search, used for rows that the read-once kernel of
// twl_prune_rows.cu does not take (a stride that is not a multiple of 4 weights or above 262144,
// or a base that is not 16-byte aligned); a build with -DTWL_PRUNE_BISECT_ONLY takes it for every
// row (a compile-time option; nothing selects it at run time).  One block per row.  The row is
// staged once in shared memory when it fits (else it is re-read from global memory / L2 each
// round).  Every round is one block reduction of the mass above the midpoint, in
// a fixed order, so all threads take the same branch.  The kept indices are compacted in
// ascending order with a block scan.
#include <stdlib.h>

#include "twl_common.cuh"
#include "twl_kernels.h"

namespace twl {
namespace {

constexpr int kPruneThreads = 1024;
constexpr int kPruneSmemFloats = 48 * 1024;  // 192 KiB of staged row

__device__ __forceinline__ float mass_at_least(const float* row, int n, float t, float* red) {
  float s = 0.f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const float x = row[i];
    s += x >= t ? x : 0.f;
  }
  return block_sum(s, red);
}

__global__ void __launch_bounds__(kPruneThreads)
    k_prune(const float* __restrict__ w, const int* __restrict__ row_len,
            const int* __restrict__ row_len_cap, int row_stride, float p, float eps, int staged,
            float* __restrict__ m_out, int* __restrict__ kept_count, int* __restrict__ kept_idx) {
  extern __shared__ float srow[];
  __shared__ float red[33];
  __shared__ int scan_sh[33];
  const int r = blockIdx.x;
  int n = row_len ? row_len[r] : row_stride;
  if (row_len_cap) n = min(n, row_len_cap[r]);
  n = max(0, min(n, row_stride));
  const float* g = w + (size_t)r * row_stride;
  const float* row = g;
  if (staged) {
    const bool vec = (reinterpret_cast<uintptr_t>(g) & 15u) == 0;
    if (vec) {
      const int n4 = n >> 2;
      for (int i = threadIdx.x; i < n4; i += blockDim.x)
        reinterpret_cast<float4*>(srow)[i] = __ldg(reinterpret_cast<const float4*>(g) + i);
      for (int i = 4 * n4 + threadIdx.x; i < n; i += blockDim.x) srow[i] = g[i];
    } else {
      for (int i = threadIdx.x; i < n; i += blockDim.x) srow[i] = g[i];
    }
    __syncthreads();
    row = srow;
  }
  float top = -INFINITY;
  for (int i = threadIdx.x; i < n; i += blockDim.x) top = fmaxf(top, row[i]);
  top = block_max(top, red);

  float m;
  if (n == 0 || p >= 1.f) {
    m = 0.f;  // p = 1 keeps every candidate: the mass test cannot resolve 1.0 in fp32
  } else if (mass_at_least(row, n, top, red) >= p) {
    m = top;
  } else {
    float lo = 0.f, hi = top;
    for (int iter = 0; iter < 64; ++iter) {
      const float width = __fsub_rn(hi, lo);
      if (width <= eps) break;
      const float mid = __fadd_rn(lo, __fmul_rn(width, 0.5f));
      if (!(lo < mid && mid < hi)) break;
      if (mass_at_least(row, n, mid, red) >= p) lo = mid;
      else hi = mid;
    }
    m = lo;
  }

  // kept = {i : W_i >= m}, ascending
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int beg = min(n, (int)threadIdx.x * per), end = min(n, beg + per);
  int cnt = 0;
  for (int i = beg; i < end; ++i) cnt += row[i] >= m;
  int total;
  int pos = block_exclusive_scan(cnt, scan_sh, &total);
  if (kept_idx) {
    int* out = kept_idx + (size_t)r * row_stride;
    for (int i = beg; i < end; ++i)
      if (row[i] >= m) out[pos++] = i;
  }
  if (threadIdx.x == 0) {
    m_out[r] = m;
    kept_count[r] = total;
  }
}

}  // namespace

cudaError_t launch_prune(const float* w, const int* row_len, const int* row_len_cap, int rows,
                         int row_stride, float p, float eps, float* m_out, int* kept_count,
                         int* kept_idx, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
#ifndef TWL_PRUNE_BISECT_ONLY  // a build option (never a run-time switch): direct bisection only
  {
    // 64 weights per thread above 16384 weights per row (no cluster up to 32768), else 32
    const cudaError_t e =
        row_stride > 16384
            ? rows64::launch_prune_rows(w, row_len, row_len_cap, rows, row_stride, p, eps, m_out,
                                        kept_count, kept_idx, s)
            : rows32::launch_prune_rows(w, row_len, row_len_cap, rows, row_stride, p, eps, m_out,
                                        kept_count, kept_idx, s);
    if (e != cudaErrorNotSupported) return e;
  }
#endif
  const int staged = row_stride <= kPruneSmemFloats;
  const size_t smem = staged ? (size_t)row_stride * sizeof(float) : 0;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k_prune, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  k_prune<<<rows, kPruneThreads, smem, s>>>(w, row_len, row_len_cap, row_stride, p, eps, staged,
                                            m_out, kept_count, kept_idx);
  return cudaGetLastError();
}

}  // namespace twl
