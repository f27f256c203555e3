// Top-p thresholds of many independent weight rows, each row read from HBM once.
//
// "Twilight: Adaptive Attention Sparsity with Hierarchical Top-p Pruning", notes page, "Key
// designs" (efficient top-p): the threshold m is found by bisection, each step testing
// mass(W >= mid) >= p, with no sort; summary, section 4.2.
//
// mass(W >= t) is a non-increasing step function of t that only changes at values of W.  The
// bisection's test at t is therefore the same as "t <= T", where T is the largest weight value v
// with mass(W >= v) >= p (T = 0 when the row's mass stays below p).  This kernel finds T, then
// bisect_scalar replays the bisection's midpoints, stopping rules and result as scalar arithmetic.
// T is a mass-weighted order statistic, found over the row held in registers; shared-memory
// atomics count every weight once for the bracket and only the few weights inside its range after
// that:
//   bracket  a count histogram of the fp32 bit patterns over [L, max W] (kNB log-spaced bins), one
//            shared add per weight (to a dummy word when outside); its estimated mass profile
//            (bin middle values) gives a key range that holds T.  A build with
//            TWL_PRUNE_SAMPLE = k > 1 counts every weight >= 4 x the mean but only one in k of
//            the others, and widens the range by the sampling variance (fewer shared adds, but
//            the wider range costs more than it saves on the rows measured).
//            L = (sum W - p) / (2 n): the weights below L sum to less than (sum - p) / 2, so T >= L.
//   exact    one pass: the weights above the range add up to the mass above it (fp32 pairwise per
//            thread, fp64 across threads); the weights inside it go to per-thread lists, then to
//            an exact histogram (count and sum of low mantissa bits per bin, so a bin's mass is an
//            exact integer in units of the range's lowest exponent).  If T lies outside the range,
//            the range moves and the pass repeats.
//   levels   a crossing bin of at most 32 weights (one CTA) is ranked by one warp; otherwise its
//            weights are histogrammed again on the next bits, until one value (or one weight,
//            whose bits follow from the bin's sums) remains.
// The fp32 part of the mass above the range is off by at most 2^-21 of it.  When the decision
// that fixed T is closer than that to p, the pass repeats with that mass summed in fp64, so the
// result is the one fp64 sums give.
//
// Layout: a CTA holds a slice of kRE * blockDim.x weights of a row in registers (kRE per
// thread, as float4 chunks strided by the block); rows longer than 32768 weights are split over
// a thread-block cluster whose CTAs merge their histograms through distributed shared memory.
// (This file is built twice: 32 weights per thread in CTAs of up to 1024 threads at 64 registers,
// and 64 weights per thread in CTAs of up to 512 threads at 128 registers (twl_prune_rows64.cu),
// which halves the per-row work that every warp repeats and suits rows above 16384 weights.)  The
// grid is persistent: each CTA (cluster) walks rows r, r + G, ..., and while it works on one row
// its threads' cp.async copies of the next row land in shared memory (every thread copies and
// later reads back only its own chunks, so the hand-off needs no barrier).
#include <mutex>

#include "twl_common.cuh"
#include "twl_kernels.h"

namespace twl {
namespace {

typedef unsigned __int128 u128;

#ifndef TWL_PRUNE_RE
#define TWL_PRUNE_RE 32
#endif
constexpr int kRE = TWL_PRUNE_RE;           // weights per thread (32 or 64)
static_assert(kRE == 32 || kRE == 64, "32 or 64 weights per thread");
constexpr int kRounds = kRE / 4;            // float4 chunks per thread
#ifndef TWL_PRUNE_MAX_THREADS
#define TWL_PRUNE_MAX_THREADS 1024
#endif
constexpr int kRMaxThreads = TWL_PRUNE_MAX_THREADS;
constexpr int kRSlice = kRE * kRMaxThreads;  // weights per CTA, at most
constexpr int kRMaxCluster = 8;
#ifndef TWL_PRUNE_NB_BITS
#define TWL_PRUNE_NB_BITS 10
#endif
#ifndef TWL_PRUNE_SAMPLE
#define TWL_PRUNE_SAMPLE 1
#endif
constexpr int kNBBits = TWL_PRUNE_NB_BITS;
constexpr int kNB = 1 << kNBBits;           // bins per histogram
static_assert(kNB >= kRMaxThreads, "the bracket scan gives every thread at least one bin");
constexpr float kHeavy = 4.f;               // weights >= kHeavy * sum / n are always counted
constexpr int kSample = TWL_PRUNE_SAMPLE;   // one in kSample of the other weights is counted
static_assert(kSample == 1 || kSample == 2 || kSample == 4, "a divisor of the 4-weight chunk");
// exact bins: count * 2^shift < 2^32 per CTA (count <= 2^15), and a range of at most
// kNB * 2^shift <= 2^27 bit patterns (16 binades) keeps a bin's integer mass below 2^59
constexpr int kMaxBinShift = kNBBits <= 10 ? 17 : 27 - kNBBits;
static_assert(kNBBits + kMaxBinShift <= 27, "exact masses fit in 64 bits");
static_assert(2 * kNBBits >= kMaxBinShift, "two refinement levels resolve an exact bin");
constexpr uint32_t kNaNBits = 0xFFFFFFFFu;  // weights past the row's length

// Optional phase clock (a probe build defines TWL_PRUNE_STAMP(slot) to record it); off by default.
#ifndef TWL_PRUNE_STAMP
#define TWL_PRUNE_STAMP(slot)
#endif

// ------------------------------------------------------------------ cluster helpers
__device__ __forceinline__ void csync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
__device__ __forceinline__ uint32_t crank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cnum() {
  uint32_t n;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(n));
  return n;
}
__device__ __forceinline__ uint32_t saddr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ uint32_t mapa(uint32_t addr, int rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ uint64_t ldc64(uint32_t addr) {
  uint64_t v;
  asm volatile("ld.shared::cluster.u64 %0, [%1];" : "=l"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t ldc32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ void stc32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t atomc_add32(uint32_t addr, uint32_t v) {
  uint32_t old;
  asm volatile("atom.shared::cluster.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(addr), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
// the sum over the cluster's CTAs of the shared u32 at `ad` (this CTA's own when C == 1)
__device__ __forceinline__ uint64_t csum32(uint32_t ad, int C) {
  if (C == 1) return lds32(ad);
  uint64_t s = 0;
#pragma unroll
  for (int q = 0; q < kRMaxCluster; ++q)
    if (q < C) s += ldc32(mapa(ad, q));
  return s;
}

// Shared-memory add and store at a shared address.
__device__ __forceinline__ void red_add_u(uint32_t ad, uint32_t v) {
  asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(ad), "r"(v) : "memory");
}
__device__ __forceinline__ void sts32(uint32_t ad, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(ad), "r"(v) : "memory");
}
// Predicated shared-memory add.
__device__ __forceinline__ void red_add(uint32_t ad, uint32_t v, bool pred) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %2, 0;\n\t@q red.shared.add.u32 [%0], %1;\n\t}" ::"r"(
          ad),
      "r"(v), "r"((uint32_t)pred)
      : "memory");
}

// Copy 16 bytes, of which `bytes` (0..16) are read from global memory and the rest zero-filled.
__device__ __forceinline__ void cp_async_n(void* smem, const void* gmem, int bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(saddr(smem)), "l"(gmem),
               "r"(bytes));
}

// ------------------------------------------------------------------ exact masses
__device__ __forceinline__ double pow2d(int k) {  // k in [-1022, 1023]
  return __longlong_as_double((long long)(k + 1023) << 52);
}
// Smallest shift with (hi >> s) - (lo >> s) < kNB.
__device__ __forceinline__ int span_shift(uint32_t lo, uint32_t hi) {
  int s = 0;
  while ((hi >> s) - (lo >> s) >= (uint32_t)kNB) ++s;
  return s;
}

// ------------------------------------------------------------------ block scans
// Exclusive prefix of 128-bit values (8 packed 16-bit counts in pass D).  sh: 33 entries.
// Two of them at once (16 rounds of counts): the same scan on a pair.
__device__ __forceinline__ u128 shfl_up_u128(u128 v, int o) {
  const uint64_t lo = __shfl_up_sync(0xffffffffu, (uint64_t)v, o);
  const uint64_t hi = __shfl_up_sync(0xffffffffu, (uint64_t)(v >> 64), o);
  return ((u128)hi << 64) | lo;
}
__device__ u128 block_excl_u128(u128 v, u128* sh, u128* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  u128 x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const u128 y = shfl_up_u128(x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  if (warp == 0) {
    u128 tt = lane < nw ? sh[lane] : (u128)0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const u128 y = shfl_up_u128(tt, o);
      if (lane >= o) tt += y;
    }
    if (lane < nw) sh[lane] = tt;
  }
  __syncthreads();
  const u128 base = warp ? sh[warp - 1] : (u128)0;
  *total = sh[nw - 1];
  __syncthreads();
  return base + x - v;
}

// ------------------------------------------------------------------ shared state
struct Cross {
  uint64_t above;  // mass (level units) of the level's bins above the crossing bin
  uint64_t mass;   // the crossing bin's mass
  uint64_t cnt;    // its weight count
  uint64_t sum;    // and low-bit sum
  int bin;         // the bin (-1: the level's mass stays below what is needed)
  int pad;
};

struct RowSh {
  u128 ush[33];
  uint64_t wtot[32];  // per-warp totals of a level scan
  double wpart[32];   // per-warp partial sums of the mass above the exact range
  float fw[32], fv[32];
  Cross cr;
  double cta_above;   // this CTA's mass above the exact range (read by the cluster)
  float m;            // the row's threshold (written by the owner of the last crossing)
  int certain;        // the last crossing is certain under the fp32 bound
  float wsum[32];
  float cta_sum;
  uint32_t top_key;   // f32_key of this CTA's largest weight (atomicMax)
  uint32_t wcnt[32];  // per-warp kept counts
  int bhi, blo;       // bracket bins (atomicMax)
  uint32_t cta_count[kRMaxCluster];  // kept weights per CTA of the cluster (written remotely)
  uint32_t gather[32];  // the crossing bin's weights, when it holds at most 32 (one CTA)
  int gcount;
  uint32_t g_t;         // their solve: T's bit pattern,
  uint64_t g_gt, g_eq;  // the mass above T and at T (units of the bin's exponent)
};

__device__ __forceinline__ uint64_t shfl_up_u64(uint64_t v, int o) {
  return __shfl_up_sync(0xffffffffu, v, o);
}

// One level in exact integer masses: bins nb-1 (largest values) .. 0; thread t owns the run
// [b0 - per + 1, b0], b0 = nb - 1 - t * per.  mass_of(b, &cnt, &sum) gives bin b's mass in the
// level's unit.  Finds the first bin, from the top, at which the mass of the bins above and
// including it reaches R (>= 1); the one thread whose run holds it records it in sh.cr (bin -1
// when the level's total stays below R).  The integer sums are exact, so exactly one thread's
// run [start, end) contains R.  Two barriers; the caller's barrier completes the histogram.
template <class F>
__device__ void level_cross(int nb, uint64_t R, F mass_of, RowSh& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int per = (nb + (int)blockDim.x - 1) / (int)blockDim.x;
  const int b0 = nb - 1 - (int)threadIdx.x * per;
  uint64_t local = 0;
  for (int e = 0; e < per && b0 - e >= 0; ++e) {
    uint64_t c, s;
    local += mass_of(b0 - e, &c, &s);
  }
  uint64_t x = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t y = shfl_up_u64(x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh.wtot[warp] = x;
  if (threadIdx.x == 0) sh.cr.bin = -1;
  __syncthreads();
  uint64_t wt = lane < nw ? sh.wtot[lane] : 0ull;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t y = shfl_up_u64(wt, o);
    if (lane >= o) wt += y;
  }
  const uint64_t wp = __shfl_sync(0xffffffffu, wt, (warp + 31) & 31);
  const uint64_t start = (warp ? wp : 0ull) + x - local;
  if (start < R && R <= start + local) {
    uint64_t run = start;
    for (int e = 0; e < per && b0 - e >= 0; ++e) {
      uint64_t c, s;
      const uint64_t mb = mass_of(b0 - e, &c, &s);
      if (run + mb >= R) {
        sh.cr.above = run;
        sh.cr.mass = mb;
        sh.cr.cnt = c;
        sh.cr.sum = s;
        sh.cr.bin = b0 - e;
        break;
      }
      run += mb;
    }
  }
  __syncthreads();
}

// Integer mass of `cnt` weights whose bit patterns share the prefix of base_key above bit sh
// (one exponent, as sh <= 23), `sum` the sum of their low sh bits, in units 2^(e_unit - 150):
// (cnt * lead + sum) << (e - e_unit), e_unit <= e (callers keep the shift small).
__device__ __forceinline__ uint64_t bin_units(uint32_t base_key, uint64_t cnt, uint64_t sum,
                                              int e_unit) {
  const int e = (int)(base_key >> 23);
  const uint64_t lead = (base_key & 0x7FFFFFu) | (e ? 0x800000u : 0u);
  return (cnt * lead + sum) << (max(e, 1) - e_unit);
}

struct PruneRowsArgs {
  const float* w;
  const int* row_len;
  const int* row_len_cap;
  int rows, stride;
  float p, eps;
  float* m_out;
  int* kept_count;
  int* kept_idx;
  int list_cap;  // per-thread entries of the exact pass's list
};

__device__ __forceinline__ int row_length(const PruneRowsArgs& a, int r) {
  int n = a.row_len ? a.row_len[r] : a.stride;
  if (a.row_len_cap) n = min(n, a.row_len_cap[r]);
  return max(0, min(n, a.stride));
}

// This thread's chunks of row r's slice into shared memory (zero-filled past the row's end).
__device__ __forceinline__ void prefetch_row(const PruneRowsArgs& a, int r, int q, float4* buf) {
  const int T = blockDim.x, t = threadIdx.x;
  const int len = row_length(a, r);
  const float* row = a.w + (size_t)r * a.stride;
  const int s0 = q * kRE * T;
#pragma unroll
  for (int k = 0; k < kRounds; ++k) {
    const int o = s0 + 4 * (k * T + t);
    const int bytes = 4 * max(0, min(4, len - o));
    cp_async_n(buf + k * T + t, bytes > 0 ? row + o : row, bytes);
  }
  cp_async_commit();
}

__device__ __forceinline__ void clear_u32(uint32_t* h, int n) {
  for (int i = threadIdx.x; i < n / 4; i += blockDim.x)
    reinterpret_cast<uint4*>(h)[i] = make_uint4(0u, 0u, 0u, 0u);
}

// Histogram of the weights whose bit pattern u has (u >> hs) == pre, binned by the next
// hs - ls bits (count, and sum of the low ls bits), and the level's crossing (masses in units of
// the prefix's exponent, so no shift).  The weights come from this thread's list (lst: shared
// address of entry 0, entries T words apart, nl of them) when the exact pass kept one, else from
// the registers.  `cnt`: shared address of kNB u32 counts, then kNB u32 sums; zero on entry.
__device__ __forceinline__ void prefix_level(const float (&x)[kRE], bool use_list, uint32_t lst,
                                             int nl, uint32_t pre, int hs, int ls, uint32_t cnt,
                                             uint64_t R, int C, RowSh& sh) {
  const uint32_t nbm = (1u << (hs - ls)) - 1u, lm = (1u << ls) - 1u;
  if (use_list) {
    for (int j = 0; j < nl; ++j) {
      const uint32_t u = lds32(lst + 4u * blockDim.x * j);
      if ((u >> hs) == pre) {
        const uint32_t ad = cnt + 4u * ((u >> ls) & nbm);
        red_add_u(ad, 1u);
        red_add_u(ad + 4u * kNB, u & lm);
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < kRE; ++i) {
      const uint32_t u = __float_as_uint(x[i]);
      const bool in = (u >> hs) == pre;  // pre is a prefix of a finite key: NaN never matches
      const uint32_t ad = cnt + 4u * ((u >> ls) & nbm);
      red_add(ad, 1u, in);
      red_add(ad + 4u * kNB, u & lm, in && lm);
    }
  }
  __syncthreads();
  if (C > 1) csync();
  const int e_unit = max((int)((pre << hs) >> 23), 1);
  auto mass = [&](int b, uint64_t* c, uint64_t* s) -> uint64_t {
    *c = csum32(cnt + 4u * b, C);
    *s = ls ? csum32(cnt + 4u * (kNB + b), C) : 0ull;
    const uint32_t key = ((pre << (hs - ls)) | (uint32_t)b) << ls;
    return bin_units(key, *c, *s, e_unit);
  };
  level_cross((int)nbm + 1, R, mass, sh);
}

// 2 kRE registers per thread: 32768 / kRE threads per SM, in CTAs of up to kRMaxThreads
#ifndef TWL_PRUNE_MIN_BLOCKS
#define TWL_PRUNE_MIN_BLOCKS (32768 / kRE / kRMaxThreads)
#endif
__global__ void __launch_bounds__(kRMaxThreads, TWL_PRUNE_MIN_BLOCKS) k_prune_rows(PruneRowsArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ RowSh sh;
  const int T = blockDim.x, t = threadIdx.x, lane = t & 31, warp = t >> 5, nw = T >> 5;
  const int C = (int)cnum(), q = (int)crank();
  const int cid = blockIdx.x / C, ncl = gridDim.x / C;
  float4* buf = reinterpret_cast<float4*>(smem);  // [8][T]
  // histogram regions of 2 x kNB u32: A (bracket counts), B (exact bins), and for a cluster C
  // (first refinement level; one CTA alone uses A, which is dead by then); the second refinement
  // level takes B (one CTA) or A (cluster: after the barrier that ends every read of A)
  uint32_t* rA = reinterpret_cast<uint32_t*>(smem + (size_t)16 * kRounds * T);
  uint32_t* rB = rA + 2 * kNB;
  uint32_t* rC = C > 1 ? rB + 2 * kNB : rA;
  uint32_t* rD = C > 1 ? rA : rB;
  const int nreg = C > 1 ? 3 : 2;
  // after the regions: 32 words that absorb the sampled adds of weights outside the window, then
  // the per-thread lists of the exact pass ((list_cap + 1) rows of T words; the last row absorbs
  // the stores of weights outside the range)
  const uint32_t a_dummy = saddr(rA + 2 * kNB * nreg) + 4u * (t & 31);
  const uint32_t a_list = saddr(rA + 2 * kNB * nreg + 32) + 4u * t;

  clear_u32(rA, 2 * kNB * nreg);
  if (t == 0) sh.top_key = 0u;
  if (cid < a.rows) prefetch_row(a, cid, q, buf);
  __syncthreads();

#pragma unroll 1
  for (int r = cid; r < a.rows; r += ncl) {
    const int len = row_length(a, r);
    const int s0 = q * kRE * T;
    TWL_PRUNE_STAMP(0);
    cp_async_wait_all();
    float x[kRE];
#pragma unroll
    for (int k = 0; k < kRounds; ++k) {
      const float4 v = buf[k * T + t];
      x[4 * k + 0] = v.x;
      x[4 * k + 1] = v.y;
      x[4 * k + 2] = v.z;
      x[4 * k + 3] = v.w;
    }
    // weights past the end become NaN, which no comparison keeps and no histogram counts (nor
    // negative, infinite or NaN weights)
    if (s0 + kRE * T > len) {
#pragma unroll
      for (int k = 0; k < kRounds; ++k)
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (s0 + 4 * (k * T + t) + j >= len) x[4 * k + j] = __uint_as_float(kNaNBits);
    }
    // pass 0: largest weight and the weight sum
    float top = -INFINITY, tsum = 0.f;
#pragma unroll
    for (int i = 0; i < kRE; ++i) {
      top = fmaxf(top, x[i]);
      tsum += fmaxf(x[i], 0.f);
    }
    top = warp_max(top);
    tsum = warp_sum(tsum);
    if (lane == 0) {
      atomicMax(&sh.top_key, f32_key(top));
      sh.wsum[warp] = tsum;
    }
    __syncthreads();  // every read of buf is done
    if (r + ncl < a.rows) prefetch_row(a, r + ncl, q, buf);
    float total = 0.f;
    uint32_t tk = 0u;
    // the per-warp sums, added by one warp-wide reduction (the same order in every warp)
    const float cta_sum = warp_sum(lane < nw ? sh.wsum[lane] : 0.f);
    if (C == 1) {
      total = cta_sum;
      tk = sh.top_key;
    } else {
      if (t == 0) sh.cta_sum = cta_sum;
      csync();
      for (int qq = 0; qq < C; ++qq) {
        tk = max(tk, ldc32(mapa(saddr(&sh.top_key), qq)));
        total += __uint_as_float(ldc32(mapa(saddr(&sh.cta_sum), qq)));
      }
    }
    // back from the order key to the float (keys of non-negative values have the top bit set)
    top = (tk & 0x80000000u) ? __uint_as_float(tk & 0x7FFFFFFFu) : __uint_as_float(~tk);
    TWL_PRUNE_STAMP(1);

    float m;
    if (len == 0 || a.p >= 1.f || !(top > 0.f)) {
      m = 0.f;  // p = 1 keeps every weight: an fp32 mass cannot resolve 1.0
    } else if (isinf(top)) {
      m = top;  // mass(W >= inf) is infinite
    } else if (total * (1.f + 0x1p-16f) < a.p) {
      // the whole row weighs less than p: no threshold reaches p, so T = 0 and the bisection
      // ends at m = 0.  The fp32 row sum is within ~80 roundings (< 2^-16 relative) of the exact
      // one, so the exact mass is below p too; every thread holds the same total.
      m = 0.f;
    } else {
      const uint32_t kt = __float_as_uint(top);
      const double P = (double)a.p;
      TWL_PRUNE_STAMP(2);
      // ---- bracket: count histogram over [L, top] (non-heavy weights: one in kSample)
      const float tot_lo = total * (1.f - 0x1p-16f);
      const float L = tot_lo > a.p ? (tot_lo - a.p) / (2.f * (float)len) : 0.f;
      const uint32_t kL = __float_as_uint(L);
      const uint32_t kH = __float_as_uint(kHeavy * (total / (float)len));
      const int s = span_shift(kL, kt);
      const uint32_t win = (kt >> s) - (uint32_t)(kNB - 1);  // bin b <-> key prefix win + b
      if constexpr (kSample == 1) {
        // every weight: one add, to its bin when it lies in [L, top], else to this lane's dummy
        // word (no branch)
        const uint32_t aH = saddr(rA);
#pragma unroll
        for (int i = 0; i < kRE; ++i) {
          const uint32_t u = __float_as_uint(x[i]);
          const bool in = u - kL <= kt - kL;
          red_add_u(in ? aH + 4u * ((u >> s) - win) : a_dummy, 1u);
        }
      } else {
        // heavy weights: all, behind one warp vote per chunk (they are rare); sampled ones: an
        // add that every thread makes, to its own dummy word when the weight is not counted
        const uint32_t aH = saddr(rA);
#pragma unroll
        for (int k = 0; k < kRounds; ++k) {
          bool hv[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t u = __float_as_uint(x[4 * k + j]);
            hv[j] = u >= kH && u <= kt;  // heavy (kH >= kL: 4x the mean is above L)
            if ((j % kSample) == 0) {
              const bool in = u - kL <= kt - kL;
              red_add_u(in && !hv[j] ? aH + 4u * ((u >> s) - win) + 4u * kNB : a_dummy, 1u);
            }
          }
          if (__any_sync(0xffffffffu, hv[0] || hv[1] || hv[2] || hv[3])) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t u = __float_as_uint(x[4 * k + j]);
              red_add(aH + 4u * ((u >> s) - win), 1u, hv[j]);
            }
          }
        }
      }
      TWL_PRUNE_STAMP(8);
      if (t == 0) {
        sh.bhi = -1;
        sh.blo = -1;
      }
      __syncthreads();
      if (C > 1) csync();
      TWL_PRUNE_STAMP(9);
      {
        // estimated mass per bin: (heavy + kSample x sampled) x the bin's middle value; the
        // variance of the sampled part sets the margin.  Thread t holds bins b0 .. b0 - per + 1.
        const int per = kNB / T;
        const int b0 = kNB - 1 - t * per;
        float le = 0.f, lv = 0.f;
        for (int e = 0; e < per; ++e) {
          const int b = b0 - e;
          const int pk = (int)win + b;
          const float ch = (float)csum32(saddr(rA + b), C);
          const float cl = kSample > 1 ? (float)csum32(saddr(rA + kNB + b), C) : 0.f;
          if (pk >= 0 && ch + cl > 0.f) {
            const float v = __uint_as_float(((uint32_t)pk << s) + ((1u << s) >> 1));
            le += (ch + (float)kSample * cl) * v;
            lv += (float)(kSample * (kSample - 1)) * cl * v * v;
          }
        }
        float xs = le;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float y = __shfl_up_sync(0xffffffffu, xs, o);
          if (lane >= o) xs += y;
        }
        const float wv = warp_sum(lv);
        if (lane == 31) sh.fw[warp] = xs;
        if (lane == 0) sh.fv[warp] = wv;
        __syncthreads();
        float ft = lane < nw ? sh.fw[lane] : 0.f;
        const float tv = warp_sum(lane < nw ? sh.fv[lane] : 0.f);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float y = __shfl_up_sync(0xffffffffu, ft, o);
          if (lane >= o) ft += y;
        }
        const float te = __shfl_sync(0xffffffffu, ft, 31);
        const float wpf = __shfl_sync(0xffffffffu, ft, (warp + 31) & 31);
        const float pf = a.p;
        const float delta = 3.f * sqrtf(tv) + te * ldexpf(1.f, s - 24) + 1e-7f * pf;
        float run = (warp ? wpf : 0.f) + (xs - le);
        int b_hi = -1, b_lo = -1;  // this thread's first bin reaching p - delta, p + delta
        for (int e = 0; e < per; ++e) {
          const int b = b0 - e;
          const int pk = (int)win + b;
          const float ch = (float)csum32(saddr(rA + b), C);
          const float cl = kSample > 1 ? (float)csum32(saddr(rA + kNB + b), C) : 0.f;
          if (pk >= 0 && ch + cl > 0.f) {
            const float v = __uint_as_float(((uint32_t)pk << s) + ((1u << s) >> 1));
            run += (ch + (float)kSample * cl) * v;
          }
          if (b_hi < 0 && run >= pf - delta) b_hi = b;
          if (b_lo < 0 && run >= pf + delta) b_lo = b;
        }
        // the highest such bin over the block: one shared atomic per warp (every thread past the
        // crossing has one, so a per-thread atomic would serialise on one word)
        b_hi = __reduce_max_sync(0xffffffffu, b_hi);
        b_lo = __reduce_max_sync(0xffffffffu, b_lo);
        if (lane == 0) {
          if (b_hi >= 0) atomicMax(&sh.bhi, b_hi);
          if (b_lo >= 0) atomicMax(&sh.blo, b_lo);
        }
      }
      __syncthreads();
      // key range [lo_key, hi_key], then aligned to whole bins of the exact histogram
      const int bhi = min(kNB - 1, max(sh.bhi, 0) + 1), blo = max(0, sh.blo - 1);
      long long lo_key = max((long long)kL, (long long)((int)win + blo) << s);
      long long hi_key = ((((long long)((int)win + bhi)) + 1) << s) - 1;
      if (hi_key > (long long)kt) hi_key = kt;
      if (lo_key > hi_key) lo_key = hi_key;
      TWL_PRUNE_STAMP(10);
      if (C == 1) clear_u32(rC, 2 * kNB);  // rC = rA: its last reads were behind the barrier
      bool found = false, exact_above = false, use_list = false, m_pending = false;
      int nlist = 0;
      uint32_t t_found = 0u;
      m = 0.f;
#pragma unroll 1
      for (int tries = 0; tries < 64 && !found; ++tries) {
        TWL_PRUNE_STAMP(3);
        if (t == 0) sh.gcount = 0;  // published by the exact pass's barriers (cluster: its csync)
        // ---- exact pass over [klo, khi]
        int sb = span_shift((uint32_t)lo_key, (uint32_t)hi_key);
        if (sb > kMaxBinShift) {  // keep the upper part; a miss moves the range down
          lo_key = hi_key - ((long long)kNB << kMaxBinShift) + 1;
          sb = span_shift((uint32_t)lo_key, (uint32_t)hi_key);
        }
        const uint32_t klo = ((uint32_t)lo_key >> sb) << sb;
        const uint32_t khi = (((uint32_t)hi_key >> sb) << sb) | ((1u << sb) - 1u);
        const float fkhi = __uint_as_float(khi);  // khi lies below the first infinite pattern
        const uint32_t fc = saddr(rB);
        double above_t;
        if (!exact_above) {
          // pairwise: quads, then a tree over the 8 quads (depth 5)
          float c[kRounds];
#pragma unroll
          for (int k = 0; k < kRounds; ++k) {
            const float y0 = x[4 * k] > fkhi ? x[4 * k] : 0.f;
            const float y1 = x[4 * k + 1] > fkhi ? x[4 * k + 1] : 0.f;
            const float y2 = x[4 * k + 2] > fkhi ? x[4 * k + 2] : 0.f;
            const float y3 = x[4 * k + 3] > fkhi ? x[4 * k + 3] : 0.f;
            c[k] = (y0 + y1) + (y2 + y3);
          }
#pragma unroll
          for (int w = kRounds / 2; w >= 1; w >>= 1)
#pragma unroll
            for (int i = 0; i < w; ++i) c[i] += c[i + w];
          above_t = (double)c[0];
        } else {
          above_t = 0.0;
#pragma unroll
          for (int i = 0; i < kRE; ++i) above_t += x[i] > fkhi ? (double)x[i] : 0.0;
        }
        const uint32_t lm = (1u << sb) - 1u, k0 = klo >> sb;
        // the weights in range go to this thread's list (a store per weight, no branch)
        const int cap = a.list_cap;
        nlist = 0;
#pragma unroll
        for (int i = 0; i < kRE; ++i) {
          const uint32_t u = __float_as_uint(x[i]);
          const bool in = u - klo <= khi - klo;
          sts32(a_list + 4u * T * (in ? min(nlist, cap) : cap), u);
          nlist += in ? 1 : 0;
        }
        // per-warp partial sums of the mass above (fixed order)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) above_t += __shfl_xor_sync(0xffffffffu, above_t, o);
        if (lane == 0) sh.wpart[warp] = above_t;
        TWL_PRUNE_STAMP(11);
        // each thread takes its histogram adds from its list, or from its registers when its list
        // overflowed (the histogram is the same either way)
        use_list = nlist <= cap;
        if (use_list) {
          for (int j = 0; j < nlist; ++j) {
            const uint32_t u = lds32(a_list + 4u * T * j);
            const uint32_t ad = fc + 4u * ((u >> sb) - k0);
            red_add_u(ad, 1u);
            red_add_u(ad + 4u * kNB, u & lm);
          }
        } else {
#pragma unroll
          for (int i = 0; i < kRE; ++i) {
            const uint32_t u = __float_as_uint(x[i]);
            const bool in = u - klo <= khi - klo;
            const uint32_t ad = fc + 4u * ((u >> sb) - k0);
            red_add(ad, 1u, in);
            red_add(ad + 4u * kNB, u & lm, in && lm);
          }
        }
        __syncthreads();  // the exact histogram and the per-warp sums are complete
        TWL_PRUNE_STAMP(12);
        double above = lane < nw ? sh.wpart[lane] : 0.0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) above += __shfl_xor_sync(0xffffffffu, above, o);
        if (C > 1) {
          if (t == 0) sh.cta_above = above;
          csync();
          above = 0.0;
          for (int qq = 0; qq < C; ++qq) {
            const uint32_t ad = mapa(saddr(&sh.cta_above), qq);
            above += __longlong_as_double((long long)ldc64(ad));
          }
        }
        // bound on the fp32 pairwise sums (depth 5): 5 * 2^-24 of the mass, rounded up
        const double err = exact_above ? 0.0 : above * 0x1p-21;
        bool up = false, redo = false, used_levels = false;
        TWL_PRUNE_STAMP(4);
        if (above - err >= P) {
          up = true;  // T lies above the range
        } else if (above >= P || above + err >= P) {
          redo = true;  // too close to call with the fp32 part
        } else {
          // masses of the exact bins in units of the range's lowest exponent (the range spans at
          // most kNB x 2^kMaxBinShift <= 2^27 patterns = 16 binades: below 2^59 per bin)
          const int e_lo = max((int)(klo >> 23), 1);
          const double unit = pow2d(e_lo - 150);
          const double need = (P - above) / unit;
          const uint64_t R = need >= 1.8e19 ? ~0ull : (uint64_t)ceil(need);
          auto mass = [&](int b, uint64_t* c, uint64_t* sm) -> uint64_t {
            *c = csum32(fc + 4u * b, C);
            *sm = sb ? csum32(fc + 4u * (kNB + b), C) : 0ull;
            return bin_units(klo + ((uint32_t)b << sb), *c, *sm, e_lo);
          };
          level_cross((int)((khi >> sb) - (klo >> sb)) + 1, max(R, (uint64_t)1), mass, sh);
          const Cross F = sh.cr;
          if (F.bin >= 0) {
            found = true;
            const uint32_t pf0 = (klo >> sb) + (uint32_t)F.bin;  // prefix of the bin at sb
            uint32_t Tbits;
            double a_gt = above + (double)F.above * unit, a_mass = (double)F.mass * unit;
            if (F.cnt == 1 || sb == 0) {
              Tbits = (pf0 << sb) | (uint32_t)F.sum;
            } else if (F.cnt <= 32) {
              // ---- few weights in the crossing bin: gather them (from the lists, into the first
              // CTA of the cluster) and rank them in one warp (exact integer masses in units of
              // the bin's exponent)
              const int e_f = max((int)((pf0 << sb) >> 23), 1);
              const int sh_f = e_f - e_lo;
              const double unit_f = pow2d(e_f - 150);
              const uint64_t R1 = ((max(R, (uint64_t)1) - F.above) + ((1ull << sh_f) - 1ull)) >> sh_f;
              const uint32_t a_gc = mapa(saddr(&sh.gcount), 0), a_ga = mapa(saddr(sh.gather), 0);
              if (use_list) {
                for (int j = 0; j < nlist; ++j) {
                  const uint32_t u = lds32(a_list + 4u * T * j);
                  if ((u >> sb) == pf0) {
                    const uint32_t g = atomc_add32(a_gc, 1u);
                    if (g < 32u) stc32(a_ga + 4u * g, u);
                  }
                }
              } else {
#pragma unroll
                for (int i = 0; i < kRE; ++i) {
                  const uint32_t u = __float_as_uint(x[i]);
                  if ((u >> sb) == pf0) {  // a finite prefix: NaN never matches
                    const uint32_t g = atomc_add32(a_gc, 1u);
                    if (g < 32u) stc32(a_ga + 4u * g, u);
                  }
                }
              }
              __syncthreads();
              if (C > 1) csync();
              if (q == 0 && warp == 0) {
                const int gc = min(sh.gcount, 32);
                const uint32_t v = lane < gc ? sh.gather[lane] : 0u;
                const bool ok = lane < gc;
                // mass of the gathered weights >= v, and > v
                uint64_t ge = 0, gt = 0;
                for (int j = 0; j < gc; ++j) {
                  const uint32_t w = __shfl_sync(0xffffffffu, v, j);
                  const uint64_t mw = (w & 0x7FFFFFu) | ((w >> 23) ? 0x800000u : 0u);
                  ge += w >= v ? mw : 0ull;
                  gt += w > v ? mw : 0ull;
                }
                // T = the largest gathered value whose mass from the top reaches R1
                const uint32_t cand = (ok && ge >= R1) ? v : 0u;
                const uint32_t tv = __reduce_max_sync(0xffffffffu, cand);
                const uint32_t at_t = __ballot_sync(0xffffffffu, ok && v == tv);  // every lane
                if (ok && v == tv && lane == __ffs(at_t) - 1) {
                  sh.g_t = tv;
                  sh.g_gt = gt;
                  sh.g_eq = ge - gt;
                }
              }
              __syncthreads();
              if (C > 1) {
                csync();
                const uint32_t a0 = mapa(saddr(&sh.g_t), 0);
                Tbits = ldc32(a0);
                const uint64_t g_gt = ldc64(mapa(saddr(&sh.g_gt), 0));
                const uint64_t g_eq = ldc64(mapa(saddr(&sh.g_eq), 0));
                a_gt += (double)g_gt * unit_f;
                a_mass = (double)g_eq * unit_f;
              } else {
                Tbits = sh.g_t;
                a_gt += (double)sh.g_gt * unit_f;
                a_mass = (double)sh.g_eq * unit_f;
              }
            } else {
              // ---- refinement levels on the crossing bin's weights (one exponent: unit 2^(e-150))
              TWL_PRUNE_STAMP(5);
              used_levels = true;
              if (C > 1) csync();  // after this no CTA reads A, which may serve level 2
              clear_u32(rD, 2 * kNB);
              const int e_f = max((int)((pf0 << sb) >> 23), 1);
              const int sh_f = e_f - e_lo;  // fine units per bin unit: 2^sh_f
              const double unit_f = pow2d(e_f - 150);
              const uint64_t R1 = ((max(R, (uint64_t)1) - F.above) + ((1ull << sh_f) - 1ull)) >> sh_f;
              const int s2 = max(0, sb - kNBBits);
              prefix_level(x, use_list, a_list, nlist, pf0, sb, s2, saddr(rC), max(R1, (uint64_t)1), C,
                           sh);
              const Cross S = sh.cr;
              const uint32_t pf1 = (pf0 << (sb - s2)) | (uint32_t)max(S.bin, 0);
              if (S.bin < 0) {  // unreachable: the finer bins sum exactly to the crossing bin
                Tbits = pf0 << sb;
              } else if (S.cnt == 1 || s2 == 0) {
                Tbits = (pf1 << s2) | (uint32_t)S.sum;
                a_gt += (double)S.above * unit_f;
                a_mass = (double)S.mass * unit_f;
              } else {
                prefix_level(x, use_list, a_list, nlist, pf1, s2, 0, saddr(rD),
                             max(R1 - S.above, (uint64_t)1), C, sh);
                const Cross V = sh.cr;
                Tbits = (pf1 << s2) | (uint32_t)max(V.bin, 0);
                a_gt += (double)S.above * unit_f;
                a_mass = (double)S.mass * unit_f;
                if (V.bin >= 0) {
                  a_gt += (double)V.above * unit_f;
                  a_mass = (double)V.mass * unit_f;
                }
              }
            }
            // T is certain unless p lies within the fp32 bound of the masses that decided it
            if (!exact_above && !(P - a_gt > err && a_gt + a_mass - P >= err)) {
              found = false;
              redo = true;
            } else {
              t_found = Tbits;
              m_pending = true;
            }
          }
        }
        if (!found) {
          // prepare the next pass: the same range with fp64 sums, or the range moved (up when the
          // mass above it reaches p, else down)
          if (C > 1) csync();  // every CTA is done reading this pass's histograms
          clear_u32(rB, 2 * kNB);
          if (used_levels) clear_u32(rC, 2 * kNB);
          if (redo) {
            exact_above = true;
          } else {
            const long long span = 2 * ((long long)khi - (long long)klo + 1);
            if (up) {
              lo_key = (long long)khi + 1;
              hi_key = min((long long)kt, (long long)khi + span);
              if (lo_key > (long long)kt) {  // cannot happen: the mass above top is zero
                found = true;
                m = top;
              }
            } else if (klo == 0u) {  // the whole row's mass is below p
              found = true;
              m = 0.f;
            } else {
              hi_key = (long long)klo - 1;
              lo_key = max(0ll, hi_key - span + 1);
            }
          }
          __syncthreads();
        }
      }
      TWL_PRUNE_STAMP(13);
      if (m_pending) {  // the scalar replay of the bisection, once per CTA
        if (t == 0) sh.m = bisect_scalar(top, __uint_as_float(t_found), a.eps);
        __syncthreads();
        m = sh.m;
      }
    }
    TWL_PRUNE_STAMP(6);

    // pass D: kept = {W >= m}
    uint64_t keepmask = 0ull;
#pragma unroll
    for (int i = 0; i < kRE; ++i) keepmask |= (x[i] >= m ? 1ull : 0ull) << i;
    if (C == 1) {
      // every read of this row's histograms and top happened before the barriers above; the
      // barriers of the count below publish the clears before the next row's adds
      clear_u32(rA, 2 * kNB * nreg);
      if (t == 0) sh.top_key = 0u;
    }
    uint32_t rbase[kRounds];
    uint32_t cta_total = 0;
    u128 pre[(kRounds + 7) / 8];
    if (a.kept_idx) {
      // ascending indices: per round k (chunks of 4 weights) the thread's count takes a 16-bit
      // field of a 128-bit word (8 rounds per word); one exclusive scan places them all
      constexpr int kWords = (kRounds + 7) / 8;
      u128 packed[kWords];
#pragma unroll
      for (int w = 0; w < kWords; ++w) packed[w] = 0;
#pragma unroll
      for (int k = 0; k < kRounds; ++k)
        packed[k / 8] |= (u128)__popcll((keepmask >> (4 * k)) & 0xFull) << (16 * (k % 8));
      u128 tot[kWords];
#pragma unroll
      for (int w = 0; w < kWords; ++w) pre[w] = block_excl_u128(packed[w], sh.ush, &tot[w]);
#pragma unroll
      for (int k = 0; k < kRounds; ++k) {
        rbase[k] = cta_total;
        cta_total += (uint32_t)(tot[k / 8] >> (16 * (k % 8))) & 0xFFFFu;
      }
    } else {
      const uint32_t wc = __reduce_add_sync(0xffffffffu, (uint32_t)__popcll(keepmask));
      if (lane == 0) sh.wcnt[warp] = wc;
      __syncthreads();
      cta_total = __reduce_add_sync(0xffffffffu, lane < nw ? sh.wcnt[lane] : 0u);
    }
    uint32_t cta_base = 0, row_total = cta_total;
    if (C > 1) {
      if (t == 0)
        for (int qq = 0; qq < C; ++qq) stc32(mapa(saddr(&sh.cta_count[q]), qq), cta_total);
      csync();  // also: every CTA has finished reading this CTA's histograms
      row_total = 0;
      for (int qq = 0; qq < C; ++qq) {
        const uint32_t c = sh.cta_count[qq];
        if (qq < q) cta_base += c;
        row_total += c;
      }
    }
    if (C > 1) {
      // every read of this CTA's histograms and top, its own and the other CTAs', happened
      // before the cluster barrier above: clear them for the next row
      clear_u32(rA, 2 * kNB * nreg);
      if (t == 0) sh.top_key = 0u;
      __syncthreads();  // cleared before the next row's histograms
    }
    if (a.kept_idx && keepmask) {
      int* out = a.kept_idx + (size_t)r * a.stride;
#pragma unroll
      for (int k = 0; k < kRounds; ++k) {
        uint32_t pos = cta_base + rbase[k] + ((uint32_t)(pre[k / 8] >> (16 * (k % 8))) & 0xFFFFu);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if ((keepmask >> (4 * k + j)) & 1ull) out[pos++] = s0 + 4 * (k * T + t) + j;
      }
    }
    TWL_PRUNE_STAMP(7);
    if (q == 0 && t == 0) {
      a.m_out[r] = m;
      a.kept_count[r] = (int)row_total;
    }
  }
  cp_async_wait_all();  // nothing is in flight at exit
}

struct RowsPlan {
  int threads, cluster, grid, list_cap;
  size_t smem;
};

// Dynamic shared memory: the prefetch buffer, the histogram regions, 32 dummy words, and the
// exact pass's lists ((list_cap + 1) x threads words).
size_t rows_smem(int threads, int cluster, int list_cap) {
  return (size_t)16 * kRounds * threads + (size_t)4 * 2 * kNB * (cluster > 1 ? 3 : 2) + 128 +
         (size_t)4 * (list_cap + 1) * threads;
}

// List entries per thread: what fits beside the CTAs an SM holds at 64 registers per thread
// (1024 / threads of them), between 4 and 16.
int rows_list_cap(int threads, int cluster) {
  const int ctas = max(1, 32768 / kRE / threads);  // CTAs per SM at 2 kRE registers per thread
  const size_t per_cta = (size_t)(227 * 1024) / ctas - 2048;  // static shared memory and reserve
  const size_t fixed = rows_smem(threads, cluster, -1);
  const long long cap = per_cta > fixed ? (long long)((per_cta - fixed) / (4 * threads)) - 1 : 0;
  return (int)min(16ll, cap);
}

}  // namespace

#ifndef TWL_PRUNE_NS
#define TWL_PRUNE_NS rows32
#endif
namespace TWL_PRUNE_NS {

// Plan for rows of `stride` weights: 0 threads when this kernel does not apply.
static RowsPlan plan_rows(int rows, int stride) {
  RowsPlan pl{0, 0, 0, 0, 0};
  if (stride < 1 || stride > kRSlice * kRMaxCluster || (stride & 3)) return pl;
  int threads = 32;
  while (threads < kRMaxThreads && threads * kRE < stride) threads <<= 1;
  const int cluster = (stride + threads * kRE - 1) / (threads * kRE);
  pl.threads = threads;
  pl.cluster = cluster;
  pl.list_cap = max(4, rows_list_cap(threads, cluster));
  pl.smem = rows_smem(threads, cluster, pl.list_cap);
  // persistent grid: as many CTAs (clusters) as are resident at once, at most one per row;
  // the residency is cached per (device, threads, cluster), under a lock for concurrent callers
  static std::mutex mu;
  static long long cache_key[32];
  static int cache_val[32];
  static int cache_n = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  const long long key = ((long long)dev << 32) | (long long)(threads * 16 + cluster);
  std::lock_guard<std::mutex> lock(mu);
  int per = -1;
  for (int i = 0; i < cache_n; ++i)
    if (cache_key[i] == key) per = cache_val[i];
  if (per < 0) {
    cudaFuncSetAttribute(k_prune_rows, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)pl.smem);
    if (cluster == 1) {
      int nb = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, k_prune_rows, threads, pl.smem) !=
          cudaSuccess)
        nb = 0;
      per = nb * num_sms();
    } else {
      if (cluster > 8)
        cudaFuncSetAttribute(k_prune_rows, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)cluster);
      cfg.blockDim = dim3((unsigned)threads);
      cfg.dynamicSmemBytes = pl.smem;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = (unsigned)cluster;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, k_prune_rows, &cfg) != cudaSuccess) n = 0;
      per = n;
    }
    cudaGetLastError();
    if (cache_n < 32) {
      cache_key[cache_n] = key;
      cache_val[cache_n] = per;
      ++cache_n;
    }
  }
  if (per <= 0) {
    pl.threads = 0;
    return pl;
  }
  pl.grid = min(rows, per) * cluster;
  return pl;
}

// Returns cudaErrorNotSupported (launching nothing) when the rows do not fit this kernel:
// a row stride that is not a multiple of 4 weights or above 262144, or a base that is not
// 16-byte aligned.
cudaError_t launch_prune_rows(const float* w, const int* row_len, const int* row_len_cap,
                              int rows, int row_stride, float p, float eps, float* m_out,
                              int* kept_count, int* kept_idx, cudaStream_t s) {
  if ((reinterpret_cast<uintptr_t>(w) & 15u) != 0) return cudaErrorNotSupported;
  const RowsPlan pl = plan_rows(rows, row_stride);
  if (pl.threads == 0) return cudaErrorNotSupported;
  PruneRowsArgs a{w,   row_len, row_len_cap, rows,     row_stride,
                  p,   eps,     m_out,       kept_count, kept_idx, pl.list_cap};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)pl.grid);
  cfg.blockDim = dim3((unsigned)pl.threads);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)pl.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaFuncSetAttribute(k_prune_rows, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)pl.smem);
  if (e != cudaSuccess) return e;
  e = cudaLaunchKernelEx(&cfg, k_prune_rows, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace TWL_PRUNE_NS
}  // namespace twl
