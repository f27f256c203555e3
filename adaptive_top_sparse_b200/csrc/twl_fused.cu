// The fused decode step: select -> INT4 estimate -> top-p prune -> group union -> attention in one
// kernel, one thread-block cluster per (sequence, kv-head) group.
//
// "Twilight: Adaptive Attention Sparsity with Hierarchical Top-p Pruning": notes page, "Overall
// framework" (select-then-prune) and "Key designs" (binary-search top-p, 4-bit K cache, head
// flattening); summary, sections 4.1-4.3 and appendices B.1-B.2 (INT4 SpGEMV once per GQA group
// over the union of the heads' pages, group-wise variable-length attention).
//
// Every dependency of the path stays inside one GQA group, so a group is processed by one cluster
// of C CTAs (up to 16 at batch 1, down to 1 when there are enough groups to fill the GPU), and the
// phases are separated by hardware cluster barriers instead of kernel boundaries:
//   1 scores   CTA r scores pages [r P/C, (r+1) P/C) of every head of the group  -> L2
//   2 top-k    one owner CTA per head selects its k pages (histogram passes over the keys, then
//              an exact ranking of the last bin)                                 -> page bitmap
//   3 union    every CTA ORs the head bitmaps; ranks come from prefix popcounts
//   4 estimate CTA r takes an even share of the union pages; a warp runs the INT4 dequant-dot
//              of two pages at a time on the tensor cores for all heads that selected them
//                                                  -> logits; per-CTA maxima -> owners' smem
//   5 prune    the owner CTA of each head normalises its weights, finds the top-p threshold and
//              writes the bitmap of kept candidate rows
//   6 union    CTA r ORs the heads' kept bits on its pages (with stats: counts are exchanged,
//              then the group's kept tokens are written in ascending order)
//   7 attend   CTA r gathers its kept K/V rows; partial (o, lse) per CTA
//   8 merge    the owner CTA of each head merges the C partials by log-sum-exp.
// Data that crosses CTAs goes through global memory (it stays in L2) with L1-bypassing loads,
// except the per-CTA logit maxima, which are stored into the owner's shared memory; the cluster
// barrier's release/acquire orders both.  Every CTA executes every barrier: no barrier sits
// behind a data-dependent branch, and a group whose sequence is invalid exits before the first
// one, uniformly across its cluster.  The score arithmetic and summation order match the staged
// kernels, so the selection is bit-identical to twl_select_pages.
#include <stdlib.h>

#include "twl_common.cuh"
#include "twl_fused.h"
#include "twl_kernels.h"

namespace twl {
namespace {

#ifndef TWL_FUSED_THREADS
#define TWL_FUSED_THREADS 512
#endif
#ifndef TWL_FUSED_NS
#define TWL_FUSED_NS fused512
#endif
constexpr int kThreads = TWL_FUSED_THREADS;  // 512, or 256 for two CTAs per SM at large batch
static_assert(kThreads == 512 || kThreads == 256, "512 or 256 threads per CTA");
constexpr int kWarps = kThreads / 32;
constexpr int kAttChunk = kThreads / 8;   // tokens gathered per attention round
constexpr int kQuarters = kThreads / 128;  // token groups of the P.V product

// Cluster barrier: arrive with release, wait with acquire semantics (orders shared, distributed
// shared and global memory accesses of the cluster's CTAs across it).
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
  uint32_t n;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(n));
  return n;
}

// Distributed shared memory: a CTA's shared address mapped into cluster CTA `rank`, and stores /
// atomics through such an address.  Ordered for the target CTA by the next cluster barrier
// (arrive has release, wait has acquire semantics).
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ uint32_t map_rank(uint32_t addr, int rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_cluster(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
// Exchange slots (shared memory, written by the other CTAs of the cluster): one per head that the
// CTA owns (heads r, r + C, ...), holding the C per-CTA maxima of the head's logits.
constexpr int kXchgSlot = 64;                // [16] floats
constexpr int kXchgBytes = 8 * kXchgSlot;    // up to 8 owned heads

// Optional phase timestamps (compile with -DTWL_PHASE_TIMING): thread 0 of the first CTA of the
// first cluster records %globaltimer at each phase boundary into the workspace header (words
// 8..63 as 64-bit values; word 1 = the cluster size launched).  Off by default.
#ifdef TWL_PHASE_TIMING
__device__ __forceinline__ void stamp(const FusedArgs& a, int slot) {
  if (blockIdx.x == 0 && threadIdx.x == 0 && a.flags) {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    reinterpret_cast<uint64_t*>(a.flags)[4 + slot] = t;
    a.flags[1] = cluster_size();
  }
}
#else
__device__ __forceinline__ void stamp(const FusedArgs&, int) {}
#endif

__device__ __forceinline__ float ldcg_f(const float* p) { return __ldcg(p); }

__device__ __forceinline__ int ldcg_i(const int* p) { return __ldcg(p); }
__device__ __forceinline__ uint32_t ldcg_u(const uint32_t* p) { return __ldcg(p); }

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// B fragments of the query for the m16n8k16 products: lane (g, t) holds the channels
// c0 = 32 t + 8 w8 (w8 = ks / 2) of its head; k-step ks pairs (c0 + 4e, c0 + 4e + 2) and
// (c0 + 4e + 1, c0 + 4e + 3), e = ks % 2, the same pairs nibble_pairs() builds from K.
// Also returns the sum of the lane's 32 query channels (for the zero-point term).
__device__ __forceinline__ float q_fragments(const uint16_t* qh, bool valid, uint32_t (&bf)[8][2]) {
  const int t = threadIdx.x & 3;
  uint32_t w[16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 v =
        valid ? *reinterpret_cast<const uint4*>(qh + 32 * t + 8 * i) : make_uint4(0, 0, 0, 0);
    w[4 * i + 0] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
  }
  float qsum = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
    qsum += f.x + f.y;
  }
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const int w8 = ks >> 1, e = ks & 1;
    bf[ks][0] = __byte_perm(w[4 * w8 + 2 * e], w[4 * w8 + 2 * e + 1], 0x5410);
    bf[ks][1] = __byte_perm(w[4 * w8 + 2 * e], w[4 * w8 + 2 * e + 1], 0x7632);
  }
  return qsum;
}

// Nibbles to fp16 without arithmetic: a byte 0000nnnn read as FP8 E4M3 (sign 0, exponent 000n3,
// mantissa n2 n1 n0) is n * 2^-9 exactly (subnormal m * 2^-9 for n < 8, (8 + m) * 2^-9 for
// n >= 8), and that is an exact fp16 value.  A word of 8 nibbles (channels c0..c0+7, low nibble
// first) gives the bytes (n0, n2, n4, n6) and (n1, n3, n5, n7); each 16-bit half converts to
// one f16x2 pair.  Products with q are therefore 2^-9 times the integer-nibble products, and the
// fp32 sums scale exactly; the epilogue multiplies by 512.
__device__ __forceinline__ uint32_t e4m3x2_lo(uint32_t y) {
  uint32_t r;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, l;\n\t}"
      : "=r"(r)
      : "r"(y));
  return r;
}
__device__ __forceinline__ uint32_t e4m3x2_hi(uint32_t y) {
  uint32_t r;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, h;\n\t}"
      : "=r"(r)
      : "r"(y));
  return r;
}
// The four A registers of k-step (w8, e) for rows g (word x0) and g + 8 (word x1).
__device__ __forceinline__ void nibble_pairs(uint32_t x0, uint32_t x1, int e, uint32_t (&av)[4]) {
  const uint32_t e0 = x0 & 0x0F0F0F0Fu, o0 = (x0 >> 4) & 0x0F0F0F0Fu;
  const uint32_t e1 = x1 & 0x0F0F0F0Fu, o1 = (x1 >> 4) & 0x0F0F0F0Fu;
  av[0] = e ? e4m3x2_hi(e0) : e4m3x2_lo(e0);
  av[1] = e ? e4m3x2_hi(e1) : e4m3x2_lo(e1);
  av[2] = e ? e4m3x2_hi(o0) : e4m3x2_lo(o0);
  av[3] = e ? e4m3x2_hi(o1) : e4m3x2_lo(o1);
}

// Bytes of the persistent bitmap region, rounded up so the scratch region after it is 128-byte
// aligned (the attention phase does 16-byte vector and cp.async accesses into it).
__host__ __device__ constexpr int bitmap_bytes(int g, int sel_words) {
  return ((4 * (2 * g + 2) * sel_words) + 127) & ~127;
}
__host__ __device__ constexpr int persistent_bytes(int g, int sel_words) {
  return bitmap_bytes(g, sel_words) + kXchgBytes;
}

// Shared-memory layout: a persistent region for the page bitmaps (phases 3-6) and one scratch
// region reused by the phases.
struct Smem {
  const int* pt;    // the sequence's page table (validated; -1 = bad entry), or nullptr
  const uint16_t* q;  // [G][128] the group's queries (fp16), staged once
  uint32_t* hbits;  // [G][nw]  head page bitmaps
  int* hpre;        // [G][nw]  exclusive prefix popcounts per word
  uint32_t* ubits;  // [nw]     union bitmap
  int* upre;        // [nw]     exclusive prefix popcounts of the union
  unsigned char* xchg;  // exchange slots of the heads this CTA owns
  unsigned char* scratch;
  int scratch_bytes;
  int nw;
};

__device__ __forceinline__ int rank_in(const uint32_t* bits, const int* pre, int j) {
  const int w = j >> 5, b = j & 31;
  return pre[w] + __popc(bits[w] & ((1u << b) - 1u));
}

// Position of the k-th (0-based) set bit of w; requires popc(w) > k.
__device__ __forceinline__ int nth_set_bit(uint32_t w, int k) {
  int pos = 0;
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) {
    const int c = __popc(w & ((1u << s) - 1u));
    if (k >= c) {
      k -= c;
      w >>= s;
      pos += s;
    }
  }
  return pos;
}

// j of the u-th set bit of the union (u < total), via binary search over the prefix table.
__device__ __forceinline__ int union_select(const uint32_t* ubits, const int* upre, int nw, int u) {
  int lo = 0, hi = nw;  // upre[lo] <= u < upre[hi] (upre[nw] = total implied)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (upre[mid] <= u) lo = mid;
    else hi = mid;
  }
  return 32 * lo + nth_set_bit(ubits[lo], u - upre[lo]);
}

// Physical page of logical page j: from the staged copy when there is one.
__device__ __forceinline__ int phys_of(const FusedArgs& a, const Smem& sm, int b, int j) {
  if (sm.pt) return sm.pt[j];
  return load_phys(a.kv.page_table, b, j, a.kv.max_pages, a.kv.num_phys, a.flags);
}

// ------------------------------------------------------------------------- phase 1: scores
// The bounds of the CTA's pages (512 B per page) are copied into shared memory in chunks with
// 16-byte cp.async spread over all threads (one memory round trip per chunk); a half-warp then
// scores a page for all G heads.
template <int G>
__device__ void phase_scores(const FusedArgs& a, int b, int kvh, int n_pages, int r, int C,
                             Smem& sm) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int half = lane >> 4, l = lane & 15;
  const int p0 = (int)((long)n_pages * r / C), p1 = (int)((long)n_pages * (r + 1) / C);
  float qv[G][8];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const uint4 raw = *reinterpret_cast<const uint4*>(
        sm.q + h * kHeadDim + 8 * l);
    unpack8(raw, qv[h]);
  }
  int* phys = reinterpret_cast<int*>(sm.scratch);
  const int cap = (sm.scratch_bytes - 128) / (4 + 512);
  const int ch = cap < 1024 ? cap : 1024;
  unsigned char* buf = sm.scratch + ((4 * ch + 127) & ~127);
#pragma unroll 1
  for (int c0 = p0; c0 < p1; c0 += ch) {
    const int cn = min(ch, p1 - c0);
    for (int i = threadIdx.x; i < cn; i += kThreads)
      phys[i] = phys_of(a, sm, b, c0 + i);
    __syncthreads();
    // 32 chunks of 16 bytes per page, spread over all threads, all in flight together
    for (int c = threadIdx.x; c < 32 * cn; c += kThreads) {
      const int i = c >> 5, k = c & 31;
      const int ph = phys[i];
      const uint16_t* src =
          ph >= 0 ? a.bounds + ((size_t)ph * a.kv.hkv + kvh) * 2 * kHeadDim + 8 * k : a.bounds;
      cp_async16(buf + 512 * i + 16 * k, src, ph >= 0);
    }
    cp_async_commit();
    cp_async_wait_all();
    __syncthreads();
    const bool ok = true;
    for (int base = 0; base < cn; base += 2 * kWarps) {  // warp-uniform trip count
      const int i0 = base + 2 * warp + half;
      const bool in = i0 < cn;
      const int ph = in ? phys[i0] : -1;
      uint4 vmn = make_uint4(0, 0, 0, 0), vmx = vmn;
      if (ph >= 0 && ok) {
        vmn = *reinterpret_cast<const uint4*>(buf + 512 * i0 + 16 * l);
        vmx = *reinterpret_cast<const uint4*>(buf + 512 * i0 + 256 + 16 * l);
      }
      float mn[8], mx[8];
      unpack8(vmn, mn);
      unpack8(vmx, mx);
      float acc[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float sc = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) sc = __fmaf_rn(qv[h][c], qv[h][c] > 0.f ? mx[c] : mn[c], sc);
        acc[h] = sc;
      }
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) {
#pragma unroll
        for (int h = 0; h < G; ++h)
          acc[h] = __fadd_rn(acc[h], __shfl_xor_sync(0xffffffffu, acc[h], off));
      }
      if (in && l < G) {
        float v = acc[0];
#pragma unroll
        for (int h = 1; h < G; ++h) v = (l == h) ? acc[h] : v;
        if (ph < 0) v = -INFINITY;
        a.scores[((size_t)b * a.hq + kvh * G + l) * a.kv.max_pages + c0 + i0] = v;
      }
    }
    __syncthreads();  // the chunk's buffer is read before the next copies land
  }
}

// ------------------------------------------------------------------------- phase 2: top-k
// Radix select of the kb largest keys (ties to the lower index) -> bitmap of selected pages.
__device__ void phase_topk_head(const FusedArgs& a, int bh, int n_pages, int kb, Smem& sm) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nw = sm.nw;
  uint32_t* out_bits = a.selbits + (size_t)bh * a.sel_words;
  int* sel_list = a.sel_pages ? a.sel_pages + (size_t)bh * a.max_budget : nullptr;
  if (n_pages <= kb) {
    for (int w = tid; w < nw; w += kThreads) {
      const int lo = 32 * w;
      uint32_t m = 0xFFFFFFFFu;
      if (lo + 32 > n_pages) m = n_pages > lo ? ((1u << (n_pages - lo)) - 1u) : 0u;
      out_bits[w] = m;
    }
    if (sel_list)
      for (int i = tid; i < n_pages; i += kThreads) sel_list[i] = i;
    if (tid == 0 && a.sel_count) a.sel_count[bh] = n_pages;
    return;
  }
  // the keys in shared memory (the launch plan guarantees room for max_pages of them)
  const float* row = a.scores + (size_t)bh * a.kv.max_pages;
  uint32_t* hist = reinterpret_cast<uint32_t*>(sm.scratch);           // 256
  int* scan_sh = reinterpret_cast<int*>(sm.scratch + 1024);           // 33
  uint32_t* state = reinterpret_cast<uint32_t*>(sm.scratch + 1200);   // 3
  uint32_t* keys = reinterpret_cast<uint32_t*>(sm.scratch + 1280);
  {
    constexpr int kB = 8;  // independent loads in flight per thread
    for (int base = 0; base < n_pages; base += kThreads * kB) {
      float v[kB];
#pragma unroll
      for (int k = 0; k < kB; ++k) {
        const int i = base + k * kThreads + tid;
        v[k] = i < n_pages ? ldcg_f(row + i) : 0.f;
      }
#pragma unroll
      for (int k = 0; k < kB; ++k) {
        const int i = base + k * kThreads + tid;
        if (i < n_pages) keys[i] = f32_key(v[k]);
      }
    }
  }
  __syncthreads();
  auto key_at = [&](int i) -> uint32_t { return keys[i]; };

  // The k-th largest key is narrowed down to a key interval [blo, bhi] holding `cand` keys, of
  // which the `remaining` largest are selected (every key above bhi is selected).  It starts as
  // [min key, max key]; each pass histograms the keys inside it into up to 4096 bins of equal key
  // width (offsets from blo, shifted right) and keeps the bin holding the k-th key.  Keys are
  // monotone in the score and roughly logarithmic in its magnitude, so one pass usually leaves a
  // handful of candidates.
  constexpr int kGatherCap = 64;
  constexpr int kBins = 4096;
  uint32_t* bhist = reinterpret_cast<uint32_t*>(sm.scratch + 1280 + 4 * n_pages);  // [kBins]
  uint32_t* gkey = bhist + kBins;                                                  // [cap]
  int* gidx = reinterpret_cast<int*>(gkey + kGatherCap);                           // [cap]
  uint32_t* sbits = reinterpret_cast<uint32_t*>(gidx + kGatherCap);                // [nw]
  const bool room = 1280 + 4 * (size_t)n_pages + 4 * kBins + 8 * kGatherCap + 4 * nw + 16 <=
                    (size_t)sm.scratch_bytes;
  uint32_t* hh = room ? bhist : hist;  // the 256-bin histogram when there is no room
  const int nbins = room ? kBins : 256;
  const int bin_bits = room ? 12 : 8;
  const int per = nbins / kThreads > 0 ? nbins / kThreads : 1;  // bins per thread in the scan
  uint32_t blo, bhi;
  {
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
    for (int i = tid; i < n_pages; i += kThreads) {
      const uint32_t k = key_at(i);
      kmin = min(kmin, k);
      kmax = max(kmax, k);
    }
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    if (lane == 0) {
      hist[2 * warp] = kmin;
      hist[2 * warp + 1] = kmax;
    }
    __syncthreads();
    kmin = 0xFFFFFFFFu;
    kmax = 0u;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      kmin = min(kmin, hist[2 * w]);
      kmax = max(kmax, hist[2 * w + 1]);
    }
    blo = kmin;
    bhi = kmax;
  }
  int remaining = kb;
  int cand = n_pages;
  __syncthreads();
  const int n_it = (n_pages + kThreads - 1) / kThreads;
#pragma unroll 1
  while ((cand > kGatherCap || !room) && blo < bhi) {
    const uint32_t range = bhi - blo;
    const int width = 32 - __clz(range);
    const int sh = width > bin_bits ? width - bin_bits : 0;
    for (int i = tid; i < nbins; i += kThreads) hh[i] = 0u;
    __syncthreads();
#pragma unroll 1
    for (int it = 0; it < n_it; ++it) {
      const int i = it * kThreads + tid;
      if (i < n_pages) {
        const uint32_t key = key_at(i);
        if (key >= blo && key <= bhi) atomicAdd(&hh[(key - blo) >> sh], 1u);
      }
    }
    __syncthreads();
    // descending scan over the bins: thread t owns bins nbins-1-per*t ... nbins-per*(t+1)
    const int b0 = nbins - 1 - per * tid;
    int mine = 0;
    for (int e = 0; e < per; ++e)
      if (b0 - e >= 0) mine += (int)hh[b0 - e];
    const int excl = block_exclusive_scan(mine, scan_sh, nullptr);
    if (excl < remaining && remaining <= excl + mine) {
      int run = excl;
      for (int e = 0; e < per; ++e) {
        const int c = (int)hh[b0 - e];
        if (run + c >= remaining) {
          state[0] = (uint32_t)(b0 - e);
          state[1] = (uint32_t)(remaining - run);
          state[2] = (uint32_t)c;
          break;
        }
        run += c;
      }
    }
    __syncthreads();
    const uint32_t bin = state[0];
    const uint32_t nlo = blo + (bin << sh);
    const uint64_t top = (uint64_t)nlo + ((1ull << sh) - 1ull);
    bhi = top < (uint64_t)bhi ? (uint32_t)top : bhi;
    blo = nlo;
    remaining = (int)state[1];
    cand = (int)state[2];
    __syncthreads();
  }
  if (room && cand <= kGatherCap) {
    for (int w = tid; w < nw; w += kThreads) sbits[w] = 0u;
    // ordered gather of the bin's keys: thread t scans a contiguous range of pages
    const int per = (n_pages + kThreads - 1) / kThreads;
    const int beg = min(n_pages, tid * per), end = min(n_pages, beg + per);
    int mine = 0;
    for (int i = beg; i < end; ++i) {
      const uint32_t key = key_at(i);
      mine += key >= blo && key <= bhi;
    }
    int slot = block_exclusive_scan(mine, scan_sh, nullptr);
    for (int i = beg; i < end && mine > 0; ++i) {
      const uint32_t key = key_at(i);
      if (key >= blo && key <= bhi) {
        gkey[slot] = key;
        gidx[slot] = i;
        ++slot;
        --mine;
      }
    }
    __syncthreads();
    for (int e = tid; e < cand; e += kThreads) {
      const uint32_t ke = gkey[e];
      const int ie = gidx[e];
      int rank = 0;
      for (int f = 0; f < cand; ++f) {
        const uint32_t kf = gkey[f];
        rank += (kf > ke || (kf == ke && gidx[f] < ie)) ? 1 : 0;
      }
      if (rank < remaining) atomicOr(&sbits[ie >> 5], 1u << (ie & 31));
    }
    __syncthreads();
    for (int base = 0; base < 32 * nw; base += kThreads) {
      const int i = base + tid;
      const bool above = i < n_pages && key_at(i) > bhi;
      const uint32_t bal = __ballot_sync(0xffffffffu, above);
      if (lane == 0 && (i >> 5) < nw) sbits[i >> 5] |= bal;
    }
    __syncthreads();
    int carry = 0;
    for (int base = 0; base < nw; base += kThreads) {
      const int w = base + tid;
      const uint32_t word = w < nw ? sbits[w] : 0u;
      if (w < nw) out_bits[w] = word;
      if (sel_list) {
        int total;
        int pos = carry + block_exclusive_scan(__popc(word), scan_sh, &total);
        carry += total;
        uint32_t x = word;
        while (x) {
          sel_list[pos++] = 32 * w + __ffs(x) - 1;
          x &= x - 1u;
        }
      }
    }
    if (tid == 0 && a.sel_count) a.sel_count[bh] = kb;
    return;
  }
  // the interval is down to one key (or there is no room for the gather): blo == bhi is the
  // k-th key itself
  // Keys above the k-th are taken; equal keys are taken in ascending page order.  One element
  // per thread per round; a warp's ballot is one 32-page word of the bitmap.
  int* wsum = scan_sh;  // [kWarps] per-warp counts, then their prefix
  int carry_eq = 0, carry_sel = 0;
  const uint32_t lt = (1u << lane) - 1u;
  for (int base = 0; base < 32 * nw; base += kThreads) {
    const int i = base + tid;
    const bool in = i < n_pages;
    const uint32_t key = in ? key_at(i) : 0u;
    const uint32_t gt = __ballot_sync(0xffffffffu, in && key > bhi);
    const uint32_t eq = __ballot_sync(0xffffffffu, in && key == blo);
    if (lane == 0) wsum[warp] = __popc(eq);
    __syncthreads();
    int eq_before = carry_eq, eq_round = 0;
    for (int w = 0; w < kWarps; ++w) {
      if (w < warp) eq_before += wsum[w];
      eq_round += wsum[w];
    }
    const bool take = in && key == blo && eq_before + __popc(eq & lt) < remaining;
    const uint32_t sel = gt | __ballot_sync(0xffffffffu, take);
    __syncthreads();
    if (lane == 0) wsum[warp] = __popc(sel);
    __syncthreads();
    int sel_before = carry_sel, sel_round = 0;
    for (int w = 0; w < kWarps; ++w) {
      if (w < warp) sel_before += wsum[w];
      sel_round += wsum[w];
    }
    const int word = i >> 5;
    if (lane == 0 && word < nw) out_bits[word] = sel;
    if (sel_list && ((sel >> lane) & 1u)) sel_list[sel_before + __popc(sel & lt)] = i;
    carry_eq += eq_round;
    carry_sel += sel_round;
    __syncthreads();
  }
  if (tid == 0 && a.sel_count) a.sel_count[bh] = kb;
}

// ------------------------------------------------------------------------- phase 3: bitmaps
template <int G>
__device__ void phase_union_bitmaps(const FusedArgs& a, int b, int kvh, Smem& sm, int* s_total,
                                    int* scan_sh) {
  const int tid = threadIdx.x, nw = sm.nw;
  for (int i = tid; i < G * nw; i += kThreads) {
    const int h = i / nw, w = i % nw;
    sm.hbits[i] = ldcg_u(a.selbits + (size_t)(b * a.hq + kvh * G + h) * a.sel_words + w);
  }
  __syncthreads();
  for (int w = tid; w < nw; w += kThreads) {
    uint32_t u = 0;
#pragma unroll
    for (int h = 0; h < G; ++h) u |= sm.hbits[h * nw + w];
    sm.ubits[w] = u;
  }
  __syncthreads();
  // exclusive prefix popcounts of the union and of every head bitmap, in one scan per round
  // of kThreads words (warp scans, then the warp totals)
  int* wtot = reinterpret_cast<int*>(sm.scratch);  // [kWarps][G + 1]
  const int lane = tid & 31, warp = tid >> 5;
  int carry[G + 1];
#pragma unroll
  for (int h = 0; h <= G; ++h) carry[h] = 0;
  for (int base = 0; base < nw; base += kThreads) {
    const int w = base + tid;
    int x[G + 1], v[G + 1];
#pragma unroll
    for (int h = 0; h <= G; ++h) {
      v[h] = w < nw ? __popc(h == 0 ? sm.ubits[w] : sm.hbits[(h - 1) * nw + w]) : 0;
      x[h] = v[h];
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
      for (int h = 0; h <= G; ++h) {
        const int y = __shfl_up_sync(0xffffffffu, x[h], o);
        if (lane >= o) x[h] += y;
      }
    }
    if (lane == 31) {
#pragma unroll
      for (int h = 0; h <= G; ++h) wtot[warp * (G + 1) + h] = x[h];
    }
    __syncthreads();
    // only the warps that hold words of this round contribute
    const int active = min(kWarps, (nw - base + 31) >> 5);
#pragma unroll
    for (int h = 0; h <= G; ++h) {
      int before = carry[h], round = 0;
      for (int ww = 0; ww < active; ++ww) {
        const int t = wtot[ww * (G + 1) + h];
        if (ww < warp) before += t;
        round += t;
      }
      if (w < nw) {
        if (h == 0) sm.upre[w] = before + x[h] - v[h];
        else sm.hpre[(h - 1) * nw + w] = before + x[h] - v[h];
      }
      carry[h] += round;
    }
    __syncthreads();
  }
  if (tid == 0) *s_total = carry[0];
  __syncthreads();
}

// ------------------------------------------------------------------------- phase 4: estimate
// The CTA's share of the union is processed in chunks: every page's logical id and physical page
// are staged (thread per page), then its INT4 tile (1 KB) and scale/zero row (64 B) are copied
// into shared memory with 16-byte cp.async over all threads; one warp then computes a page.
template <int G>
__device__ void phase_estimate(const FusedArgs& a, int b, int kvh, int n, int U, int r, int C,
                               Smem& sm) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gr = lane >> 2, t = lane & 3;
  const int nw = sm.nw;
  const float inv_sqrt_d = 0.08838834764831845f;
  const int u0 = (int)((long)U * r / C), u1 = (int)((long)U * (r + 1) / C);
  float* red = reinterpret_cast<float*>(sm.scratch);  // [kWarps][8]
  const int cap = (sm.scratch_bytes - 1024 - 256) / (8 + 1088);
  const int ch = cap < 1024 ? cap : 1024;
  int* pj = reinterpret_cast<int*>(sm.scratch + 1024);  // [ch]
  int* pph = pj + ch;                                    // [ch]
  unsigned char* tiles = sm.scratch + ((1024 + 8 * ch + 127) & ~127);  // [ch][1024] nibbles
  unsigned char* szs = tiles + 1024 * ch;                              // [ch][64] scale/zero
  uint32_t bf[8][2];
  const bool head_ok = gr < G;
  const uint16_t* qh = sm.q + (head_ok ? gr : 0) * kHeadDim;
  float qs_part = q_fragments(qh, head_ok, bf);
  qs_part += __shfl_xor_sync(0xffffffffu, qs_part, 1);
  qs_part += __shfl_xor_sync(0xffffffffu, qs_part, 2);
  const float qsum0 = __shfl_sync(0xffffffffu, qs_part, (2 * t) * 4);
  const float qsum1 = __shfl_sync(0xffffffffu, qs_part, (2 * t + 1) * 4);
  // running max of this lane's two heads over its rows
  float rm[2] = {-INFINITY, -INFINITY};

#pragma unroll 1
  for (int c0 = u0; c0 < u1; c0 += ch) {
    const int cn = min(ch, u1 - c0);
    for (int i = threadIdx.x; i < cn; i += kThreads) {
      const int j = union_select(sm.ubits, sm.upre, nw, c0 + i);
      pj[i] = j;
      pph[i] = phys_of(a, sm, b, j);
    }
    __syncthreads();
    if (c0 == u0) stamp(a, 25);
      // 68 chunks of 16 bytes per page (64 of nibbles, 4 of scale/zero), spread over all threads
    for (int c = threadIdx.x; c < 68 * cn; c += kThreads) {
      const int i = c / 68, k = c - 68 * i;
      const int ph = pph[i];
      const size_t tile = ph >= 0 ? ((size_t)ph * a.kv.hkv + kvh) * kPage : 0;
      if (k < 64)
        cp_async16(tiles + 1024 * i + 16 * k, a.k_int4 + tile * (kHeadDim / 2) + 16 * k, ph >= 0);
      else
        cp_async16(szs + 64 * i + 16 * (k - 64), a.k_sz + tile * 2 + 8 * (k - 64), ph >= 0);
    }
    cp_async_commit();
    cp_async_wait_all();
    __syncthreads();
    if (c0 == u0) stamp(a, 26);
      const bool ok = true;
    // two pages per warp iteration: their mma chains and epilogues are independent
#pragma unroll 1
    for (int i0 = 2 * warp; i0 < cn; i0 += 2 * kWarps) {
      float accp[2][4];
      int jp[2];
      bool badp[2];
      uint32_t szp[2][2];
#pragma unroll
      for (int pp = 0; pp < 2; ++pp) {
        const int i = i0 + pp;
        const bool in = i < cn;
        jp[pp] = in ? pj[i] : 0;
        badp[pp] = !in || pph[i] < 0 || !ok;
        uint4 x0 = make_uint4(0, 0, 0, 0), x1 = x0;
        szp[pp][0] = szp[pp][1] = 0;
        if (!badp[pp]) {
          const uint4* tp = reinterpret_cast<const uint4*>(tiles + 1024 * i);
          x0 = tp[lane];
          x1 = tp[32 + lane];
          const uint32_t* sp = reinterpret_cast<const uint32_t*>(szs + 64 * i);
          szp[pp][0] = sp[gr];
          szp[pp][1] = sp[gr + 8];
        }
        const uint32_t r0[4] = {x0.x, x0.y, x0.z, x0.w};
        const uint32_t r1[4] = {x1.x, x1.y, x1.z, x1.w};
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const int w8 = ks >> 1, e = ks & 1;
          uint32_t av[4];
          nibble_pairs(r0[w8], r1[w8], e, av);
          mma_16816(acc, av, bf[ks][0], bf[ks][1]);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) accp[pp][k] = acc[k];
      }
#pragma unroll
      for (int pp = 0; pp < 2; ++pp) {
        if (i0 + pp >= cn) break;  // warp-uniform
        const int j = jp[pp];
        const bool bad = badp[pp];
        const int rows = page_rows(n, j);
        const uint32_t sz0 = szp[pp][0], sz1 = szp[pp][1];
        const float s0 = __half2float(__ushort_as_half((unsigned short)(sz0 & 0xFFFFu)));
        const float z0 = __half2float(__ushort_as_half((unsigned short)(sz0 >> 16)));
        const float s1 = __half2float(__ushort_as_half((unsigned short)(sz1 & 0xFFFFu)));
        const float z1 = __half2float(__ushort_as_half((unsigned short)(sz1 >> 16)));
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int hl = 2 * t + e;
          if (hl >= G) continue;
          const uint32_t* hb = sm.hbits + hl * nw;
          if (!((hb[j >> 5] >> (j & 31)) & 1u)) continue;
          const int bh = b * a.hq + kvh * G + hl;
          const int rk = rank_in(hb, sm.hpre + hl * nw, j);
          const float qsum = e ? qsum1 : qsum0;
          const size_t obase = (size_t)bh * a.cand_stride + (size_t)rk * kPage;
#pragma unroll
          for (int rr = 0; rr < 2; ++rr) {
            const int row = gr + 8 * rr;
            if (row >= rows) continue;
            const float sv = rr ? s1 : s0, zv = rr ? z1 : z0;
            const float lg =
                bad ? -INFINITY : (sv * (accp[pp][2 * rr + e] * 512.f) + zv * qsum) * inv_sqrt_d;
            a.logits[obase + row] = lg;
            if (a.cand_tok) a.cand_tok[obase + row] = kPage * j + row;
            rm[e] = fmaxf(rm[e], lg);
          }
        }
      }
    }
    __syncthreads();  // the chunk's tiles are read before the next copies land
    }
  stamp(a, 21);
  // the CTA's max per head (over the 8 row-lanes of each head, then over the warps), pushed to
  // the head's owner
#pragma unroll
  for (int e = 0; e < 2; ++e) {
#pragma unroll
    for (int off = 4; off < 32; off <<= 1)
      rm[e] = fmaxf(rm[e], __shfl_xor_sync(0xffffffffu, rm[e], off));
  }
  if (lane < 4) {
#pragma unroll
    for (int e = 0; e < 2; ++e) red[warp * 8 + 2 * lane + e] = rm[e];
  }
  __syncthreads();
  if (threadIdx.x < G) {
    const int hl = threadIdx.x;
    float m = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) m = fmaxf(m, red[w * 8 + hl]);
    st_cluster(map_rank(smem_addr(sm.xchg + (hl / C) * kXchgSlot + 4 * r), hl % C), m);
  }
}

// ------------------------------------------------------------------------- phase 5: prune
__device__ float block_sum_fixed(float v, float* red) {
  // sum over the block in a fixed order; every thread receives the total
  v = warp_sum(v);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) t += red[w];
  return t;
}

// Weight in fixed point (units of 2^-48; W <= 1): integer sums are exact up to the conversion and
// independent of the order of the terms, so the live-set masses do not depend on the order in
// which the other CTAs pushed the entries.
__device__ __forceinline__ long long w_fixed(float w) { return __float2ll_rn(w * 281474976710656.f); }

// Threshold from the live set {W >= L} (n <= kThreads values lw, fixed-point copies lq).  Every
// test of the search at mid > L counts only live weights, and mass(W >= t) is a non-increasing
// step function of t, so "mid <= L or mass(W >= mid) >= p" is the same test as "mid <= T" with
// T = max(L, the largest live weight v with mass(W >= v) >= p).  T comes from all pairwise
// comparisons at once (4, 2 or 1 threads per value); the search itself is then a scalar loop that
// every thread runs (same inputs, same result).
__device__ float top_p_from_live(const float* lw, const long long* lq, int n, float L, float p,
                                 float eps, float top, float* red) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long P = __double2ll_ru((double)p * 281474976710656.0);
  const int tpv = n <= kThreads / 4 ? 4 : (n <= kThreads / 2 ? 2 : 1);
  const int i = tid / tpv, part = tid % tpv;
  long long mass = 0;
  float vi = 0.f;
  if (i < n) {
    vi = lw[i];
#pragma unroll 4
    for (int j = part; j < n; j += tpv) mass += lw[j] >= vi ? lq[j] : 0ll;
  }
  if (tpv >= 2) mass += __shfl_xor_sync(0xffffffffu, mass, 1);
  if (tpv >= 4) mass += __shfl_xor_sync(0xffffffffu, mass, 2);
  float t = (i < n && mass >= P) ? vi : 0.f;
  t = warp_max(t);
  __syncthreads();
  if (lane == 0) red[warp] = t;
  __syncthreads();
  float Tp = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) Tp = fmaxf(Tp, red[w]);
  return bisect_scalar(top, fmaxf(L, Tp), eps);
}

// Bisection of the notes page's "Key designs" (efficient top-p), three levels per block
// reduction: the seven midpoints the sequential search could visit next are computed exactly as it
// would compute them (mid = lo + (hi - lo) * 0.5 in fp32), their masses are summed in one pass, and
// the search then walks the tree taking the same decisions, stopping rules included.  Each mass is
// the same per-thread sum and the same block reduction as a one-threshold pass, so every decision
// is the one the one-midpoint-per-pass loop with this reduction would take.
// The same search over all nc weights (shared memory or global), three levels of the bisection
// tree per round: every round sums the masses of the 7 candidate midpoints below (lo, hi) at once.
__device__ float bisect_block(const float* W, bool staged, int nc, float top, float p, float eps,
                              float* red, float* ctl) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // ctl[0..6] thresholds, ctl[8] lo, ctl[9] hi, ctl[10] done, ctl[11] m, ctl[12] steps taken
  if (tid == 0) {
    ctl[10] = 0.f;
    ctl[0] = top;
    for (int k = 1; k < 7; ++k) ctl[k] = INFINITY;
    ctl[8] = 0.f;
    ctl[9] = top;
    ctl[11] = 0.f;
    ctl[12] = 0.f;
  }
  __syncthreads();
  bool first = true;
#pragma unroll 1
  while (ctl[10] == 0.f) {
    float th[7];
#pragma unroll
    for (int k = 0; k < 7; ++k) th[k] = ctl[k];
    float tmin = th[0];
#pragma unroll
    for (int k = 1; k < 7; ++k) tmin = fminf(tmin, th[k]);
    float acc[7];
#pragma unroll
    for (int k = 0; k < 7; ++k) acc[k] = 0.f;
#pragma unroll 1
    for (int i = tid; i < nc; i += kThreads) {
      const float x = staged ? W[i] : ldcg_f(W + i);
      if (x >= tmin) {  // below every threshold of this round: contributes to no mass
#pragma unroll
        for (int k = 0; k < 7; ++k) acc[k] += x >= th[k] ? x : 0.f;
      }
    }
#pragma unroll
    for (int k = 0; k < 7; ++k) acc[k] = warp_sum(acc[k]);
    if (lane == 0) {
#pragma unroll
      for (int k = 0; k < 7; ++k) red[warp * 8 + k] = acc[k];
    }
    __syncthreads();
    if (warp == 0) {
      float t = 0.f;
      if (lane < 7) {
#pragma unroll
        for (int w = 0; w < kWarps; ++w) t += red[w * 8 + lane];
      }
      float ms[7];
#pragma unroll
      for (int k = 0; k < 7; ++k) ms[k] = __shfl_sync(0xffffffffu, t, k);
      if (lane == 0) {
        float lo = ctl[8], hi = ctl[9];
        int steps = (int)ctl[12];
        int done = 0;
        if (first) {
          // the single-threshold test at max W
          if (ms[0] >= p) {
            ctl[11] = top;
            done = 1;
          }
        } else {
          // walk the 3-level tree rooted at (lo, hi); node n's midpoint is th[n - 1]
          int node = 1;
#pragma unroll
          for (int level = 0; level < 3; ++level) {
            if (done) break;
            if (__fsub_rn(hi, lo) <= eps) {
              done = 1;
              break;
            }
            float mid = th[0], mass = ms[0];
#pragma unroll
            for (int n = 2; n < 8; ++n)
              if (node == n) {
                mid = th[n - 1];
                mass = ms[n - 1];
              }
            if (!(lo < mid && mid < hi) || steps >= 64) {
              done = 1;
              break;
            }
            if (mass >= p) {
              lo = mid;
              node = 2 * node + 1;
            } else {
              hi = mid;
              node = 2 * node;
            }
            ++steps;
          }
          if (done) ctl[11] = lo;
        }
        if (!done) {
          // next round: the tree of midpoints below (lo, hi), computed as the search would
          float nlo[8], nhi[8], nmid[8];
          nlo[1] = lo;
          nhi[1] = hi;
          nmid[1] = mid_of(lo, hi);
#pragma unroll
          for (int n = 2; n < 8; ++n) {
            const int par = n >> 1;
            nlo[n] = (n & 1) ? nmid[par] : nlo[par];
            nhi[n] = (n & 1) ? nhi[par] : nmid[par];
            nmid[n] = mid_of(nlo[n], nhi[n]);
          }
#pragma unroll
          for (int n = 1; n < 8; ++n) ctl[n - 1] = nmid[n];
        }
        ctl[8] = lo;
        ctl[9] = hi;
        ctl[10] = done ? 1.f : 0.f;
        ctl[12] = (float)steps;
      }
    }
    first = false;
    __syncthreads();
  }
  const float m = ctl[11];
  __syncthreads();
  return m;
}

// Top-p of one head, run by its owner CTA.  M is the largest of the C per-CTA maxima pushed into
// this CTA's exchange slot; W_i = exp(l_i - M) / S with S summed in a fixed order (per thread over
// its rows, then over the block).  Only weights >= L = (1 - p) / (2 nc) can decide a test above
// L (the weights below L sum to less than nc L = (1 - p) / 2, so the mass above any t <= L
// exceeds p): the threshold comes from that live set when it is small (the common case), else
// from the three-level search over every weight.
__device__ void phase_prune_head(const FusedArgs& a, int hl, int bh, int nc, int C, Smem& sm) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float* red = reinterpret_cast<float*>(sm.scratch);                  // [kWarps][8]
  float* ctl = reinterpret_cast<float*>(sm.scratch + 4 * kWarps * 8);   // search state
  int* scan_sh2 = reinterpret_cast<int*>(sm.scratch + 768);             // 33 ints
  uint32_t* top_u = reinterpret_cast<uint32_t*>(sm.scratch + 1000);     // block max of W
  float* lw = reinterpret_cast<float*>(sm.scratch + 1024);              // [kThreads] live W
  int* li = reinterpret_cast<int*>(sm.scratch + 1024 + 4 * kThreads);   // [kThreads] their rows
  long long* lq = reinterpret_cast<long long*>(sm.scratch + 1024 + 8 * kThreads);  // fixed point
  unsigned char* tail = sm.scratch + 1024 + 16 * kThreads;
  const int tail_off = (int)(tail - sm.scratch);
  const bool staged = tail_off + 4 * nc <= sm.scratch_bytes;

  const float* part = reinterpret_cast<const float*>(sm.xchg + (hl / C) * kXchgSlot);
  float pm[16];
#pragma unroll
  for (int rr = 0; rr < 16; ++rr) pm[rr] = rr < C ? part[rr] : -INFINITY;
  float M = -INFINITY;
#pragma unroll
  for (int rr = 0; rr < 16; ++rr) M = fmaxf(M, pm[rr]);
  const bool empty = !(M > -INFINITY);
  stamp(a, 17);

  const float p = a.p, eps = a.eps;
  const bool use_bound = nc > 0 && p < 1.f && (1.f - p) >= 1e-3f;
  const float L = use_bound ? (1.f - p) / (2.f * (float)nc) : 0.f;
  float* lrow = a.logits + (size_t)bh * a.cand_stride;
  float* wout = a.weights_out ? a.weights_out + (size_t)bh * a.cand_stride : nullptr;
  if (tid == 0) *top_u = 0u;

  // Weights: in registers (row i = k * kThreads + tid) when nc <= kThreads * kR, else in shared
  // memory (or in place in the logits row when they do not fit).
  constexpr int kR = 16;
  const bool in_regs = nc <= kThreads * kR;
  float wr[kR];
  float* W = staged ? reinterpret_cast<float*>(tail) : lrow;
  float esum = 0.f;
  if (in_regs) {
#pragma unroll
    for (int k = 0; k < kR; ++k) {
      const int i = k * kThreads + tid;
      wr[k] = i < nc ? ldcg_f(lrow + i) : 0.f;
    }
#pragma unroll
    for (int k = 0; k < kR; ++k) {
      const int i = k * kThreads + tid;
      const float e = (i < nc && !empty) ? __expf(wr[k] - M) : 0.f;
      wr[k] = e;
      esum += e;
    }
  } else {
    constexpr int kB = 8;
#pragma unroll 1
    for (int base = 0; base < nc; base += kThreads * kB) {
      float v[kB];
#pragma unroll
      for (int k = 0; k < kB; ++k) {
        const int i = base + k * kThreads + tid;
        v[k] = i < nc ? ldcg_f(lrow + i) : 0.f;
      }
#pragma unroll
      for (int k = 0; k < kB; ++k) {
        const int i = base + k * kThreads + tid;
        if (i < nc) {
          const float e = empty ? 0.f : __expf(v[k] - M);
          W[i] = e;
          esum += e;
        }
      }
    }
  }
  const float S = block_sum_fixed(esum, red);
  const float inv = S > 0.f ? 1.f / S : 0.f;
  stamp(a, 18);
  // W = e / S, the largest weight, the live count
  float top = 0.f;
  int cntl = 0;
  if (in_regs) {
#pragma unroll
    for (int k = 0; k < kR; ++k) {
      const int i = k * kThreads + tid;
      wr[k] *= inv;
      top = fmaxf(top, wr[k]);
      cntl += (i < nc && wr[k] >= L) ? 1 : 0;
    }
  } else {
#pragma unroll 1
    for (int i = tid; i < nc; i += kThreads) {
      const float w = (staged ? W[i] : ldcg_f(W + i)) * inv;
      W[i] = w;
      top = fmaxf(top, w);
      cntl += w >= L ? 1 : 0;
    }
  }
  top = warp_max(top);
  if (lane == 0) atomicMax(top_u, __float_as_uint(top));  // W >= 0: the bits order as the values
  int nlive = 0;
  int pos = block_exclusive_scan(cntl, scan_sh2, &nlive);  // its barriers also publish top_u
  top = __uint_as_float(*top_u);
  stamp(a, 19);
  const bool from_live = use_bound && nlive <= kThreads;
  if (from_live) {
    if (in_regs) {
#pragma unroll
      for (int k = 0; k < kR; ++k) {
        const int i = k * kThreads + tid;
        if (i < nc && wr[k] >= L) {
          lw[pos] = wr[k];
          li[pos] = i;
          lq[pos] = w_fixed(wr[k]);
          ++pos;
        }
      }
    } else {
      for (int i = tid; i < nc; i += kThreads) {
        const float w = staged ? W[i] : ldcg_f(W + i);
        if (w >= L) {
          lw[pos] = w;
          li[pos] = i;
          lq[pos] = w_fixed(w);
          ++pos;
        }
      }
    }
  }
  if (wout) {  // the weights output: every candidate
    if (in_regs) {
#pragma unroll
      for (int k = 0; k < kR; ++k) {
        const int i = k * kThreads + tid;
        if (i < nc) wout[i] = wr[k];
      }
    } else {
      for (int i = tid; i < nc; i += kThreads) wout[i] = staged ? W[i] : ldcg_f(W + i);
    }
  }
  if (in_regs && !from_live && nc > 0 && p < 1.f) {  // the block search reads every weight
#pragma unroll
    for (int k = 0; k < kR; ++k) {
      const int i = k * kThreads + tid;
      if (i < nc) W[i] = wr[k];
    }
  }
  __syncthreads();  // the live set (or the weights) complete
  float m;
  if (nc == 0 || p >= 1.f) m = 0.f;  // keep every candidate
  else if (from_live) m = top_p_from_live(lw, lq, nlive, L, p, eps, top, red);
  else m = bisect_block(W, staged, nc, top, p, eps, red, ctl);
  stamp(a, 20);
  if (tid == 0) {
    if (a.threshold) a.threshold[bh] = m;
    if (a.cand_count) a.cand_count[bh] = nc;
  }
  // kept-row bitmap of this head: bit i = (W_i >= m)
  uint32_t* kb_out = a.keptbits + (size_t)bh * a.kept_words;
  const int kw = (nc + 31) >> 5;
  uint32_t* kbits = reinterpret_cast<uint32_t*>(tail);
  int cnt = 0;
  if (from_live && m >= L && tail_off + 4 * kw <= sm.scratch_bytes) {
    // every kept candidate is live
    for (int w = tid; w < kw; w += kThreads) kbits[w] = 0u;
    __syncthreads();
    if (tid < nlive && lw[tid] >= m) atomicOr(&kbits[li[tid] >> 5], 1u << (li[tid] & 31));
    __syncthreads();
    for (int w = tid; w < kw; w += kThreads) {
      const uint32_t x = kbits[w];
      kb_out[w] = x;
      cnt += __popc(x);
    }
  } else if (in_regs) {
#pragma unroll
    for (int k = 0; k < kR; ++k) {
      const int i = k * kThreads + tid;
      const bool keep = i < nc && wr[k] >= m;
      const uint32_t bal = __ballot_sync(0xffffffffu, keep);
      if (lane == 0 && k * kThreads + 32 * warp < nc) kb_out[k * kWarps + warp] = bal;
      cnt += keep;
    }
  } else {
#pragma unroll 1
    for (int base = 0; base < nc; base += kThreads) {
      const int i = base + tid;
      const bool keep = i < nc && (staged ? W[i] : ldcg_f(W + i)) >= m;
      const uint32_t bal = __ballot_sync(0xffffffffu, keep);
      if (lane == 0 && base + 32 * warp < nc) kb_out[(base >> 5) + warp] = bal;
      cnt += keep;
    }
  }
  if (a.kept_count) {  // only when the caller asks for it
    const float total = block_sum_fixed((float)cnt, red);
    if (tid == 0) a.kept_count[bh] = (int)total;
  }
}

// ------------------------------------------------------------------------- phase 6: kept union
// Per page of this CTA's union share: 16-bit mask of rows kept by any head of the group.
// The kept rows of union page j: the OR over the group's heads that selected j of their 16-row
// pieces of the kept-row bitmaps (the candidate rows of a head are its selected pages' rows in
// ascending page order), cut to the page's valid rows.
template <int G>
__device__ __forceinline__ uint32_t union_row_mask(const FusedArgs& a, int b, int kvh, int n, int j,
                                                   const Smem& sm) {
  const int nw = sm.nw;
  uint32_t words[G];
  int shift[G];
#pragma unroll
  for (int hl = 0; hl < G; ++hl) {  // every head's word in flight before combining
    const uint32_t* hb = sm.hbits + hl * nw;
    words[hl] = 0u;
    shift[hl] = 0;
    if ((hb[j >> 5] >> (j & 31)) & 1u) {
      const int rk = rank_in(hb, sm.hpre + hl * nw, j);
      words[hl] = ldcg_u(a.keptbits + (size_t)(b * a.hq + kvh * G + hl) * a.kept_words + (rk >> 1));
      shift[hl] = 16 * (rk & 1);
    }
  }
  uint32_t m = 0;
#pragma unroll
  for (int hl = 0; hl < G; ++hl) m |= (words[hl] >> shift[hl]) & 0xFFFFu;
  const int rows = page_rows(n, j);
  return m & (rows >= 16 ? 0xFFFFu : ((1u << rows) - 1u));
}

template <int G>
__device__ int phase_kept_rows(const FusedArgs& a, int b, int kvh, int n, int U, int r, int C,
                               Smem& sm, uint16_t* rowmask, int* scan_sh) {
  const int tid = threadIdx.x, nw = sm.nw;
  const int u0 = (int)((long)U * r / C), u1 = (int)((long)U * (r + 1) / C);
  int cnt = 0;
  for (int u = u0 + tid; u < u1; u += kThreads) {
    const int j = union_select(sm.ubits, sm.upre, nw, u);
    const uint32_t m = union_row_mask<G>(a, b, kvh, n, j, sm);
    rowmask[u - u0] = (uint16_t)m;
    cnt += __popc(m);
  }
  int total;
  block_exclusive_scan(cnt, scan_sh, &total);
  return total;
}

// Kept rows of this CTA's union share for attention without a global list: per page (in union
// order) its 16-bit row mask, the exclusive prefix of kept rows, and its physical page.
// Returns the number of kept rows of the share.
template <int G>
__device__ int phase_kept_rows_local(const FusedArgs& a, int b, int kvh, int n, int U, int r,
                                     int C, Smem& sm, uint16_t* rowmask, int* pfx, int* pph,
                                     int* scan_sh) {
  const int tid = threadIdx.x, nw = sm.nw;
  const int u0 = (int)((long)U * r / C), u1 = (int)((long)U * (r + 1) / C);
  int carry = 0;
#pragma unroll 1
  for (int ub = u0; ub < u1; ub += kThreads) {
    const int u = ub + tid;
    uint32_t m = 0;
    if (u < u1) {
      const int j = union_select(sm.ubits, sm.upre, nw, u);
      pph[u - u0] = phys_of(a, sm, b, j);
      m = union_row_mask<G>(a, b, kvh, n, j, sm);
      rowmask[u - u0] = (uint16_t)m;
    }
      int total;
    const int ex = block_exclusive_scan(__popc(m), scan_sh, &total);
      if (u < u1) pfx[u - u0] = carry + ex;
    carry += total;
  }
  __syncthreads();
  return carry;
}

template <int G>
__device__ void phase_write_union(const FusedArgs& a, int gi, int U, int r, int C, int base,
                                  Smem& sm, const uint16_t* rowmask, int* scan_sh) {
  const int tid = threadIdx.x, nw = sm.nw;
  const int u0 = (int)((long)U * r / C), u1 = (int)((long)U * (r + 1) / C);
  int* out = a.union_tok + (size_t)gi * a.union_stride;
  // pages are handled in rounds of kThreads; thread order = page order
  int carry = base;
  for (int ub = u0; ub < u1; ub += kThreads) {
    const int u = ub + tid;
    const uint32_t m = u < u1 ? rowmask[u - u0] : 0u;
    int total;
    int pos = carry + block_exclusive_scan(__popc(m), scan_sh, &total);
    carry += total;
    if (m) {
      const int j = union_select(sm.ubits, sm.upre, nw, u);
      uint32_t mm = m;
      while (mm) {
        out[pos++] = kPage * j + __ffs(mm) - 1;
        mm &= mm - 1u;
      }
    }
  }
}

// ------------------------------------------------------------------------- phase 7: attention
// Thread layout: token slot t = tid / 8 (kAttChunk per round), sub-lane s = tid % 8 owns channels
// [8s, 8s+8) and [64+8s, 64+8s+8).  For P.V: channel d = tid % 128, token group tid / 128.
// kLocal: tokens of this CTA's own union share, from (rowmask, pfx, pph) in shared memory;
// otherwise an even share [T r / C, T (r+1) / C) of the group's global ascending list.
template <int G, bool kLocal>
__device__ void phase_attend(const FusedArgs& a, int b, int kvh, int gi, int n, int T, int r, int C,
                             Smem& sm, const uint16_t* rowmask = nullptr, const int* pfx = nullptr,
                             const int* pph = nullptr, int npg = 0) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ts = tid >> 3, s8 = tid & 7;
  const int d = tid & 127, quarter = tid >> 7;
  unsigned char* sp = sm.scratch;
  constexpr int kKV = kAttChunk * 256;  // bytes of one staged K (or V) chunk
  uint4* ks = reinterpret_cast<uint4*>(sp);                              // [kAttChunk][16]
  uint4* vs = reinterpret_cast<uint4*>(sp + kKV);                        // [kAttChunk][16]
  float* ps = reinterpret_cast<float*>(sp + 2 * kKV);                    // [G][kAttChunk]
  float* red = reinterpret_cast<float*>(sp + 2 * kKV + G * kAttChunk * 4);  // [kWarps][G]
  uint32_t* rowidx =
      reinterpret_cast<uint32_t*>(sp + 2 * kKV + G * kAttChunk * 4 + kWarps * G * 4);  // [kAttChunk]
  float* opart = reinterpret_cast<float*>(sp + 2 * kKV + G * kAttChunk * 4 + kWarps * G * 4 +
                                          kAttChunk * 4);  // [kQuarters][G][128]
  const int t0 = kLocal ? 0 : (int)((long)T * r / C), t1 = kLocal ? T : (int)((long)T * (r + 1) / C);
  const int* ulist = a.union_tok + (size_t)gi * a.union_stride;

  float qv[G][16];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const uint16_t* qh = sm.q + h * kHeadDim;
    float f[8];
    unpack8(*reinterpret_cast<const uint4*>(qh + 8 * s8), f);
#pragma unroll
    for (int i = 0; i < 8; ++i) qv[h][i] = f[i];
    unpack8(*reinterpret_cast<const uint4*>(qh + 64 + 8 * s8), f);
#pragma unroll
    for (int i = 0; i < 8; ++i) qv[h][8 + i] = f[i];
  }
  float M[G], L[G], O[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    M[h] = -INFINITY;
    L[h] = 0.f;
    O[h] = 0.f;
  }
  for (int cb = t0; cb < t1; cb += kAttChunk) {
    const int nt = min(kAttChunk, t1 - cb);
    if (tid < kAttChunk) {
      uint32_t ri = 0xFFFFFFFFu;
      if (tid < nt) {
        if (kLocal) {
          // page of local token t: the last page whose exclusive prefix is <= t
          const int t = cb + tid;
          int lo = 0, hi = npg;
          while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (pfx[mid] <= t) lo = mid;
            else hi = mid;
          }
          const int row = nth_set_bit(rowmask[lo], t - pfx[lo]);
          const int ph = pph[lo];
          if (ph >= 0) ri = (uint32_t)(((size_t)ph * a.kv.hkv + kvh) * kPage + row);
        } else {
          const int tk = ldcg_i(ulist + cb + tid);
          if (tk >= 0 && tk < n) {
            const int ph = load_phys(a.kv.page_table, b, tk >> 4, a.kv.max_pages, a.kv.num_phys,
                                     a.flags);
            if (ph >= 0) ri = (uint32_t)(((size_t)ph * a.kv.hkv + kvh) * kPage + (tk & 15));
          } else {
            raise_flag(a.flags, TWL_FLAG_BAD_INDEX);
          }
        }
      }
      rowidx[tid] = ri;
    }
    __syncthreads();
    // gather kAttChunk rows of K and V: 2 x 16 x kAttChunk 16-byte chunks, 4 per thread
#pragma unroll
    for (int it = 0; it < 2; ++it) {
      const int c = tid + it * kThreads;  // 0 .. 16 kAttChunk - 1
      const int tt = c >> 4, ch = c & 15;
      const uint32_t ri = rowidx[tt];
      const bool ok = ri != 0xFFFFFFFFu;
      const size_t off = ok ? (size_t)ri * kHeadDim + 8 * ch : 0;
      cp_async16(&ks[tt * 16 + ch], a.kv.k + off, ok);
      cp_async16(&vs[tt * 16 + ch], a.kv.v + off, ok);
    }
    cp_async_commit();
    cp_async_wait_all();
    __syncthreads();
    // scores
    const bool tok_ok = ts < nt && rowidx[ts] != 0xFFFFFFFFu;
    float sc[G];
    {
      float k0[8], k1[8];
      unpack8(ks[ts * 16 + s8], k0);
      unpack8(ks[ts * 16 + 8 + s8], k1);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) acc = fmaf(qv[h][i], k0[i], acc);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc = fmaf(qv[h][8 + i], k1[i], acc);
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        acc += __shfl_xor_sync(0xffffffffu, acc, 4);
        sc[h] = tok_ok ? acc * a.sm_scale : -INFINITY;
      }
    }
    // chunk max per head
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float m = sc[h];
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
      if (lane == 0) red[warp * G + h] = m;
    }
    __syncthreads();
    float scale[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float cm = -INFINITY;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) cm = fmaxf(cm, red[w * G + h]);
      const float nm = fmaxf(M[h], cm);
      scale[h] = (nm > -INFINITY && M[h] > -INFINITY) ? __expf(M[h] - nm) : (nm > -INFINITY ? 0.f : 1.f);
      M[h] = nm;
      const float pv = (tok_ok && nm > -INFINITY) ? __expf(sc[h] - nm) : 0.f;
      if (s8 == 0) ps[h * kAttChunk + ts] = pv;
    }
    __syncthreads();
    // P.V for channel d over tokens quarter, quarter + kQuarters, ...
    const __half* vh = reinterpret_cast<const __half*>(vs);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float acc = 0.f, lsum = 0.f;
      for (int tt = quarter; tt < nt; tt += kQuarters) {
        const float pv = ps[h * kAttChunk + tt];
        acc = fmaf(pv, __half2float(vh[tt * kHeadDim + d]), acc);
        lsum += pv;
      }
      O[h] = O[h] * scale[h] + acc;
      L[h] = L[h] * scale[h] + lsum;
    }
    __syncthreads();
  }
  // combine the token groups, write this CTA's partial: M, L, O (unnormalised)
#pragma unroll
  for (int h = 0; h < G; ++h) opart[(quarter * G + h) * kHeadDim + d] = O[h];
  float* lpart = reinterpret_cast<float*>(ps);  // reuse: [kQuarters][G]
  if (d == 0) {
#pragma unroll
    for (int h = 0; h < G; ++h) lpart[quarter * G + h] = L[h];
  }
  __syncthreads();
  float* part = a.part_att + ((size_t)gi * C + r) * G * (kHeadDim + 2);
  if (quarter == 0) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float o = 0.f, l = 0.f;
#pragma unroll
      for (int qq = 0; qq < kQuarters; ++qq) {
        o += opart[(qq * G + h) * kHeadDim + d];
        l += lpart[qq * G + h];
      }
      part[h * (kHeadDim + 2) + 2 + d] = o;
      if (d == 0) {
        part[h * (kHeadDim + 2) + 0] = M[h];
        part[h * (kHeadDim + 2) + 1] = l;
      }
    }
  }
}

// ------------------------------------------------------------------------- phase 8: merge
__device__ void phase_merge_head(const FusedArgs& a, int gi, int bh, int hl, int G, int C) {
  const int tid = threadIdx.x;
  if (tid >= kHeadDim) return;
  float pm[16], pl[16], po[16];
#pragma unroll
  for (int rr = 0; rr < 16; ++rr) {  // every partial's loads in flight together
    pm[rr] = -INFINITY;
    pl[rr] = 0.f;
    po[rr] = 0.f;
    if (rr < C) {
      const float* part =
          a.part_att + ((size_t)gi * C + rr) * G * (kHeadDim + 2) + hl * (kHeadDim + 2);
      pm[rr] = ldcg_f(part);
      pl[rr] = ldcg_f(part + 1);
      po[rr] = ldcg_f(part + 2 + tid);
    }
  }
  float Mx = -INFINITY;
#pragma unroll
  for (int rr = 0; rr < 16; ++rr)
    if (pl[rr] > 0.f) Mx = fmaxf(Mx, pm[rr]);
  float o = 0.f, l = 0.f;
  if (Mx > -INFINITY) {
#pragma unroll
    for (int rr = 0; rr < 16; ++rr) {
      if (!(pl[rr] > 0.f)) continue;
      const float wgt = __expf(pm[rr] - Mx);
      o = fmaf(wgt, po[rr], o);
      l = fmaf(wgt, pl[rr], l);
    }
  }
  const bool any = l > 0.f;
  a.o[(size_t)bh * kHeadDim + tid] = any ? o / l : 0.f;
  if (tid == 0) a.lse[bh] = any ? Mx + __logf(l) : -INFINITY;
}

template <int G>
__host__ __device__ constexpr size_t attend_smem_bytes() {
  return 2 * kAttChunk * 256 + G * kAttChunk * 4 + kWarps * G * 4 + kAttChunk * 4 +
         kQuarters * G * kHeadDim * 4;
}

// The local attention path needs room for the largest share of the cluster (so every CTA takes
// the same branch and executes the same barriers).
__device__ __forceinline__ bool local_fits_all(const FusedArgs& a, int U, int C, int att_bytes,
                                               int scratch_bytes) {
  (void)a;
  const int max_share = (U + C - 1) / C;
  return att_bytes + 10 * max_share + 64 <= scratch_bytes;
}

// ------------------------------------------------------------------------- the kernel
template <int G>
__global__ void __launch_bounds__(kThreads, 512 / kThreads) k_decode_fused(FusedArgs a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  __shared__ int scan_sh[33];
  __shared__ int s_total;
  __shared__ int s_nc[8];

  const int C = (int)cluster_size();
  const int r = (int)cluster_rank();
  const int gi = blockIdx.x / C;
  const int b = gi / a.kv.hkv, kvh = gi % a.kv.hkv;
  const int tid = threadIdx.x;
  // wait for the previous grid in the stream (launched programmatically), then let the next one
  // be scheduled: it will in turn wait for this grid to complete before touching memory
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");

  const Seq sq = load_seq(a.kv.seq_lens, b, a.kv.max_pages, a.flags, r == 0 && tid == 0);
  const int n_pages = sq.pages;
  if (n_pages == 0) {  // invalid sequence: uniform across the cluster, before any barrier
    if (r == 0) {
      for (int i = tid; i < G * kHeadDim; i += kThreads)
        a.o[((size_t)b * a.hq + kvh * G) * kHeadDim + i] = 0.f;
      if (tid < G) {
        a.lse[(size_t)b * a.hq + kvh * G + tid] = -INFINITY;
        if (a.sel_count) a.sel_count[b * a.hq + kvh * G + tid] = 0;
        if (a.cand_count) a.cand_count[b * a.hq + kvh * G + tid] = 0;
        if (a.kept_count) a.kept_count[b * a.hq + kvh * G + tid] = 0;
      }
      if (tid == 0 && a.union_count) a.union_count[gi] = 0;
    }
    return;
  }
  int kb = a.budget_pages > 0 ? a.budget_pages : (n_pages + a.budget_div - 1) / a.budget_div;
  kb = min(min(kb, n_pages), a.max_budget);

  Smem sm;
  sm.nw = (n_pages + 31) >> 5;
  {
    __shared__ __align__(16) uint16_t s_q[8 * kHeadDim];
    const uint4* src = reinterpret_cast<const uint4*>(a.q + ((size_t)b * a.hq + kvh * G) * kHeadDim);
    for (int i = tid; i < G * kHeadDim / 8; i += kThreads) reinterpret_cast<uint4*>(s_q)[i] = src[i];
    sm.q = s_q;
  }
  {
    unsigned char* p = smem_raw;
    sm.hbits = reinterpret_cast<uint32_t*>(p);
    p += 4 * G * a.sel_words;
    sm.hpre = reinterpret_cast<int*>(p);
    p += 4 * G * a.sel_words;
    sm.ubits = reinterpret_cast<uint32_t*>(p);
    p += 4 * a.sel_words;
    sm.upre = reinterpret_cast<int*>(p);
    sm.xchg = smem_raw + bitmap_bytes(G, a.sel_words);
    p = smem_raw + persistent_bytes(G, a.sel_words);
    sm.pt = nullptr;
    if (a.pt_smem) {  // the sequence's page table, validated once
      int* pt = reinterpret_cast<int*>(p);
      for (int j = tid; j < n_pages; j += kThreads)
        pt[j] = load_phys(a.kv.page_table, b, j, a.kv.max_pages, a.kv.num_phys, a.flags);
      sm.pt = pt;
      p += (4 * a.kv.max_pages + 127) & ~127;
    }
    sm.scratch = p;  // 128-byte aligned
    sm.scratch_bytes = a.smem_bytes - (int)(p - smem_raw);
  }
  __syncthreads();

  // 1: scores
  stamp(a, 0);
  phase_scores<G>(a, b, kvh, n_pages, r, C, sm);
  stamp(a, 1);
  cluster_sync();
  stamp(a, 2);
  // 2: top-k of the heads this CTA owns
  for (int hl = r; hl < G; hl += C) phase_topk_head(a, b * a.hq + kvh * G + hl, n_pages, kb, sm);
  stamp(a, 3);
  cluster_sync();
  stamp(a, 4);
  // 3: bitmaps, union, ranks (every CTA)
  phase_union_bitmaps<G>(a, b, kvh, sm, &s_total, scan_sh);
  const int U = s_total;
  if (tid < G) {
    // candidate rows of each head: its kb pages' rows; the last selected page (the highest set
    // bit of the head bitmap) may be partial
    const uint32_t* hb = sm.hbits + tid * sm.nw;
    int jl = -1;
    for (int w = sm.nw - 1; w >= 0; --w)
      if (hb[w]) {
        jl = 32 * w + 31 - __clz(hb[w]);
        break;
      }
    s_nc[tid] = (kb > 0 && jl >= 0) ? kPage * (kb - 1) + page_rows(sq.n, jl) : 0;
  }
  __syncthreads();
  stamp(a, 5);
  // 4: INT4 estimate over this CTA's share of the union; partials and candidate lists to owners
  phase_estimate<G>(a, b, kvh, sq.n, U, r, C, sm);
  stamp(a, 6);
  cluster_sync();
  stamp(a, 7);
  // 5: top-p of the heads this CTA owns
  if (kb > 0)
    for (int hl = r; hl < G; hl += C) {
      phase_prune_head(a, hl, b * a.hq + kvh * G + hl, s_nc[hl], C, sm);
      __syncthreads();
    }
  stamp(a, 8);
  cluster_sync();
  stamp(a, 9);
  // 6-7: kept rows of this CTA's union pages, then attention over them.  The group's ordered
  // union list is only built when the caller asks for it (counts exchanged, list written, then
  // attention over even shares of it); otherwise every CTA attends over its own kept rows.
  const int share = (int)((long)U * (r + 1) / C) - (int)((long)U * r / C);
  const int att_bytes = (int)attend_smem_bytes<G>();
  const bool local_fits = att_bytes + 10 * share + 64 <= sm.scratch_bytes;
  if (!a.want_union && local_fits_all(a, U, C, att_bytes, sm.scratch_bytes)) {
    unsigned char* base = sm.scratch + att_bytes;
    int* pfx = reinterpret_cast<int*>(base);
    int* pph = pfx + share;
    uint16_t* rowmask = reinterpret_cast<uint16_t*>(pph + share);
    const int T = phase_kept_rows_local<G>(a, b, kvh, sq.n, U, r, C, sm, rowmask, pfx, pph, scan_sh);
    stamp(a, 10);
    phase_attend<G, true>(a, b, kvh, gi, sq.n, T, r, C, sm, rowmask, pfx, pph, share);
  } else {
    (void)local_fits;
    uint16_t* rowmask = reinterpret_cast<uint16_t*>(sm.scratch);
    const int local = phase_kept_rows<G>(a, b, kvh, sq.n, U, r, C, sm, rowmask, scan_sh);
    if (tid == 0) a.union_part[(size_t)gi * C + r] = local;
    stamp(a, 10);
    cluster_sync();
    stamp(a, 11);
    int base = 0, T = 0;
    for (int rr = 0; rr < C; ++rr) {
      const int c = ldcg_i(a.union_part + (size_t)gi * C + rr);
      if (rr < r) base += c;
      T += c;
    }
    phase_write_union<G>(a, gi, U, r, C, base, sm, rowmask, scan_sh);
    if (r == 0 && tid == 0 && a.union_count) a.union_count[gi] = T;
    stamp(a, 12);
    cluster_sync();
    stamp(a, 13);
    phase_attend<G, false>(a, b, kvh, gi, sq.n, T, r, C, sm);
  }
  stamp(a, 14);
  cluster_sync();
  stamp(a, 15);
  // 8: merge per head
  for (int hl = r; hl < G; hl += C) phase_merge_head(a, gi, b * a.hq + kvh * G + hl, hl, G, C);
  stamp(a, 16);
}


}  // namespace

namespace TWL_FUSED_NS {

FusedPlan plan_fused(int batch, int hq, int hkv, int max_pages, int max_budget) {
  FusedPlan pl{};
  const int g = hq / hkv;
  const int groups = batch * hkv;
  pl.sel_words = (max_pages + 31) / 32;
  pl.cand_stride = kPage * max_budget;
  pl.union_stride = kPage * max_pages;
  // cluster size: enough CTAs to fill the GPU, at most 16
  const int sms = num_sms();
  int c = 1;
  const int per_sm = 512 / kThreads;  // CTAs that fit on one SM
  while (c < 16 && groups * (c + 1) <= per_sm * sms) ++c;
  // TWL_FUSED_CLUSTER=1..16 forces the cluster size (used by the tests to cover several sizes)
  if (const char* env = getenv("TWL_FUSED_CLUSTER")) {
    const int f = atoi(env);
    if (f >= 1 && f <= 16) c = f;
  }
  pl.cluster = c;
  pl.pt_smem = max_pages <= 8192;
  const size_t persistent = (size_t)persistent_bytes(g, pl.sel_words) +
                            (pl.pt_smem ? ((size_t)4 * max_pages + 127) / 128 * 128 : 0);
  size_t scratch = 0;
  switch (g) {
    case 1: scratch = attend_smem_bytes<1>(); break;
    case 2: scratch = attend_smem_bytes<2>(); break;
    case 4: scratch = attend_smem_bytes<4>(); break;
    default: scratch = attend_smem_bytes<8>(); break;
  }
  // top-k keys and staged weights when they fit in what is left
  size_t cap = (kThreads == 256 ? 110 : 220) * 1024;  // two 256-thread CTAs share an SM
  // TWL_FUSED_SMEM_KB=N caps the dynamic shared memory per CTA (N >= 64; below ~110 two CTAs fit
  // on one SM)
  if (const char* env = getenv("TWL_FUSED_SMEM_KB")) {
    const int kb = atoi(env);
    if (kb >= 64 && kb < 220) cap = (size_t)kb * 1024;
  }
  size_t want = scratch;
  const size_t topk_need = 1280 + (size_t)4 * max_pages + 4 * kWarps * 512 + 2048;
  want = want > topk_need ? want : topk_need;
  const size_t local_need = scratch + (size_t)10 * max_pages + 64;
  want = want > local_need ? want : local_need;
  const size_t prune_need = 1024 + (size_t)16 * kThreads + (size_t)4 * pl.cand_stride;
  want = want > prune_need ? want : prune_need;
  want = want > (size_t)2 * pl.union_stride / 16 + 16 ? want : (size_t)2 * pl.union_stride / 16 + 16;
  // the bulk-copy chunks of the scoring and estimate phases take whatever is left: ask for the
  // full capacity (one CTA per SM in any case)
  want = cap - persistent;
  pl.smem_bytes = (int)(persistent + want);
  pl.ok = persistent + scratch <= cap && persistent + (size_t)2 * max_pages <= cap &&
          persistent + 1280 + (size_t)4 * max_pages <= cap;  // the top-k keys
  return pl;
}

size_t fused_workspace_bytes(int batch, int hq, int hkv, int max_pages, int max_budget) {
  const FusedPlan pl = plan_fused(batch, hq, hkv, max_pages, max_budget);
  const int g = hq / hkv;
  const size_t bh = (size_t)batch * hq, groups = (size_t)batch * hkv;
  // cluster-dependent parts are sized for the largest cluster (16)
  size_t s = 0;
  auto add = [&](size_t bytes) { s += (bytes + 255) & ~(size_t)255; };
  add(bh * max_pages * 4);                    // scores
  add(bh * pl.sel_words * 4);                 // selected-page bitmaps
  add(bh * (size_t)pl.cand_stride * 4);       // logits / weights
  add(groups * 16 * 4);                       // union counts per CTA
  add(groups * (size_t)pl.union_stride * 4);  // union token lists
  add(groups * 16 * g * (kHeadDim + 2) * 4);  // attention partials
  add(bh * (size_t)((pl.cand_stride + 31) / 32) * 4);  // kept-row bitmaps
  return s;
}

void carve_fused(FusedArgs& a, char* ws, const FusedPlan& pl, int batch, int hq, int hkv,
                 int max_pages) {
  const int g = hq / hkv;
  const size_t bh = (size_t)batch * hq, groups = (size_t)batch * hkv;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = ws + off;
    off += (bytes + 255) & ~(size_t)255;
    return p;
  };
  a.scores = reinterpret_cast<float*>(take(bh * max_pages * 4));
  a.selbits = reinterpret_cast<uint32_t*>(take(bh * pl.sel_words * 4));
  a.logits = reinterpret_cast<float*>(take(bh * (size_t)pl.cand_stride * 4));
  a.union_part = reinterpret_cast<int*>(take(groups * 16 * 4));
  int* ulist = reinterpret_cast<int*>(take(groups * (size_t)pl.union_stride * 4));
  if (!a.union_tok) a.union_tok = ulist;
  a.part_att = reinterpret_cast<float*>(take(groups * 16 * g * (kHeadDim + 2) * 4));
  a.kept_words = (pl.cand_stride + 31) / 32;
  a.keptbits = reinterpret_cast<uint32_t*>(take(bh * (size_t)a.kept_words * 4));
}

cudaError_t launch_fused(const FusedArgs& a, const FusedPlan& pl, cudaStream_t s) {
  const int g = a.hq / a.kv.hkv;
  const int groups = a.kv.batch * a.kv.hkv;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(groups * pl.cluster));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = (size_t)pl.smem_bytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)pl.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // programmatic dependent launch: this grid may be scheduled while the previous kernel in the
  // stream finishes; it waits for that kernel (griddepcontrol.wait) before touching memory
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
#define TWL_FUSED(G)                                                                            \
  do {                                                                                          \
    cudaError_t e = cudaFuncSetAttribute(k_decode_fused<G>,                                     \
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,           \
                                         pl.smem_bytes);                                        \
    if (e != cudaSuccess) return e;                                                             \
    if (pl.cluster > 8) {                                                                       \
      e = cudaFuncSetAttribute(k_decode_fused<G>,                                               \
                               cudaFuncAttributeNonPortableClusterSizeAllowed, 1);              \
      if (e != cudaSuccess) return e;                                                           \
    }                                                                                           \
    e = cudaLaunchKernelEx(&cfg, k_decode_fused<G>, a);                                         \
    if (e != cudaSuccess) return e;                                                             \
  } while (0)
  switch (g) {
    case 1: TWL_FUSED(1); break;
    case 2: TWL_FUSED(2); break;
    case 4: TWL_FUSED(4); break;
    case 8: TWL_FUSED(8); break;
    default: return cudaErrorInvalidValue;
  }
#undef TWL_FUSED
  return cudaGetLastError();
}

// Active clusters of size c the device can hold at once for this kernel (0 if none / error).
static int active_clusters(int g, int c, int smem_bytes) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)c);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = (size_t)smem_bytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)c;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  cudaError_t e = cudaErrorInvalidValue;
#define TWL_FIT(G)                                                                              \
  do {                                                                                          \
    cudaFuncSetAttribute(k_decode_fused<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,        \
                         smem_bytes);                                                           \
    if (c > 8)                                                                                  \
      cudaFuncSetAttribute(k_decode_fused<G>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1); \
    e = cudaOccupancyMaxActiveClusters(&n, k_decode_fused<G>, &cfg);                            \
  } while (0)
  switch (g) {
    case 1: TWL_FIT(1); break;
    case 2: TWL_FIT(2); break;
    case 4: TWL_FIT(4); break;
    default: TWL_FIT(8); break;
  }
#undef TWL_FIT
  if (e != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

// Cluster size for `groups` groups: the largest c <= want (any size up to 16) whose clusters for
// every group can be resident at once; if none can, the c that keeps the most CTAs resident.
int fit_cluster(int g, int want, int groups, int smem_bytes) {
  int best = 1, best_ctas = 0;
  for (int c = want; c >= 1; --c) {
    const int n = c == 1 ? groups : active_clusters(g, c, smem_bytes);
    if (n >= groups) return c;
    if (n * c > best_ctas) {
      best_ctas = n * c;
      best = c;
    }
  }
  return best;
}

}  // namespace TWL_FUSED_NS
}  // namespace twl
