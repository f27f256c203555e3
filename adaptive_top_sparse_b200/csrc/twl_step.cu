// The decode step of hierarchical top-p sparse attention as ONE persistent grid over every SM.
//
// "Twilight: Adaptive Attention Sparsity with Hierarchical Top-p Pruning": notes page, "Overall
// framework" (a conservative selector, then top-p pruning of its tokens) and "Key designs"
// (binary-search top-p, 4-bit K cache, head flattening for load balancing); summary, sections
// 4.1-4.3 and appendices B.1-B.2 (INT4 SpGEMV once per GQA group over the union of the heads'
// pages, group-wise variable-length attention).
//
// Every dependency of the path stays inside one (sequence, kv-head) group, but the work of a group
// is far from uniform: page scoring and the INT4 estimate stream megabytes, top-k and top-p are
// per-head searches over a few kilobytes, attention scales with the kept tokens (which differ
// ~50x between heads).  So the step is cut into work items, each a job for one CTA:
//   score   a chunk of a group's pages, scored for all G heads       -> order keys  (L2)
//   top-k   one q-head's k best pages                                -> page bitmap (L2)
//           the last top-k item of a group forms the union of its heads' pages and, per union
//           page, its physical page and its rank in each head's selection
//   est     a slice of the union: INT4 dequant-dot on the tensor cores -> logits per head (L2)
//   prune   one q-head: softmax, top-p threshold m by bisection     -> kept-row bitmap (L2)
//           the last prune item of a group lists the group's kept tokens (the union over heads)
//   attend  a slice of that list: fp16 K/V rows gathered, partial (max, sum, o) per head
//           the last attend item of a group merges the partials by log-sum-exp -> o, lse
// Items are numbered so that an item depends only on lower-numbered items; the grid is launched
// with every CTA resident, and each CTA takes the next free number (one atomic).  The lowest
// unfinished item therefore always has a CTA working on it, so the waits below always end; each
// is still bounded (TWL_FLAG_TIMEOUT), after which the launch finishes without the missing work.
// A dependency is a per-group counter in the workspace: producers add to it after a release
// fence, consumers poll it with acquire loads and read the produced data through L2.  The last
// CTA to leave clears the counters for the next launch on the workspace.
//
// The arithmetic (score order, INT4 products, softmax and threshold search, attention) is the
// same as the staged kernels', so the selections are bit-identical to twl_select_pages.
//
// This file is built twice: with 512-thread CTAs, one per SM (namespace step, the default), and
// with 256-thread CTAs, two per SM (twl_step_256.cu: namespace step256), for batches with more
// groups than SMs, where two resident items per SM hide each other's latency.
#include "twl_common.cuh"
#include "twl_step.h"

#ifndef TWL_STEP_THREADS
#define TWL_STEP_THREADS 512
#endif
#ifndef TWL_STEP_NS
#define TWL_STEP_NS step
#endif

namespace twl {
namespace TWL_STEP_NS {
using namespace ::twl::step;  // the argument types and constants of twl_step.h
namespace {

constexpr int kThreads = TWL_STEP_THREADS;
static_assert(kThreads == 512 || kThreads == 256, "512 or 256 threads per CTA");
constexpr int kCtasPerSm = 512 / kThreads;  // resident CTAs per SM the build is sized for
constexpr int kWarps = kThreads / 32;
constexpr uint32_t kSpinLimit = 1u << 22;  // polls (>= 64 ns apart) before a wait gives up
                                           // (the default of Args::spin_limit)

struct Shared {
  int flag;
  int next;
  int total;
  int jlast;
  int scan[64];
  uint32_t state[4];
  int att[2][4];       // attention producers: the chunk taken (slot, group, first, end page)
  int att_desc[3][4];  // attention ring: per buffer (tokens, slot, group, flags)
  int att_last;        // attention consumers: this chunk completed its group
  int att_prod_ok;     // attention producers: the wait for a free buffer succeeded
  __align__(8) uint64_t att_full[3];   // attention ring: buffer filled (producers -> consumers)
  __align__(8) uint64_t att_empty[3];  // attention ring: buffer consumed (consumers -> producers)
  unsigned long long t_ready;    // trace builds: when the item's wait ended
  unsigned long long marks[10];  // trace builds: points inside the item
};

// Trace build (compile with -DTWL_STEP_TRACE; never in the shipped library): thread 0 of every CTA
// records, per item, (index, CTA, start, wait end, 10 marks, end) in %globaltimer nanoseconds and
// the SM clock at start and end into a region
// at the start of the step's workspace region (before its other arrays).
#ifdef TWL_STEP_TRACE
__device__ __forceinline__ unsigned long long now_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
#define TRACE_MARK(sh, k)                                  \
  do {                                                     \
    if (threadIdx.x == 0) (sh).marks[(k)] = now_ns();      \
  } while (0)
#else
#define TRACE_MARK(sh, k) \
  do {                    \
  } while (0)
#endif

// ------------------------------------------------------------------------------ synchronisation
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t* counter(const Args& a, int which, int g) {
  return a.sync + kSyncHead + which * a.groups + g;
}

// Wait (whole CTA) until *ctr >= target.  False when the wait gave up: the launch was aborted
// by another CTA's timeout, or this one timed out (it then raises the flag and aborts).
__device__ bool block_wait(const Args& a, Shared& sh, const uint32_t* ctr, uint32_t target) {
  if (threadIdx.x == 0) {
    int ok = 1;
    uint32_t it = 0;
    while (ld_acquire(ctr) < target) {
      if ((++it & 31u) == 0u) {
        if (ld_acquire(a.sync + kAbort) != 0u) {
          ok = 0;
          break;
        }
        if (it >= a.spin_limit) {
          raise_flag(a.flags, TWL_FLAG_TIMEOUT);
          atomicExch(a.sync + kAbort, 1u);
          ok = 0;
          break;
        }
      }
      __nanosleep(64);
    }
    sh.flag = ok;
#ifdef TWL_STEP_TRACE
    sh.t_ready = now_ns();
#endif
  }
  __syncthreads();
  const bool ok = sh.flag != 0;
  __syncthreads();
  return ok;
}

// The CTA's results are complete: count this item with a release reduction.  The block barrier
// orders every thread's writes before thread 0's release (release is cumulative), so a consumer
// that acquires the counter sees them.
__device__ __forceinline__ void red_release_add(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t atom_acq_rel_add(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v)
               : "memory");
  return old;
}

__device__ void block_signal(uint32_t* ctr) {
  __syncthreads();
  if (threadIdx.x == 0) red_release_add(ctr, 1u);
}

// As block_signal; true in every thread of the CTA whose item brought the count to `total`.  Its
// atomic is acquire-release, so that CTA then sees every other item's results.
__device__ bool block_signal_last(Shared& sh, uint32_t* ctr, uint32_t total) {
  __syncthreads();
  if (threadIdx.x == 0) sh.flag = atom_acq_rel_add(ctr, 1u) + 1u == total;
  __syncthreads();
  const bool last = sh.flag != 0;
  __syncthreads();
  return last;
}

__device__ __forceinline__ float ldcg_f(const float* p) { return __ldcg(p); }
__device__ __forceinline__ int ldcg_i(const int* p) { return __ldcg(p); }
__device__ __forceinline__ uint32_t ldcg_u(const uint32_t* p) { return __ldcg(p); }
__device__ __forceinline__ int4 ldcg_i4(const int4* p) { return __ldcg(p); }
__device__ __forceinline__ uint32_t saddr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
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

__device__ __forceinline__ int group_of(const Args& a, int bh) {
  return (bh / a.hq) * a.kv.hkv + (bh % a.hq) / a.g;
}

// ------------------------------------------------------------------------------ scores
// Pages [c * chunk, (c + 1) * chunk) of the group's sequence, scored for every head of the group.
// The chunk's page-table entries are staged first; the page bounds (512 B per page) are then
// copied with 16-byte cp.async in passes of up to kScorePass pages, two passes in flight (every
// copy of a pass is issued at once: measured the fastest way to pull tens of kilobytes per SM).
// A half-warp scores a page: lane l holds channels 8l..8l+7 of the min and max rows and of each
// head's query, so the score is the fixed order of the staged selector (8 channels per lane left
// to right, then the pairs (l, l+8), (l, l+4), (l, l+2), (l, l+1)).
constexpr int kScorePass = kThreads == 512 ? 176 : 64;

// Packed fp32 FMA on two lanes (a.x*b.x + c.x, a.y*b.y + c.y), each lane rounded as fmaf.
__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b,
                                                   unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ unsigned long long pack2(float x, float y) {
  return (unsigned long long)__float_as_uint(x) | ((unsigned long long)__float_as_uint(y) << 32);
}

// The score of the half-warp's page for every head, in the fixed order: lane l's partial sum of
// channels 8l..8l+7 (from +0, left to right), then the pairs (l, l^8), (l, l^4), (l, l^2),
// (l, l^1).  Each term is q_c * max_c (q_c > 0) or q_c * min_c: written as fma(q+, max, acc)
// followed by fma(q-, min, acc), one of which adds an exact zero, so the sum rounds exactly as
// acc + t_c.  Two heads share each packed FMA.  The tree exchanges halves of the head set at
// each level (every sum still pairs the same two partial sums), so lane l ends with the score of
// head l / (16 / G) when l is a multiple of 16 / G.
template <int G, int NV>
__device__ __forceinline__ float score_tree(float (&v)[NV], int l) {
  // exchange tree over offsets 8, 4, 2, 1 (within the half-warp)
  int n = G;
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) {
    if (n > 1) {
      const bool up = (l & o) != 0;
      const int half = n / 2;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (i < half) {
          const float send = up ? v[i] : v[i + half];
          const float keep = up ? v[i + half] : v[i];
          v[i] = __fadd_rn(keep, __shfl_xor_sync(0xffffffffu, send, o));
        }
      }
      n = half;
    } else {
      v[0] = __fadd_rn(v[0], __shfl_xor_sync(0xffffffffu, v[0], o));
    }
  }
  return v[0];
}

template <int G>
__device__ __forceinline__ float page_score(const unsigned long long (&qp)[(G + 1) / 2][8],
                                            const unsigned long long (&qn)[(G + 1) / 2][8],
                                            const float (&mn)[8], const float (&mx)[8], int l) {
  constexpr int GP = (G + 1) / 2;
  float v[2 * GP];
#pragma unroll
  for (int hp = 0; hp < GP; ++hp) {
    unsigned long long acc = 0ull;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      acc = fma2(qp[hp][k], pack2(mx[k], mx[k]), acc);
      acc = fma2(qn[hp][k], pack2(mn[k], mn[k]), acc);
    }
    v[2 * hp] = __uint_as_float((uint32_t)acc);
    v[2 * hp + 1] = __uint_as_float((uint32_t)(acc >> 32));
  }
  return score_tree<G>(v, l);
}

// The same for eight heads (the packed (q+, q-) pairs would take 128 registers): the term is
// selected per head and added with one scalar FMA (the same rounding).
__device__ __forceinline__ float page_score8(const float (&qv)[8][8], const float (&mn)[8],
                                             const float (&mx)[8], int l) {
  float v[8];
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    float acc = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) acc = __fmaf_rn(qv[h][k], qv[h][k] > 0.f ? mx[k] : mn[k], acc);
    v[h] = acc;
  }
  return score_tree<8>(v, l);
}

template <int G>
__device__ void item_score(const Args& a, Shared& sh, int g, int c, unsigned char* smem) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int half = lane >> 4, l = lane & 15;
  const int b = g / a.kv.hkv, kvh = g - b * a.kv.hkv;
  // the chunk's page-table entries are read before the sequence length is known (entries past
  // the sequence are in the table, only ignored), so the two loads overlap
  const int p0 = c * a.s_chunk, pmax = min(a.kv.max_pages, p0 + a.s_chunk);
  int* pt = reinterpret_cast<int*>(smem);
  unsigned char* buf = smem + ((4 * a.s_chunk + 127) & ~127);
  for (int i = tid; i < pmax - p0; i += kThreads)
    pt[i] = a.kv.page_table[(size_t)b * a.kv.max_pages + p0 + i];
  const Seq sq = load_seq(a.kv.seq_lens, b, a.kv.max_pages, a.flags, c == 0 && tid == 0);
  const int p1 = min(sq.pages, pmax);
  const int n = p1 - p0;
  if (n > 0) {
    for (int i = tid; i < n; i += kThreads) {
      const int ph = pt[i];
      if (ph < 0 || ph >= a.kv.num_phys) {
        raise_flag(a.flags, TWL_FLAG_BAD_INDEX);
        pt[i] = -1;
      }
    }
    constexpr int GP = (G + 1) / 2;
    constexpr bool kPacked = G <= 4;
    // (q+, q-) of heads (2i, 2i+1), channels 8l..8l+7 (packed form), or q itself (eight heads)
    unsigned long long qp[kPacked ? GP : 1][8], qn[kPacked ? GP : 1][8];
    float q8[kPacked ? 1 : 8][8];
    if constexpr (!kPacked) {
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(
                                    a.q + ((size_t)b * a.hq + kvh * G + h) * kHeadDim) + l);
        unpack8(raw, q8[h]);
      }
    } else {
      float qv[2 * GP][8];
#pragma unroll
      for (int h = 0; h < 2 * GP; ++h) {
        if (h < G) {
          const uint4 raw = __ldg(reinterpret_cast<const uint4*>(
                                      a.q + ((size_t)b * a.hq + kvh * G + h) * kHeadDim) + l);
          unpack8(raw, qv[h]);
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k) qv[h][k] = 0.f;
        }
      }
#pragma unroll
      for (int hp = 0; hp < GP; ++hp)
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float x = qv[2 * hp][k], y = qv[2 * hp + 1][k];
          qp[hp][k] = pack2(x > 0.f ? x : 0.f, y > 0.f ? y : 0.f);
          qn[hp][k] = pack2(x > 0.f ? 0.f : x, y > 0.f ? 0.f : y);
        }
    }
    (void)qp;
    (void)qn;
    (void)q8;
    __syncthreads();
    TRACE_MARK(sh, 0);
    const int npass = (n + kScorePass - 1) / kScorePass;
    auto issue = [&](int k) {
      unsigned char* dst = buf + (k & 1) * kScorePass * 512;
      const int i0 = k * kScorePass, cn = min(kScorePass, n - i0);
      for (int q = tid; q < 32 * cn; q += kThreads) {
        const int i = q >> 5, part = q & 31;
        const int ph = pt[i0 + i];
        const uint16_t* src = a.bounds + ((size_t)(ph < 0 ? 0 : ph) * a.kv.hkv + kvh) * 2 * kHeadDim;
        cp_async16(dst + 512 * i + 16 * part, src + 8 * part, ph >= 0);
      }
      cp_async_commit();
    };
    issue(0);
    if (npass > 1) issue(1);
    uint32_t* krow = a.keys + ((size_t)b * a.hq + kvh * G) * a.kv.max_pages + p0;
#pragma unroll 1
    for (int k = 0; k < npass; ++k) {
      if (k + 1 < npass) asm volatile("cp.async.wait_group 1;\n" ::: "memory");
      else cp_async_wait_all();
      __syncthreads();
      TRACE_MARK(sh, 1);
      const unsigned char* src = buf + (k & 1) * kScorePass * 512;
      const int i0 = k * kScorePass, cn = min(kScorePass, n - i0);
#pragma unroll 1
      for (int base = 0; base < cn; base += 2 * kWarps) {  // warp-uniform trip count
        const int ip = base + 2 * warp + half;
        const bool in = ip < cn;
        const int ph = in ? pt[i0 + ip] : -1;
        const uint4* rowp = reinterpret_cast<const uint4*>(src + 512 * ip);
        uint4 vmn = make_uint4(0, 0, 0, 0), vmx = vmn;
        if (ph >= 0) {
          vmn = rowp[l];
          vmx = rowp[16 + l];
        }
        float mn[8], mx[8];
        unpack8(vmn, mn);
        unpack8(vmx, mx);
        float v;
        if constexpr (kPacked) v = page_score<G>(qp, qn, mn, mx, l);
        else v = page_score8(q8, mn, mx, l);
        constexpr int kStride = 16 / G;  // lanes per head after the exchange tree
        if (in && (l % kStride) == 0) {
          if (ph < 0) v = -INFINITY;
          krow[(size_t)(l / kStride) * a.kv.max_pages + i0 + ip] = f32_key(v);
        }
      }
      __syncthreads();  // the pass's buffer is read before it is refilled
      if (k + 2 < npass) issue(k + 2);
    }
  }
  block_signal(counter(a, kCntScore, g));
}

// ------------------------------------------------------------------------------ top-k
// The kb largest keys of one head (ties to the lower page) -> bitmap of its selected pages.
// The k-th largest key is narrowed to a key interval [blo, bhi] holding `cand` keys, of which the
// `remaining` largest are selected (every key above bhi is).  Each pass histograms the keys inside
// the interval into up to 4096 bins of equal key width and keeps the bin holding the k-th key;
// float keys are roughly logarithmic in the score, so one pass usually leaves a handful.  A bin of
// at most 64 keys is ranked exactly; an interval down to one key takes its equal keys in page
// order.  Writes the bitmap (sbits, shared) and returns nothing; sh.jlast = the last selected page.
__device__ void topk_bits(const uint32_t* keys, int n_pages, int kb, uint32_t* sbits,
                          unsigned char* scratch, int scratch_bytes, Shared& sh) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nw = (n_pages + 31) >> 5;
  constexpr int kGatherCap = 64;
  constexpr int kBins = 4096;
  constexpr int kPerT = kBins / kThreads;  // bins per thread in the scan (8 or 16)
  // the bins, one padding word after every kPerT (bin b at word b + b / kPerT), so that the
  // scan's per-thread runs of kPerT bins start kPerT + 1 words apart and load free of bank
  // conflicts
  uint32_t* hh = reinterpret_cast<uint32_t*>(scratch);  // [kBins + kBins / kPerT]
  uint32_t* gkey = hh + kBins + kBins / kPerT;          // [kGatherCap]
  int* gidx = reinterpret_cast<int*>(gkey + kGatherCap);  // [kGatherCap]
  (void)scratch_bytes;
  uint32_t blo, bhi;
  {
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
    for (int i = tid; i < n_pages; i += kThreads) {
      const uint32_t k = keys[i];
      kmin = min(kmin, k);
      kmax = max(kmax, k);
    }
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    if (lane == 0) {
      hh[2 * warp] = kmin;
      hh[2 * warp + 1] = kmax;
    }
    __syncthreads();
    kmin = 0xFFFFFFFFu;
    kmax = 0u;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      kmin = min(kmin, hh[2 * w]);
      kmax = max(kmax, hh[2 * w + 1]);
    }
    blo = kmin;
    bhi = kmax;
  }
  int remaining = kb;
  int cand = n_pages;
  __syncthreads();
#pragma unroll 1
  while (cand > kGatherCap && blo < bhi) {
    const uint32_t range = bhi - blo;
    const int width = 32 - __clz(range);
    const int sh_ = width > 12 ? width - 12 : 0;
    for (int i = tid; i < kBins + kBins / kPerT; i += kThreads) hh[i] = 0u;
    __syncthreads();
    for (int i = tid; i < n_pages; i += kThreads) {
      const uint32_t key = keys[i];
      if (key >= blo && key <= bhi) {
        const uint32_t b = (key - blo) >> sh_;
        atomicAdd(&hh[b + b / kPerT], 1u);
      }
    }
    __syncthreads();
    // descending scan over the bins: thread t owns bins kBins-1-kPerT*t ... kBins-kPerT*(t+1)
    const int b0 = kBins - 1 - kPerT * tid;
    int mine = 0;
#pragma unroll
    for (int e = 0; e < kPerT; ++e) mine += (int)hh[(b0 - e) + (b0 - e) / kPerT];
    const int excl = block_exclusive_scan(mine, sh.scan, nullptr);
    if (excl < remaining && remaining <= excl + mine) {
      int run = excl;
      for (int e = 0; e < kPerT; ++e) {
        const int c = (int)hh[(b0 - e) + (b0 - e) / kPerT];
        if (run + c >= remaining) {
          sh.state[0] = (uint32_t)(b0 - e);
          sh.state[1] = (uint32_t)(remaining - run);
          sh.state[2] = (uint32_t)c;
          break;
        }
        run += c;
      }
    }
    __syncthreads();
    const uint32_t bin = sh.state[0];
    const uint32_t nlo = blo + (bin << sh_);
    const uint64_t top = (uint64_t)nlo + ((1ull << sh_) - 1ull);
    bhi = top < (uint64_t)bhi ? (uint32_t)top : bhi;
    blo = nlo;
    remaining = (int)sh.state[1];
    cand = (int)sh.state[2];
    __syncthreads();
  }
  for (int w = tid; w < nw; w += kThreads) sbits[w] = 0u;
  if (cand <= kGatherCap) {
    // ordered gather of the interval's keys: thread t scans a contiguous range of pages
    const int per = (n_pages + kThreads - 1) / kThreads;
    const int beg = min(n_pages, tid * per), end = min(n_pages, beg + per);
    int mine = 0;
    for (int i = beg; i < end; ++i) {
      const uint32_t key = keys[i];
      mine += key >= blo && key <= bhi;
    }
    int slot = block_exclusive_scan(mine, sh.scan, nullptr);
    for (int i = beg; i < end && mine > 0; ++i) {
      const uint32_t key = keys[i];
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
      const bool above = i < n_pages && keys[i] > bhi;
      const uint32_t bal = __ballot_sync(0xffffffffu, above);
      if (lane == 0 && (i >> 5) < nw) atomicOr(&sbits[i >> 5], bal);
    }
    __syncthreads();
    return;
  }
  // the interval is down to one key (blo == bhi, the k-th key itself): keys above it are taken,
  // equal keys in ascending page order.  One element per thread per round; a warp's ballot is
  // one 32-page word of the bitmap.
  int* wsum = sh.scan;
  int carry_eq = 0;
  const uint32_t lt = (1u << lane) - 1u;
  for (int base = 0; base < 32 * nw; base += kThreads) {
    const int i = base + tid;
    const bool in = i < n_pages;
    const uint32_t key = in ? keys[i] : 0u;
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
    if (lane == 0 && (i >> 5) < nw) sbits[i >> 5] = sel;
    carry_eq += eq_round;
    __syncthreads();
  }
}

// One q-head's selection: bitmap -> workspace, candidate count, optional stats.
template <int G>
__device__ void item_topk(const Args& a, Shared& sh, int bh, unsigned char* smem, int smem_bytes) {
  const int tid = threadIdx.x;
  const int g = group_of(a, bh);
  const bool ready = block_wait(a, sh, counter(a, kCntScore, g), (uint32_t)a.s_per);
  const int b = bh / a.hq;
  uint32_t* sbits = reinterpret_cast<uint32_t*>(smem);                            // [sel_words]
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem + 4 * ((a.sel_words + 31) & ~31));
  unsigned char* scratch = reinterpret_cast<unsigned char*>(keys) + 4 * ((a.kv.max_pages + 31) & ~31);
  const int scratch_bytes = smem_bytes - (int)(scratch - smem);
  // the key row is loaded up to max_pages while the sequence length is read (keys past the
  // sequence are never used)
  {
    const uint32_t* row = a.keys + (size_t)bh * a.kv.max_pages;
    constexpr int kB = 8;  // independent loads in flight per thread
    for (int base = 0; base < a.kv.max_pages; base += kThreads * kB) {
      uint32_t v[kB];
#pragma unroll
      for (int k = 0; k < kB; ++k) {
        const int i = base + k * kThreads + tid;
        v[k] = i < a.kv.max_pages ? ldcg_u(row + i) : 0u;
      }
#pragma unroll
      for (int k = 0; k < kB; ++k) {
        const int i = base + k * kThreads + tid;
        if (i < a.kv.max_pages) keys[i] = v[k];
      }
    }
  }
  const Seq sq = load_seq(a.kv.seq_lens, b, a.kv.max_pages, a.flags, false);
  const int n_pages = ready ? sq.pages : 0;
  int kb = a.budget_pages > 0 ? a.budget_pages : (n_pages + a.budget_div - 1) / a.budget_div;
  kb = min(min(kb, n_pages), a.max_budget);
  const int nw = (n_pages + 31) >> 5;
  __syncthreads();
  TRACE_MARK(sh, 0);
  if (n_pages > 0 && n_pages <= kb) {
    for (int w = tid; w < nw; w += kThreads) {
      const int lo = 32 * w;
      sbits[w] = lo + 32 <= n_pages ? 0xFFFFFFFFu : ((1u << (n_pages - lo)) - 1u);
    }
    __syncthreads();
  } else if (n_pages > 0) {
    topk_bits(keys, n_pages, kb, sbits, scratch, scratch_bytes, sh);
  }
  TRACE_MARK(sh, 1);
  // bitmap and per-word exclusive prefix counts out (a page's rank in the selection is
  // hpre[w] + popc(bits[w] below it)); the last selected page fixes the candidate count (only it
  // can be partial); the ascending list when asked
  uint32_t* out = a.selbits + (size_t)bh * a.sel_words;
  int* pre = a.hpre + (size_t)bh * a.sel_words;
  int* list = a.sel_pages ? a.sel_pages + (size_t)bh * a.max_budget : nullptr;
  int carry = 0, jlast = -1;
  for (int base = 0; base < nw; base += kThreads) {
    const int w = base + tid;
    const uint32_t x = w < nw ? sbits[w] : 0u;
    int total;
    int pos = carry + block_exclusive_scan(__popc(x), sh.scan, &total);
    carry += total;
    if (w < nw) {
      out[w] = x;
      pre[w] = pos;
      if (x) jlast = 32 * w + 31 - __clz(x);
    }
    if (list) {
      uint32_t y = x;
      while (y) {
        list[pos++] = 32 * w + __ffs(y) - 1;
        y &= y - 1u;
      }
    }
  }
  if (tid == 0) sh.jlast = -1;
  __syncthreads();
  if (jlast >= 0) atomicMax(&sh.jlast, jlast);
  __syncthreads();
  if (tid == 0) {
    const int jl = sh.jlast;
    const int nc = (kb > 0 && jl >= 0) ? kPage * (kb - 1) + page_rows(sq.n, jl) : 0;
    a.ncand[bh] = nc;
    if (a.sel_count) a.sel_count[bh] = kb;
  }
}

// ------------------------------------------------------------------------------ INT4 estimate
// B fragments of the query for the m16n8k16 products: lane (gr, t) holds the channels
// c0 = 32 t + 8 w8 (w8 = ks / 2) of head gr; k-step ks pairs (c0 + 4e, c0 + 4e + 2) and
// (c0 + 4e + 1, c0 + 4e + 3), e = ks % 2, the same pairs nibble_pairs() builds from K.
// Returns the sum of the lane's 32 query channels (for the zero-point term).
__device__ __forceinline__ float q_fragments(const uint16_t* qh, bool valid, uint32_t (&bf)[8][2]) {
  const int t = threadIdx.x & 3;
  uint32_t w[16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 v = valid ? __ldg(reinterpret_cast<const uint4*>(qh + 32 * t + 8 * i))
                          : make_uint4(0, 0, 0, 0);
    w[4 * i + 0] = v.x;
    w[4 * i + 1] = v.y;
    w[4 * i + 2] = v.z;
    w[4 * i + 3] = v.w;
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
// first) gives the bytes (n0, n2, n4, n6) and (n1, n3, n5, n7); each 16-bit half converts to one
// f16x2 pair.  Products with q are 2^-9 times the integer-nibble products and the fp32 sums scale
// exactly; the epilogue multiplies by 512.
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
// The four A registers of k-step (w8, e) for rows gr (word x0) and gr + 8 (word x1).
__device__ __forceinline__ void nibble_pairs(uint32_t x0, uint32_t x1, int e, uint32_t (&av)[4]) {
  const uint32_t e0 = x0 & 0x0F0F0F0Fu, o0 = (x0 >> 4) & 0x0F0F0F0Fu;
  const uint32_t e1 = x1 & 0x0F0F0F0Fu, o1 = (x1 >> 4) & 0x0F0F0F0Fu;
  av[0] = e ? e4m3x2_hi(e0) : e4m3x2_lo(e0);
  av[1] = e ? e4m3x2_hi(e1) : e4m3x2_lo(e1);
  av[2] = e ? e4m3x2_hi(o0) : e4m3x2_lo(o0);
  av[3] = e ? e4m3x2_hi(o1) : e4m3x2_lo(o1);
}

// Logical pages [c * chunk, (c + 1) * chunk) of group g, in sub-ranges of up to kEstMeta pages:
// the union of the heads' selections over the sub-range comes from their bitmaps, and every union
// page's (logical page, physical page, rank in each head's selection) is staged; the rank is the
// head's published prefix count of its bitmap word plus the set bits below the page.  The INT4
// tiles (1 KB) and scale/zero rows (64 B) of those pages are then copied with 16-byte cp.async in
// passes of kEstPass pages, two in flight.  A warp computes two pages at a time, the page as the
// M = 16 tile of m16n8k16 and the group's heads as N.  Logit slot of (head h, page j, row r) =
// 16 * (rank of j in h's selection) + r.
constexpr int kEstPass = kThreads == 512 ? 80 : 32;
constexpr int kEstMeta = 480;  // a multiple of kEstPass, and of 32
static_assert(kEstMeta % kEstPass == 0 && kEstMeta % 32 == 0, "estimate sub-range");

template <int G>
__device__ void item_estimate(const Args& a, Shared& sh, int g, int e, unsigned char* smem) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gr = lane >> 2, t = lane & 3;
  // (a test of the timeout path makes this wait unreachable: stall_estimate)
  const bool ready = block_wait(a, sh, counter(a, kCntTopK, g),
                                a.stall_estimate ? 0xFFFFFFFFu : (uint32_t)a.g);
  const int b = g / a.kv.hkv, kvh = g - b * a.kv.hkv;
  const Seq sq = load_seq(a.kv.seq_lens, b, a.kv.max_pages, a.flags, false);
  const int p0 = e * a.e_chunk, p1 = ready ? min(sq.pages, p0 + a.e_chunk) : 0;
  if (p0 < p1) {
    const float inv_sqrt_d = 0.08838834764831845f;
    constexpr int kM = 2 + G;  // ints of metadata per page
    constexpr int kW = kEstMeta / 32 + 1;  // bitmap words a sub-range touches
    int* meta = reinterpret_cast<int*>(smem);
    uint32_t* hb = reinterpret_cast<uint32_t*>(meta + kM * kEstMeta);  // [G][kW]
    int* hp = reinterpret_cast<int*>(hb + G * kW);                     // [G][kW]
    uint32_t* ub = reinterpret_cast<uint32_t*>(hp + G * kW);           // [kW]
    int* upre = reinterpret_cast<int*>(ub + kW);                       // [kW + 1]
    unsigned char* buf = smem + ((4 * (kM * kEstMeta + (2 * G + 2) * kW + 1) + 127) & ~127);
    const size_t row0 = (size_t)b * a.hq + kvh * G;
    uint32_t bf[8][2];
    const bool head_ok = gr < G;
    const uint16_t* qh = a.q + ((size_t)b * a.hq + kvh * G + (head_ok ? gr : 0)) * kHeadDim;
    float qs_part = q_fragments(qh, head_ok, bf);
    qs_part += __shfl_xor_sync(0xffffffffu, qs_part, 1);
    qs_part += __shfl_xor_sync(0xffffffffu, qs_part, 2);
    const float qsum0 = __shfl_sync(0xffffffffu, qs_part, (2 * t) * 4);
    const float qsum1 = __shfl_sync(0xffffffffu, qs_part, (2 * t + 1) * 4);
#pragma unroll 1
    for (int j0 = p0; j0 < p1; j0 += kEstMeta) {
      const int j1 = min(p1, j0 + kEstMeta);
      const int w0 = j0 >> 5, nwr = ((j1 - 1) >> 5) - w0 + 1;
      for (int i = tid; i < G * nwr; i += kThreads) {
        const int h = i / nwr, wi = i - h * nwr;
        hb[h * kW + wi] = ldcg_u(a.selbits + (row0 + h) * a.sel_words + w0 + wi);
        hp[h * kW + wi] = ldcg_i(a.hpre + (row0 + h) * a.sel_words + w0 + wi);
      }
      __syncthreads();
      if (warp == 0) {  // union words cut to [j0, j1), and their exclusive prefix counts
        uint32_t u = 0;
        if (lane < nwr) {
#pragma unroll
          for (int h = 0; h < G; ++h) u |= hb[h * kW + lane];
          const int lo = 32 * (w0 + lane);
          if (lo < j0) u &= ~((1u << (j0 - lo)) - 1u);
          if (lo + 32 > j1) u &= j1 - lo >= 32 ? 0xFFFFFFFFu : ((1u << (j1 - lo)) - 1u);
          ub[lane] = u;
        }
        int x = __popc(u);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += y;
        }
        if (lane < nwr) upre[lane] = x - __popc(u);
        if (lane == 31) upre[kW] = x;
      }
      __syncthreads();
      const int n = upre[kW];
      for (int jj = j0 + tid; jj < j1; jj += kThreads) {
        const int wi = (jj >> 5) - w0, bit = jj & 31;
        const uint32_t below = (1u << bit) - 1u;
        const uint32_t uw = ub[wi];
        if ((uw >> bit) & 1u) {
          int* mm = meta + kM * (upre[wi] + __popc(uw & below));
          mm[0] = jj;
          mm[1] = load_phys(a.kv.page_table, b, jj, a.kv.max_pages, a.kv.num_phys, a.flags);
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const uint32_t x = hb[h * kW + wi];
            mm[2 + h] = ((x >> bit) & 1u) ? hp[h * kW + wi] + __popc(x & below) : -1;
          }
        }
      }
      __syncthreads();
      TRACE_MARK(sh, 0);
      const int npass = (n + kEstPass - 1) / kEstPass;
      auto issue = [&](int k) {
        unsigned char* tl = buf + (k & 1) * kEstPass * 1088;
        unsigned char* sz = tl + kEstPass * 1024;
        const int i0 = k * kEstPass, cn = min(kEstPass, n - i0);
        // 68 chunks of 16 bytes per page (64 of nibbles, 4 of scale/zero)
        for (int q = tid; q < 68 * cn; q += kThreads) {
          const int i = q / 68, kk = q - 68 * i;
          const int ph = meta[(i0 + i) * kM + 1];
          const size_t tile = ph >= 0 ? ((size_t)ph * a.kv.hkv + kvh) * kPage : 0;
          if (kk < 64)
            cp_async16(tl + 1024 * i + 16 * kk, a.k_int4 + tile * (kHeadDim / 2) + 16 * kk, ph >= 0);
          else
            cp_async16(sz + 64 * i + 16 * (kk - 64), a.k_sz + tile * 2 + 8 * (kk - 64), ph >= 0);
        }
        cp_async_commit();
      };
      issue(0);
      if (npass > 1) issue(1);
#pragma unroll 1
      for (int k = 0; k < npass; ++k) {
        if (k + 1 < npass) asm volatile("cp.async.wait_group 1;\n" ::: "memory");
        else cp_async_wait_all();
        __syncthreads();
        TRACE_MARK(sh, 1);
        const unsigned char* tl = buf + (k & 1) * kEstPass * 1088;
        const unsigned char* sz = tl + kEstPass * 1024;
        const int i0 = k * kEstPass, cn = min(kEstPass, n - i0);
#pragma unroll 1
        for (int ib = 2 * warp; ib < cn; ib += 2 * kWarps) {  // warp-uniform
          float accp[2][4];
          uint32_t szp[2][2];
#pragma unroll
          for (int pp = 0; pp < 2; ++pp) {
            const int ip = ib + pp;
            uint4 x0 = make_uint4(0, 0, 0, 0), x1 = x0;
            szp[pp][0] = szp[pp][1] = 0;
            if (ip < cn && meta[(i0 + ip) * kM + 1] >= 0) {
              const uint4* tp = reinterpret_cast<const uint4*>(tl + 1024 * ip);
              x0 = tp[lane];
              x1 = tp[32 + lane];
              const uint32_t* sp = reinterpret_cast<const uint32_t*>(sz + 64 * ip);
              szp[pp][0] = sp[gr];
              szp[pp][1] = sp[gr + 8];
            }
            const uint32_t r0[4] = {x0.x, x0.y, x0.z, x0.w};
            const uint32_t r1[4] = {x1.x, x1.y, x1.z, x1.w};
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
              const int w8 = ks >> 1, e2 = ks & 1;
              uint32_t av[4];
              nibble_pairs(r0[w8], r1[w8], e2, av);
              mma_16816(acc, av, bf[ks][0], bf[ks][1]);
            }
#pragma unroll
            for (int k2 = 0; k2 < 4; ++k2) accp[pp][k2] = acc[k2];
          }
#pragma unroll
          for (int pp = 0; pp < 2; ++pp) {
            const int ip = ib + pp;
            if (ip >= cn) break;  // warp-uniform
            const int* mm = meta + (i0 + ip) * kM;
            const int j = mm[0];
            const bool bad = mm[1] < 0;
            const int rows = page_rows(sq.n, j);
            const uint32_t sz0 = szp[pp][0], sz1 = szp[pp][1];
            const float s0 = __half2float(__ushort_as_half((unsigned short)(sz0 & 0xFFFFu)));
            const float z0 = __half2float(__ushort_as_half((unsigned short)(sz0 >> 16)));
            const float s1 = __half2float(__ushort_as_half((unsigned short)(sz1 & 0xFFFFu)));
            const float z1 = __half2float(__ushort_as_half((unsigned short)(sz1 >> 16)));
#pragma unroll
            for (int e2 = 0; e2 < 2; ++e2) {
              const int hl = 2 * t + e2;
              if (hl >= G) continue;
              const int rk = mm[2 + hl];
              if (rk < 0) continue;
              const int bh = b * a.hq + kvh * G + hl;
              const float qsum = e2 ? qsum1 : qsum0;
              const size_t obase = (size_t)bh * a.cand_stride + (size_t)rk * kPage;
#pragma unroll
              for (int rr = 0; rr < 2; ++rr) {
                const int row = gr + 8 * rr;
                if (row >= rows) continue;
                const float sv = rr ? s1 : s0, zv = rr ? z1 : z0;
                const float lg =
                    bad ? -INFINITY
                        : (sv * (accp[pp][2 * rr + e2] * 512.f) + zv * qsum) * inv_sqrt_d;
                a.logits[obase + row] = lg;
                if (a.cand_tok) a.cand_tok[obase + row] = kPage * j + row;
              }
            }
          }
        }
        __syncthreads();  // the pass's buffer is read before it is refilled
        if (k + 2 < npass) issue(k + 2);
      }
    }
  }
  block_signal(counter(a, kCntEst, g));
}

// ------------------------------------------------------------------------------ prune
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
// do not depend on the order of the terms.
__device__ __forceinline__ long long w_fixed(float w) { return __float2ll_rn(w * 281474976710656.f); }

// Sum over the block of one 64-bit value per thread (exact; every thread receives the total).
// `sh64` needs kWarps words.
__device__ unsigned long long block_sum_u64(unsigned long long v, unsigned long long* sh64) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) sh64[warp] = v;
  __syncthreads();
  unsigned long long t = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) t += sh64[w];
  return t;
}

// Exclusive prefix sum over the block of one 64-bit value per thread (thread order); *total gets
// the block total.  `sh64` needs kWarps + 1 words.
__device__ unsigned long long block_excl_u64(unsigned long long v, unsigned long long* sh64,
                                             unsigned long long* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) sh64[warp] = x;
  __syncthreads();
  unsigned long long before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const unsigned long long t = sh64[w];
    if (w < warp) before += t;
    all += t;
  }
  if (total) *total = all;
  return before + x - v;
}

// T among n <= kThreads weights gv (fixed-point copies gq) given the exact mass `above` of the
// weights above them: the largest v with above + mass(gv >= v) >= P (0 when none), by comparing
// all pairs at once (4, 2 or 1 threads per value).  Cheaper than refine_threshold up to a few
// hundred weights (its cost grows as n^2; the refinement's is about three block scans).
__device__ float rank_pairwise(const float* gv, const long long* gq, int n,
                               unsigned long long above, long long P, float* red) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tpv = n <= kThreads / 4 ? 4 : (n <= kThreads / 2 ? 2 : 1);
  const int i = tid / tpv, part = tid % tpv;
  unsigned long long mass = 0;
  float vi = 0.f;
  if (i < n) {
    vi = gv[i];
#pragma unroll 4
    for (int j = part; j < n; j += tpv) mass += gv[j] >= vi ? (unsigned long long)gq[j] : 0ull;
  }
  if (tpv >= 2) mass += __shfl_xor_sync(0xffffffffu, mass, 1);
  if (tpv >= 4) mass += __shfl_xor_sync(0xffffffffu, mass, 2);
  float t = (i < n && above + mass >= (unsigned long long)P) ? vi : 0.f;
  t = warp_max(t);
  __syncthreads();
  if (lane == 0) red[warp] = t;
  __syncthreads();
  float T = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) T = fmaxf(T, red[w]);
  __syncthreads();  // red is read before it is reused
  return T;
}
constexpr int kPairwiseMax = 384;  // rank_pairwise up to this many weights, refine_threshold above
constexpr int kHBins = 2048;                 // bins of the exact histograms
constexpr int kHPer = kHBins / kThreads;     // bins per thread in their scans (4 or 8)
constexpr int kPadBins = kHBins + kHBins / kHPer;  // words per part of a padded histogram

// T among n <= kThreads weights gv (fixed-point copies gq, units of 2^-48) whose keys (float
// bits) lie in [lo, hi], given the exact mass `above` of the weights with keys above hi: the
// largest value v with above + mass(gv >= v) >= P, or 0 when even all of them fall short.  The
// keys are histogrammed into up to kHBins bins of equal key width with exact masses (each
// fixed-point weight, < 2^49, summed as three 16-bit parts in 32-bit shared atomics: no overflow
// for n <= 2^15); a descending scan finds the bin where the mass from the top first reaches P, and
// the search narrows to that bin until it is a single key: at most three levels for 32-bit keys.
// A crossing bin holds mass, so the key found is one of the weights.  `bins` needs 3 * kHBins
// 32-bit words, `sh64` kWarps + 1.
__device__ float refine_threshold(const float* gv, const long long* gq, int n, uint32_t lo,
                                  uint32_t hi, unsigned long long above, long long P,
                                  uint32_t* bins, Shared& sh, unsigned long long* sh64) {
  const int tid = threadIdx.x;
  const bool mine = tid < n;
  const uint32_t u = mine ? __float_as_uint(gv[tid]) : 0u;
  const unsigned long long q = mine ? (unsigned long long)gq[tid] : 0ull;
#pragma unroll 1
  for (int level = 0; level < 4; ++level) {
    const uint32_t width = hi - lo;
    const int bits = 32 - __clz(width);
    const int s = bits > 11 ? bits - 11 : 0;
    const int nb = (int)(width >> s) + 1;
    // bin b at word b + b / kHPer of each part (the scan's runs of kHPer bins load
    // conflict-free)
    for (int i = tid; i < kPadBins; i += kThreads) {
      bins[i] = 0u;
      bins[kPadBins + i] = 0u;
      bins[2 * kPadBins + i] = 0u;
    }
    __syncthreads();
    if (mine && u >= lo && u <= hi) {
      const int b = (int)((u - lo) >> s);
      const int bp = b + b / kHPer;
      atomicAdd(&bins[bp], (uint32_t)(q & 0xFFFFu));
      atomicAdd(&bins[kPadBins + bp], (uint32_t)((q >> 16) & 0xFFFFu));
      atomicAdd(&bins[2 * kPadBins + bp], (uint32_t)(q >> 32));
    }
    __syncthreads();
    // descending scan: thread t holds bins nb-1-kHPer t .. nb-kHPer(t+1)
    unsigned long long mb[kHPer], tot = 0;
#pragma unroll
    for (int e = 0; e < kHPer; ++e) {
      const int b = nb - 1 - kHPer * tid - e, bp = b + b / kHPer;
      mb[e] = b >= 0 ? (unsigned long long)bins[bp] + ((unsigned long long)bins[kPadBins + bp] << 16) +
                           ((unsigned long long)bins[2 * kPadBins + bp] << 32)
                     : 0ull;
      tot += mb[e];
    }
    if (tid == 0) sh.state[3] = 0xFFFFFFFFu;
    unsigned long long run = above + block_excl_u64(tot, sh64, nullptr);
#pragma unroll
    for (int e = 0; e < kHPer; ++e) {
      const int b = nb - 1 - kHPer * tid - e;
      if (b >= 0 && run < (unsigned long long)P && run + mb[e] >= (unsigned long long)P) {
        sh.state[3] = (uint32_t)b;
        sh64[kWarps] = run;  // mass above the crossing bin
      }
      run += mb[e];
    }
    __syncthreads();
    const uint32_t bx = sh.state[3];
    const unsigned long long ab = sh64[kWarps];
    __syncthreads();  // read before the next level (or the caller) writes them
    if (bx == 0xFFFFFFFFu) return 0.f;
    above = ab;
    lo = lo + (bx << s);
    const uint64_t top_key = (uint64_t)lo + ((1ull << s) - 1ull);
    hi = top_key < (uint64_t)hi ? (uint32_t)top_key : hi;
    if (lo == hi) return __uint_as_float(lo);
  }
  return 0.f;
}

// T for a large live set: the largest weight value v with mass(W >= v) >= p, masses exact in
// fixed point (units of 2^-48).  The masses of the weights with float bit patterns in [lo, hi]
// are summed into up to 2048 bins of equal key width, exactly and independently of the order of
// the adds: each fixed-point weight is split into four 12-bit parts summed in 32-bit shared
// atomics (no overflow for up to 2^20 weights; measured faster than one 64-bit atomic).  A
// descending scan finds the bin where the mass from the top first reaches p, and T lies in it.
// If that bin holds at most kThreads weights they are gathered and refined exactly
// (refine_threshold), a single-key bin is T itself, and otherwise the bin is histogrammed again
// on its finer bits.  Returns 0 when even all counted weights fall
// short of p.  Weights come from registers (row k * kThreads + tid) or from W (shared or global);
// `mass` needs 4 * 2048 32-bit words, gv / gq kThreads entries each.
template <int kR>
__device__ float threshold_by_bins(const float (&wr)[kR], bool in_regs, const float* W,
                                   bool staged, int nc, uint32_t lo, uint32_t hi, long long P,
                                   unsigned long long* mass, float* gv, long long* gq, Shared& sh,
                                   unsigned long long* sh64, float* red) {
  const int tid = threadIdx.x;
  unsigned long long above = 0;  // exact mass of the weights with keys above hi
// BODY runs with `w` bound to each of this thread's weights (registers or W)
#define TWL_FOR_EACH_WEIGHT(BODY)                                           \
  do {                                                                      \
    if (in_regs) {                                                          \
      _Pragma("unroll") for (int k_ = 0; k_ < kR; ++k_) {                   \
        if (k_ * kThreads + tid < nc) {                                     \
          const float w = wr[k_];                                           \
          BODY;                                                             \
        }                                                                   \
      }                                                                     \
    } else {                                                                \
      for (int i_ = tid; i_ < nc; i_ += kThreads) {                         \
        const float w = staged ? W[i_] : __ldcg(W + i_);                    \
        BODY;                                                               \
      }                                                                     \
    }                                                                       \
  } while (0)
  int n = 0;
#pragma unroll 1
  for (int level = 0; level < 4; ++level) {
    const uint32_t width = hi - lo;
    const int bits = 32 - __clz(width);
    const int s = bits > 11 ? bits - 11 : 0;
    const int nb = (int)(width >> s) + 1;
    // [4][kPadBins] 12-bit part sums; bin b at word b + b / kHPer of each part (the scan's runs
    // of kHPer bins load conflict-free)
    uint32_t* part = reinterpret_cast<uint32_t*>(mass);
    for (int i = tid; i < 4 * kPadBins; i += kThreads) part[i] = 0u;
    __syncthreads();
    TWL_FOR_EACH_WEIGHT({
      const uint32_t u = __float_as_uint(w);
      if (u >= lo && u <= hi) {
        const int b = (int)((u - lo) >> s);
        const int bp = b + b / kHPer;
        const unsigned long long q = (unsigned long long)w_fixed(w);
        atomicAdd(&part[bp], (uint32_t)(q & 0xFFFu));
        atomicAdd(&part[kPadBins + bp], (uint32_t)((q >> 12) & 0xFFFu));
        atomicAdd(&part[2 * kPadBins + bp], (uint32_t)((q >> 24) & 0xFFFu));
        atomicAdd(&part[3 * kPadBins + bp], (uint32_t)(q >> 36));
      }
    });
    __syncthreads();
    // descending scan: thread t holds bins nb-1-kHPer t .. nb-kHPer(t+1)
    unsigned long long mb[kHPer], mine = 0;
#pragma unroll
    for (int e = 0; e < kHPer; ++e) {
      const int b = nb - 1 - kHPer * tid - e, bp = b + b / kHPer;
      mb[e] = 0ull;
      if (b >= 0)
        mb[e] = (unsigned long long)part[bp] + ((unsigned long long)part[kPadBins + bp] << 12) +
                ((unsigned long long)part[2 * kPadBins + bp] << 24) +
                ((unsigned long long)part[3 * kPadBins + bp] << 36);
      mine += mb[e];
    }
    if (tid == 0) sh.state[3] = 0xFFFFFFFFu;
    unsigned long long run = above + block_excl_u64(mine, sh64, nullptr);
#pragma unroll
    for (int e = 0; e < kHPer; ++e) {
      const int b = nb - 1 - kHPer * tid - e;
      if (b >= 0 && run < (unsigned long long)P && run + mb[e] >= (unsigned long long)P) {
        sh.state[3] = (uint32_t)b;
        sh64[kWarps] = run;  // mass above the crossing bin
      }
      run += mb[e];
    }
    __syncthreads();
    const uint32_t bx = sh.state[3];
    if (bx == 0xFFFFFFFFu) return 0.f;  // the counted weights never reach p
    above = sh64[kWarps];
    const uint32_t nlo = lo + (bx << s);
    const uint64_t top_key = (uint64_t)nlo + ((1ull << s) - 1ull);
    hi = top_key < (uint64_t)hi ? (uint32_t)top_key : hi;
    lo = nlo;
    if (lo == hi) return __uint_as_float(lo);  // one key value: T itself
    int c = 0;
    TWL_FOR_EACH_WEIGHT({
      const uint32_t u = __float_as_uint(w);
      c += (u >= lo && u <= hi) ? 1 : 0;
    });
    int pos = block_exclusive_scan(c, sh.scan, &n);
    if (n <= kThreads) {  // gather the crossing bin's weights and rank them exactly
      TWL_FOR_EACH_WEIGHT({
        const uint32_t u = __float_as_uint(w);
        if (u >= lo && u <= hi) {
          gv[pos] = w;
          gq[pos] = w_fixed(w);
          ++pos;
        }
      });
      break;
    }
  }
  __syncthreads();
  if (n > kThreads) return 0.f;  // not reached: four levels narrow any 32-bit key range
  return n <= kPairwiseMax ? rank_pairwise(gv, gq, n, above, P, red)
                           : refine_threshold(gv, gq, n, lo, hi, above, P,
                                              reinterpret_cast<uint32_t*>(mass), sh, sh64);
#undef TWL_FOR_EACH_WEIGHT
}

constexpr int kBandBins = 8192;
constexpr int kBandPer = kBandBins / kThreads;  // bins per thread in the band's scan (16 or 32)
// the histogram scratch of the prune item: the band's padded bins (kBandBins + kBandBins /
// kBandPer words), the exact bins' 4 x kPadBins parts, or the refinement's 3 x kPadBins
constexpr int kHistBytes =
    4 * (4 * kPadBins > kBandBins + kBandBins / kBandPer + 32 ? 4 * kPadBins
                                                             : kBandBins + kBandBins / kBandPer + 32);
// The same T, located first with approximate bin masses (kBandBins bins, one shared integer
// atomic per weight, the weight truncated to units of 2^-30) and then
// proven exactly: with the bin where the approximate mass from the top first reaches p, the band of
// that bin and its two neighbours is checked in fixed point (the exact mass above the band is below p
// and, with the band, reaches p), and the band's weights are refined exactly (refine_threshold).  The approximate
// sums only choose where to look; the threshold is exact or the exact histogram search runs
// instead.
// Returns false when the check fails (or the band holds more than kThreads weights).
template <int kR>
__device__ bool threshold_by_band(const float (&wr)[kR], bool in_regs, const float* W,
                                  bool staged, int nc, uint32_t lo, uint32_t hi, long long P,
                                  float* fmass, float* gv, long long* gq, Shared& sh,
                                  unsigned long long* sh64, float* red, float* T_out) {
  const int tid = threadIdx.x;
// BODY runs with `w` bound to each of this thread's weights (registers or W)
#define TWL_FOR_EACH_WEIGHT(BODY)                                           \
  do {                                                                      \
    if (in_regs) {                                                          \
      _Pragma("unroll") for (int k_ = 0; k_ < kR; ++k_) {                   \
        if (k_ * kThreads + tid < nc) {                                     \
          const float w = wr[k_];                                           \
          BODY;                                                             \
        }                                                                   \
      }                                                                     \
    } else {                                                                \
      for (int i_ = tid; i_ < nc; i_ += kThreads) {                         \
        const float w = staged ? W[i_] : __ldcg(W + i_);                    \
        BODY;                                                               \
      }                                                                     \
    }                                                                       \
  } while (0)
  // kBandBins bins of equal key width (kBandPer per thread in the scan)
  const uint32_t width = hi - lo;
  const int bits = 32 - __clz(width);
  const int s = bits > 13 ? bits - 13 : 0;
  const int nb = (int)(width >> s) + 1;
  uint32_t* imass = reinterpret_cast<uint32_t*>(fmass);
  // bin b lives at word b + b / kBandPer: a thread's kBandPer bins of the scan below then start
  // kBandPer + 1 words after the previous thread's, so the scan's loads are free of bank
  // conflicts
  for (int i = tid; i < nb + nb / kBandPer + 1; i += kThreads) imass[i] = 0u;
  __syncthreads();
  // bin masses in units of 2^-30, truncated (a weight loses < 2^-30; W <= 1 and the weights sum
  // to about 1, so the sums and their prefix stay below 2^31)
  TWL_FOR_EACH_WEIGHT({
    const uint32_t u = __float_as_uint(w);
    if (u >= lo && u <= hi) {
      const uint32_t b = (u - lo) >> s;
      atomicAdd(&imass[b + b / kBandPer], (uint32_t)(w * 1073741824.f));
    }
  });
  __syncthreads();
  // descending integer scan (thread t holds bins nb-1-kBandPer t .. nb-kBandPer(t+1)): the
  // crossing bin
  int mb[kBandPer], mine = 0;
#pragma unroll
  for (int e = 0; e < kBandPer; ++e) {
    const int b = nb - 1 - kBandPer * tid - e;
    mb[e] = b >= 0 ? (int)imass[b + b / kBandPer] : 0;
    mine += mb[e];
  }
  if (tid == 0) sh.state[3] = 0xFFFFFFFFu;
  int run = block_exclusive_scan(mine, sh.scan, nullptr);
  const int p30 = (int)(P >> 18);  // P in units of 2^-30
#pragma unroll
  for (int e = 0; e < kBandPer; ++e) {
    const int b = nb - 1 - kBandPer * tid - e;
    if (b >= 0 && run < p30 && run + mb[e] >= p30) sh.state[3] = (uint32_t)b;
    run += mb[e];
  }
  __syncthreads();
  const uint32_t bx = sh.state[3];
  bool ok = bx != 0xFFFFFFFFu;
  float T = 0.f;
  if (ok) {
    // the band: the crossing bin and its two neighbours
    const uint32_t blo_bin = bx > 0 ? bx - 1 : 0, bhi_bin = bx + 1;
    const uint32_t band_lo = lo + (blo_bin << s);
    const uint64_t bh_top = (uint64_t)lo + ((uint64_t)(bhi_bin + 1) << s) - 1;
    const uint32_t band_hi = bh_top < (uint64_t)hi ? (uint32_t)bh_top : hi;
    // exact: the mass above the band, and the band's weights
    unsigned long long above_t = 0;
    int c = 0;
    TWL_FOR_EACH_WEIGHT({
      const uint32_t u = __float_as_uint(w);
      if (u > band_hi && u <= hi) above_t += (unsigned long long)w_fixed(w);
      c += (u >= band_lo && u <= band_hi) ? 1 : 0;
    });
    unsigned long long above = 0;
    above = block_sum_u64(above_t, sh64);
    int n = 0;
    int pos = block_exclusive_scan(c, sh.scan, &n);
    ok = n <= kThreads && above < (unsigned long long)P;  // uniform
    TRACE_MARK(sh, 8);
    if (ok) {
      TWL_FOR_EACH_WEIGHT({
        const uint32_t u = __float_as_uint(w);
        if (u >= band_lo && u <= band_hi) {
          gv[pos] = w;
          gq[pos] = w_fixed(w);
          ++pos;
        }
      });
      __syncthreads();
      // rank the band exactly (the approximate bins are no longer needed: their space is reused)
      T = n <= kPairwiseMax ? rank_pairwise(gv, gq, n, above, P, red)
                            : refine_threshold(gv, gq, n, band_lo, band_hi, above, P,
                                               reinterpret_cast<uint32_t*>(fmass), sh, sh64);
      // no band weight reaching p means T lies below the band
      ok = T > 0.f;
    }
  }
  __syncthreads();
#undef TWL_FOR_EACH_WEIGHT
  *T_out = T;
  return ok;
}

// Top-p of one q-head over its nc candidates.  W_i = exp(l_i - M) / S with M the largest logit
// and S summed in a fixed order (per thread over its rows, then over the block).  Only weights
// >= L = (1 - p) / (2 nc) can decide a test above L (the weights below L sum to less than
// nc L = (1 - p) / 2, so the mass above any t <= L exceeds p): the threshold comes from that
// live set when it fits one value per thread, else from the three-level search over every
// weight.  Output: the kept-row bitmap of the head (bit i = W_i >= m) and the optional stats.
__device__ void item_prune(const Args& a, Shared& sh, int bh, unsigned char* smem,
                           int smem_bytes) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = group_of(a, bh);
  const bool ready = block_wait(a, sh, counter(a, kCntEst, g), (uint32_t)a.e_per);
  const int nc = ready ? ldcg_i(a.ncand + bh) : 0;
  float* red = reinterpret_cast<float*>(smem);                       // [kWarps][8]
  uint32_t* top_u = reinterpret_cast<uint32_t*>(smem + 4 * kWarps * 8);
  unsigned long long* sh64 = reinterpret_cast<unsigned long long*>(smem + 640);  // [kWarps + 1]
  float* lw = reinterpret_cast<float*>(smem + 1024);                 // [kThreads] live W
  int* li = reinterpret_cast<int*>(smem + 1024 + 4 * kThreads);      // [kThreads] their rows
  long long* lq = reinterpret_cast<long long*>(smem + 1024 + 8 * kThreads);  // fixed point
  unsigned char* tail = smem + 1024 + 16 * kThreads;
  const int tail_off = (int)(tail - smem);
  // weights staged in shared memory when they fit beside the histogram scratch of the large
  // live-set search (5 * 2048 words)
  const bool staged = tail_off + ((4 * nc + 127) & ~127) + kHistBytes +
                          4 * (((nc + 31) >> 5) + 32) + 8 * (a.sel_words + 32) <=
                      smem_bytes;

  // the head's selected-page bitmap and its prefix counts (for the page masks at the end), copied
  // into shared memory now so that their latency overlaps the softmax
  const Seq sq = load_seq(a.kv.seq_lens, bh / a.hq, a.kv.max_pages, a.flags, false);
  const int nw = (sq.pages + 31) >> 5;
  const int kw = (nc + 31) >> 5;
  uint32_t* kws = reinterpret_cast<uint32_t*>(tail + (staged ? ((4 * nc + 127) & ~127) : 0) +
                                              kHistBytes);
  uint32_t* sb = kws + ((kw + 31) & ~31);
  int* sp = reinterpret_cast<int*>(sb + ((nw + 31) & ~31));
  {
    const int n4 = (nw + 3) >> 2;  // 16-byte pieces (rows are sel_words, a multiple of 4, long)
    for (int w = tid; w < 2 * n4; w += kThreads) {
      const bool second = w >= n4;
      const int ww = 4 * (second ? w - n4 : w);
      const void* src = second ? (const void*)(a.hpre + (size_t)bh * a.sel_words + ww)
                               : (const void*)(a.selbits + (size_t)bh * a.sel_words + ww);
      cp_async16(second ? (void*)(sp + ww) : (void*)(sb + ww), src, true);
    }
    cp_async_commit();
  }

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
  float mloc = -INFINITY;
  if (in_regs) {
#pragma unroll
    for (int k = 0; k < kR; ++k) {
      const int i = k * kThreads + tid;
      wr[k] = i < nc ? ldcg_f(lrow + i) : -INFINITY;
      mloc = fmaxf(mloc, wr[k]);
    }
  } else {
    constexpr int kB = 8;
#pragma unroll 1
    for (int base = 0; base < nc; base += kThreads * kB) {
      float v[kB];
#pragma unroll
      for (int k = 0; k < kB; ++k) {
        const int i = base + k * kThreads + tid;
        v[k] = i < nc ? ldcg_f(lrow + i) : -INFINITY;
      }
#pragma unroll
      for (int k = 0; k < kB; ++k) {
        const int i = base + k * kThreads + tid;
        if (i < nc) {
          if (staged) W[i] = v[k];
          mloc = fmaxf(mloc, v[k]);
        }
      }
    }
  }
  TRACE_MARK(sh, 0);
  const float M = block_max(mloc, red);
  const bool empty = !(M > -INFINITY);
  float esum = 0.f;
  if (in_regs) {
#pragma unroll
    for (int k = 0; k < kR; ++k) {
      const int i = k * kThreads + tid;
      const float e = (i < nc && !empty) ? __expf(wr[k] - M) : 0.f;
      wr[k] = e;
      esum += e;
    }
  } else {
#pragma unroll 1
    for (int i = tid; i < nc; i += kThreads) {
      const float e = empty ? 0.f : __expf((staged ? W[i] : ldcg_f(lrow + i)) - M);
      W[i] = e;
      esum += e;
    }
  }
  const float S = block_sum_fixed(esum, red);
  const float inv = S > 0.f ? 1.f / S : 0.f;
  TRACE_MARK(sh, 1);
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
  int pos = block_exclusive_scan(cntl, sh.scan, &nlive);  // its barriers also publish top_u
  top = __uint_as_float(*top_u);
  TRACE_MARK(sh, 2);
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
  __syncthreads();  // the live set (or the weights) complete
  // histogram scratch, after the staged weights
  unsigned long long* hist =
      reinterpret_cast<unsigned long long*>(tail + (staged ? ((4 * nc + 127) & ~127) : 0));
  float m;
  if (nc == 0 || p >= 1.f) {
    m = 0.f;  // keep every candidate
  } else if (from_live) {
    // Every test of the search at mid > L counts only live weights, and mass(W >= t) is a
    // non-increasing step function of t, so "mid <= L or mass(W >= mid) >= p" is the same test
    // as "mid <= T" with T = max(L, the largest live weight v with mass(W >= v) >= p).
    const long long P = __double2ll_ru((double)p * 281474976710656.0);
    const float T =
        nlive <= kPairwiseMax
            ? rank_pairwise(lw, lq, nlive, 0ull, P, red)
            : refine_threshold(lw, lq, nlive, __float_as_uint(L), __float_as_uint(top), 0ull, P,
                               reinterpret_cast<uint32_t*>(hist), sh, sh64);
    m = bisect_scalar(top, fmaxf(L, T), eps);
  } else {
    // the threshold from exact bin masses over the weights >= L
    const long long P = __double2ll_ru((double)p * 281474976710656.0);
    float T = 0.f;
    if (!threshold_by_band<kR>(wr, in_regs, W, staged, nc, __float_as_uint(L),
                               __float_as_uint(top), P, reinterpret_cast<float*>(hist), lw, lq,
                               sh, sh64, red, &T))
    {
      TRACE_MARK(sh, 9);
      T = threshold_by_bins<kR>(wr, in_regs, W, staged, nc, __float_as_uint(L),
                                __float_as_uint(top), P, hist, lw, lq, sh, sh64, red);
    }
    m = bisect_scalar(top, fmaxf(L, T), eps);
  }
  TRACE_MARK(sh, 3);
  if (tid == 0) {
    if (a.threshold) a.threshold[bh] = m;
    if (a.cand_count) a.cand_count[bh] = nc;
  }
  // kept-row bitmap of this head (kws): bit i = (W_i >= m), in shared memory (after the staged
  // weights and the histogram scratch)
  int cnt = 0;
  if (from_live && m >= L) {
    // every kept candidate is live
    for (int w = tid; w < kw; w += kThreads) kws[w] = 0u;
    __syncthreads();
    if (tid < nlive && lw[tid] >= m) atomicOr(&kws[li[tid] >> 5], 1u << (li[tid] & 31));
    __syncthreads();
    for (int w = tid; w < kw; w += kThreads) cnt += __popc(kws[w]);
  } else if (in_regs) {
#pragma unroll
    for (int k = 0; k < kR; ++k) {
      const int i = k * kThreads + tid;
      const bool keep = i < nc && wr[k] >= m;
      const uint32_t bal = __ballot_sync(0xffffffffu, keep);
      if (lane == 0 && k * kThreads + 32 * warp < nc) kws[k * kWarps + warp] = bal;
      cnt += keep;
    }
  } else {
#pragma unroll 1
    for (int base = 0; base < nc; base += kThreads) {
      const int i = base + tid;
      const bool keep = i < nc && (staged ? W[i] : ldcg_f(W + i)) >= m;
      const uint32_t bal = __ballot_sync(0xffffffffu, keep);
      if (lane == 0 && base + 32 * warp < nc) kws[(base >> 5) + warp] = bal;
      cnt += keep;
    }
  }
  if (a.kept_count) {  // only when the caller asks for it
    const float total = block_sum_fixed((float)cnt, red);
    if (tid == 0) a.kept_count[bh] = (int)total;
  }
  // the head's kept rows of each selected page, ORed into the group's page masks (two pages per
  // word); the page of selection rank r is the r-th set bit of the head's bitmap, found from its
  // per-word prefix counts
  cp_async_wait_all();  // the bitmap and prefix counts copied at the start
  __syncthreads();
  uint32_t* pm = a.pmask + (size_t)g * a.pm_words;
  const int kbp = (nc + kPage - 1) / kPage;  // selected pages of the head
  for (int r = tid; r < kbp; r += kThreads) {
    const uint32_t mk = (kws[r >> 1] >> (16 * (r & 1))) & 0xFFFFu;
    if (mk == 0u) continue;
    int lo = 0, hi = nw;  // the last word whose prefix is <= r
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (sp[mid] <= r) lo = mid;
      else hi = mid;
    }
    const int j = 32 * lo + nth_set_bit(sb[lo], r - sp[lo]);
    atomicOr(pm + (j >> 1), mk << (16 * (j & 1)));
  }
}

// ------------------------------------------------------------------------------ kept tokens
// Run by the CTA whose prune item completed its group: for every union page (ascending) the OR of
// the 16-row pieces of the kept bitmaps of the heads that selected it, cut to the page's valid
// rows; the kept rows are listed in ascending token order as K/V row indices (and token ids when
// the caller asks for the union).
template <int G>
__device__ void build_kept(const Args& a, Shared& sh, int g, unsigned char* smem) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = g / a.kv.hkv, kvh = g - b * a.kv.hkv;
  const Seq sq = load_seq(a.kv.seq_lens, b, a.kv.max_pages, a.flags, false);
  const bool aborted = ld_acquire(a.sync + kAbort) != 0u;
  const int n_pages = aborted ? 0 : sq.pages;
  const int nw2 = (n_pages + 1) >> 1;
  int4* kp = a.kpages + (size_t)g * a.kv.max_pages;
  uint32_t* pm = a.pmask + (size_t)g * a.pm_words;
  TRACE_MARK(sh, 4);
  // thread per mask word (two logical pages): the kept rows of the group's heads, cut to the valid
  // rows of pages the table can place (the word is cleared for the next launch); every page with
  // a kept row becomes one entry (K/V row index of its row 0, row mask, logical page, kept tokens
  // before it), in page order
  const int* ptab = a.kv.page_table + (size_t)b * a.kv.max_pages;
  int* spre = reinterpret_cast<int*>(smem);  // kept tokens before each kept page
  int npg = 0, ntok = 0;
#pragma unroll 1
  for (int base = 0; base < nw2; base += kThreads) {
    const int w2 = base + tid;
    uint32_t m32 = 0;
    int ph[2] = {-1, -1};
    if (w2 < nw2) {
      m32 = ldcg_u(pm + w2);
      ph[0] = ptab[2 * w2];
      ph[1] = 2 * w2 + 1 < n_pages ? ptab[2 * w2 + 1] : -1;
    }
    if (m32) pm[w2] = 0u;
    uint32_t mk[2] = {m32 & 0xFFFFu, m32 >> 16};
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int j = 2 * w2 + e;
      if (mk[e]) {
        const int rows = page_rows(sq.n, j);
        mk[e] &= rows >= 16 ? 0xFFFFu : ((1u << rows) - 1u);
        if (ph[e] < 0 || ph[e] >= a.kv.num_phys) mk[e] = 0u;  // never attended (flagged before)
      }
    }
    TRACE_MARK(sh, 5);
    // two scans at once (pages, tokens): warp shuffles, then the warp totals
    int cp = (mk[0] != 0u) + (mk[1] != 0u), ct = __popc(mk[0]) + __popc(mk[1]);
    int xp = cp, xt = ct;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int yp = __shfl_up_sync(0xffffffffu, xp, o);
      const int yt = __shfl_up_sync(0xffffffffu, xt, o);
      if (lane >= o) {
        xp += yp;
        xt += yt;
      }
    }
    __syncthreads();
    if (lane == 31) {
      sh.scan[warp] = xp;
      sh.scan[kWarps + warp] = xt;
    }
    __syncthreads();
    int bp = npg, bt = ntok, ap = 0, at = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const int vp = sh.scan[w], vt = sh.scan[kWarps + w];
      if (w < warp) {
        bp += vp;
        bt += vt;
      }
      ap += vp;
      at += vt;
    }
    int q = bp + xp - cp, tq = bt + xt - ct;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      if (mk[e]) {
        const int j = 2 * w2 + e;
        kp[q] = make_int4((int)(((size_t)ph[e] * a.kv.hkv + kvh) * kPage), (int)mk[e], j, tq);
        spre[q] = tq;
        if (a.union_tok) {  // the ascending union of kept tokens, when the caller asks for it
          uint32_t mm = mk[e];
          int t = tq;
          while (mm) {
            a.union_tok[(size_t)g * kPage * a.kv.max_pages + t++] = kPage * j + __ffs(mm) - 1;
            mm &= mm - 1u;
          }
        }
        ++q;
        tq += __popc(mk[e]);
      }
    }
    npg += ap;
    ntok += at;
  }
  TRACE_MARK(sh, 7);
  // publish the group's kept pages to the attention queue in nch chunks of about equal token
  // counts: page q opens chunk floor(pre(q) nch / ntok).  A chunk is cut to about ntok /
  // att_chunks tokens (the group's share of the workers), at least kAttChunkTok and
  // at most kAttChunkMax (+15 at a page edge).  As a page holds at most 16 tokens and a chunk
  // about ntok / nch >= kAttChunkTok / 2 = 64, consecutive pages open consecutive chunks and none
  // is empty.  One empty chunk when nothing is kept, so the merge still writes the outputs.
  int tgt = (ntok + a.att_chunks - 1) / a.att_chunks;
  tgt = tgt < kAttChunkTok ? kAttChunkTok : (tgt > kAttChunkMax ? kAttChunkMax : tgt);
  const int nch = ntok > 0 ? (ntok + tgt - 1) / tgt : 1;
  if (tid == 0) {
    if (a.union_count) a.union_count[g] = ntok;
    sh.total = (int)atomicAdd(a.sync + kQAlloc, (uint32_t)nch);
  }
  __syncthreads();  // also orders the staged prefix counts
  const int base = sh.total;
  for (int q = tid; q < npg; q += kThreads) {
    const int c = (int)((long long)spre[q] * nch / ntok);
    const int cp = q > 0 ? (int)((long long)spre[q - 1] * nch / ntok) : -1;
    if (c != cp) {
      if (base + c < a.q_cap) {
        int* e = a.qtab + 4 * (size_t)(base + c);
        e[0] = g;
        e[1] = q;
      }
      if (c > 0 && base + c - 1 < a.q_cap) a.qtab[4 * (size_t)(base + c - 1) + 2] = q;
    }
  }
  if (tid == 0) {
    if (base + nch - 1 < a.q_cap) {
      int* e = a.qtab + 4 * (size_t)(base + nch - 1);
      e[2] = npg;
      if (npg == 0) {
        e[0] = g;
        e[1] = 0;
      }
    }
    a.cbase[2 * g] = base;
    a.cbase[2 * g + 1] = nch;
  }
  __syncthreads();  // the chunk entries, counts and kept pages before the valid flags
  if (tid == 0) {
    // one release fence for everything the block wrote (it observed all of it at the barrier),
    // then plain stores of the flags
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
    for (int c = 0; c < nch && base + c < a.q_cap; ++c)
      asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(a.qvalid + base + c), "r"(1u)
                   : "memory");
    asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(a.sync + kQGroups), "r"(1u)
                 : "memory");
  }
  TRACE_MARK(sh, 6);
}

// ------------------------------------------------------------------------------ attention
// The attention work list ([Notes] "Key designs", load balancing: the heads' kept tokens differ
// ~50x, so each group's kept pages are cut into chunks that any CTA takes).  A worker is warp-
// specialised: the upper half of the warps produce, the lower half consume (8 and 8 in the
// 512-thread build, 4 and 4 in the 256-thread one), and the two sides meet only at mbarriers
// on a ring of pass buffers, so that the copies of later passes are issued while earlier ones are
// computed.
//   * Producers take the chunks from the queue (ticket, wait until published), expand a chunk's
//     kept pages to the K/V row index of every kept token (thread per page), and copy each pass
//     of up to kAttPass tokens (256 B of K and of V per token, with 16-byte cp.async, each row's
//     16-byte pieces XOR-swizzled by the row number so that ldmatrix reads are free of bank
//     conflicts; the group's query rows too) into the next free buffer, with a descriptor (tokens,
//     chunk, group, first / last pass of the chunk).  The buffer's full barrier completes when
//     every producer thread's copies have landed.
//   * Consumer warp w takes the 16-token tile w of a pass, on the tensor cores (mma.m16n8k16,
//     fp16 in, fp32 accumulate): S^T = K Q^T takes the tile's tokens as the M rows and the heads
//     (G <= 8) as N; the weights are moved by shuffles into the B operand of O^T += V^T P^T, which
//     takes 16 channels as M (eight tiles), the 16 tokens as K and the heads as N.  P is split into
//     an fp16 head and an fp16 tail (p - head), two products, so its rounding stays near 2^-22 of
//     the weights.  Each warp keeps its own running (max, sum, o) of its lanes' heads (2t, 2t+1),
//     and frees the buffer through its empty barrier.
//   * At a chunk's last pass the consumers merge the warps' states into the chunk's partial
//     [G][128 o, max, sum, -, -]; the chunk that completes its group merges the group's
//     partials (log-sum-exp, in chunk order) into o and lse.
constexpr int kAttCons = kThreads / 2;          // consumer threads (the first half of the warps)
constexpr int kAttProd = kThreads - kAttCons;    // producer threads (the second half)
constexpr int kAttConsWarps = kAttCons / 32;
constexpr int kAttPass = 16 * kAttConsWarps;     // tokens per pass: one 16-token tile per consumer
constexpr int kAttIdx = kAttChunkMax + 16;
constexpr int kAttPartStride = kHeadDim + 4;  // floats per head of a chunk partial
constexpr int kAttBufBytes = kAttPass * 512 + 8 * 256;  // K rows | V rows | query rows
constexpr uint32_t kMbarLimit = 1u << 22;      // polls of an mbarrier before a wait gives up
// pass buffers in the ring (three when the merge scratch and the CTAs an SM holds leave room)
template <int G>
constexpr int att_bufs() {
  return (G >= 8 || kThreads < 512) ? 2 : 3;
}
// shared memory of a worker: [bufs][kAttBufBytes] | [2][kAttIdx] row indices | scratch of the
// consumers ([warps][2 G] max, sum | [warps][G][128] o)
template <int G>
constexpr int att_scratch_off() {
  return att_bufs<G>() * kAttBufBytes + 2 * ((4 * kAttIdx + 127) & ~127);
}
template <int G>
constexpr int att_merge_floats();
template <int G>
constexpr int att_smem() {
  return att_scratch_off<G>() +
         4 * (kAttConsWarps * (2 * G + G * kHeadDim) > att_merge_floats<G>()
                  ? kAttConsWarps * (2 * G + G * kHeadDim)
                  : att_merge_floats<G>());
}
enum { kDescEnd = 1, kDescFirst = 2, kDescLast = 4 };

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ void bar_named(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(saddr(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_inval(uint64_t* b) {
  asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(saddr(b)) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(saddr(b)) : "memory");
}
// arrives once every cp.async this thread issued before has landed
__device__ __forceinline__ void mbar_arrive_cp(uint64_t* b) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(saddr(b)) : "memory");
}
// one bounded poll (the thread may be suspended up to about a microsecond inside it)
__device__ __forceinline__ bool mbar_test(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(saddr(b)), "r"(parity), "r"(1000u)
      : "memory");
  return ok != 0u;
}
// One thread: wait (bounded) for the phase of parity `parity` of b; false when the wait gave up
// (which flags a timeout and aborts the step).  The ring's waits do not give up on an abort of
// the step by others: the producers end the ring themselves (an end descriptor), so that every
// consumer warp leaves at the same pass and the consumers' named barriers stay matched.
__device__ bool mbar_wait(const Args& a, uint64_t* b, uint32_t parity) {
#pragma unroll 1
  for (uint32_t it = 0;; ++it) {
    if (mbar_test(b, parity)) return true;
    if (it >= kMbarLimit) {
      raise_flag(a.flags, TWL_FLAG_TIMEOUT);
      atomicExch(a.sync + kAbort, 1u);
      return false;
    }
  }
}

// Consumer warp: one 16-token tile of a pass (cn tokens; K rows at kb, V rows at vb, the query
// rows at qs) folded into the warp's running state of its lanes' heads (2t, 2t+1): max m[], sum
// l[] (of this lane's tokens only) and O^T (channels 16 mt + gr (+8), heads 2t, 2t+1).
template <int G>
__device__ __forceinline__ void attend_tile(const unsigned char* kb, const unsigned char* vb,
                                            const unsigned char* qs, int cn, float sc_scale,
                                            float (&m)[2], float (&l)[2], float (&ot)[8][4]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gr = lane >> 2, t = lane & 3;  // mma fragment row / column pair
  const int tok0 = 16 * warp;
  if (tok0 >= cn) return;  // warp-uniform
  const int mrow = lane & 7, mat = lane >> 3;
  // S^T = K Q^T: A = the tile's K rows (ldmatrix), B = the query rows (head gr; zero for heads
  // >= G)
  const bool head_ok = gr < G;
  const unsigned char* qh = qs + 256 * (head_ok ? gr : 0);
  float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const int tk = tok0 + mrow + 8 * (mat >> 1), ch = 2 * ks + (mat & 1);
    uint32_t kf[4];
    ldsm_x4(kf, saddr(kb + 256 * tk + 16 * (ch ^ (tk & 7))));
    const uint32_t ka[4] = {kf[0], kf[2], kf[1], kf[3]};
    const uint32_t q0 = head_ok ? *reinterpret_cast<const uint32_t*>(qh + 32 * ks + 4 * t) : 0u;
    const uint32_t q1 = head_ok ? *reinterpret_cast<const uint32_t*>(qh + 32 * ks + 16 + 4 * t) : 0u;
    mma_16816(s, ka, q0, q1);
  }
  // s[0], s[1]: token tok0 + gr, heads 2t, 2t + 1; s[2], s[3]: token tok0 + gr + 8
  const bool v0 = tok0 + gr < cn, v1 = tok0 + gr + 8 < cn;
  float x[4];
  x[0] = v0 ? s[0] * sc_scale : -INFINITY;
  x[1] = v0 ? s[1] * sc_scale : -INFINITY;
  x[2] = v1 ? s[2] * sc_scale : -INFINITY;
  x[3] = v1 ? s[3] * sc_scale : -INFINITY;
  float f[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    float mx = fmaxf(x[e], x[2 + e]);
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    const float nm = fmaxf(m[e], mx);  // finite: token tok0 is valid
    f[e] = m[e] > -INFINITY ? __expf(m[e] - nm) : 0.f;
    m[e] = nm;
    x[e] = v0 ? __expf(x[e] - nm) : 0.f;
    x[2 + e] = v1 ? __expf(x[2 + e] - nm) : 0.f;
    l[e] = l[e] * f[e] + (x[e] + x[2 + e]);
  }
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    ot[mt][0] *= f[0];
    ot[mt][1] *= f[1];
    ot[mt][2] *= f[0];
    ot[mt][3] *= f[1];
  }
  // P^T as the B operand (k = tokens, n = head gr): tokens 2t, 2t + 8 of head gr are held by
  // lane 8t + gr / 2, tokens 2t + 1, 2t + 9 by lane 8t + 4 + gr / 2 (component gr & 1)
  const int sa = 8 * t + (gr >> 1), sb = sa + 4;
  const bool odd = gr & 1;
  float pa0 = __shfl_sync(0xffffffffu, x[0], sa), pa1 = __shfl_sync(0xffffffffu, x[1], sa);
  float pa2 = __shfl_sync(0xffffffffu, x[2], sa), pa3 = __shfl_sync(0xffffffffu, x[3], sa);
  float pb0 = __shfl_sync(0xffffffffu, x[0], sb), pb1 = __shfl_sync(0xffffffffu, x[1], sb);
  float pb2 = __shfl_sync(0xffffffffu, x[2], sb), pb3 = __shfl_sync(0xffffffffu, x[3], sb);
  const float p_t0 = odd ? pa1 : pa0, p_t8 = odd ? pa3 : pa2;  // tokens 2t, 2t + 8
  const float p_t1 = odd ? pb1 : pb0, p_t9 = odd ? pb3 : pb2;  // tokens 2t + 1, 2t + 9
  const uint32_t bh0 = pack_f16x2(p_t0, p_t1), bh1 = pack_f16x2(p_t8, p_t9);
  const float2 h0 = __half22float2(*reinterpret_cast<const __half2*>(&bh0));
  const float2 h1 = __half22float2(*reinterpret_cast<const __half2*>(&bh1));
  const uint32_t bl0 = pack_f16x2(p_t0 - h0.x, p_t1 - h0.y);
  const uint32_t bl1 = pack_f16x2(p_t8 - h1.x, p_t9 - h1.y);
  // O^T += V^T P^T over the eight 16-channel tiles (A from ldmatrix.trans of the V rows)
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    const int tk = tok0 + mrow + 8 * (mat >> 1);
    const int ch = 2 * mt + (mat & 1);
    uint32_t va[4];
    ldsm_x4_t(va, saddr(vb + 256 * tk + 16 * (ch ^ (tk & 7))));
    mma_16816(ot[mt], va, bh0, bh1);
    mma_16816(ot[mt], va, bl0, bl1);
  }
}

// Consumers (256 threads): the warps' states of a finished chunk -> its partial [G][o(128), max,
// sum] in a.part (slot c).  scr: the consumers' scratch.
template <int G>
__device__ void attend_finish(const Args& a, int c, const float (&m)[2], float (&l)[2],
                              const float (&ot)[8][4], float* scr) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gr = lane >> 2, t = lane & 3;
  float* wm = scr;                           // [kAttConsWarps][G]
  float* wl = wm + kAttConsWarps * G;        // [kAttConsWarps][G]
  float* wo = wl + kAttConsWarps * G;        // [kAttConsWarps][G][128]
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    l[e] += __shfl_xor_sync(0xffffffffu, l[e], 4);
    l[e] += __shfl_xor_sync(0xffffffffu, l[e], 8);
    l[e] += __shfl_xor_sync(0xffffffffu, l[e], 16);
    const int h = 2 * t + e;
    if (gr == 0 && h < G) {
      wm[warp * G + h] = m[e];
      wl[warp * G + h] = l[e];
    }
  }
#pragma unroll
  for (int mt = 0; mt < 8; ++mt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int h = 2 * t + (e & 1), ch = 16 * mt + gr + 8 * (e >> 1);
      if (h < G) wo[(warp * G + h) * kHeadDim + ch] = ot[mt][e];
    }
  bar_named(2, kAttCons);
  float* part = a.part + (size_t)c * G * kAttPartStride;
  for (int i = tid; i < G * kHeadDim; i += kAttCons) {
    const int h = i / kHeadDim, d = i - h * kHeadDim;
    float mxw = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAttConsWarps; ++w) mxw = fmaxf(mxw, wm[w * G + h]);
    float ov = 0.f, lv = 0.f;
    if (mxw > -INFINITY) {
#pragma unroll
      for (int w = 0; w < kAttConsWarps; ++w) {
        const float mw = wm[w * G + h];
        if (!(mw > -INFINITY)) continue;
        const float fw = __expf(mw - mxw);
        ov = fmaf(fw, wo[(w * G + h) * kHeadDim + d], ov);
        lv = fmaf(fw, wl[w * G + h], lv);
      }
    }
    part[h * kAttPartStride + d] = ov;
    if (d == 0) {
      part[h * kAttPartStride + kHeadDim] = mxw;
      part[h * kAttPartStride + kHeadDim + 1] = lv;
    }
  }
}

// Consumers (256 threads), in the CTA whose chunk completed group g: log-sum-exp merge of the
// group's nch chunk partials (slots c0 ...) -> o, lse of every head (o = 0, lse = -inf when
// nothing was kept).  The max of every (chunk, head) is staged in shared memory in one round of
// loads; warp h turns head h's into chunk weights exp(max_c - max) and the head's total;
// then each float4 of o is summed by kAttCons / (32 G) threads over interleaved chunks, or each
// thread sums whole float4 columns when there are more columns than threads (their loads are
// independent of the sums, so they stay in flight together) and their sums are added in a fixed
// order.  scr: the consumers' scratch (kAttMergeFloats floats at least).
constexpr int kAttMaxChunks = 512;  // chunks of one group at most (16 * kMaxPages / kAttChunkMax)
template <int G>
constexpr int att_merge_floats() {
  return kAttMaxChunks * G + 16 + 4 * kAttCons;
}
// o and lse of head h of group (b, kvh) from the merged float4 column c4 of o (sum acc of the
// weighted chunk partials) and the head's max and total in hs.
template <int G>
__device__ __forceinline__ void merge_store(const Args& a, int b, int kvh, int h, int c4,
                                            const float4& acc, const float* hs) {
  const float lt = hs[G + h];
  const bool any = lt > 0.f;
  const size_t bh = (size_t)b * a.hq + kvh * G + h;
  float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
  if (any) o = make_float4(acc.x / lt, acc.y / lt, acc.z / lt, acc.w / lt);
  reinterpret_cast<float4*>(a.o + bh * kHeadDim)[c4] = o;
  if (c4 == 0) a.lse[bh] = any ? hs[h] + __logf(lt) : -INFINITY;
}

template <int G>
__device__ void merge_group(const Args& a, int g, int c0, int nch, float* scr) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = g / a.kv.hkv, kvh = g - b * a.kv.hkv;
  const float* part = a.part + (size_t)c0 * G * kAttPartStride;
  float4* red = reinterpret_cast<float4*>(scr);      // [kAttCons]
  float* hs = scr + 4 * kAttCons;                    // [G] head max, [G] head total
  float* wm = hs + 16;                               // [nch][G] chunk max, then its weight
  for (int i = tid; i < nch * G; i += kAttCons) {
    const float* pp = part + (size_t)i * kAttPartStride + kHeadDim;
    const float l = ldcg_f(pp + 1), m = ldcg_f(pp);
    wm[i] = l > 0.f ? m : -INFINITY;
  }
  bar_named(2, kAttCons);
  for (int hw = warp; hw < G; hw += kAttConsWarps) {  // warp hw: head hw
    float mx = -INFINITY;
    for (int c = lane; c < nch; c += 32) mx = fmaxf(mx, wm[c * G + hw]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float tot = 0.f;
    for (int c = lane; c < nch; c += 32) {
      const float m = wm[c * G + hw];
      const float w = m > -INFINITY ? __expf(m - mx) : 0.f;
      wm[c * G + hw] = w;
      if (w > 0.f)
        tot = fmaf(w, ldcg_f(part + (size_t)(c * G + hw) * kAttPartStride + kHeadDim + 1), tot);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
    if (lane == 0) {
      hs[hw] = mx;
      hs[G + hw] = tot;
    }
  }
  bar_named(2, kAttCons);
  constexpr int kCols = G * kHeadDim / 4;
  if constexpr (kAttCons >= kCols) {
    constexpr int kPer = kAttCons / kCols;
    const int col = tid % kCols, r = tid / kCols, h = col / (kHeadDim / 4);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
    for (int c = r; c < nch; c += kPer) {
      const float w = wm[c * G + h];
      const float4 v = __ldcg(reinterpret_cast<const float4*>(part + (size_t)(c * G + h) *
                                                                        kAttPartStride) +
                              (col % (kHeadDim / 4)));
      acc.x = fmaf(w, v.x, acc.x);
      acc.y = fmaf(w, v.y, acc.y);
      acc.z = fmaf(w, v.z, acc.z);
      acc.w = fmaf(w, v.w, acc.w);
    }
    red[tid] = acc;
    bar_named(2, kAttCons);
    if (r == 0) {
#pragma unroll
      for (int k = 1; k < kPer; ++k) {
        const float4 v = red[k * kCols + col];
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      merge_store<G>(a, b, kvh, h, col % (kHeadDim / 4), acc, hs);
    }
  } else {
    // more float4 columns than consumer threads: each thread sums whole columns
    for (int col = tid; col < kCols; col += kAttCons) {
      const int h = col / (kHeadDim / 4);
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
      for (int c = 0; c < nch; ++c) {
        const float w = wm[c * G + h];
        const float4 v = __ldcg(reinterpret_cast<const float4*>(part + (size_t)(c * G + h) *
                                                                          kAttPartStride) +
                                (col % (kHeadDim / 4)));
        acc.x = fmaf(w, v.x, acc.x);
        acc.y = fmaf(w, v.y, acc.y);
        acc.z = fmaf(w, v.z, acc.z);
        acc.w = fmaf(w, v.w, acc.w);
      }
      merge_store<G>(a, b, kvh, h, col % (kHeadDim / 4), acc, hs);
    }
  }
  bar_named(2, kAttCons);  // the scratch is reused
}

// Thread 0: the state of queue ticket c: 1 = its chunk is published, -1 = there is none (every
// group has published and c is past the end, or the step was aborted), 0 = not yet.
__device__ __forceinline__ int ticket_state(const Args& a, int c) {
  if (c < a.q_cap && ld_acquire(a.qvalid + c) != 0u) return 1;
  if (ld_acquire(a.sync + kQGroups) >= (uint32_t)a.groups &&
      (uint32_t)c >= ld_acquire(a.sync + kQAlloc))
    return -1;
  if (ld_acquire(a.sync + kAbort) != 0u) return -1;
  return 0;
}

// Thread 0: wait (bounded) until ticket c is decided; 1 = published, -1 = none.
__device__ int ticket_wait(const Args& a, int c) {
#pragma unroll 1
  for (uint32_t it = 0;; ++it) {
    const int st = ticket_state(a, c);
    if (st != 0) return st;
    if (it >= a.spin_limit) {
      raise_flag(a.flags, TWL_FLAG_TIMEOUT);
      atomicExch(a.sync + kAbort, 1u);
      return -1;
    }
    __nanosleep(64);
  }
}

// Producers (the upper half of the warps): take chunks until the queue is done, copy their
// passes into the ring, then post the end.  The next chunk is prepared while the current one's passes are issued, one
// step per pass (take its queue ticket; see it published and read its entry; expand its pages
// into the other row-index stage), so a chunk switch leaves no gap in the copies.
template <int G>
__device__ void attend_produce(const Args& a, Shared& sh, unsigned char* smem) {
  constexpr int NB = att_bufs<G>();
  const int pt = threadIdx.x - kAttCons;
  uint32_t* idx_base = reinterpret_cast<uint32_t*>(smem + NB * kAttBufBytes);  // [2][kAttIdx]
  int ticket = -1;  // thread pt == 0: the ticket of the chunk being prepared
  // expand chunk (group g, pages [p0, p1)) into stage s; returns its token count
  auto expand = [&](int s, int g, int p0, int p1) {
    uint32_t* idx = idx_base + s * kAttIdx;
    const int4* kp = a.kpages + (size_t)g * a.kv.max_pages;
    int n = 0, tb = 0;
    if (p1 > p0) {
      const int4 f = ldcg_i4(kp + p0), ls = ldcg_i4(kp + p1 - 1);
      tb = f.w;
      n = ls.w + __popc((uint32_t)ls.y) - tb;
    }
    for (int q = p0 + pt; q < p1; q += kAttProd) {
      const int4 en = ldcg_i4(kp + q);
      uint32_t mk = (uint32_t)en.y;
      int pos = en.w - tb;
      while (mk) {
        idx[pos++] = (uint32_t)en.x + (uint32_t)(__ffs(mk) - 1);
        mk &= mk - 1u;
      }
    }
    bar_named(1, kAttProd);
    return n;
  };
  // thread 0 has the ticket's state st (1 published, -1 none, 0 not yet): share it and, when
  // published, the chunk's entry (slot, group, first page, end page) through stage s
  auto share = [&](int s, int st) {
    if (pt == 0) {
      sh.att[s][0] = st > 0 ? ticket : (st < 0 ? -1 : -2);
      if (st > 0) {
        const int* e = a.qtab + 4 * (size_t)ticket;
        sh.att[s][1] = ldcg_i(e);
        sh.att[s][2] = ldcg_i(e + 1);
        sh.att[s][3] = ldcg_i(e + 2);
      }
    }
    bar_named(1, kAttProd);
  };
  // the first chunk, waited for
  if (pt == 0) {
    ticket = (int)atomicAdd(a.sync + kQNext, 1u);
  }
  share(0, pt == 0 ? ticket_wait(a, ticket) : 0);
  int cs = 0;                 // stage of the current chunk
  int c = sh.att[0][0], g = sh.att[0][1];
  int n = c >= 0 ? expand(0, g, sh.att[0][2], sh.att[0][3]) : 0;
  // preparation of the next chunk (stage cs ^ 1): 0 nothing yet, 1 ticket taken, 2 published and
  // entry read, 3 expanded, -1 none left (the same value in every producer thread)
  int prep = 0, c2 = -1, g2 = 0, n2 = 0;
  auto prep_step = [&](bool wait) {
    const int s = cs ^ 1;
    if (prep == 0) {
      if (pt == 0) ticket = (int)atomicAdd(a.sync + kQNext, 1u);
      prep = 1;
      if (!wait) return;
    }
    if (prep == 1) {
      int st = 0;
      if (pt == 0) st = wait ? ticket_wait(a, ticket) : ticket_state(a, ticket);
      share(s, st);
      const int v = sh.att[s][0];
      bar_named(1, kAttProd);  // read before stage s's entry can be written again
      if (v == -2) return;     // not published yet
      if (v < 0) {
        prep = -1;
        return;
      }
      c2 = v;
      g2 = sh.att[s][1];
      prep = 2;
      if (!wait) {
        // the entry stays in stage s until the expansion below
        return;
      }
    }
    if (prep == 2) {
      n2 = expand(s, g2, sh.att[s][2], sh.att[s][3]);
      prep = 3;
    }
  };
  int j = 0;  // passes posted
  bool ok = true;
#pragma unroll 1
  for (;;) {
    const int np = c >= 0 ? (n > 0 ? (n + kAttPass - 1) / kAttPass : 1) : 1;
    const int b_ = g / a.kv.hkv, kvh = g - b_ * a.kv.hkv;
    const uint32_t* idx = idx_base + cs * kAttIdx;
#pragma unroll 1
    for (int k = 0; k < np; ++k, ++j) {
      const int bs = j % NB, u = j / NB;
#ifdef TWL_STEP_TRACE
      const unsigned long long tp0 = now_ns();
#endif
      if (u > 0) {  // the buffer's previous pass consumed (thread 0 waits for all)
        if (pt == 0) sh.att_prod_ok = mbar_wait(a, &sh.att_empty[bs], (uint32_t)((u - 1) & 1));
        bar_named(1, kAttProd);
        ok = sh.att_prod_ok != 0;
        bar_named(1, kAttProd);
        if (!ok) break;
      }
#ifdef TWL_STEP_TRACE
      const unsigned long long tp1 = now_ns();
#endif
      unsigned char* kb = smem + bs * kAttBufBytes;
      unsigned char* vb = kb + kAttPass * 256;
      unsigned char* qb = kb + kAttPass * 512;
      if (c >= 0) {
        const int cn = min(kAttPass, n - k * kAttPass);
        const int rows = (cn + 15) & ~15;  // rows past cn in the last tile read zeros
        const uint32_t* ix = idx + k * kAttPass;
        for (int q = pt; q < 32 * rows; q += kAttProd) {
          const int i = q >> 5, part = q & 31;
          const bool okr = i < cn;
          const size_t off = okr ? (size_t)ix[i] * kHeadDim : 0;
          if (part < 16)
            cp_async16(kb + 256 * i + 16 * (part ^ (i & 7)), a.kv.k + off + 8 * part, okr);
          else
            cp_async16(vb + 256 * i + 16 * ((part - 16) ^ (i & 7)),
                       a.kv.v + off + 8 * (part - 16), okr);
        }
        if (pt < G * 16) {
          const int row = pt >> 4, piece = pt & 15;
          cp_async16(qb + 256 * row + 16 * piece,
                     a.q + ((size_t)b_ * a.hq + kvh * G + row) * kHeadDim + 8 * piece, true);
        }
        if (pt == 0) {
          sh.att_desc[bs][0] = cn;
          sh.att_desc[bs][1] = c;
          sh.att_desc[bs][2] = g;
          sh.att_desc[bs][3] = (k == 0 ? kDescFirst : 0) | (k == np - 1 ? kDescLast : 0);
        }
      } else if (pt == 0) {
        sh.att_desc[bs][3] = kDescEnd;
      }
      mbar_arrive_cp(&sh.att_full[bs]);
      if (pt == 0) mbar_arrive(&sh.att_full[bs]);
#ifdef TWL_STEP_TRACE
      if (pt == 0 && a.trace && j < 16) {
        unsigned long long* pr = a.trace + 17 * (size_t)a.n_items + 96 * (size_t)blockIdx.x + 6 * j;
        pr[0] = tp0;
        pr[1] = tp1;
        pr[2] = now_ns();
      }
#endif
      // one step of the next chunk's preparation while this pass's copies fly
      if (c >= 0 && prep >= 0 && prep < 3) prep_step(false);
    }
    if (c < 0 || !ok) break;
    // switch to the next chunk, finishing its preparation (waiting now if it must)
#pragma unroll 1
    while (prep >= 0 && prep < 3) prep_step(true);
    cs ^= 1;
    c = prep == 3 ? c2 : -1;
    g = g2;
    n = n2;
    prep = 0;
  }
  cp_async_wait_all();
}

// Consumers (the lower half of the warps): compute the posted passes until the end; at a
// chunk's last pass write its partial, count it, and merge the group when it is the last.
template <int G>
__device__ void attend_consume(const Args& a, Shared& sh, unsigned char* smem) {
  constexpr int NB = att_bufs<G>();
  const int tid = threadIdx.x, lane = tid & 31;
  float* scr = reinterpret_cast<float*>(smem + att_scratch_off<G>());
  const float sc_scale = a.sm_scale;
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  float ot[8][4];
#pragma unroll
  for (int mt = 0; mt < 8; ++mt)
#pragma unroll
    for (int e = 0; e < 4; ++e) ot[mt][e] = 0.f;
#pragma unroll 1
  for (int j = 0;; ++j) {
    const int bs = j % NB, u = j / NB;
#ifdef TWL_STEP_TRACE
    const unsigned long long tc0 = now_ns();
#endif
    int got = 0;
    if (lane == 0) got = mbar_wait(a, &sh.att_full[bs], (uint32_t)(u & 1));
    got = __shfl_sync(0xffffffffu, got, 0);
    if (!got) break;
    // the other lanes acquire the phase too (it is complete: the poll returns at once)
    if (lane != 0) mbar_test(&sh.att_full[bs], (uint32_t)(u & 1));
    const int flags = sh.att_desc[bs][3];
    if (flags & kDescEnd) break;
    const int cn = sh.att_desc[bs][0], c = sh.att_desc[bs][1], g = sh.att_desc[bs][2];
#ifdef TWL_STEP_TRACE
    const unsigned long long tc1 = now_ns();
#endif
    if (flags & kDescFirst) {
      m[0] = m[1] = -INFINITY;
      l[0] = l[1] = 0.f;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) ot[mt][e] = 0.f;
    }
    const unsigned char* kb = smem + bs * kAttBufBytes;
    attend_tile<G>(kb, kb + kAttPass * 256, kb + kAttPass * 512, cn, sc_scale, m, l, ot);
    __syncwarp();
    if (lane == 0) mbar_arrive(&sh.att_empty[bs]);
#ifdef TWL_STEP_TRACE
    if (tid == 0 && a.trace && j < 16) {
      unsigned long long* pr = a.trace + 17 * (size_t)a.n_items + 96 * (size_t)blockIdx.x + 6 * j;
      pr[3] = tc0;
      pr[4] = tc1;
      pr[5] = now_ns();
    }
#endif
    if (!(flags & kDescLast)) continue;
    attend_finish<G>(a, c, m, l, ot, scr);
    const int c0 = ldcg_i(a.cbase + 2 * g), nch = ldcg_i(a.cbase + 2 * g + 1);
    bar_named(2, kAttCons);  // every consumer's partial writes before the count
    if (tid == 0) sh.att_last = atom_acq_rel_add(counter(a, kCntAttend, g), 1u) + 1u == (uint32_t)nch;
    bar_named(2, kAttCons);
    if (sh.att_last) merge_group<G>(a, g, c0, nch, scr);
  }
}

// A worker of the attention queue (one per CTA, after its other items).
template <int G>
__device__ void attend_worker(const Args& a, Shared& sh, unsigned char* smem) {
  constexpr int NB = att_bufs<G>();
  if (threadIdx.x == 0) {
    for (int i = 0; i < NB; ++i) {
      mbar_init(&sh.att_full[i], kAttProd + 1);
      mbar_init(&sh.att_empty[i], kAttCons / 32);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x >= kAttCons) attend_produce<G>(a, sh, smem);
  else attend_consume<G>(a, sh, smem);
  __syncthreads();
  if (threadIdx.x == 0)
    for (int i = 0; i < NB; ++i) {
      mbar_inval(&sh.att_full[i]);
      mbar_inval(&sh.att_empty[i]);
    }
}

// ------------------------------------------------------------------------------ the kernel
template <int G>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) k_step(const __grid_constant__ Args a) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ Shared sh;
  // wait for the previous grid in the stream (launched programmatically), then let the next one
  // be scheduled: it will in turn wait for this grid to complete before touching memory
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");
  int idx = blockIdx.x;
#pragma unroll 1
  while (idx < a.n_items) {
#ifdef TWL_STEP_TRACE
    unsigned long long t_start = 0, c_start = 0;
    if (threadIdx.x == 0) {
      t_start = now_ns();
      c_start = clock64();
      sh.t_ready = 0;
      for (int m = 0; m < 10; ++m) sh.marks[m] = 0;
    }
#endif
    int phase = -1, g = 0, sub = 0;
#pragma unroll 1
    for (int s = 0; s < a.nseg; ++s) {
      const Segment& sg = a.seg[s];
      const int cnt = (sg.g1 - sg.g0) * sg.per;
      if (idx < sg.first + cnt) {
        const int l = idx - sg.first;
        phase = sg.phase;
        g = sg.g0 + l / sg.per;
        sub = l - (l / sg.per) * sg.per;
        break;
      }
    }
    const int b = g / a.kv.hkv, kvh = g - b * a.kv.hkv;
    switch (phase) {
      case kScore:
        item_score<G>(a, sh, g, sub, smem);
        break;
      case kTopK:
        item_topk<G>(a, sh, b * a.hq + kvh * G + sub, smem, a.smem_bytes);
        block_signal(counter(a, kCntTopK, g));
        break;
      case kEst:
        item_estimate<G>(a, sh, g, sub, smem);
        break;
      case kPrune:
        item_prune(a, sh, b * a.hq + kvh * G + sub, smem, a.smem_bytes);
        if (block_signal_last(sh, counter(a, kCntPrune, g), (uint32_t)G))
          build_kept<G>(a, sh, g, smem);
        break;
      case kAttend:
        attend_worker<G>(a, sh, smem);
        break;
      default:
        break;
    }
#ifdef TWL_STEP_TRACE
    __syncthreads();
    if (threadIdx.x == 0 && a.trace) {
      unsigned long long* tr = a.trace + 17 * (size_t)idx;
      tr[0] = (unsigned long long)idx;
      tr[1] = blockIdx.x;
      tr[2] = t_start;
      tr[3] = sh.t_ready;
      for (int m = 0; m < 10; ++m) tr[4 + m] = sh.marks[m];
      tr[14] = now_ns();
      tr[15] = c_start;
      tr[16] = clock64();
    }
#endif
    // the next free item, taken only now: a CTA never holds an item it cannot start
    if (threadIdx.x == 0) sh.next = (int)(gridDim.x + atomicAdd(a.sync + kNext, 1u));
    __syncthreads();
    idx = sh.next;
    __syncthreads();
  }
  // leaving: the last CTA out clears the synchronisation words for the next launch
  __syncthreads();
  if (threadIdx.x == 0) sh.flag = atom_acq_rel_add(a.sync + kExit, 1u) + 1u == gridDim.x;
  __syncthreads();
  if (sh.flag) {
    const int used = min(a.q_cap, (int)ldcg_u(a.sync + kQAlloc));
    for (int i = threadIdx.x; i < used; i += kThreads) a.qvalid[i] = 0u;
    // an aborted launch may leave page masks that no kept-list build consumed
    if (ldcg_u(a.sync + kAbort) != 0u)
      for (size_t i = threadIdx.x; i < (size_t)a.groups * a.pm_words; i += kThreads)
        a.pmask[i] = 0u;
    const int nwords = kSyncHead + kCounters * a.groups;
    for (int i = threadIdx.x; i < nwords; i += kThreads) a.sync[i] = 0u;
  }
}

}  // namespace

// ---------------------------------------------------------------------------------- host side
namespace {

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }
int round32(int x) { return (x + 31) & ~31; }

template <int G>
const void* kernel_of() {
  return reinterpret_cast<const void*>(&k_step<G>);
}
const void* kernel_for(int g) {
  switch (g) {
    case 1: return kernel_of<1>();
    case 2: return kernel_of<2>();
    case 4: return kernel_of<4>();
    case 8: return kernel_of<8>();
    default: return nullptr;
  }
}

// Shared memory each item kind needs (bytes).
int smem_need(int g, int max_pages, int max_budget, int s_chunk) {
  const int sw = round32((max_pages + 31) / 32);
  const int topk = 4 * sw + 4 * round32(max_pages) + 4 * (4096 + 512) + 8 * 64 + 64;
  const int kept_words = (16 * max_budget + 31) / 32;
  const int prune = 1024 + 16 * kThreads + kHistBytes + 4 * round32(kept_words) +
                    8 * round32(sw) + 128;  // + staged weights when they fit
  const int score = ((4 * s_chunk + 127) & ~127) + 2 * kScorePass * 512;
  const int est_kw = kEstMeta / 32 + 1;
  const int est = ((4 * ((2 + g) * kEstMeta + (2 * g + 2) * est_kw + 1) + 127) & ~127) +
                  2 * kEstPass * 1088;
  int need = topk;
  const int att = g == 1 ? att_smem<1>() : g == 2 ? att_smem<2>() : g == 4 ? att_smem<4>()
                                                                        : att_smem<8>();
  for (int x : {prune, score, est, att}) need = need > x ? need : x;
  return need;
}

// Dynamic shared memory per CTA: everything the device grants one block beyond the static part
// (the estimate's stages and the staged weights use what the minimum leaves).
int smem_avail(int g) {
  int dev = 0, optin = 0, per_sm = 0;
  cudaGetDevice(&dev);
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    optin = 227 * 1024;
  if (cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) !=
      cudaSuccess)
    per_sm = 228 * 1024;
  cudaFuncAttributes fa{};
  const void* k = kernel_for(g);
  size_t stat = 1024;
  if (k && cudaFuncGetAttributes(&fa, k) == cudaSuccess) stat = fa.sharedSizeBytes;
  cudaGetLastError();
  // kCtasPerSm CTAs share the SM's shared memory, 1 KB of it reserved per CTA
  long long avail = (long long)per_sm / kCtasPerSm - 1024;
  avail = avail < optin ? avail : optin;
  return (int)(avail - (long long)stat - (kCtasPerSm == 1 ? 1024 : 0)) & ~127;
}

}  // namespace

Plan plan(int batch, int hq, int hkv, int max_pages, int max_budget) {
  Plan pl{};
  const int g = hq / hkv;
  const int groups = batch * hkv;
  pl.sel_words = ((max_pages + 31) / 32 + 3) & ~3;  // rows of whole 16-byte pieces
  pl.cand_stride = kPage * max_budget;
  pl.kept_words = (pl.cand_stride + 31) / 32;
  // the CTAs of the grid: kCtasPerSm per SM, every CTA resident ("sms" below counts CTAs)
  const int sms = num_sms() * kCtasPerSm;
  pl.grid = sms;
  pl.smem_bytes = smem_avail(g);
  // work list: score chunks so the pages fill every CTA (one wave when the groups are few and
  // short, about four otherwise); estimate and attention slices likewise per group
  const long long total_pages = (long long)groups * max_pages;
  if (groups <= sms / 2 && total_pages <= (long long)sms * 512) {
    pl.s_per = sms / groups;
  } else {
    const long long chunk = (total_pages + 4ll * sms - 1) / (4ll * sms);
    pl.s_per = (int)((max_pages + chunk - 1) / chunk);
  }
  pl.s_per = pl.s_per < 1 ? 1 : (pl.s_per > max_pages ? max_pages : pl.s_per);
  if ((max_pages + pl.s_per - 1) / pl.s_per > 4096) pl.s_per = (max_pages + 4095) / 4096;
  pl.s_chunk = (max_pages + pl.s_per - 1) / pl.s_per;
  pl.s_per = (max_pages + pl.s_chunk - 1) / pl.s_chunk;
  pl.ok = smem_need(g, max_pages, max_budget, pl.s_chunk) <= pl.smem_bytes;
  const long long est_pages = (long long)groups * (max_pages < 2 * max_budget ? max_pages
                                                                             : 2 * max_budget);
  long long waves = (est_pages + (long long)sms * 128 - 1) / ((long long)sms * 128);
  waves = waves < 1 ? 1 : (waves > 4 ? 4 : waves);
  if (waves == 1 && groups <= sms) pl.e_per = sms / groups;
  else pl.e_per = (int)((waves * sms + groups - 1) / groups);
  pl.e_per = pl.e_per < 1 ? 1 : (pl.e_per > 64 ? 64 : pl.e_per);
  pl.e_chunk = (max_pages + pl.e_per - 1) / pl.e_per;  // logical pages per estimate item
  pl.e_per = (max_pages + pl.e_chunk - 1) / pl.e_chunk;
  // attention chunks: at most one per kAttChunkTok kept tokens of each group plus one, and the
  // numbers the workers take past the end
  pl.q_cap = groups * (1 + (kPage * max_pages + kAttChunkTok - 1) / kAttChunkTok) + sms + 32;
  pl.att_chunks = sms / groups;
  pl.att_chunks = pl.att_chunks < 1 ? 1 : pl.att_chunks;
  return pl;
}

namespace {
struct Layout {
  size_t sync, keys, selbits, ncand, hpre, logits, pmask, kpages,
      qtab, qvalid, cbase, part, trace, total;
};
Layout layout(const Plan& pl, int batch, int hq, int hkv, int max_pages) {
  const int g = hq / hkv;
  const size_t bh = (size_t)batch * hq, groups = (size_t)batch * hkv;
  Layout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align_up(bytes);
    return o;
  };
#ifdef TWL_STEP_TRACE
  L.trace = take(8 * 17 * (size_t)(groups * (pl.s_per + 2 * g + pl.e_per) + pl.grid) +
                 8 * 96 * (size_t)pl.grid);
#endif
  L.sync = take(4 * (kSyncHead + kCounters * groups));
  L.keys = take(4 * bh * max_pages);
  L.selbits = take(4 * bh * pl.sel_words);
  L.ncand = take(4 * bh);
  L.hpre = take(4 * bh * pl.sel_words);
  L.logits = take(4 * bh * pl.cand_stride);
  L.pmask = take(4 * groups * (size_t)((max_pages + 1) / 2));
  L.kpages = take(16 * groups * (size_t)max_pages);
  L.qtab = take(16 * (size_t)pl.q_cap);
  L.qvalid = take(4 * (size_t)pl.q_cap);
  L.cbase = take(8 * groups);
  L.part = take(4 * (size_t)pl.q_cap * g * kAttPartStride);
  L.total = off;
  return L;
}
}  // namespace

size_t workspace_bytes(int batch, int hq, int hkv, int max_pages, int max_budget) {
  const Plan pl = plan(batch, hq, hkv, max_pages, max_budget);
  return layout(pl, batch, hq, hkv, max_pages).total;
}

namespace {
uint32_t g_spin_limit = kSpinLimit;  // test knobs (twl_test_set_waits)
int g_stall_estimate = 0;
}  // namespace

void set_test_waits(uint32_t spin_limit, int stall_estimate) {
  g_spin_limit = spin_limit > 0 ? spin_limit : kSpinLimit;
  g_stall_estimate = stall_estimate != 0;
}

void carve(Args& a, char* ws, const Plan& pl, int batch, int hq, int hkv, int max_pages) {
  const Layout L = layout(pl, batch, hq, hkv, max_pages);
  a.sync = reinterpret_cast<uint32_t*>(ws + L.sync);
  a.keys = reinterpret_cast<uint32_t*>(ws + L.keys);
  a.selbits = reinterpret_cast<uint32_t*>(ws + L.selbits);
  a.ncand = reinterpret_cast<int*>(ws + L.ncand);
  a.hpre = reinterpret_cast<int*>(ws + L.hpre);
  a.logits = reinterpret_cast<float*>(ws + L.logits);
  a.pmask = reinterpret_cast<uint32_t*>(ws + L.pmask);
  a.pm_words = (max_pages + 1) / 2;
  a.kpages = reinterpret_cast<int4*>(ws + L.kpages);
  a.qtab = reinterpret_cast<int*>(ws + L.qtab);
  a.qvalid = reinterpret_cast<uint32_t*>(ws + L.qvalid);
  a.cbase = reinterpret_cast<int*>(ws + L.cbase);
  a.part = reinterpret_cast<float*>(ws + L.part);
#ifdef TWL_STEP_TRACE
  a.trace = reinterpret_cast<unsigned long long*>(ws + L.trace);
#endif
  const int g = hq / hkv;
  a.g = g;
  a.groups = batch * hkv;
  a.sel_words = pl.sel_words;
  a.cand_stride = pl.cand_stride;
  a.kept_words = pl.kept_words;
  a.s_per = pl.s_per;
  a.s_chunk = pl.s_chunk;
  a.e_per = pl.e_per;
  a.e_chunk = pl.e_chunk;
  a.q_cap = pl.q_cap;
  a.att_chunks = pl.att_chunks;
  a.spin_limit = g_spin_limit;
  a.stall_estimate = g_stall_estimate;
  a.smem_bytes = pl.smem_bytes;
  // the work list, kind by kind (every item depends only on items of earlier kinds)
  // the work list, kind by kind (every item depends only on items of earlier kinds); the last
  // kind is one attention worker per CTA
  const int per[4] = {pl.s_per, g, pl.e_per, g};
  int first = 0;
  a.nseg = 0;
  for (int ph = kScore; ph <= kPrune; ++ph) {
    Segment& s = a.seg[a.nseg++];
    s.phase = ph;
    s.g0 = 0;
    s.g1 = a.groups;
    s.per = per[ph];
    s.first = first;
    first += a.groups * per[ph];
  }
  Segment& w = a.seg[a.nseg++];
  w.phase = kAttend;
  w.g0 = 0;
  w.g1 = 1;
  w.per = pl.grid;
  w.first = first;
  a.n_items = first + pl.grid;
}

cudaError_t launch(const Args& a, const Plan& pl, cudaStream_t s) {
  const void* k = kernel_for(a.g);
  if (!k) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       pl.smem_bytes);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, kThreads, pl.smem_bytes);
  if (e != cudaSuccess) return e;
  if (per_sm < kCtasPerSm) return cudaErrorInvalidConfiguration;  // not every CTA resident
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)pl.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = (size_t)pl.smem_bytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  // programmatic dependent launch: this grid may be scheduled while the previous kernel in the
  // stream finishes; it waits for that kernel (griddepcontrol.wait) before touching memory
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  void* params[] = {const_cast<Args*>(&a)};
  e = cudaLaunchKernelExC(&cfg, k, params);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace TWL_STEP_NS
}  // namespace twl
