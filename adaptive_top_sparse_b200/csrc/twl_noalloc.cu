// twl_sparse_decode_noalloc: twl_sparse_decode for callers that cannot allocate device memory.
//
// Some callers have no way to hand the library a workspace: code that runs inside a host
// framework which owns every byte of device memory and exposes no allocator to plug-ins, code
// with a hard real-time budget that may not call cudaMalloc (it can synchronise the whole device),
// and integrations whose memory plan is fixed before the first call.  For them this entry point
// takes its scratch from one file-scope device array instead of a caller workspace.
//
// The array is statically sized (kNoAllocScratchBytes) and is part of the library image: every
// GPU that loads libtwl.so holds it until the process exits.  Requests whose split-KV partials do
// not fit are rejected with TWL_ERR_SCRATCH_LIMIT before anything is launched.  The device
// address of the array is looked up once per device (cudaGetSymbolAddress, with that device
// current) on the first call made on that device; make that first call before any stream capture.
// The looked-up address belongs to the device's primary context as it was at that first call: it
// does not survive cudaDeviceReset (which unloads the library image from the device), nor does it
// serve a different context made current on the same device; such callers must not use this entry
// point afterwards.
// All calls share the array, so calls that overlap on the GPU (different streams, or different
// host threads) race on it.  Nothing in it needs to start at zero: the partials are written before
// they are read, and the device flags of its 256-byte header are not reported to the caller.
// This entry point allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
#include <cuda_runtime.h>

#include <mutex>

#include "twl.h"
#include "twl_kernels.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_twl_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device (looked up once per device).
// In host code the array's name is only a host-side handle: passing it to a kernel would fault or
// read the wrong memory, so the address must come from cudaGetSymbolAddress.
twl_status scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return TWL_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return TWL_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_twl_noalloc_scratch) != cudaSuccess || p == nullptr)
      return TWL_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return TWL_OK;
}

}  // namespace

extern "C" size_t twl_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

extern "C" twl_status twl_sparse_decode_noalloc(const void* q, int32_t num_q_heads,
                                                const twl_paged_kv* kv, const int32_t* tok,
                                                const int32_t* tok_count, int32_t tok_stride,
                                                float sm_scale, float* o, float* lse,
                                                twl_stream_t stream) {
  // the argument checks of twl_sparse_decode first, so a malformed request gets the same
  // status as there (not TWL_ERR_SCRATCH_LIMIT)
  twl::KV k;
  const twl_status chk = twl::check_sparse_decode_args(q, num_q_heads, kv, tok, tok_count,
                                                       tok_stride, sm_scale, o, lse, &k);
  if (chk != TWL_OK) return chk;
  const size_t need = twl_workspace_bytes(TWL_OP_SPARSE_DECODE, kv->batch, num_q_heads,
                                          kv->num_kv_heads, 0, 0, 0, tok_stride);
  if (need == 0) return TWL_ERR_INVALID_ARG;
  if (need > kNoAllocScratchBytes) return TWL_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  const twl_status st = scratch_for_current_device(&scratch);
  if (st != TWL_OK) return st;
  return twl_sparse_decode(q, num_q_heads, kv, tok, tok_count, tok_stride, sm_scale, o, lse,
                           scratch, kNoAllocScratchBytes, stream);
}
