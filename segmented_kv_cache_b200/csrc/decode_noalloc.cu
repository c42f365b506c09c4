// Decode entry point for callers that cannot allocate device memory.
//
// seg_attn_decode needs a scratch buffer for its split-K partials, which the
// caller normally allocates.  Some callers cannot: a plugin hosted by another
// runtime that owns every device allocation and hands out no allocator, or a
// latency-critical serving loop that must not call cudaMalloc once it is
// running (cudaMalloc may synchronise the device and stall every stream).
// For them this file keeps the scratch in one fixed device array that lives in
// the library image itself.
//
// Limits and rules (also stated in include/seg_attn.h):
//   - The array holds kNoAllocScratchBytes (64 MiB).  Every GPU on which the
//     library's module is loaded keeps that memory until the process exits.
//   - A call whose table needs more scratch than that is rejected with
//     SEG_ATTN_ERR_WORKSPACE before anything is launched.
//   - All calls share the one array and it keeps whatever the last call left
//     in it.  Nothing in it has to start at zero: every partial the merge
//     kernel reads was written earlier by the same call.  Calls that overlap
//     on the GPU (other streams, other host threads) race on the array; the
//     caller must order them, e.g. by issuing them on one stream.
//   - The first call on each device asks the runtime for the array's device
//     address (cudaGetSymbolAddress) with that device current and remembers
//     it.  Make that first call before any stream capture is started.  The
//     remembered address is only valid while the device's primary context
//     lives: a cudaDeviceReset reloads the module, possibly elsewhere, so the
//     entry point must not be used on that device again in the process.
//   - Nothing here calls cudaMalloc, cudaFree or an allocating library routine.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "seg_attn.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 64ull << 20;
constexpr int kMaxDevices = 64;

// Split-K partials of seg_attn_decode_noalloc.  In host code this name is only
// a host-side handle: its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once).
int scratch_on_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return SEG_ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return SEG_ATTN_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return SEG_ATTN_OK;
}

}  // namespace

extern "C" int seg_attn_decode_noalloc(const void* q, const void* k_pool, const void* v_pool,
                                       void* out, float* lse, const void* dev_table,
                                       const seg_attn_table_desc* desc, float softmax_scale,
                                       void* stream) {
  if (!desc || desc->magic != SEG_ATTN_TABLE_MAGIC) return SEG_ATTN_ERR_INVALID_ARG;
  if (desc->workspace_bytes > kNoAllocScratchBytes) return SEG_ATTN_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (desc->workspace_bytes > 0) {
    const int rc = scratch_on_current_device(&scratch);
    if (rc != SEG_ATTN_OK) return rc;
  }
  return seg_attn_decode(q, k_pool, v_pool, out, lse, dev_table, desc, softmax_scale, scratch,
                         scratch ? kNoAllocScratchBytes : 0, stream);
}
