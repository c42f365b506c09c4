// C-ABI entry points of segment linear attention: argument checks, then kernel
// launches on the caller's stream.  Nothing here allocates, frees or synchronises.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "seg_la.h"
#include "seg_la_internal.h"

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int la_check(const void* q, const void* k, const void* v, const float* g, const void* out,
             const float* state_pool, const void* dev_table, const seg_la_table_desc* desc,
             float scale, int mode) {
  if (!desc || desc->magic != SEG_LA_TABLE_MAGIC || desc->version != SEG_LA_TABLE_VERSION ||
      desc->mode != mode)
    return SEG_ATTN_ERR_INVALID_ARG;
  if (!isfinite(scale)) return SEG_ATTN_ERR_INVALID_ARG;
  if (desc->batch > 0 && (!dev_table || !aligned16(dev_table))) return SEG_ATTN_ERR_INVALID_ARG;
  if (desc->total_q > 0 &&
      (!q || !k || !v || !g || !out || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
       !aligned16(out) || (reinterpret_cast<uintptr_t>(g) & 3)))
    return SEG_ATTN_ERR_INVALID_ARG;
  if (desc->batch > 0 && desc->num_state_slots > 0 && (!state_pool || !aligned16(state_pool)))
    return SEG_ATTN_ERR_INVALID_ARG;
  return SEG_ATTN_OK;
}

segla::Launch make_launch(const void* q, const void* k, const void* v, const float* g, void* out,
                          float* state_pool, const void* dev_table,
                          const seg_la_table_desc* desc, float scale, void* workspace) {
  segla::Launch a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.g = g;
  a.out = out;
  a.state_pool = state_pool;
  a.tab = segla::make_table(dev_table, *desc);
  a.desc = desc;
  a.scale = scale;
  a.workspace = workspace;
  return a;
}

}  // namespace

extern "C" int seg_la_prefill(const void* q, const void* k, const void* v, const float* g,
                              void* out, float* state_pool, const void* dev_table,
                              const seg_la_table_desc* desc, float scale, void* workspace,
                              size_t workspace_bytes, void* stream) {
  int rc = la_check(q, k, v, g, out, state_pool, dev_table, desc, scale, SEG_ATTN_MODE_PREFILL);
  if (rc != SEG_ATTN_OK) return rc;
  if (desc->workspace_bytes > 0 &&
      (!workspace || workspace_bytes < desc->workspace_bytes || !aligned16(workspace)))
    return SEG_ATTN_ERR_WORKSPACE;
  if (desc->batch == 0) return SEG_ATTN_OK;
  return segla::launch_la_prefill(
      make_launch(q, k, v, g, out, state_pool, dev_table, desc, scale, workspace),
      static_cast<cudaStream_t>(stream));
}

extern "C" int seg_la_decode(const void* q, const void* k, const void* v, const float* g,
                             void* out, float* state_pool, const void* dev_table,
                             const seg_la_table_desc* desc, float scale, void* stream) {
  int rc = la_check(q, k, v, g, out, state_pool, dev_table, desc, scale, SEG_ATTN_MODE_DECODE);
  if (rc != SEG_ATTN_OK) return rc;
  if (desc->batch == 0) return SEG_ATTN_OK;
  return segla::launch_la_decode(
      make_launch(q, k, v, g, out, state_pool, dev_table, desc, scale, nullptr),
      static_cast<cudaStream_t>(stream));
}
