// C-ABI compute entry points: argument checks, then kernel launches on the
// caller's stream.  Nothing here allocates, frees or synchronises.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "seg_attn.h"
#include "seg_attn_internal.h"
#include "seg_la_internal.h"

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int check_common(const void* q, const void* k_pool, const void* v_pool, const void* out,
                 const float* lse, const void* dev_table, const seg_attn_table_desc* desc,
                 float scale, int mode) {
  if (!desc || desc->magic != SEG_ATTN_TABLE_MAGIC || desc->version != SEG_ATTN_TABLE_VERSION)
    return SEG_ATTN_ERR_INVALID_ARG;
  if (desc->mode != mode) return SEG_ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return SEG_ATTN_ERR_INVALID_ARG;
  if (desc->total_q > 0) {
    if (!q || !out || !aligned16(q) || !aligned16(out)) return SEG_ATTN_ERR_INVALID_ARG;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3)) return SEG_ATTN_ERR_INVALID_ARG;
  }
  if (desc->total_k > 0 && (!k_pool || !v_pool || !aligned16(k_pool) || !aligned16(v_pool)))
    return SEG_ATTN_ERR_INVALID_ARG;
  if (desc->num_work > 0 && (!dev_table || !aligned16(dev_table)))
    return SEG_ATTN_ERR_INVALID_ARG;
  return SEG_ATTN_OK;
}

char* at(void* base, size_t off) { return static_cast<char*>(base) + off; }

// The pass over the shared prefixes (prefill kernel, every piece a partial; on
// an FP8 cache the FP8 prefill kernel with the same scales as the rest).
int launch_group_pass(const void* q, const void* k_pool, const void* v_pool, const float* k_scale,
                      const float* v_scale, bool fp8, const void* dev_table,
                      const seg_attn_table_desc& desc, const segattn::WorkspaceLayout& ws_at,
                      void* workspace, float scale, cudaStream_t stream) {
  if (desc.num_group_work == 0) return SEG_ATTN_OK;
  const seg_attn_table_desc gd = segattn::group_pass_desc(desc);
  segattn::PrefillLaunch a;
  a.q = q;
  a.k_pool = k_pool;
  a.v_pool = v_pool;
  a.out = nullptr;  // every piece writes to the workspace
  a.lse = nullptr;
  a.tab = segattn::make_view(dev_table, gd);
  a.desc = &gd;
  a.scale = scale;
  a.part_o = reinterpret_cast<float*>(at(workspace, ws_at.group_o));
  a.part_lse = reinterpret_cast<float*>(at(workspace, ws_at.group_lse));
  a.fp8 = fp8;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  return segattn::launch_prefill(a, stream);
}

int launch_cascade(const void* dev_table, const seg_attn_table_desc& desc,
                   const segattn::WorkspaceLayout& ws_at, void* workspace, void* out, float* lse,
                   cudaStream_t stream) {
  segattn::CascadeLaunch c;
  c.dev_table = dev_table;
  c.desc = &desc;
  c.main_o = reinterpret_cast<const float*>(at(workspace, ws_at.main_o));
  c.main_lse = reinterpret_cast<const float*>(at(workspace, ws_at.main_lse));
  c.group_o = reinterpret_cast<const float*>(at(workspace, ws_at.group_o));
  c.group_lse = reinterpret_cast<const float*>(at(workspace, ws_at.group_lse));
  c.out = out;
  c.lse = lse;
  return segattn::launch_cascade_merge(c, stream);
}

}  // namespace

namespace {

int prefill_common(const void* q, const void* k_pool, const void* v_pool, const float* k_scale,
                   const float* v_scale, bool fp8, void* out, float* lse, const void* dev_table,
                   const seg_attn_table_desc* desc, float softmax_scale, void* workspace,
                   size_t workspace_bytes, void* stream) {
  int rc = check_common(q, k_pool, v_pool, out, lse, dev_table, desc, softmax_scale,
                        SEG_ATTN_MODE_PREFILL);
  if (rc != SEG_ATTN_OK) return rc;
  if (fp8 && desc->total_k > 0 &&
      (!k_scale || !v_scale || (reinterpret_cast<uintptr_t>(k_scale) & 3) ||
       (reinterpret_cast<uintptr_t>(v_scale) & 3)))
    return SEG_ATTN_ERR_INVALID_ARG;
  if (desc->workspace_bytes > 0 &&
      (!workspace || workspace_bytes < desc->workspace_bytes || !aligned16(workspace)))
    return SEG_ATTN_ERR_WORKSPACE;
  if (desc->num_work == 0 && desc->num_group_work == 0) return SEG_ATTN_OK;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const segattn::WorkspaceLayout ws_at = segattn::workspace_layout(*desc, false);
  if (desc->shared) {
    rc = launch_group_pass(q, k_pool, v_pool, k_scale, v_scale, fp8, dev_table, *desc, ws_at,
                           workspace, softmax_scale, st);
    if (rc != SEG_ATTN_OK) return rc;
  }
  if (desc->num_work > 0) {
    segattn::PrefillLaunch a;
    a.q = q;
    a.k_pool = k_pool;
    a.v_pool = v_pool;
    a.out = out;
    a.lse = lse;
    a.tab = segattn::make_view(dev_table, *desc);
    a.desc = desc;
    a.scale = softmax_scale;
    a.part_o = desc->num_parts > 0 ? reinterpret_cast<float*>(at(workspace, ws_at.main_o)) : nullptr;
    a.part_lse =
        desc->num_parts > 0 ? reinterpret_cast<float*>(at(workspace, ws_at.main_lse)) : nullptr;
    a.fp8 = fp8;
    a.k_scale = k_scale;
    a.v_scale = v_scale;
    rc = segattn::launch_prefill(a, st);
    if (rc != SEG_ATTN_OK) return rc;
  }
  if (desc->shared) return launch_cascade(dev_table, *desc, ws_at, workspace, out, lse, st);
  return SEG_ATTN_OK;
}

}  // namespace

extern "C" int seg_attn_prefill(const void* q, const void* k_pool, const void* v_pool, void* out,
                                float* lse, const void* dev_table, const seg_attn_table_desc* desc,
                                float softmax_scale, void* workspace, size_t workspace_bytes,
                                void* stream) {
  return prefill_common(q, k_pool, v_pool, nullptr, nullptr, false, out, lse, dev_table, desc,
                        softmax_scale, workspace, workspace_bytes, stream);
}

extern "C" int seg_attn_prefill_fp8(const void* q, const void* k_pool, const void* v_pool,
                                    const float* k_scale, const float* v_scale, void* out,
                                    float* lse, const void* dev_table,
                                    const seg_attn_table_desc* desc, float softmax_scale,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  return prefill_common(q, k_pool, v_pool, k_scale, v_scale, true, out, lse, dev_table, desc,
                        softmax_scale, workspace, workspace_bytes, stream);
}

namespace {

int decode_common(const void* q, const void* k_pool, const void* v_pool, const float* k_scale,
                  const float* v_scale, bool fp8, void* out, float* lse, const void* dev_table,
                  const seg_attn_table_desc* desc, float softmax_scale, void* workspace,
                  size_t workspace_bytes, void* stream) {
  int rc = check_common(q, k_pool, v_pool, out, lse, dev_table, desc, softmax_scale,
                        SEG_ATTN_MODE_DECODE);
  if (rc != SEG_ATTN_OK) return rc;
  if (fp8 && desc->total_k > 0 &&
      (!k_scale || !v_scale || (reinterpret_cast<uintptr_t>(k_scale) & 3) ||
       (reinterpret_cast<uintptr_t>(v_scale) & 3)))
    return SEG_ATTN_ERR_INVALID_ARG;
  if (desc->workspace_bytes > 0 &&
      (!workspace || workspace_bytes < desc->workspace_bytes || !aligned16(workspace)))
    return SEG_ATTN_ERR_WORKSPACE;
  if (desc->num_work == 0) return SEG_ATTN_OK;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const segattn::WorkspaceLayout ws_at =
      segattn::workspace_layout(*desc, desc->workspace_bytes > 0);
  if (desc->shared) {
    rc = launch_group_pass(q, k_pool, v_pool, k_scale, v_scale, fp8, dev_table, *desc, ws_at,
                           workspace, softmax_scale, st);
    if (rc != SEG_ATTN_OK) return rc;
  }
  segattn::DecodeLaunch a;
  a.q = q;
  a.k_pool = k_pool;
  a.v_pool = v_pool;
  a.out = out;
  a.lse = lse;
  a.tab = segattn::make_view(dev_table, *desc);
  a.desc = desc;
  a.scale = softmax_scale;
  a.part_o = desc->workspace_bytes > 0 ? reinterpret_cast<float*>(at(workspace, ws_at.main_o))
                                       : nullptr;
  a.part_lse = desc->workspace_bytes > 0
                   ? reinterpret_cast<float*>(at(workspace, ws_at.main_lse))
                   : nullptr;
  a.fp8 = fp8;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  rc = segattn::launch_decode(a, st);
  if (rc != SEG_ATTN_OK) return rc;
  if (desc->shared) return launch_cascade(dev_table, *desc, ws_at, workspace, out, lse, st);
  return SEG_ATTN_OK;
}

}  // namespace

extern "C" int seg_attn_decode(const void* q, const void* k_pool, const void* v_pool, void* out,
                               float* lse, const void* dev_table, const seg_attn_table_desc* desc,
                               float softmax_scale, void* workspace, size_t workspace_bytes,
                               void* stream) {
  return decode_common(q, k_pool, v_pool, nullptr, nullptr, false, out, lse, dev_table, desc,
                       softmax_scale, workspace, workspace_bytes, stream);
}

extern "C" int seg_attn_decode_fp8(const void* q, const void* k_pool, const void* v_pool,
                                   const float* k_scale, const float* v_scale, void* out,
                                   float* lse, const void* dev_table,
                                   const seg_attn_table_desc* desc, float softmax_scale,
                                   void* workspace, size_t workspace_bytes, void* stream) {
  return decode_common(q, k_pool, v_pool, k_scale, v_scale, true, out, lse, dev_table, desc,
                       softmax_scale, workspace, workspace_bytes, stream);
}

extern "C" int seg_attn_wait_selftest(int wait_us, void* stream) {
  if (wait_us < 1 || wait_us > 1000000) return SEG_ATTN_ERR_INVALID_ARG;
  return segattn::launch_wait_selftest(wait_us, static_cast<cudaStream_t>(stream));
}

extern "C" int seg_attn_stall_test(int withhold_k_tile, int wait_us) {
  if (wait_us < 1 || wait_us > 1000000) return SEG_ATTN_ERR_INVALID_ARG;
  return segattn::set_stall_test(withhold_k_tile, wait_us);
}

extern "C" int seg_attn_order_test(int delay_ns) {
  if (delay_ns < 0 || delay_ns > 1000000) return SEG_ATTN_ERR_INVALID_ARG;
  return segattn::set_order_test(delay_ns);
}

extern "C" int seg_attn_take_device_error(int* value) {
  if (!value) return SEG_ATTN_ERR_INVALID_ARG;
  int wait_err = 0, append_err = 0;
  int rc = segattn::take_device_error(&wait_err);
  if (rc != SEG_ATTN_OK) return rc;
  rc = segattn::take_append_error(&append_err);
  if (rc != SEG_ATTN_OK) return rc;
  int la_err = 0;
  rc = segla::take_la_error(&la_err);
  if (rc != SEG_ATTN_OK) return rc;
  *value = (wait_err ? 1 : 0) | (append_err ? 2 : 0) | (la_err ? 4 : 0);
  return SEG_ATTN_OK;
}
