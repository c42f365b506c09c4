// KV append: copy the K/V rows of new tokens into their slots of the pool.
//
// Each slot's row is kv_heads * head_dim contiguous bf16 values in both pools,
// so the copy is one 16-byte vector per thread, coalesced on both sides.  The
// caller gets the slots from the segment allocator (seg_attn_pool_append).  A
// slot outside the pool is skipped and flagged in a device error word; nothing
// is written out of bounds.
#include <cuda_runtime.h>
#include <stdint.h>

#include "seg_attn.h"
#include "seg_attn_internal.h"

namespace segattn {

__device__ int g_append_error;  // non-zero once a slot out of range was skipped

namespace {

__global__ void __launch_bounds__(256) kv_append_kernel(const uint4* __restrict__ k_new,
                                                        const uint4* __restrict__ v_new,
                                                        const int32_t* __restrict__ slots,
                                                        int64_t n_tokens, int row_vecs,
                                                        uint4* k_pool, uint4* v_pool,
                                                        int64_t num_slots) {
  const int64_t total = n_tokens * row_vecs;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t tok = i / row_vecs;
    const int v = (int)(i - tok * row_vecs);
    const int32_t s = __ldg(slots + tok);
    if (s < 0 || s >= num_slots) {
      if (v == 0) atomicOr(&g_append_error, 1);
      continue;
    }
    const int64_t dst = (int64_t)s * row_vecs + v;
    k_pool[dst] = __ldg(k_new + i);
    v_pool[dst] = __ldg(v_new + i);
  }
}

// FP8 pools: one thread writes 16 E4M3 codes (one 16-byte vector) of a slot's
// row from 16 bf16 inputs; code = RNE(x / scale[head]) saturated to +-448.
// The first element of each pair lands in the low byte.
__device__ __forceinline__ uint32_t quant_pair(uint32_t bf16x2, float scale) {
  const float lo = __uint_as_float(bf16x2 << 16) / scale;
  const float hi = __uint_as_float(bf16x2 & 0xffff0000u) / scale;
  unsigned short code;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(code) : "f"(hi), "f"(lo));
  return code;
}

__global__ void __launch_bounds__(256) kv_append_fp8_kernel(
    const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
    const int32_t* __restrict__ slots, int64_t n_tokens, int row_vecs, int head_dim,
    const float* __restrict__ k_scale, const float* __restrict__ v_scale, uint4* k_pool,
    uint4* v_pool, int64_t num_slots) {
  const int64_t total = n_tokens * row_vecs;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t tok = i / row_vecs;
    const int v = (int)(i - tok * row_vecs);
    const int32_t s = __ldg(slots + tok);
    if (s < 0 || s >= num_slots) {
      if (v == 0) atomicOr(&g_append_error, 1);
      continue;
    }
    const int head = (16 * v) / head_dim;
    const float ks = __ldg(k_scale + head), vs = __ldg(v_scale + head);
    const int64_t dst = (int64_t)s * row_vecs + v;
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      const uint4* src = which == 0 ? k_new : v_new;
      const float sc = which == 0 ? ks : vs;
      const uint4 a = __ldg(src + 2 * i), b = __ldg(src + 2 * i + 1);
      uint4 out;
      out.x = quant_pair(a.x, sc) | (quant_pair(a.y, sc) << 16);
      out.y = quant_pair(a.z, sc) | (quant_pair(a.w, sc) << 16);
      out.z = quant_pair(b.x, sc) | (quant_pair(b.y, sc) << 16);
      out.w = quant_pair(b.z, sc) | (quant_pair(b.w, sc) << 16);
      (which == 0 ? k_pool : v_pool)[dst] = out;
    }
  }
}

}  // namespace

int take_append_error(int* value) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_append_error, sizeof(int)) != cudaSuccess) return SEG_ATTN_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_append_error, &zero, sizeof(int)) != cudaSuccess) return SEG_ATTN_ERR_CUDA;
  *value = v;
  return SEG_ATTN_OK;
}

}  // namespace segattn

extern "C" int seg_attn_kv_append(const void* k_new, const void* v_new, const int32_t* slots,
                                  int64_t n_tokens, int kv_heads, int head_dim, void* k_pool,
                                  void* v_pool, int64_t num_slots, void* stream) {
  if (n_tokens < 0 || kv_heads <= 0 || head_dim <= 0 || num_slots < 0)
    return SEG_ATTN_ERR_INVALID_ARG;
  const int64_t row_bytes = (int64_t)kv_heads * head_dim * 2;
  if (row_bytes % 16 != 0 || row_bytes / 16 > INT32_MAX) return SEG_ATTN_ERR_UNSUPPORTED;
  if (n_tokens == 0) return SEG_ATTN_OK;
  auto aligned = [](const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  if (!aligned(k_new) || !aligned(v_new) || !aligned(k_pool) || !aligned(v_pool) || !slots ||
      (reinterpret_cast<uintptr_t>(slots) & 3))
    return SEG_ATTN_ERR_INVALID_ARG;
  const int row_vecs = (int)(row_bytes / 16);
  const int64_t total = n_tokens * row_vecs;
  const int64_t want = (total + 255) / 256;
  const int blocks = (int)(want < 148 * 16 ? want : 148 * 16);
  segattn::kv_append_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), slots, n_tokens,
      row_vecs, static_cast<uint4*>(k_pool), static_cast<uint4*>(v_pool), num_slots);
  return cudaGetLastError() == cudaSuccess ? SEG_ATTN_OK : SEG_ATTN_ERR_CUDA;
}

extern "C" int seg_attn_kv_append_fp8(const void* k_new, const void* v_new, const int32_t* slots,
                                      int64_t n_tokens, int kv_heads, int head_dim,
                                      const float* k_scale, const float* v_scale, void* k_pool,
                                      void* v_pool, int64_t num_slots, void* stream) {
  if (n_tokens < 0 || kv_heads <= 0 || head_dim <= 0 || num_slots < 0)
    return SEG_ATTN_ERR_INVALID_ARG;
  if (head_dim % 16 != 0) return SEG_ATTN_ERR_UNSUPPORTED;
  if (n_tokens == 0) return SEG_ATTN_OK;
  auto aligned = [](const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  if (!aligned(k_new) || !aligned(v_new) || !aligned(k_pool) || !aligned(v_pool) || !slots ||
      (reinterpret_cast<uintptr_t>(slots) & 3) || !k_scale || !v_scale ||
      (reinterpret_cast<uintptr_t>(k_scale) & 3) || (reinterpret_cast<uintptr_t>(v_scale) & 3))
    return SEG_ATTN_ERR_INVALID_ARG;
  const int64_t row_vecs = (int64_t)kv_heads * head_dim / 16;  // 16 codes per vector
  if (row_vecs > INT32_MAX) return SEG_ATTN_ERR_UNSUPPORTED;
  const int64_t total = n_tokens * row_vecs;
  const int64_t want = (total + 255) / 256;
  const int blocks = (int)(want < 148 * 16 ? want : 148 * 16);
  segattn::kv_append_fp8_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), slots, n_tokens,
      (int)row_vecs, head_dim, k_scale, v_scale, static_cast<uint4*>(k_pool),
      static_cast<uint4*>(v_pool), num_slots);
  return cudaGetLastError() == cudaSuccess ? SEG_ATTN_OK : SEG_ATTN_ERR_CUDA;
}
