// Segment linear attention decode (simple GLA, one token per request) for sm_100a.
//
// Per request and head the step reads the fp32 state S (128 x 128, 64 KiB),
// applies S' = exp(g) S + k^T v, writes S' back and emits o = scale * S'^T q.
// That is 6 flops per 8 bytes of state traffic: the kernel streams the state
// through the SMs with 128-bit loads and stores and does the arithmetic on the
// FP32 pipe (the tensor cores would not help an HBM-bound update).
// Grid: (request, head, column half); 256 threads, each owning one 4-column
// group of 8 rows, so every warp reads and writes whole 256-byte row pieces.
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "seg_la_internal.h"

namespace segla {
namespace {

constexpr int kThreads = 256;
constexpr int kCols = kDim / 2;             // columns per CTA
constexpr int kGroups = kCols / 4;          // 4-column groups per CTA (16)
constexpr int kRowSets = kThreads / kGroups;  // threads sharing a column group (16)
constexpr int kRowsPerThread = kDim / kRowSets;  // 8

struct DecodeParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const float* g;
  __nv_bfloat16* out;
  float* pool;
  Table tab;
  float scale;
  int heads;
};

__device__ __forceinline__ float4 load_stream(const float* p) {
  float4 x;
  asm volatile("ld.global.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];\n"
               : "=f"(x.x), "=f"(x.y), "=f"(x.z), "=f"(x.w)
               : "l"(p));
  return x;
}

__global__ void __launch_bounds__(kThreads) la_decode_kernel(const DecodeParams p) {
  __shared__ float sq[kDim], sk[kDim];
  __shared__ float4 red[kRowSets][kGroups];
  const int r = blockIdx.x, h = blockIdx.y, half = blockIdx.z;
  const int tid = threadIdx.x;
  const int cg = tid % kGroups, rs = tid / kGroups;
  const int j0 = half * kCols + 4 * cg;
  const int tok = __ldg(p.tab.q_offsets + r);
  const int in = __ldg(p.tab.in_slot + r), out = __ldg(p.tab.out_slot + r);
  const int64_t qrow = ((int64_t)tok * p.heads + h) * kDim;

  // state rows of this thread first, so the loads are in flight while q, k, v arrive
  float4 s[kRowsPerThread];
  const float* src = in >= 0 ? p.pool + ((int64_t)in * p.heads + h) * kDim * kDim : nullptr;
#pragma unroll
  for (int m = 0; m < kRowsPerThread; ++m)
    s[m] = src ? load_stream(src + (int64_t)(rs + kRowSets * m) * kDim + j0)
               : make_float4(0.f, 0.f, 0.f, 0.f);
  if (tid < kDim) {
    sq[tid] = __bfloat162float(p.q[qrow + tid]);
    sk[tid] = __bfloat162float(p.k[qrow + tid]);
  }
  const uint2 vb = *reinterpret_cast<const uint2*>(p.v + qrow + j0);
  const float v0 = __uint_as_float(vb.x << 16), v1 = __uint_as_float(vb.x & 0xffff0000u);
  const float v2 = __uint_as_float(vb.y << 16), v3 = __uint_as_float(vb.y & 0xffff0000u);
  const float decay = expf(__ldg(p.g + (int64_t)tok * p.heads + h));
  __syncthreads();

  float* dst = out >= 0 ? p.pool + ((int64_t)out * p.heads + h) * kDim * kDim : nullptr;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int m = 0; m < kRowsPerThread; ++m) {
    const int i = rs + kRowSets * m;
    const float ki = sk[i], qi = sq[i];
    float4 x = s[m];
    x.x = fmaf(decay, x.x, ki * v0);
    x.y = fmaf(decay, x.y, ki * v1);
    x.z = fmaf(decay, x.z, ki * v2);
    x.w = fmaf(decay, x.w, ki * v3);
    acc.x = fmaf(qi, x.x, acc.x);
    acc.y = fmaf(qi, x.y, acc.y);
    acc.z = fmaf(qi, x.z, acc.z);
    acc.w = fmaf(qi, x.w, acc.w);
    if (dst) *reinterpret_cast<float4*>(dst + (int64_t)i * kDim + j0) = x;
  }
  red[rs][cg] = acc;
  __syncthreads();
  if (tid < kCols) {  // column j0' = half * 64 + tid: sum over the 16 row sets
    const int grp = tid / 4, lane4 = tid % 4;
    float sum = 0.f;
#pragma unroll
    for (int k2 = 0; k2 < kRowSets; ++k2) {
      const float4 a = red[k2][grp];
      sum += lane4 == 0 ? a.x : lane4 == 1 ? a.y : lane4 == 2 ? a.z : a.w;
    }
    p.out[qrow + half * kCols + tid] = __float2bfloat16_rn(p.scale * sum);
  }
}

}  // namespace

int launch_la_decode(const Launch& a, cudaStream_t stream) {
  const seg_la_table_desc& d = *a.desc;
  if (d.batch == 0) return SEG_ATTN_OK;
  DecodeParams p;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.k = static_cast<const __nv_bfloat16*>(a.k);
  p.v = static_cast<const __nv_bfloat16*>(a.v);
  p.g = a.g;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.pool = a.state_pool;
  p.tab = a.tab;
  p.scale = a.scale;
  p.heads = d.heads;
  la_decode_kernel<<<dim3(d.batch, d.heads, 2), kThreads, 0, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? SEG_ATTN_OK : SEG_ATTN_ERR_CUDA;
}

}  // namespace segla
