// Merge for shared prefixes (prefix caching, Flood README "Roadmap").
//
// With a shared-prefix table the attention of one output row (query, head) is
// computed in two disjoint parts: the group's prefix keys, by the prefill
// kernel over the group's packed queries, and the request's own keys, by the
// usual prefill or decode kernel.  Every part leaves a normalised partial
// output O_j and the log2 of its sum of exponentials lse_j; the full result is
//   O = sum_j 2^(lse_j - M) O_j / sum_j 2^(lse_j - M),  lse = M + log2 sum_j 2^(lse_j - M)
// with M = max_j lse_j -- the per-block partial + per-request reduction of the
// FlashAccel article ("data layout optimisation") applied across the two
// passes.  One warp per (row, head); each lane owns D/32 consecutive columns.
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "seg_attn_internal.h"

namespace segattn {
namespace {

struct CascadeParams {
  const int4* cascade;        // [n][2]: row, request, prefix item, row in group | suffix item, row in request
  const int4* citem;          // first slot, pieces, first query of the item
  const int32_t* req_chunks;  // decode: [B+1]
  const float* main_o;
  const float* main_lse;
  const float* group_o;
  const float* group_lse;
  __nv_bfloat16* out;
  float* lse;
  int q_heads, group, qpt, decode;
};

template <int D>
__global__ void __launch_bounds__(128) cascade_merge_kernel(const CascadeParams p) {
  constexpr int PER = D / 32;
  const int head = blockIdx.y * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (head >= p.q_heads) return;
  const int4 e0 = p.cascade[2 * blockIdx.x], e1 = p.cascade[2 * blockIdx.x + 1];
  const int row = e0.x, req = e0.y;
  const int g = head / p.group, hh = head % p.group;
  // packed row of query `local` (counted from the item's first query) in a prefill item
  auto item_row = [&](int local) {
    const int t = local / p.qpt;
    return t * kTileRows + (local - t * p.qpt) * p.group + hh;
  };
  int pre_slot = 0, pre_parts = 0, pre_row = 0;
  if (e0.z >= 0) {
    const int4 ci = p.citem[e0.z + g];
    pre_slot = ci.x;
    pre_parts = ci.y;
    pre_row = item_row(e0.w - ci.z);
  }
  int own_first = 0, own_parts = 0, own_row = 0;
  if (p.decode) {
    own_first = __ldg(p.req_chunks + req);
    own_parts = __ldg(p.req_chunks + req + 1) - own_first;
  } else {
    const int4 ci = p.citem[e1.x + g];
    own_first = ci.x;
    own_parts = ci.y;
    own_row = item_row(e1.y - ci.z);
  }
  const int n = pre_parts + own_parts;
  // partial j: prefix pieces first, then the request's own pieces or chunks
  auto index = [&](int j) -> int64_t {
    if (j < pre_parts) return (int64_t)(pre_slot + j) * kItemRows + pre_row;
    j -= pre_parts;
    if (p.decode) return (int64_t)(own_first + j) * p.q_heads + head;
    return (int64_t)(own_first + j) * kItemRows + own_row;
  };
  auto lse_of = [&](int j) { return j < pre_parts ? p.group_lse[index(j)] : p.main_lse[index(j)]; };
  auto o_of = [&](int j) { return (j < pre_parts ? p.group_o : p.main_o) + index(j) * D; };

  float M = -INFINITY;
  for (int j = lane; j < n; j += 32) M = fmaxf(M, lse_of(j));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  const float Mb = M == -INFINITY ? 0.f : M;
  float acc[PER], L = 0.f;
#pragma unroll
  for (int c = 0; c < PER; ++c) acc[c] = 0.f;
  for (int j = 0; j < n; ++j) {
    const float w = exp2f(lse_of(j) - Mb);
    L += w;
    const float* po = o_of(j) + lane * PER;
    // PER is 2 (d = 64) or 4 (d = 128): 8-byte pairs fit both, and a lane's
    // columns start 8-byte aligned in either case
#pragma unroll
    for (int c = 0; c < PER; c += 2) {
      const float2 x = *reinterpret_cast<const float2*>(po + c);
      acc[c] += w * x.x;
      acc[c + 1] += w * x.y;
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  __nv_bfloat16* orow = p.out + ((int64_t)row * p.q_heads + head) * D + lane * PER;
#pragma unroll
  for (int c = 0; c < PER; c += 2) {
    __nv_bfloat162 v = __floats2bfloat162_rn(acc[c] * inv, acc[c + 1] * inv);
    *reinterpret_cast<__nv_bfloat162*>(orow + c) = v;
  }
  if (p.lse && lane == 0)
    p.lse[(int64_t)row * p.q_heads + head] =
        L > 0.f ? (Mb + log2f(L)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace

int launch_cascade_merge(const CascadeLaunch& a, cudaStream_t stream) {
  const seg_attn_table_desc& d = *a.desc;
  if (d.num_cascade == 0) return SEG_ATTN_OK;
  const int32_t* t = static_cast<const int32_t*>(a.dev_table);
  CascadeParams p;
  p.cascade = reinterpret_cast<const int4*>(t + d.off_cascade);
  p.citem = reinterpret_cast<const int4*>(t + d.off_citem);
  p.req_chunks = t + d.off_req_chunks;
  p.main_o = a.main_o;
  p.main_lse = a.main_lse;
  p.group_o = a.group_o;
  p.group_lse = a.group_lse;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.lse = a.lse;
  p.q_heads = d.q_heads;
  p.group = d.q_heads / d.kv_heads;
  p.qpt = d.queries_per_tile;
  p.decode = d.mode == SEG_ATTN_MODE_DECODE;
  const dim3 grid(d.num_cascade, (d.q_heads + 3) / 4);
  if (d.head_dim == 128)
    cascade_merge_kernel<128><<<grid, 128, 0, stream>>>(p);
  else
    cascade_merge_kernel<64><<<grid, 128, 0, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? SEG_ATTN_OK : SEG_ATTN_ERR_CUDA;
}

}  // namespace segattn
