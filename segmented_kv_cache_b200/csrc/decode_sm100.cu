// Decode SegmentAttention for sm_100a: split-K over chunks of logical keys,
// then a log-sum-exp merge of the chunk partials.
//
// Decode (one query per request) reads every K/V byte once and does 8 flop
// per byte with 8 packed query heads, so it is HBM-bound; with scalar FMAs the
// 4096 flop per (key, kv head) would nearly saturate the FP32 pipe at full
// HBM rate.  The two small products therefore run on the tensor cores with
// the packed heads as the N = 8 side of mma.m16n8k16:
//   S^T[16 keys x 8 heads]   = K[16 keys x d] . Q^T[d x 8 heads]
//   O^T[d x 8 heads]        += V^T[d x 16 keys] . P^T[16 keys x 8 heads]
// K and V go straight from HBM into the mma operand registers with 128-bit
// loads (no shared-memory staging): the contraction index d is permuted so a
// thread's four K words of a k-step come from one 16-byte chunk, and the
// output row index of O^T is permuted so a thread's V words come from two
// 16-byte chunks per key.  P^T operands are made from the S^T accumulators
// with one movmatrix transpose per 8x8 block.  The online softmax (running
// max and normaliser per head; Ascend FlashAttention article, "bottleneck 2")
// is reduced across lanes with warp shuffles.  Chunks are the per-block
// partial attentions of the FlashAccel article ("data layout optimisation");
// the merge kernel reduces them per request.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>
#include <stdint.h>

#include "seg_attn_internal.h"

namespace segattn {
namespace {

constexpr int kDecodeWarps = 4;
constexpr int kDecodeThreads = kDecodeWarps * 32;
constexpr int kWarpKeys = 32;  // keys per warp iteration: two m16 blocks

__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_16816_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// two E4M3 codes (low byte = first element) -> f16x2 (low half = first element)
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
  uint32_t y;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(y) : "h"(static_cast<unsigned short>(two_codes)));
  return y;
}

__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t x) {
  __half2 h = __floats2half2_rn(__uint_as_float(x << 16), __uint_as_float(x & 0xffff0000u));
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t transpose8x8(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ uint4 load_stream(const __nv_bfloat16* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t word(const uint4& v, int w) {
  return w == 0 ? v.x : (w == 1 ? v.y : (w == 2 ? v.z : v.w));
}

struct SegCursor {
  const int32_t* kstart;
  const int32_t* start;
  int seg, seg_end;  // current segment, one past the request's last
  __device__ __forceinline__ void advance_to(int j) {
    while (seg + 1 < seg_end && __ldg(kstart + seg + 1) <= j) ++seg;
  }
  __device__ __forceinline__ int slot_of(int j) const {
    int s = seg;
    while (s + 1 < seg_end && __ldg(kstart + s + 1) <= j) ++s;
    return __ldg(start + s) + (j - __ldg(kstart + s));
  }
};

struct DecodeParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const uint8_t* k8;      // FP8 variant: E4M3 pools and per-kv-head scales
  const uint8_t* v8;
  const float* k_scale;
  const float* v_scale;
  __nv_bfloat16* out;
  float* lse;
  TableView tab;
  float* part_o;
  float* part_lse;
  float scale_log2;
  int q_heads, kv_heads, group;
  // query heads per CTA: hs = min(group, 8) packed heads (the mma's N = 8 side);
  // a group larger than 8 is covered by `slices` = group / 8 CTAs per (chunk, kv
  // head), adjacent in the grid so the siblings' K/V reads hit L2
  int hs, slices;
};

// Merge the four warps' (m, l, O) of this chunk through shared memory and write
// either the final bf16 output (single-chunk request) or the fp32 partial.
template <int D>
__device__ __forceinline__ void write_chunk_result(const DecodeParams& p, float (&sm_o)[kDecodeWarps][8][D],
                                                   float (&sm_m)[kDecodeWarps][8],
                                                   float (&sm_l)[kDecodeWarps][8], int req, int chunk,
                                                   int h0, int n_chunks, float out_scale) {
  constexpr int PER_THREAD = 8 * D / kDecodeThreads;  // outputs per thread
  const int hh = threadIdx.x / (D / PER_THREAD);
  const int d0 = (threadIdx.x % (D / PER_THREAD)) * PER_THREAD;
  if (hh >= p.hs) return;
  float mw[kDecodeWarps], M = -INFINITY;
#pragma unroll
  for (int w = 0; w < kDecodeWarps; ++w) {
    mw[w] = sm_m[w][hh];
    M = fmaxf(M, mw[w]);
  }
  const float Mb = M == -INFINITY ? 0.f : M;
  float L = 0.f, acc[PER_THREAD];
#pragma unroll
  for (int e = 0; e < PER_THREAD; ++e) acc[e] = 0.f;
#pragma unroll
  for (int w = 0; w < kDecodeWarps; ++w) {
    const float a = exp2f(mw[w] - Mb);
    L += a * sm_l[w][hh];
#pragma unroll
    for (int e = 0; e < PER_THREAD; ++e) acc[e] += a * sm_o[w][hh][d0 + e];
  }
  const float inv = L > 0.f ? out_scale / L : 0.f;
  const int head = h0 + hh;
  const float lse2 = L > 0.f ? Mb + log2f(L) : -INFINITY;
  if (n_chunks == 1) {
    const int tok = __ldg(p.tab.q_offsets + req);
    __nv_bfloat16* orow = p.out + ((int64_t)tok * p.q_heads + head) * D + d0;
#pragma unroll
    for (int e = 0; e < PER_THREAD; e += 4) {
      uint2 v;
      v.x = pack_bf16(acc[e] * inv, acc[e + 1] * inv);
      v.y = pack_bf16(acc[e + 2] * inv, acc[e + 3] * inv);
      *reinterpret_cast<uint2*>(orow + e) = v;
    }
    if (p.lse && d0 == 0) p.lse[(int64_t)tok * p.q_heads + head] = lse2 * 0.69314718055994531f;
  } else {
    float* prow = p.part_o + ((int64_t)chunk * p.q_heads + head) * D + d0;
#pragma unroll
    for (int e = 0; e < PER_THREAD; e += 4)
      *reinterpret_cast<float4*>(prow + e) =
          make_float4(acc[e] * inv, acc[e + 1] * inv, acc[e + 2] * inv, acc[e + 3] * inv);
    if (d0 == 0) p.part_lse[(int64_t)chunk * p.q_heads + head] = lse2;
  }
}

// One CTA per (chunk, kv head); four warps take interleaved 32-key blocks.
template <int D>
__global__ void __launch_bounds__(kDecodeThreads, 2) decode_chunk_kernel(const DecodeParams p) {
  constexpr int KSTEPS = D / 16;  // k-steps of the QK product, m-tiles of the PV product
  constexpr int KCH = D / 32;     // 16-byte K chunks per row per thread
  constexpr int VCH = D / 64;     // 16-byte V chunks per key per thread
  __shared__ float sm_o[kDecodeWarps][8][D];
  __shared__ float sm_m[kDecodeWarps][8];
  __shared__ float sm_l[kDecodeWarps][8];

  const int chunk = blockIdx.x / p.slices;
  const int4 item = p.tab.work[chunk];
  const int req = item.x, k_begin = item.y, k_end = item.z, n_chunks = item.w;
  const int g = blockIdx.y;
  const int h0 = g * p.group + (blockIdx.x - chunk * p.slices) * 8;  // first query head here
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = lane >> 2, qd = lane & 3;
  const int64_t kv_stride = (int64_t)p.kv_heads * D;  // elements between consecutive slots

  // Q^T operand fragments of the packed heads (head h0 + r; zero pad past hs).
  uint32_t qf[KSTEPS][2];
  {
    const int tok = __ldg(p.tab.q_offsets + req);
    const __nv_bfloat16* qrow = p.q + ((int64_t)tok * p.q_heads + h0 + r) * D;
#pragma unroll
    for (int t = 0; t < KCH; ++t) {
      uint4 w = make_uint4(0, 0, 0, 0);
      if (r < p.hs) w = *reinterpret_cast<const uint4*>(qrow + 8 * (qd + 4 * t));
      qf[2 * t][0] = w.x;
      qf[2 * t][1] = w.y;
      qf[2 * t + 1][0] = w.z;
      qf[2 * t + 1][1] = w.w;
    }
  }

  float o[KSTEPS][4];
#pragma unroll
  for (int i = 0; i < KSTEPS; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  SegCursor cur;
  cur.kstart = p.tab.seg_kstart;
  cur.start = p.tab.seg_start;
  cur.seg = __ldg(p.tab.seg_offsets + req);
  cur.seg_end = __ldg(p.tab.seg_offsets + req + 1);

  const __nv_bfloat16* kbase = p.k + (int64_t)g * D;
  const __nv_bfloat16* vbase = p.v + (int64_t)g * D;

  for (int jb = k_begin + warp * kWarpKeys; jb < k_end; jb += kDecodeWarps * kWarpKeys) {
    cur.advance_to(jb);
    const int seg_lo = __ldg(cur.kstart + cur.seg);
    const int seg_hi = seg_lo + __ldg(p.tab.seg_len + cur.seg);
    const bool fast = jb + kWarpKeys <= seg_hi;
    const int base_slot = __ldg(cur.start + cur.seg) - seg_lo;
    auto slot = [&](int j) { return fast ? base_slot + j : cur.slot_of(j); };

    // ---- issue all loads of this 32-key block
    uint4 kw[2][2][KCH];  // [block][row r / r+8][chunk]
    uint4 vw[2][4][VCH];  // [block][key 2q,2q+1,2q+8,2q+9][chunk]
#pragma unroll
    for (int b = 0; b < 2; ++b) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int j = jb + 16 * b + r + 8 * h;
        if (j < k_end) {
          const __nv_bfloat16* row = kbase + (int64_t)slot(j) * kv_stride;
#pragma unroll
          for (int t = 0; t < KCH; ++t) kw[b][h][t] = load_stream(row + 8 * (qd + 4 * t));
        } else {
#pragma unroll
          for (int t = 0; t < KCH; ++t) kw[b][h][t] = make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = jb + 16 * b + 2 * qd + (e & 1) + 8 * (e >> 1);
        if (j < k_end) {
          const __nv_bfloat16* row = vbase + (int64_t)slot(j) * kv_stride;
#pragma unroll
          for (int c = 0; c < VCH; ++c) vw[b][e][c] = load_stream(row + 64 * c + 8 * r);
        } else {
#pragma unroll
          for (int c = 0; c < VCH; ++c) vw[b][e][c] = make_uint4(0, 0, 0, 0);
        }
      }
    }

    // ---- S^T = K Q^T for both 16-key blocks
    float s[2][4];
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      s[b][0] = s[b][1] = s[b][2] = s[b][3] = 0.f;
#pragma unroll
      for (int t = 0; t < KCH; ++t) {
        mma_16816(s[b], kw[b][0][t].x, kw[b][1][t].x, kw[b][0][t].y, kw[b][1][t].y, qf[2 * t][0],
                  qf[2 * t][1]);
        mma_16816(s[b], kw[b][0][t].z, kw[b][1][t].z, kw[b][0][t].w, kw[b][1][t].w,
                  qf[2 * t + 1][0], qf[2 * t + 1][1]);
      }
    }
    // ---- scale, mask, block max per head (heads 2qd, 2qd+1 of this thread)
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int b = 0; b < 2; ++b) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const bool ok = jb + 16 * b + r + 8 * h < k_end;
        s[b][2 * h] = ok ? s[b][2 * h] * p.scale_log2 : -INFINITY;
        s[b][2 * h + 1] = ok ? s[b][2 * h + 1] * p.scale_log2 : -INFINITY;
        mx0 = fmaxf(mx0, s[b][2 * h]);
        mx1 = fmaxf(mx1, s[b][2 * h + 1]);
      }
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float base0 = mn0 == -INFINITY ? 0.f : mn0;
    const float base1 = mn1 == -INFINITY ? 0.f : mn1;
    const float a0 = exp2f(m0 - base0), a1 = exp2f(m1 - base1);
    m0 = mn0;
    m1 = mn1;
    l0 *= a0;
    l1 *= a1;
#pragma unroll
    for (int i = 0; i < KSTEPS; ++i) {
      o[i][0] *= a0;
      o[i][2] *= a0;
      o[i][1] *= a1;
      o[i][3] *= a1;
    }
    // ---- P, then O^T += V^T P^T
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      const float p00 = exp2f(s[b][0] - base0), p01 = exp2f(s[b][1] - base1);
      const float p10 = exp2f(s[b][2] - base0), p11 = exp2f(s[b][3] - base1);
      l0 += p00 + p10;
      l1 += p01 + p11;
      const uint32_t pb0 = transpose8x8(pack_bf16(p00, p01));  // keys 0-7
      const uint32_t pb1 = transpose8x8(pack_bf16(p10, p11));  // keys 8-15
#pragma unroll
      for (int i = 0; i < KSTEPS; ++i) {
        const int c = i >> 2, w = i & 3;
        const uint32_t x0 = word(vw[b][0][c], w), x1 = word(vw[b][1][c], w);
        const uint32_t x2 = word(vw[b][2][c], w), x3 = word(vw[b][3][c], w);
        mma_16816(o[i], __byte_perm(x0, x1, 0x5410), __byte_perm(x0, x1, 0x7632),
                  __byte_perm(x2, x3, 0x5410), __byte_perm(x2, x3, 0x7632), pb0, pb1);
      }
    }
  }

  // ---- warp totals, then merge the four warps through shared memory
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }
  if (r == 0) {
    sm_m[warp][2 * qd] = m0;
    sm_m[warp][2 * qd + 1] = m1;
    sm_l[warp][2 * qd] = l0;
    sm_l[warp][2 * qd + 1] = l1;
  }
#pragma unroll
  for (int i = 0; i < KSTEPS; ++i) {
    const int d0 = 64 * (i >> 2) + 8 * r + 2 * (i & 3);  // O^T rows r and r+8 of m-tile i
    sm_o[warp][2 * qd][d0] = o[i][0];
    sm_o[warp][2 * qd + 1][d0] = o[i][1];
    sm_o[warp][2 * qd][d0 + 1] = o[i][2];
    sm_o[warp][2 * qd + 1][d0 + 1] = o[i][3];
  }
  __syncthreads();

  write_chunk_result<D>(p, sm_o, sm_m, sm_l, req, chunk, h0, n_chunks, 1.f);
}

// FP8 (E4M3) KV cache: same split-K structure, half the bytes.  The E4M3
// codes go from HBM into registers with 16-byte loads and are widened in
// pairs to f16 mma operands (cvt.rn.f16x2.e4m3x2); queries and P are f16.
// The K scale of the kv head is folded into the softmax scale and the V scale
// is applied to the output, so the MMAs see the raw code values.
// K fragment layout: a thread's 16-byte chunk of a K row holds four k-steps
// (4 values each: the (2q, 2q+1) and (2q+8, 2q+9) slots); its V chunk holds
// D/8 consecutive values of one key, O^T row of m-tile i = (D/8)*r + 2i (+1).
constexpr int kWarpKeys8 = 32;  // keys per warp iteration (3 CTAs per SM fit in registers)

template <int D>
__global__ void __launch_bounds__(kDecodeThreads, 3) decode_chunk_fp8_kernel(const DecodeParams p) {
  constexpr int KSTEPS = D / 16;  // k-steps of QK, m-tiles of PV
  constexpr int KCH = D / 64;     // 16-byte K chunks per row per thread
  constexpr int VB = D / 8;       // V bytes per key per thread
  constexpr int NB = kWarpKeys8 / 16;
  __shared__ float sm_o[kDecodeWarps][8][D];
  __shared__ float sm_m[kDecodeWarps][8];
  __shared__ float sm_l[kDecodeWarps][8];

  const int chunk = blockIdx.x / p.slices;
  const int4 item = p.tab.work[chunk];
  const int req = item.x, k_begin = item.y, k_end = item.z, n_chunks = item.w;
  const int g = blockIdx.y;
  const int h0 = g * p.group + (blockIdx.x - chunk * p.slices) * 8;  // first query head here
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = lane >> 2, qd = lane & 3;
  const int64_t kv_stride = (int64_t)p.kv_heads * D;  // bytes between consecutive slots
  const float sl2 = p.scale_log2 * __ldg(p.k_scale + g);
  const float v_scale = __ldg(p.v_scale + g);

  uint32_t qf[KSTEPS][2];  // f16 Q^T fragments of head h0 + r (zero past hs)
  {
    const int tok = __ldg(p.tab.q_offsets + req);
    const __nv_bfloat16* qrow = p.q + ((int64_t)tok * p.q_heads + h0 + r) * D;
#pragma unroll
    for (int t = 0; t < KCH; ++t) {
      uint4 w0 = make_uint4(0, 0, 0, 0), w1 = make_uint4(0, 0, 0, 0);
      if (r < p.hs) {
        w0 = *reinterpret_cast<const uint4*>(qrow + 16 * (qd + 4 * t));
        w1 = *reinterpret_cast<const uint4*>(qrow + 16 * (qd + 4 * t) + 8);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint4& w = u < 2 ? w0 : w1;
        qf[4 * t + u][0] = bf16x2_to_f16x2(word(w, (2 * u) % 4));
        qf[4 * t + u][1] = bf16x2_to_f16x2(word(w, (2 * u + 1) % 4));
      }
    }
  }

  float o[KSTEPS][4];
#pragma unroll
  for (int i = 0; i < KSTEPS; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  SegCursor cur;
  cur.kstart = p.tab.seg_kstart;
  cur.start = p.tab.seg_start;
  cur.seg = __ldg(p.tab.seg_offsets + req);
  cur.seg_end = __ldg(p.tab.seg_offsets + req + 1);
  const uint8_t* kbase = p.k8 + (int64_t)g * D;
  const uint8_t* vbase = p.v8 + (int64_t)g * D;

  for (int jb = k_begin + warp * kWarpKeys8; jb < k_end; jb += kDecodeWarps * kWarpKeys8) {
    cur.advance_to(jb);
    const int seg_lo = __ldg(cur.kstart + cur.seg);
    const int seg_hi = seg_lo + __ldg(p.tab.seg_len + cur.seg);
    const bool fast = jb + kWarpKeys8 <= seg_hi;
    const int base_slot = __ldg(cur.start + cur.seg) - seg_lo;
    auto slot = [&](int j) { return fast ? base_slot + j : cur.slot_of(j); };

    uint4 kw[NB][2][KCH];  // [block][row r / r+8][chunk]
    uint4 vw[NB][4];       // [block][key 2q, 2q+1, 2q+8, 2q+9]
#pragma unroll
    for (int b = 0; b < NB; ++b) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int j = jb + 16 * b + r + 8 * h;
        if (j < k_end) {
          const uint8_t* row = kbase + (int64_t)slot(j) * kv_stride;
#pragma unroll
          for (int t = 0; t < KCH; ++t)
            kw[b][h][t] = *reinterpret_cast<const uint4*>(row + 16 * (qd + 4 * t));
        } else {
#pragma unroll
          for (int t = 0; t < KCH; ++t) kw[b][h][t] = make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = jb + 16 * b + 2 * qd + (e & 1) + 8 * (e >> 1);
        vw[b][e] = make_uint4(0, 0, 0, 0);
        if (j < k_end) {
          const uint8_t* row = vbase + (int64_t)slot(j) * kv_stride + VB * r;
          if constexpr (VB == 16) {
            vw[b][e] = *reinterpret_cast<const uint4*>(row);
          } else {
            const uint2 x = *reinterpret_cast<const uint2*>(row);
            vw[b][e].x = x.x;
            vw[b][e].y = x.y;
          }
        }
      }
    }

    float s[NB][4];
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      s[b][0] = s[b][1] = s[b][2] = s[b][3] = 0.f;
#pragma unroll
      for (int t = 0; t < KCH; ++t)
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t x0 = word(kw[b][0][t], u), x1 = word(kw[b][1][t], u);
          mma_16816_f16(s[b], e4m3x2_to_f16x2(x0), e4m3x2_to_f16x2(x1),
                        e4m3x2_to_f16x2(x0 >> 16), e4m3x2_to_f16x2(x1 >> 16), qf[4 * t + u][0],
                        qf[4 * t + u][1]);
        }
    }
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const bool ok = jb + 16 * b + r + 8 * h < k_end;
        s[b][2 * h] = ok ? s[b][2 * h] * sl2 : -INFINITY;
        s[b][2 * h + 1] = ok ? s[b][2 * h + 1] * sl2 : -INFINITY;
        mx0 = fmaxf(mx0, s[b][2 * h]);
        mx1 = fmaxf(mx1, s[b][2 * h + 1]);
      }
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float base0 = mn0 == -INFINITY ? 0.f : mn0;
    const float base1 = mn1 == -INFINITY ? 0.f : mn1;
    const float a0 = exp2f(m0 - base0), a1 = exp2f(m1 - base1);
    m0 = mn0;
    m1 = mn1;
    l0 *= a0;
    l1 *= a1;
#pragma unroll
    for (int i = 0; i < KSTEPS; ++i) {
      o[i][0] *= a0;
      o[i][2] *= a0;
      o[i][1] *= a1;
      o[i][3] *= a1;
    }
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const float p00 = exp2f(s[b][0] - base0), p01 = exp2f(s[b][1] - base1);
      const float p10 = exp2f(s[b][2] - base0), p11 = exp2f(s[b][3] - base1);
      l0 += p00 + p10;
      l1 += p01 + p11;
      const uint32_t pb0 = transpose8x8(pack_f16(p00, p01));  // keys 0-7
      const uint32_t pb1 = transpose8x8(pack_f16(p10, p11));  // keys 8-15
#pragma unroll
      for (int w = 0; w < VB / 4; ++w) {
        const uint32_t x0 = word(vw[b][0], w), x1 = word(vw[b][1], w);
        const uint32_t x2 = word(vw[b][2], w), x3 = word(vw[b][3], w);
        const uint32_t lo01 = __byte_perm(x0, x1, 0x5140), hi01 = __byte_perm(x0, x1, 0x7362);
        const uint32_t lo23 = __byte_perm(x2, x3, 0x5140), hi23 = __byte_perm(x2, x3, 0x7362);
        mma_16816_f16(o[2 * w], e4m3x2_to_f16x2(lo01), e4m3x2_to_f16x2(lo01 >> 16),
                      e4m3x2_to_f16x2(lo23), e4m3x2_to_f16x2(lo23 >> 16), pb0, pb1);
        mma_16816_f16(o[2 * w + 1], e4m3x2_to_f16x2(hi01), e4m3x2_to_f16x2(hi01 >> 16),
                      e4m3x2_to_f16x2(hi23), e4m3x2_to_f16x2(hi23 >> 16), pb0, pb1);
      }
    }
  }

#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }
  if (r == 0) {
    sm_m[warp][2 * qd] = m0;
    sm_m[warp][2 * qd + 1] = m1;
    sm_l[warp][2 * qd] = l0;
    sm_l[warp][2 * qd + 1] = l1;
  }
#pragma unroll
  for (int i = 0; i < KSTEPS; ++i) {
    const int d0 = VB * r + 2 * i;  // O^T rows r and r+8 of m-tile i
    sm_o[warp][2 * qd][d0] = o[i][0];
    sm_o[warp][2 * qd + 1][d0] = o[i][1];
    sm_o[warp][2 * qd][d0 + 1] = o[i][2];
    sm_o[warp][2 * qd + 1][d0 + 1] = o[i][3];
  }
  __syncthreads();
  write_chunk_result<D>(p, sm_o, sm_m, sm_l, req, chunk, h0, n_chunks, v_scale);
}

// Merge the chunk partials of each multi-chunk request (one warp per head).
template <int D>
__global__ void __launch_bounds__(128) decode_merge_kernel(const DecodeParams p) {
  const int req = blockIdx.x;
  const int head = blockIdx.y * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int c0 = __ldg(p.tab.req_chunks + req), c1 = __ldg(p.tab.req_chunks + req + 1);
  if (c1 - c0 <= 1 || head >= p.q_heads) return;
  float M = -INFINITY;
  for (int c = c0 + lane; c < c1; c += 32) M = fmaxf(M, p.part_lse[(int64_t)c * p.q_heads + head]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  const float Mb = M == -INFINITY ? 0.f : M;
  constexpr int PER = D / 32;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  float L = 0.f;
  for (int c = c0; c < c1; ++c) {
    const float w = exp2f(p.part_lse[(int64_t)c * p.q_heads + head] - Mb);
    L += w;
    const float* prow = p.part_o + ((int64_t)c * p.q_heads + head) * D + lane * PER;
#pragma unroll
    for (int e = 0; e < PER; e += 2) {
      const float2 x = *reinterpret_cast<const float2*>(prow + e);
      acc[e] += w * x.x;
      acc[e + 1] += w * x.y;
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  const int tok = __ldg(p.tab.q_offsets + req);
  __nv_bfloat16* orow = p.out + ((int64_t)tok * p.q_heads + head) * D + lane * PER;
#pragma unroll
  for (int e = 0; e < PER; e += 2)
    *reinterpret_cast<uint32_t*>(orow + e) = pack_bf16(acc[e] * inv, acc[e + 1] * inv);
  if (p.lse && lane == 0)
    p.lse[(int64_t)tok * p.q_heads + head] =
        L > 0.f ? (Mb + log2f(L)) * 0.69314718055994531f : -INFINITY;
}

template <int D>
int launch_decode_d(const DecodeLaunch& a, cudaStream_t stream) {
  const seg_attn_table_desc& d = *a.desc;
  DecodeParams p;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.k = static_cast<const __nv_bfloat16*>(a.k_pool);
  p.v = static_cast<const __nv_bfloat16*>(a.v_pool);
  p.k8 = static_cast<const uint8_t*>(a.k_pool);
  p.v8 = static_cast<const uint8_t*>(a.v_pool);
  p.k_scale = a.k_scale;
  p.v_scale = a.v_scale;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.lse = a.lse;
  p.tab = a.tab;
  p.part_o = a.part_o;
  p.part_lse = a.part_lse;
  p.scale_log2 = (float)((double)a.scale * 1.4426950408889634);
  p.q_heads = d.q_heads;
  p.kv_heads = d.kv_heads;
  p.group = d.q_heads / d.kv_heads;
  p.hs = p.group < 8 ? p.group : 8;
  p.slices = p.group / p.hs;
  const dim3 grid(d.num_work * p.slices, d.kv_heads);
  if (a.fp8)
    decode_chunk_fp8_kernel<D><<<grid, kDecodeThreads, 0, stream>>>(p);
  else
    decode_chunk_kernel<D><<<grid, kDecodeThreads, 0, stream>>>(p);
  if (cudaGetLastError() != cudaSuccess) return SEG_ATTN_ERR_CUDA;
  // a shared-prefix table leaves every merge to the cascade merge
  if (d.workspace_bytes > 0 && !d.shared) {
    decode_merge_kernel<D><<<dim3(d.batch, (d.q_heads + 3) / 4), 128, 0, stream>>>(p);
    if (cudaGetLastError() != cudaSuccess) return SEG_ATTN_ERR_CUDA;
  }
  return SEG_ATTN_OK;
}

}  // namespace

int launch_decode(const DecodeLaunch& a, cudaStream_t stream) {
  if (a.desc->num_work == 0) return SEG_ATTN_OK;
  return a.desc->head_dim == 128 ? launch_decode_d<128>(a, stream) : launch_decode_d<64>(a, stream);
}

}  // namespace segattn
