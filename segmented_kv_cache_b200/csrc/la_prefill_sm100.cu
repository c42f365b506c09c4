// Segment linear attention prefill (simple GLA, chunked form) for sm_100a.
//
// A request's tokens are cut into chunks of 128.  With G_t the running sum of
// the log-decays g inside a chunk, the recurrence S <- exp(g_t) S + k_t^T v_t
// over a chunk is equivalent to
//   S_next = exp(G_last) S + U,   U = (K * exp(G_last - G))^T V,
//   out    = scale * ((Q K^T . D) V + exp(G_t) Q S),  D[t][s] = exp(G_t - G_s), s <= t
// (the chunked form of gated linear attention).  Three kernels:
//   la_chunk_state_kernel  per (chunk, head): U with one 128x128x128 tcgen05 MMA
//                          (A = the scaled K tile used transposed, B = V);
//   la_scan_kernel         per (request, head): the state entering each chunk,
//                          stored as a bf16 tile, and the final state;
//   la_chunk_out_kernel    per (chunk, head): Q K^T, Q S_c and P V on the tensor
//                          cores (P = Q K^T . D, written to tensor memory as bf16
//                          by the math warps), combined in the epilogue.  P V runs
//                          before the entering state is known, and Q S_c then goes
//                          into the columns of S and P, which P V has read: 256
//                          tensor-memory columns and 97 KB of shared memory (S_c
//                          lands where K was), so two CTAs share an SM.
// Tiles come in with TMA (128 tokens x 64 columns per box, 128-byte swizzle),
// accumulators live in tensor memory.  Warp roles: warp 0 lane 0 issues the
// copies and the MMAs, warp 1 owns the tensor memory (and in the output pass
// loads the entering state once the scan has finished), warps 2-5 (one TMEM lane
// quadrant each) do the per-row arithmetic.  Every mbarrier wait gives up after
// one second and flags a device error instead of hanging.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "ptx_sm100.cuh"
#include "seg_la_internal.h"

namespace segla {

__device__ int g_la_error;  // non-zero once a bounded wait gave up

namespace {

using namespace segattn::ptx;

constexpr int kThreads = 192;
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr uint32_t kHalf = 128 * 128;  // one 128-row x 64-column bf16 box (16 KiB)
constexpr uint32_t kTile = 2 * kHalf;  // 128 x 128 bf16 tile
constexpr float kLog2e = 1.4426950408889634f;

struct Params {
  __nv_bfloat16* out;
  const float* g;
  float* pool;
  Table tab;
  float* u;             // [units][d][d] fp32
  __nv_bfloat16* s_in;  // [units][d][d] bf16
  float* gamma;         // [units]
  float scale;
  int heads;
};

// Running sum G of the chunk's log-decays (row t = this math thread), in the log2
// domain, shared through `g2` [128]; rows past the chunk's end add nothing.
// Runs on the 128 math threads only (named barrier 1).
__device__ __forceinline__ float chunk_log2_decay(const Params& p, int row0, int len, int h,
                                                  int t, float* g2, float* warp_sum) {
  const int lane = t & 31, w = t >> 5;
  float x = t < len ? __ldg(p.g + (int64_t)(row0 + t) * p.heads + h) * kLog2e : 0.f;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) warp_sum[w] = x;
  named_barrier(1, 128);
  for (int k = 0; k < w; ++k) x += warp_sum[k];
  g2[t] = x;
  named_barrier(1, 128);
  return x;
}

template <int NCOLS>
__device__ __forceinline__ void math_row_index(int warp, int lane, int& t, uint32_t& lane_base,
                                               uint32_t tmem) {
  const int quad = warp & 3;
  t = quad * 32 + lane;
  lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
}

// ---------------------------------------------------------------- pass 1
__global__ void __launch_bounds__(kThreads) la_chunk_state_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint8_t* sK = sm;
  uint8_t* sV = sm + kTile;
  __shared__ uint64_t kv_full, k_ready, mma_done;
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;
  __shared__ float g2[kChunk], warp_sum[4];

  grid_launch_dependents();  // the scan may launch now; it waits for this grid's results
  const int c = blockIdx.x, h = blockIdx.y;
  const int4 ch = p.tab.chunks[c];
  const int row0 = ch.y, len = ch.z;
  const int unit = c * p.heads + h;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&kv_full, 1);
    mbar_init(&k_ready, 128);
    mbar_init(&mma_done, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&tmem_slot, 128);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      mbar_expect_tx(&kv_full, 2 * kTile);
      for (int hh = 0; hh < 2; ++hh) {
        tma_load_3d(sK + hh * kHalf, &tm_k, &kv_full, 64 * hh, h, row0);
        tma_load_3d(sV + hh * kHalf, &tm_v, &kv_full, 64 * hh, h, row0);
      }
      // U = (K')^T V: A = K' read transposed (MN-major), B = V (MN-major)
      bool ok = mbar_wait(&kv_full, 0, &abort_flag, kWaitNs) &&
                mbar_wait(&k_ready, 0, &abort_flag, kWaitNs);
      if (ok) {
        tc_fence_after();
        constexpr uint32_t idesc = idesc_bf16_f32_ab(128, 128, true, true);
        const uint32_t ka = smem_u32(sK), va = smem_u32(sV);
#pragma unroll
        for (int k = 0; k < kChunk / 16; ++k)
          mma_ss(tmem, sdesc_sw128(ka + k * 2048, kHalf, 1024),
                 sdesc_sw128(va + k * 2048, kHalf, 1024), idesc, k > 0 ? 1u : 0u);
      }
      mma_commit(&mma_done);
      mbar_wait(&mma_done, 0, nullptr, kWaitNs);
      if (!ok) mbar_wait(&kv_full, 0, nullptr, kWaitNs);  // no copy left in flight
    }
    __syncwarp();
  } else if (warp >= 2) {
    int t;
    uint32_t lane_base;
    math_row_index<128>(warp, lane, t, lane_base, tmem);
    const float gt = chunk_log2_decay(p, row0, len, h, t, g2, warp_sum);
    const float glast = g2[len - 1];
    const float w = t < len ? ex2(glast - gt) : 0.f;
    if (t == 0) p.gamma[unit] = ex2(glast);
    // K row t *= exp(G_last - G_t): the row's 16-byte pieces are permuted by the
    // swizzle but stay inside the row, so scaling in place is layout-blind.  Thread
    // t starts at piece t & 7, so the 8 rows of one shared-memory phase use 8
    // different banks.
    bool ok = mbar_wait(&kv_full, 0, &abort_flag, kWaitNs);
    if (ok) {
      for (int hh = 0; hh < 2; ++hh) {
        uint4* row = reinterpret_cast<uint4*>(sK + hh * kHalf + t * 128);
#pragma unroll
        for (int e0 = 0; e0 < 8; ++e0) {
          const int e = e0 ^ (t & 7);
          uint4 x = row[e];
          uint32_t* wd = reinterpret_cast<uint32_t*>(&x);
#pragma unroll
          for (int u2 = 0; u2 < 4; ++u2) {
            __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&wd[u2]);
            float2 f = __bfloat1622float2(b);
            b = __floats2bfloat162_rn(f.x * w, f.y * w);
            wd[u2] = *reinterpret_cast<uint32_t*>(&b);
          }
          row[e] = x;
        }
      }
      fence_proxy_async_smem();
    }
    mbar_arrive(&k_ready);
    ok = ok && mbar_wait(&mma_done, 0, &abort_flag, kWaitNs);
    if (ok) {
      tc_fence_after();
      // Row t of U (key index i = t) is 128 fp32 columns = 32 pieces of 16 bytes.
      // The K and V tiles are idle once the MMA is done: row t goes there at
      // 512 * t, piece c at position (c & ~7) | ((c ^ t) & 7), and then each warp
      // writes its own 32 rows out, one whole 512-byte row per store instruction.
      uint4* stage = reinterpret_cast<uint4*>(sm);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t a[2][32];
        tmem_ld64(lane_base + 64 * half, a);
        tmem_wait_ld(a[0]);
        tmem_wait_ld(a[1]);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int c = 16 * half + j;
          const uint32_t* w4 = &a[j >> 3][4 * (j & 7)];
          stage[32 * t + ((c & ~7) | ((c ^ t) & 7))] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
      }
      __syncwarp();
      const int r0 = t - lane;
      uint4* dst = reinterpret_cast<uint4*>(p.u + ((int64_t)unit * kDim + r0) * kDim);
#pragma unroll 4
      for (int r = 0; r < 32; ++r)
        dst[32 * r + lane] = stage[32 * (r0 + r) + ((lane & ~7) | ((lane ^ (r0 + r)) & 7))];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
  if (threadIdx.x == 0 && abort_flag) atomicOr(&g_la_error, 1);
}

// ---------------------------------------------------------------- pass 2
// One CTA per (request, head, 1024-element slice of the state); each thread
// carries 4 consecutive elements through the request's chunks in fp32.
__global__ void __launch_bounds__(256) la_scan_kernel(const Params p) {
  // the output pass may launch now (it waits for this grid before it reads the
  // entering states); this pass needs every U of the state pass
  grid_launch_dependents();
  grid_dependency_wait();
  const int r = blockIdx.x / p.heads, h = blockIdx.x % p.heads;
  const int e = (blockIdx.y * 256 + threadIdx.x) * 4;
  const int in = __ldg(p.tab.in_slot + r), out = __ldg(p.tab.out_slot + r);
  const int c0 = __ldg(p.tab.req_chunks + r), c1 = __ldg(p.tab.req_chunks + r + 1);
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
  if (in >= 0) s = *reinterpret_cast<const float4*>(p.pool + ((int64_t)in * p.heads + h) * kDim * kDim + e);
  for (int c = c0; c < c1; ++c) {
    const int64_t unit = (int64_t)c * p.heads + h;
    const float4 u = *reinterpret_cast<const float4*>(p.u + unit * kDim * kDim + e);
    const float gm = p.gamma[unit];
    __nv_bfloat162 lo = __floats2bfloat162_rn(s.x, s.y), hi = __floats2bfloat162_rn(s.z, s.w);
    uint2 packed;
    packed.x = *reinterpret_cast<uint32_t*>(&lo);
    packed.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(p.s_in + unit * kDim * kDim + e) = packed;
    s.x = fmaf(gm, s.x, u.x);
    s.y = fmaf(gm, s.y, u.y);
    s.z = fmaf(gm, s.z, u.z);
    s.w = fmaf(gm, s.w, u.w);
  }
  if (out >= 0) *reinterpret_cast<float4*>(p.pool + ((int64_t)out * p.heads + h) * kDim * kDim + e) = s;
}

// ---------------------------------------------------------------- pass 3
__global__ void __launch_bounds__(kThreads, 2) la_chunk_out_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_s,
    const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = sm;
  uint8_t* sK = sm + kTile;
  uint8_t* sV = sm + 2 * kTile;
  uint8_t* sS = sK;  // the entering state, loaded once Q K^T has read K
  __shared__ uint64_t qk_full, s_full, v_full, qk_done, p_full, mma_done;
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;
  __shared__ float g2[kChunk], warp_sum[4];

  const int c = blockIdx.x, h = blockIdx.y;
  const int4 ch = p.tab.chunks[c];
  const int row0 = ch.y, len = ch.z;
  const int unit = c * p.heads + h;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&qk_full, 1);
    mbar_init(&s_full, 1);
    mbar_init(&v_full, 1);
    mbar_init(&qk_done, 1);
    mbar_init(&p_full, 128);
    mbar_init(&mma_done, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&tmem_slot, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  // tensor memory: S = Q K^T, then P over it, then Q S_c [0,128); P V [128,256)
  const uint32_t tS = tmem, tI = tmem, tO = tmem + 128;

  if (warp == 0) {
    if (lane == 0) {
      mbar_expect_tx(&qk_full, 2 * kTile);
      mbar_expect_tx(&v_full, kTile);
      for (int hh = 0; hh < 2; ++hh) {
        tma_load_3d(sQ + hh * kHalf, &tm_q, &qk_full, 64 * hh, h, row0);
        tma_load_3d(sK + hh * kHalf, &tm_k, &qk_full, 64 * hh, h, row0);
      }
      for (int hh = 0; hh < 2; ++hh) tma_load_3d(sV + hh * kHalf, &tm_v, &v_full, 64 * hh, h, row0);
      const uint32_t qa = smem_u32(sQ), ka = smem_u32(sK), va = smem_u32(sV), sa = smem_u32(sS);
      constexpr uint32_t id_qk = idesc_bf16_f32(128, 128, false);  // B = K, K-major
      constexpr uint32_t id_mn = idesc_bf16_f32(128, kDim, true);  // B MN-major (S_c, V)
      bool ok = mbar_wait(&qk_full, 0, &abort_flag, kWaitNs);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < kDim / 16; ++k) {
          const uint32_t off = (k >> 2) * kHalf + (k & 3) * 32;
          mma_ss(tS, sdesc_sw128(qa + off, 16, 1024), sdesc_sw128(ka + off, 16, 1024), id_qk,
                 k > 0 ? 1u : 0u);
        }
        mma_commit(&qk_done);
      }
      // P V needs nothing from the scan; Q S_c follows once the entering state has
      // landed (warp 1 loads it), into the columns of S and P: tensor-core operations
      // of one CTA run in issue order, so P V has read P by then
      ok = ok && mbar_wait(&v_full, 0, &abort_flag, kWaitNs) &&
           mbar_wait(&p_full, 0, &abort_flag, kWaitNs);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < kChunk / 16; ++k)
          mma_ts(tO, tS + 8 * k, sdesc_sw128(va + k * 2048, kHalf, 1024), id_mn, k > 0 ? 1u : 0u);
      }
      ok = ok && mbar_wait(&s_full, 0, &abort_flag, kWaitNs);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < kDim / 16; ++k) {
          const uint32_t aoff = (k >> 2) * kHalf + (k & 3) * 32;
          mma_ss(tI, sdesc_sw128(qa + aoff, 16, 1024), sdesc_sw128(sa + k * 2048, kHalf, 1024),
                 id_mn, k > 0 ? 1u : 0u);
        }
      }
      mma_commit(&mma_done);
      mbar_wait(&mma_done, 0, nullptr, kWaitNs);
      if (!ok) {  // leave no copy in flight (warp 1 waits for the state's)
        mbar_wait(&qk_full, 0, nullptr, kWaitNs);
        mbar_wait(&v_full, 0, nullptr, kWaitNs);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // Only the entering state comes from the scan: everything else runs while the
      // scan is still going when this grid was launched as its programmatic
      // dependent.  It lands where K was, once the Q K^T products have read K.
      grid_dependency_wait();
      if (mbar_wait(&qk_done, 0, &abort_flag, kWaitNs)) {
        mbar_expect_tx(&s_full, kTile);
        for (int hh = 0; hh < 2; ++hh)
          tma_load_3d(sS + hh * kHalf, &tm_s, &s_full, 64 * hh, 0, unit);
        mbar_wait(&s_full, 0, nullptr, kWaitNs);  // no copy left in flight at exit
      }
    }
    __syncwarp();
  } else if (warp >= 2) {
    int t;
    uint32_t lane_base;
    math_row_index<128>(warp, lane, t, lane_base, tmem);
    const float gt = chunk_log2_decay(p, row0, len, h, t, g2, warp_sum);
    const bool row_valid = t < len;
    bool ok = __all_sync(0xffffffffu, mbar_wait(&qk_done, 0, &abort_flag, kWaitNs));
    if (ok) {
      tc_fence_after();
      // P[t][s] = S[t][s] * exp(G_t - G_s) for s <= t (rows past the chunk: 0):
      // the whole S row in one load, the 64 packed bf16 pairs back in one store
      uint32_t a[4][32], pk[4][16];
      tmem_ld128(tS + (lane_base - tmem), a);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) tmem_wait_ld(a[cc]);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int s0 = 32 * cc + 2 * e;
          const float p0 =
              (row_valid && s0 <= t) ? __uint_as_float(a[cc][2 * e]) * ex2(gt - g2[s0]) : 0.f;
          const float p1 = (row_valid && s0 + 1 <= t)
                               ? __uint_as_float(a[cc][2 * e + 1]) * ex2(gt - g2[s0 + 1])
                               : 0.f;
          __nv_bfloat162 b = __floats2bfloat162_rn(p0, p1);
          pk[cc][e] = *reinterpret_cast<uint32_t*>(&b);
        }
      }
      tmem_st64(tS + (lane_base - tmem), pk);
      tmem_wait_st();
    }
    tc_fence_before();
    mbar_arrive(&p_full);
    ok = ok && __all_sync(0xffffffffu, mbar_wait(&mma_done, 0, &abort_flag, kWaitNs));
    if (ok) {
      tc_fence_after();
      // Row t of out is 128 bf16 = 16 pieces of 16 bytes.  The Q tile is idle once
      // every MMA is done: row t goes there at 256 * t, piece c at position
      // (c & 8) | ((c ^ t) & 7), and each warp then writes its own 32 rows out, two
      // whole 256-byte rows per store instruction (rows past the chunk stay unwritten).
      const float decay_t = ex2(gt);
      uint4* stage = reinterpret_cast<uint4*>(sQ);
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t a[32], b[32];
        tmem_ld32(tI + (lane_base - tmem) + 32 * q4, a);
        tmem_ld32(tO + (lane_base - tmem) + 32 * q4, b);
        tmem_wait_ld(a);
        tmem_wait_ld(b);
#pragma unroll
        for (int j = 0; j < 4; ++j) {  // piece c = 4 * q4 + j: columns 8c .. 8c + 7
          uint32_t wd[4];
#pragma unroll
          for (int u2 = 0; u2 < 4; ++u2) {
            const int e = 8 * j + 2 * u2;
            const float o0 = p.scale * fmaf(decay_t, __uint_as_float(a[e]), __uint_as_float(b[e]));
            const float o1 =
                p.scale * fmaf(decay_t, __uint_as_float(a[e + 1]), __uint_as_float(b[e + 1]));
            __nv_bfloat162 v2 = __floats2bfloat162_rn(o0, o1);
            wd[u2] = *reinterpret_cast<uint32_t*>(&v2);
          }
          const int c = 4 * q4 + j;
          stage[16 * t + ((c & 8) | ((c ^ t) & 7))] = make_uint4(wd[0], wd[1], wd[2], wd[3]);
        }
      }
      __syncwarp();
      const int r0 = t - lane, c = lane & 15;
#pragma unroll 4
      for (int r2 = 0; r2 < 16; ++r2) {
        const int r = r0 + 2 * r2 + (lane >> 4);
        if (r < len)
          reinterpret_cast<uint4*>(p.out + ((int64_t)(row0 + r) * p.heads + h) * kDim)[c] =
              stage[16 * r + ((c & 8) | ((c ^ r) & 7))];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
  if (threadIdx.x == 0 && abort_flag) atomicOr(&g_la_error, 1);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 3D bf16 map over [n2][n1][128] with a 64 x 1 x 128 box along dims (0, 1, 2) or
// a 64 x 128 x 1 box (`rows_in_dim1`).
bool encode3(CUtensorMap* map, const void* base, uint64_t n1, uint64_t n2, bool rows_in_dim1) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)kDim, n1, n2};
  const cuuint64_t strides[2] = {(cuuint64_t)kDim * 2, (cuuint64_t)n1 * kDim * 2};
  const cuuint32_t box[3] = {64, rows_in_dim1 ? 128u : 1u, rows_in_dim1 ? 1u : 128u};
  const cuuint32_t elem[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

int launch_la_prefill(const Launch& a, cudaStream_t stream) {
  const seg_la_table_desc& d = *a.desc;
  const Workspace ws = prefill_workspace(d);
  char* w = static_cast<char*>(a.workspace);
  Params p;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.g = a.g;
  p.pool = a.state_pool;
  p.tab = a.tab;
  p.u = reinterpret_cast<float*>(w + ws.u);
  p.s_in = reinterpret_cast<__nv_bfloat16*>(w + ws.s_in);
  p.gamma = reinterpret_cast<float*>(w + ws.gamma);
  p.scale = a.scale;
  p.heads = d.heads;
  const int units = d.num_chunks * d.heads;
  if (d.num_chunks > 0) {
    CUtensorMap tq, tk, tv, ts;
    if (!encode3(&tq, a.q, d.heads, d.total_q, false) || !encode3(&tk, a.k, d.heads, d.total_q, false) ||
        !encode3(&tv, a.v, d.heads, d.total_q, false) || !encode3(&ts, p.s_in, kDim, units, true))
      return SEG_ATTN_ERR_CUDA;
    constexpr int smem1 = 2 * kTile + 1024, smem3 = 3 * kTile + 1024;
    // The output pass fits two CTAs per SM; a grid that fills at most one CTA per SM
    // asks for more shared memory than two could share, so no SM takes two of them
    // while others idle.
    constexpr int kSms = 148, smem3_spread = 4 * kTile + 1024;
    const int smem3_launch = units <= kSms ? smem3_spread : smem3;
    // function attributes are per device: set them for the current one on every call
    if (cudaFuncSetAttribute(la_chunk_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem1) != cudaSuccess ||
        cudaFuncSetAttribute(la_chunk_out_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem3_spread) != cudaSuccess)
      return SEG_ATTN_ERR_CUDA;
    const dim3 grid(d.num_chunks, d.heads);
    la_chunk_state_kernel<<<grid, kThreads, smem1, stream>>>(tk, tv, p);
    if (cudaGetLastError() != cudaSuccess) return SEG_ATTN_ERR_CUDA;
    // the scan and the output pass are programmatic dependents of the pass before
    // them: each launches while its predecessor still runs and waits for it only
    // where it reads that predecessor's results
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.stream = stream;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(d.batch * d.heads, kDim * kDim / 1024);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    if (cudaLaunchKernelEx(&cfg, la_scan_kernel, p) != cudaSuccess) return SEG_ATTN_ERR_CUDA;
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem3_launch;
    if (cudaLaunchKernelEx(&cfg, la_chunk_out_kernel, tq, tk, tv, ts, p) != cudaSuccess)
      return SEG_ATTN_ERR_CUDA;
  } else if (d.batch > 0) {
    // no tokens: the scan still moves every state from its input to its output slot
    la_scan_kernel<<<dim3(d.batch * d.heads, kDim * kDim / 1024), 256, 0, stream>>>(p);
  }
  return cudaGetLastError() == cudaSuccess ? SEG_ATTN_OK : SEG_ATTN_ERR_CUDA;
}

int take_la_error(int* value) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_la_error, sizeof(int)) != cudaSuccess) return SEG_ATTN_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_la_error, &zero, sizeof(int)) != cudaSuccess) return SEG_ATTN_ERR_CUDA;
  *value = v;
  return SEG_ATTN_OK;
}

}  // namespace segla
