// Chunked-prefill SegmentAttention for sm_100a (tcgen05 + TMEM + TMA).
//
// Work item = (request, kv head g, two query tiles).  A query tile is 128
// rows of (query, head) pairs: 128/G consecutive queries x the G query heads
// that share kv head g, so every K/V byte fetched serves all G heads, and a
// small chunk (few new queries per request) still fills the 128 rows.  The
// two tiles share each K/V tile, which halves L2->SM traffic per flop.
//
// K/V tiles are 128 consecutive *logical* keys.  Segments (Flood README,
// "Introduction": contiguous runs in a shared slot pool) make every row's
// slot known up front, so the producer warp gathers the tile row by row with
// TMA gather4 (four pool rows per instruction) straight into the 128-byte
// swizzled layout the tensor cores read; keys past the end of the request
// are clamped to its last key and masked.  A tile whose 128 keys are 128
// consecutive pool slots (the common case: segments are long) is instead
// loaded as two tiled boxes, which the TMA engine moves far faster than 64
// four-row gathers.
//
// Warp roles (10 warps; 12 over an FP8 cache, see below):
//   warp 0       TMA producer: Q tiles once, then a K ring and a V ring
//                (stages per variant below), K tile i + 1 before V tile i.
//   warp 1       TMEM allocator and MMA issuer: the whole warp runs the issue
//                loop, one elected lane executes each tcgen05.mma / commit.
//   warps 2-5    softmax for query tile 0, warps 6-9 for tile 1: one thread
//                per row (its TMEM lane); online softmax (running max m and
//                normaliser l, as in the Ascend FlashAttention article,
//                "bottleneck 2") in registers, O rescaled in TMEM only when
//                the max grows by more than 2^8 (the final O / l uses the same
//                reference max, so the result is unchanged), epilogue O / l ->
//                bf16 and lse.
// Two query tiles (the usual item):
//                  S   = Q_t K^T   (SS: Q tile and K stage from shared memory)
//                  O_t += P_t V    (TS: P from tensor memory, V MN-major)
// and the two tiles take turns on one S buffer.  A softmax thread loads its
// whole S row, releases the buffer (the other tile's QK can go), and writes P
// into tensor-memory columns of its own, so the next K tile's S of a query
// tile is computed while this tile's softmax still runs, and no MMA writes
// tensor memory that an earlier MMA reads (such a write waits for the tensor
// pipe to drain).  P stays out of shared memory, whose bandwidth the SS QK,
// the V reads of PV and the TMA writes already share.
// TMEM columns: O0 [0,128) O1 [128,256) S [256,384) P0 [384,448) P1 [448,512).
// One query tile: S double-buffered, each buffer with a P region of its own, so
// the QK that refills an S buffer never overwrites what the PV before it reads.
// TMEM columns: O [0,128) P0 [128,192) P1 [192,256) S0 [256,384) S1 [384,512).
// Over an FP8 cache two more warps widen the E4M3 codes to f16: with two query
// tiles in place, inside the ring slot whose second half the codes were loaded
// into; with one, from staging tiles of their own.
// Every mbarrier wait is bounded (1 s); a timeout stops all roles of the CTA,
// drains in-flight copies and MMAs, frees TMEM and flags a device error.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include <atomic>
#include <mutex>
#include <type_traits>

#include "ptx_sm100.cuh"
#include "seg_attn_internal.h"

namespace segattn {

__device__ int g_device_error;  // non-zero once a bounded wait gave up

namespace {

constexpr int kThreads = 320;
// FP8 cache: two more warps (10, 11) widen E4M3 code tiles to f16 in shared memory
constexpr int kThreadsFp8 = 384;
constexpr int kConvThreads = 64;
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // default limit of a bounded wait
// Stall test (off by default): the K tile at which every later prefill CTA's
// producer stops loading (-1: none), and the limit of its bounded waits.
std::atomic<int> g_stall_tile{-1};
std::atomic<uint64_t> g_stall_wait_ns{kWaitLimitNs};
// Order test (off by default): every softmax warp of a one-tile item sleeps this
// long after it signals P of the item's last K tile.
std::atomic<int> g_order_delay_ns{0};
constexpr float kRescaleLog2 = 8.0f;
constexpr uint32_t kHalfBytes = 128 * 128;  // 128 rows x 64 bf16 (one swizzle-128B panel)

struct PrefillParams {
  __nv_bfloat16* out;
  float* lse;
  TableView tab;
  float scale_log2;
  int q_heads, kv_heads, group, qpt, causal;
  float* part_o;    // split items: [slot][kItemRows][D], O / l of the piece
  float* part_lse;  // split items: [slot][kItemRows], log2 of the piece's sum of exp
  int work_base;    // first work item of this launch
  const float* k_scale;  // FP8 cache: [kv_heads] dequantisation scales (value = code * scale)
  const float* v_scale;
  uint64_t wait_ns;      // limit of every bounded wait (1 s unless a stall test shortens it)
  int withhold_tile;     // stall test: the producer stops before loading this K tile (-1: off)
  int p_delay_ns;        // order test: one-tile softmax sleep after the last P is signalled (0: off)
};

// Query region + K ring + V ring + barriers + alignment slack.  The query
// region is one Q tile (SINGLE) or the two P tiles, which hold the two Q tiles
// until the softmax threads have moved them to tensor memory.  The d = 64
// variant asks for more than half the SM's shared memory as well, so one CTA
// owns an SM and its 512 tensor-memory columns.
// K/V ring depths (stages of K, of V).  Over a bf16 cache the one-tile kernel
// spends the second query tile's space on a third K and V stage; the two-tile
// kernels, whose P tiles live in tensor memory, have room for a third K stage:
// their QK of a K tile runs a softmax ahead of the PV of the previous one, so K
// tiles are wanted earlier than V tiles.  The one-tile kernel over an FP8 cache
// keeps two of each beside its code staging tiles.
template <bool SINGLE, bool FP8>
constexpr int ring_k() {
  return SINGLE && FP8 ? 2 : 3;
}
template <bool SINGLE, bool FP8>
constexpr int ring_v() {
  return SINGLE && !FP8 ? 3 : 2;
}

// Two query tiles: P in tensor memory columns of its own (so no MMA ever writes
// tensor memory that an earlier MMA reads), one S buffer the two tiles take
// turns on.  One query tile: S double-buffered, a P region per S buffer.  Queries
// stay in shared memory as the TMA loaded them in both.
template <bool SINGLE, bool FP8>
constexpr bool two_tiles() {
  return !SINGLE;
}

// FP8 cache, two query tiles: a K/V tile's E4M3 codes land in the second half of
// its ring slot and are widened to f16 there (no staging tiles, which leaves the
// shared memory the tensor-memory query layout needs).  One query tile: codes
// are staged in tiles of their own and widened into the ring.
template <bool SINGLE, bool FP8>
constexpr bool widen_in_place() {
  return FP8 && !SINGLE;
}
template <int D, bool SINGLE, bool FP8>
constexpr size_t staging_bytes() {
  return FP8 && !widen_in_place<SINGLE, FP8>() ? 2 * (size_t)kTileKeys * D : 0;
}

template <int D, bool SINGLE, bool FP8>
constexpr size_t query_region_bytes() {
  return (SINGLE ? 1 : 2) * (D / 64) * (size_t)kHalfBytes;
}

// The one-tile FP8 variant adds one staging tile of raw codes each for K and V.
template <int D, bool SINGLE, bool FP8>
constexpr size_t prefill_smem_bytes() {
  constexpr size_t need = query_region_bytes<D, SINGLE, FP8>() +
                          (ring_k<SINGLE, FP8>() + ring_v<SINGLE, FP8>()) * (D / 64) *
                              (size_t)kHalfBytes +
                          staging_bytes<D, SINGLE, FP8>() + 256 + 1024;
  static_assert(need <= 227 * 1024, "shared memory per CTA");
  return need < 120 * 1024 ? 120 * 1024 : need;
}

// Three-input maximum (one instruction on sm_100).
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Packed fp32 pairs: one instruction does two fmaf / two adds, each rounded as
// the scalar one would be.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Eight bf16 (one 16-byte chunk) -> eight f16 in place; exact for |x| in
// [2^-14, 65504], rounded below (f16 subnormals), infinite above.
__device__ __forceinline__ void bf16x8_to_f16x8(uint4& v) {
  uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i)
    w[i] = ptx::pack_f16x2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u));
}

// One tile of E4M3 codes (kTileKeys rows of D bytes, plain row-major) -> f16
// in the 128-byte-swizzled K-major layout the tensor cores read (the layout a
// tiled TMA load of a bf16 tile produces): row r, 16-byte chunk c of 64-column
// half h lands at h * kHalfBytes + r * 128 + ((c ^ (r & 7)) * 16).  Thread ct
// owns one 16-code column j of rows r0, r0 + step, ... with step a multiple of
// 8, so the swizzle phase r & 7 and both store offsets are fixed per thread and
// the unrolled loop needs no address arithmetic.
template <int D>
__device__ __forceinline__ void widen_tile(const uint8_t* src, uint8_t* dst, int ct) {
  constexpr int kCols = D / 16;                   // 16-code units per row
  constexpr int kRowStep = kConvThreads / kCols;  // 8 (d = 128) or 16 (d = 64)
  static_assert(kRowStep % 8 == 0, "rows of one thread must share the swizzle phase");
  const int j = ct % kCols, r0 = ct / kCols;
  const int sw = r0 & 7, c0 = (j & 3) * 2;
  const uint8_t* s = src + r0 * D + 16 * j;
  uint8_t* d = dst + (j >> 2) * kHalfBytes + r0 * 128;
  const int o0 = (c0 ^ sw) << 4, o1 = ((c0 + 1) ^ sw) << 4;
#pragma unroll
  for (int k = 0; k < kTileKeys / kRowStep; ++k) {
    const uint4 w = *reinterpret_cast<const uint4*>(s + k * kRowStep * D);
    uint4 lo, hi;
    lo.x = ptx::e4m3x2_to_f16x2(w.x);
    lo.y = ptx::e4m3x2_to_f16x2(w.x >> 16);
    lo.z = ptx::e4m3x2_to_f16x2(w.y);
    lo.w = ptx::e4m3x2_to_f16x2(w.y >> 16);
    hi.x = ptx::e4m3x2_to_f16x2(w.z);
    hi.y = ptx::e4m3x2_to_f16x2(w.z >> 16);
    hi.z = ptx::e4m3x2_to_f16x2(w.w);
    hi.w = ptx::e4m3x2_to_f16x2(w.w >> 16);
    *reinterpret_cast<uint4*>(d + k * kRowStep * 128 + o0) = lo;
    *reinterpret_cast<uint4*>(d + k * kRowStep * 128 + o1) = hi;
  }
}

// In-place variant: the codes of one tile sit in the second half of the ring slot
// (rows of D bytes) and are widened into the whole slot, in the layout above.  A
// row's f16 output overwrites code bytes that other threads read, so every thread
// first loads all of its codes, the 64 widening threads meet at named barrier 1,
// and only then write.
template <int D>
__device__ __forceinline__ void widen_tile_in_place(uint8_t* slot, int ct) {
  constexpr int kCols = D / 16;
  constexpr int kRowStep = kConvThreads / kCols;
  constexpr int kRows = kTileKeys / kRowStep;
  static_assert(kRowStep % 8 == 0, "rows of one thread must share the swizzle phase");
  const int j = ct % kCols, r0 = ct / kCols;
  const uint8_t* s = slot + (D / 64) * kHalfBytes / 2 + r0 * D + 16 * j;
  uint4 w[kRows];
#pragma unroll
  for (int k = 0; k < kRows; ++k) w[k] = *reinterpret_cast<const uint4*>(s + k * kRowStep * D);
  ptx::named_barrier(1, kConvThreads);
  const int sw = r0 & 7, c0 = (j & 3) * 2;
  uint8_t* d = slot + (j >> 2) * kHalfBytes + r0 * 128;
  const int o0 = (c0 ^ sw) << 4, o1 = ((c0 + 1) ^ sw) << 4;
#pragma unroll
  for (int k = 0; k < kRows; ++k) {
    uint4 lo, hi;
    lo.x = ptx::e4m3x2_to_f16x2(w[k].x);
    lo.y = ptx::e4m3x2_to_f16x2(w[k].x >> 16);
    lo.z = ptx::e4m3x2_to_f16x2(w[k].y);
    lo.w = ptx::e4m3x2_to_f16x2(w[k].y >> 16);
    hi.x = ptx::e4m3x2_to_f16x2(w[k].z);
    hi.y = ptx::e4m3x2_to_f16x2(w[k].z >> 16);
    hi.z = ptx::e4m3x2_to_f16x2(w[k].w);
    hi.w = ptx::e4m3x2_to_f16x2(w[k].w >> 16);
    *reinterpret_cast<uint4*>(d + k * kRowStep * 128 + o0) = lo;
    *reinterpret_cast<uint4*>(d + k * kRowStep * 128 + o1) = hi;
  }
}

// SINGLE: every item of the launch has queries in its first query tile only
// (the planner lists those items last and launches them separately, so each
// instantiation keeps its own register allocation).
// FP8: the pools hold E4M3 codes (value = code * scale of the kv head).  Code
// tiles are staged by TMA as raw bytes and widened to f16 (exact) by warps 10
// and 11 into the K/V rings; queries are converted bf16 -> f16 in shared memory
// and P is f16, so every product is f16 x f16 -> f32.  The K scale is folded
// into the softmax scale, the V scale into the output.
template <int D, bool SINGLE, bool FP8, bool TMA_OUT>
__global__ void __launch_bounds__(FP8 ? kThreadsFp8 : kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_k3,
                   const __grid_constant__ CUtensorMap tm_v3, const __grid_constant__ CUtensorMap tm_o,
                   const PrefillParams p) {
  using namespace ptx;
  constexpr int HALVES = D / 64;
  constexpr uint32_t TILE = HALVES * kHalfBytes;
  constexpr int KSTEPS = D / 16;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  constexpr int RK = ring_k<SINGLE, FP8>(), RV = ring_v<SINGLE, FP8>();
  // Q tiles at sQ + t * TILE.  Two query tiles (QT): P_t in tensor memory columns
  // [384 + 64 t, 448 + 64 t).
  constexpr bool QT = two_tiles<SINGLE, FP8>();
  constexpr uint32_t QSTRIDE = TILE;
  uint8_t* sQ = sm;
  uint8_t* sK = sm + query_region_bytes<D, SINGLE, FP8>();
  uint8_t* sV = sK + RK * TILE;
  constexpr bool INPLACE = widen_in_place<SINGLE, FP8>();
  uint8_t* sStK = sV + RV * TILE;           // FP8, one tile: raw code tile of K
  uint8_t* sStV = sStK + kTileKeys * D;     // FP8, one tile: raw code tile of V
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + RV * TILE + staging_bytes<D, SINGLE, FP8>());
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [RK]
  uint64_t* k_empty = bars + 4;   // [RK]
  uint64_t* v_full = bars + 7;    // [RV]
  uint64_t* v_empty = bars + 10;  // [RV]
  uint64_t* s_full = bars + 13;   // [2] per query tile (S buffer)
  uint64_t* p_full = bars + 15;   // [2]
  uint64_t* o_full = bars + 17;   // [2]
  uint64_t* mma_done = bars + 19;
  uint64_t* kst_full = bars + 20;   // FP8, one tile: code staging of K filled (TMA bytes)
  uint64_t* kst_empty = bars + 21;  // FP8, one tile: code staging of K read by the converters
  uint64_t* vst_full = bars + 22;
  uint64_t* vst_empty = bars + 23;
  uint64_t* code_k = bars + 20;     // FP8 in place: [RK] codes landed in a K ring slot
  uint64_t* code_v = bars + 30;     // FP8 in place: [RV] the same for V
  uint64_t* q_conv = bars + 24;     // FP8: queries converted to f16 in place
  uint64_t* s_free = bars + 25;     // two tiles: the shared S buffer read by its softmax
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 28);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // limit of every bounded wait, read only when a wait checks it
  volatile uint64_t* wait_limit = reinterpret_cast<volatile uint64_t*>(bars + 29);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // piece: keys tiles [kt0, kt1) of item (request, kv head g, query tiles from q0);
  // slot >= 0 when the item is split and this piece writes a partial result.  The
  // row also carries the request's first query row, queries, keys and the segment
  // of the piece's first key, so no dependent table load precedes the first copies.
  const int item = p.work_base + blockIdx.x;
  const int4 w0 = p.tab.work[4 * item], w1 = p.tab.work[4 * item + 1];
  const int4 w2 = p.tab.work[4 * item + 2], w3 = p.tab.work[4 * item + 3];
  const int g = w0.y, q0 = w0.z, kt0 = w0.w, slot = w1.y;
  const int n_tiles = w1.x - kt0;
  const int tok0 = w2.x, q_len = w2.y, k_len = w2.z;
  // Only query tile 0 holds queries (a short chunk, or the packed queries of a
  // small shared-prefix group): tile 1 is skipped and its S columns become a
  // second S buffer of tile 0, so the next tile's S = QK^T overlaps this tile's
  // softmax.
  constexpr bool single = SINGLE;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    // FP8: the rings are filled by the converter threads, not by TMA
    for (int s = 0; s < RK; ++s) {
      mbar_init(k_full + s, FP8 ? kConvThreads : 1);
      mbar_init(k_empty + s, 1);
    }
    for (int s = 0; s < RV; ++s) {
      mbar_init(v_full + s, FP8 ? kConvThreads : 1);
      mbar_init(v_empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(s_full + s, 1);
      mbar_init(p_full + s, 128);
      mbar_init(o_full + s, 1);
    }
    mbar_init(mma_done, 1);
    mbar_init(s_free, 4);  // one arrival per softmax warp of the tile that read S
    mbar_init(q_conv, (SINGLE ? 1 : 2) * 128);
    if (INPLACE) {
      for (int s = 0; s < RK; ++s) mbar_init(code_k + s, 1);
      for (int s = 0; s < RV; ++s) mbar_init(code_v + s, 1);
    } else if (FP8) {
      mbar_init(kst_full, 1);
      mbar_init(kst_empty, kConvThreads);
      mbar_init(vst_full, 1);
      mbar_init(vst_empty, kConvThreads);
    }
    *abort_flag = 0;
    *wait_limit = p.wait_ns;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    prefetch_tensormap(&tm_k3);
    prefetch_tensormap(&tm_v3);
    prefetch_tensormap(&tm_o);
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int k_issued = 0, v_issued = 0;
    if (n_tiles > 0) {
      // bf16 cache: when the table gives the slot of a first K tile that lies inside
      // one segment, that tile goes with the query tiles, ahead of any table lookup
      // (a stage of the fresh ring is free)
      const bool k0_early = !FP8 && w3.x >= 0 && p.withhold_tile != 0;
      if (lane == 0) {
        const int q_tiles = single ? 1 : 2;
        mbar_expect_tx(q_full, q_tiles * TILE);
        for (int t = 0; t < q_tiles; ++t)
          for (int h = 0; h < HALVES; ++h)
            tma_load_3d(sQ + t * QSTRIDE + h * kHalfBytes, &tm_q, q_full, 64 * h, g * p.group,
                        tok0 + q0 + t * p.qpt);
        if (k0_early) {
          mbar_expect_tx(k_full, TILE);
          for (int h = 0; h < HALVES; ++h)
            tma_load_3d(sK + h * kHalfBytes, &tm_k3, k_full, 64 * h, g, w3.x);
        }
      }
      int seg = w2.w;
      const int seg_end = w1.w;
      // Pool rows of K tile i: lane l holds logical keys 4l .. 4l + 3 (keys past the
      // request are clamped to its last key).  Most tiles are 128 consecutive pool
      // slots (segments are long): one tiled box per 64-column half; tiles that
      // straddle a segment boundary or the end of the request are gathered row by
      // row.  Tiles are visited in increasing order (the segment cursor only moves on).
      struct TileRows {
        int rows[4];
        int slot0;
        bool contiguous;
      };
      auto tile_rows = [&](int i, TileRows& tr) {
        // the usual case: all 128 keys inside the segment of the first one, i.e. 128
        // consecutive pool slots -- one lookup, the same on every lane
        {
          const int j0 = (kt0 + i) * kTileKeys;
          while (seg + 1 < seg_end && __ldg(p.tab.seg_kstart + seg + 1) <= j0) ++seg;
          const int ks = __ldg(p.tab.seg_kstart + seg);
          if (j0 + kTileKeys <= ks + __ldg(p.tab.seg_len + seg)) {
            tr.slot0 = __ldg(p.tab.seg_start + seg) + (j0 - ks);
            tr.contiguous = true;
            return;
          }
        }
        int slot_first = 0;
        bool run = true;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = min((kt0 + i) * kTileKeys + 4 * lane + e, k_len - 1);
          while (seg + 1 < seg_end && __ldg(p.tab.seg_kstart + seg + 1) <= j) ++seg;
          const int slot = __ldg(p.tab.seg_start + seg) + (j - __ldg(p.tab.seg_kstart + seg));
          tr.rows[e] = slot * p.kv_heads + g;
          if (e == 0) slot_first = slot;
        }
        tr.slot0 = __shfl_sync(0xffffffffu, slot_first, 0);
#pragma unroll
        for (int e = 0; e < 4; ++e) run &= tr.rows[e] == (tr.slot0 + 4 * lane + e) * p.kv_heads + g;
        tr.contiguous = __all_sync(0xffffffffu, run);
      };
      auto load_tile = [&](const TileRows& tr, uint8_t* dst, const CUtensorMap* tiled,
                           const CUtensorMap* rowmap, uint64_t* bar) {
        if (lane == 0) mbar_expect_tx(bar, TILE);
        __syncwarp();
        if (tr.contiguous) {
          if (lane == 0)
            for (int h = 0; h < HALVES; ++h)
              tma_load_3d(dst + h * kHalfBytes, tiled, bar, 64 * h, g, tr.slot0);
        } else {
#pragma unroll
          for (int h = 0; h < HALVES; ++h)
            tma_gather4(dst + h * kHalfBytes + lane * 512, rowmap, bar, 64 * h, tr.rows[0],
                        tr.rows[1], tr.rows[2], tr.rows[3]);
        }
      };
      // FP8: raw code rows (D bytes each) into the staging tile, no swizzle
      auto load_codes = [&](const TileRows& tr, uint8_t* dst, const CUtensorMap* tiled,
                            const CUtensorMap* rowmap, uint64_t* bar) {
        if (lane == 0) mbar_expect_tx(bar, kTileKeys * D);
        __syncwarp();
        if (tr.contiguous) {
          if (lane == 0) tma_load_3d(dst, tiled, bar, 0, g, tr.slot0);
        } else {
          tma_gather4(dst + lane * 4 * D, rowmap, bar, 0, tr.rows[0], tr.rows[1], tr.rows[2],
                      tr.rows[3]);
        }
      };
      auto load_k = [&](int i, const TileRows& tr) -> bool {
        // stall test: stop loading here, as a copy that never lands would; the
        // consumers' bounded waits then give up and the CTA drains and exits
        if (i == p.withhold_tile) return false;
        const int st = i % RK;
        if (!__all_sync(0xffffffffu, mbar_wait(k_empty + st, ((i / RK) & 1) ^ 1, abort_flag,
                                               wait_limit, true)))
          return false;
        if (INPLACE)  // codes into the slot's second half, widened there by warps 10-11
          load_codes(tr, sK + st * TILE + TILE / 2, &tm_k3, &tm_k, code_k + st);
        else
          load_tile(tr, sK + st * TILE, &tm_k3, &tm_k, k_full + st);
        ++k_issued;
        return true;
      };
      auto load_v = [&](int i, const TileRows& tr) -> bool {
        const int st = i % RV;
        if (!__all_sync(0xffffffffu, mbar_wait(v_empty + st, ((i / RV) & 1) ^ 1, abort_flag,
                                               wait_limit, true)))
          return false;
        if (INPLACE)
          load_codes(tr, sV + st * TILE + TILE / 2, &tm_v3, &tm_v, code_v + st);
        else
          load_tile(tr, sV + st * TILE, &tm_v3, &tm_v, v_full + st);
        ++v_issued;
        return true;
      };
      if (FP8 && !INPLACE) {
        // codes of K tile i, then of V tile i, through one staging tile each
        for (int i = 0; i < n_tiles; ++i) {
          TileRows tr;
          tile_rows(i, tr);
          if (i == p.withhold_tile) break;  // stall test (see load_k)
          if (!__all_sync(0xffffffffu, mbar_wait(kst_empty, (i & 1) ^ 1, abort_flag, wait_limit, true))) break;
          load_codes(tr, sStK, &tm_k3, &tm_k, kst_full);
          ++k_issued;
          if (!__all_sync(0xffffffffu, mbar_wait(vst_empty, (i & 1) ^ 1, abort_flag, wait_limit, true))) break;
          load_codes(tr, sStV, &tm_v3, &tm_v, vst_full);
          ++v_issued;
        }
        // never leave the CTA with copies in flight (a staged copy is issued only
        // after the converters read the previous one, so the last is enough)
        if (k_issued > 0) mbar_wait(kst_full, (k_issued - 1) & 1, nullptr, wait_limit);
        if (v_issued > 0) mbar_wait(vst_full, (v_issued - 1) & 1, nullptr, wait_limit);
      } else {
        // K tile i + 1 before V tile i: the MMA warp takes them in that order
        TileRows cur, nxt;
        tile_rows(0, cur);
        if (k0_early) ++k_issued;
        bool run = k0_early || load_k(0, cur);
        for (int i = 0; run && i < n_tiles; ++i) {
          if (i + 1 < n_tiles) {
            tile_rows(i + 1, nxt);
            if (!(run = load_k(i + 1, nxt))) break;
          }
          if (!(run = load_v(i, cur))) break;
          cur = nxt;
        }
        // never leave the CTA with copies in flight (the copies' own barriers: in
        // place, the ring slots' full barriers wait for the widening threads too)
        for (int s = 0; s < RK; ++s)
          if (k_issued > s) {
            const int last = s + RK * ((k_issued - 1 - s) / RK);
            mbar_wait((INPLACE ? code_k : k_full) + s, (last / RK) & 1, nullptr, wait_limit);
          }
        for (int s = 0; s < RV; ++s)
          if (v_issued > s) {
            const int last = s + RV * ((v_issued - 1 - s) / RV);
            mbar_wait((INPLACE ? code_v : v_full) + s, (last / RV) & 1, nullptr, wait_limit);
          }
      }
      if (lane == 0) mbar_wait(q_full, 0, nullptr, wait_limit);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the issue loop on warp-uniform values; one elected lane
    // executes each tcgen05.mma / commit.
    if (n_tiles > 0) {
      // The issue loop is one warp sharing its sub-partition with two softmax warps,
      // so every instruction on it adds latency to the period: a complete phase is
      // taken on the first try (uniform across the warp, no vote), and several
      // barriers get independent first tries whose latencies overlap; the bounded
      // wait runs only when a phase is not complete yet.
      auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
        if (mbar_try_wait(smem_u32(bar), parity)) return true;
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, wait_limit, true)) != 0;
      };
      auto ready = [&](uint64_t* bar, uint32_t parity) { return mbar_try_wait(smem_u32(bar), parity); };
      const uint32_t idesc_qk =
          FP8 ? idesc_f16_f32(128, 128, false) : idesc_bf16_f32(128, 128, false);
      const uint32_t idesc_pv = FP8 ? idesc_f16_f32(128, D, true) : idesc_bf16_f32(128, D, true);
      const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      const uint32_t tS0 = tmem + 256, tO0 = tmem, tP0 = tmem + 384;
      // S buffer `sb` = Q tile `qt` . K stage `st`^T;  O tile `ot` += P (in S buffer `sb`) . V stage `st`
      // Shared-memory descriptors are built once: a ring stage or P tile moves the
      // start address (16-byte units, the low 14 bits) by a multiple of its size,
      // and each 16-deep K step by a constant.  Building them per MMA inside the
      // issue loop measured ~1.8x slower MMA issue than the tensor core's rate.
      const uint64_t dq = sdesc_sw128(q_addr, 16, 1024), dk = sdesc_sw128(k_addr, 16, 1024);
      const uint64_t dv = sdesc_sw128(v_addr, kHalfBytes, 1024);
      constexpr uint32_t kTileU = TILE >> 4;
      // K-step k of a K-major operand: panel k / 4, 32 bytes per step inside it
      auto kstep = [](int k) -> uint32_t { return ((k >> 2) * kHalfBytes + (k & 3) * 32) >> 4; };
      // S buffer `sb` = Q tile `qt` . K stage `st`^T;  O tile `ot` += P (in S buffer `sb`) . V stage `st`
      auto issue_qk = [&](int qt, int sb, int st) {
        const uint64_t a0 = dq + qt * kTileU, b0 = dk + st * kTileU;
        const uint32_t d = tS0 + 128 * sb;
#pragma unroll
        for (int k = 0; k < KSTEPS; ++k)
          mma_ss_warp(d, a0 + kstep(k), b0 + kstep(k), idesc_qk, k > 0 ? 1u : 0u);
      };
      // one tile: O += P (region `sb`, columns [128 + 64 sb, 192 + 64 sb)) . V stage `st`
      auto issue_pv = [&](int ot, int sb, int st, bool acc) {
        const uint64_t b0 = dv + st * kTileU;
        const uint32_t d = tO0 + 128 * ot, a = tmem + 128 + 64 * sb;
#pragma unroll
        for (int k = 0; k < kTileKeys / 16; ++k)
          mma_ts_warp(d, a + 8 * k, b0 + ((k * 2048) >> 4), idesc_pv, (acc || k > 0) ? 1u : 0u);
      };
      // two tiles: S = Q tile `qt` . K stage `st`^T into the shared S buffer (SS);
      // O tile `ot` += P tile `ot` (its own tensor-memory columns) . V stage `st` (TS)
      auto issue_qk_t = [&](int qt, int st) {
        const uint64_t a0 = dq + qt * kTileU, b0 = dk + st * kTileU;
#pragma unroll
        for (int k = 0; k < KSTEPS; ++k)
          mma_ss_warp(tS0, a0 + kstep(k), b0 + kstep(k), idesc_qk, k > 0 ? 1u : 0u);
      };
      auto issue_pv_s = [&](int ot, int st, bool acc) {
        const uint64_t b0 = dv + st * kTileU;
        const uint32_t d = tO0 + 128 * ot, a = tP0 + 64 * ot;
#pragma unroll
        for (int k = 0; k < kTileKeys / 16; ++k)
          mma_ts_warp(d, a + 8 * k, b0 + ((k * 2048) >> 4), idesc_pv, (acc || k > 0) ? 1u : 0u);
      };
      // FP8: the softmax threads convert the query tiles to f16 in place first
      bool ok = wait_all(FP8 ? q_conv : q_full, 0) && wait_all(k_full + 0, 0);
      if (single) {
        // one query tile, S double-buffered: K tile i uses S buffer and P region i & 1.
        // While the softmax works on buffer i & 1, S of tile i + 1 is already in the
        // other one; right after PV(i), S of tile i + 2 goes into buffer i & 1 (the PV
        // reads P region i & 1, not the S columns).  Tensor-core operations of one CTA
        // run in issue order, so S of tile i + 2 being complete also means PV(i) is, and
        // the softmax may then overwrite P region i & 1.
        if (ok) {
          tc_fence_after();
          issue_qk(0, 0, 0);
          mma_commit_warp(s_full + 0);
          mma_commit_warp(k_empty + 0);
        }
        if (ok && n_tiles > 1 && (ok = wait_all(k_full + 1, 0))) {
          tc_fence_after();
          issue_qk(0, 1, 1);
          mma_commit_warp(s_full + 1);
          mma_commit_warp(k_empty + 1);
        }
        // S buffer of tile i: i & 1; its ring stages: i % RK, i % RV
        for (int i = 0; ok && i < n_tiles; ++i) {
          const int b = i & 1, vs = i % RV;
          const uint32_t ph = (i >> 1) & 1;
          if (!(ok = wait_all(v_full + vs, (i / RV) & 1))) break;
          if (!(ok = wait_all(p_full + b, ph))) break;
          tc_fence_after();
          issue_pv(0, b, vs, i > 0);
          mma_commit_warp(o_full + 0);
          mma_commit_warp(v_empty + vs);
          if (i + 2 < n_tiles) {
            const int ks = (i + 2) % RK;
            if (!(ok = wait_all(k_full + ks, ((i + 2) / RK) & 1)))
              break;
            tc_fence_after();
            issue_qk(0, b, ks);
            mma_commit_warp(s_full + b);
            mma_commit_warp(k_empty + ks);
          }
        }
      } else {
        // Two tiles, one S buffer.  Use u of the buffer is QK of K tile u / 2 for
        // query tile u % 2; it may start once the softmax has read use u - 1
        // (completion u - 1 of s_free).  Per K tile i the order is
        //   QK_0(i + 1), PV_0(i), QK_1(i + 1), PV_1(i)
        // so the S of a query tile's next K tile is ready when its softmax
        // finishes the current one.
        if (ok) {
          tc_fence_after();
          issue_qk_t(0, 0);
          mma_commit_warp(s_full + 0);
        }
        if (ok && (ok = wait_all(s_free, 0))) {
          tc_fence_after();
          issue_qk_t(1, 0);
          mma_commit_warp(s_full + 1);
          mma_commit_warp(k_empty + 0);
        }
        for (int i = 0; ok && i < n_tiles; ++i) {
          const int st = i % RV;  // V stage of K tile i
          const uint32_t ph = (i / RV) & 1;
          const bool more = i + 1 < n_tiles;
          const int st1 = (i + 1) % RK;  // K stage of K tile i + 1
          const uint32_t ph1 = ((i + 1) / RK) & 1;
          if (more) {
            // use 2i + 2 waits for completion 2i + 1 (tile 1 read S of K tile i)
            if (!(ready(k_full + st1, ph1) & ready(s_free, 1)) &&
                !(ok = wait_all(k_full + st1, ph1) && wait_all(s_free, 1)))
              break;
            tc_fence_after();
            issue_qk_t(0, st1);
            mma_commit_warp(s_full + 0);
          }
          if (!(ready(v_full + st, ph) & ready(p_full + 0, i & 1)) &&
              !(ok = wait_all(v_full + st, ph) && wait_all(p_full + 0, i & 1)))
            break;
          tc_fence_after();
          issue_pv_s(0, st, i > 0);
          mma_commit_warp(o_full + 0);
          if (more) {
            // use 2i + 3 waits for completion 2i + 2 (tile 0 read S of K tile i + 1)
            if (!(ok = wait_all(s_free, 0)))
              break;
            tc_fence_after();
            issue_qk_t(1, st1);
            mma_commit_warp(s_full + 1);
            mma_commit_warp(k_empty + st1);
          }
          if (!(ok = wait_all(p_full + 1, i & 1))) break;
          tc_fence_after();
          issue_pv_s(1, st, i > 0);
          mma_commit_warp(o_full + 1);
          mma_commit_warp(v_empty + st);
        }
      }
      // all MMAs finished before tensor memory is released
      mma_commit_warp(mma_done);
      mbar_wait(mma_done, 0, nullptr, wait_limit);
    }
    __syncwarp();
  } else if (FP8 && warp >= 10) {
    // ------------------------------------------------------------ FP8 code widening
    // E4M3 tile -> f16 K (V) ring slot, then make the generic-proxy writes
    // visible to the tensor cores before signalling the ring slot full.
    const int ct = threadIdx.x - 10 * 32;
    bool ok = true;
    if (INPLACE) {
      // codes in the slot's second half, in the producer's order: K tile 0, then
      // K tile i + 1 before V tile i.  The 64 threads agree on every wait's outcome
      // at a barrier (all or none go on), since the widening meets at another one.
      auto widen = [&](uint8_t* slot, uint64_t* landed, uint32_t parity, uint64_t* full) -> bool {
        const bool got = mbar_wait(landed, parity, abort_flag, wait_limit);
        if (!named_barrier_and(1, kConvThreads, got)) return false;
        widen_tile_in_place<D>(slot, ct);
        fence_proxy_async_smem();
        mbar_arrive(full);
        return true;
      };
      if (n_tiles > 0) ok = widen(sK, code_k, 0, k_full);
      for (int i = 0; ok && i < n_tiles; ++i) {
        if (i + 1 < n_tiles) {
          const int sk = (i + 1) % RK;
          if (!(ok = widen(sK + sk * TILE, code_k + sk, ((i + 1) / RK) & 1, k_full + sk))) break;
        }
        const int sv = i % RV;
        ok = widen(sV + sv * TILE, code_v + sv, (i / RV) & 1, v_full + sv);
      }
    }
    for (int i = 0; !INPLACE && ok && i < n_tiles; ++i) {
      const int sk = i % RK, sv = i % RV;
      if (!(ok = mbar_wait(kst_full, i & 1, abort_flag, wait_limit) &&
                 mbar_wait(k_empty + sk, ((i / RK) & 1) ^ 1, abort_flag, wait_limit)))
        break;
      widen_tile<D>(sStK, sK + sk * TILE, ct);
      fence_proxy_async_smem();
      mbar_arrive(k_full + sk);
      mbar_arrive(kst_empty);
      if (!(ok = mbar_wait(vst_full, i & 1, abort_flag, wait_limit) &&
                 mbar_wait(v_empty + sv, ((i / RV) & 1) ^ 1, abort_flag, wait_limit)))
        break;
      widen_tile<D>(sStV, sV + sv * TILE, ct);
      fence_proxy_async_smem();
      mbar_arrive(v_full + sv);
      mbar_arrive(vst_empty);
    }
  } else if (!single || warp < 6) {
    // ------------------------------------------------------------ softmax + epilogue
    const int t = (warp - 2) >> 2;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const int qi = q0 + t * p.qpt + row / p.group;
    const int head = g * p.group + row % p.group;
    const bool row_valid = qi < q_len;
    const int vis = p.causal ? min(k_len, k_len - q_len + qi + 1) : k_len;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    uint32_t tS = lane_base + 256 + 128 * t;  // S buffer of the current K tile (SINGLE)
    if (QT) tS = lane_base + 256;             // two tiles: the shared S buffer
    const uint32_t tO = lane_base + 128 * t;
    // P of the current K tile: two tiles, this tile's region; one tile, the region of
    // the current S buffer (set per K tile)
    uint32_t tP = lane_base + 384 + 64 * t;
    // FP8: scores are q . code * k_scale, so the K scale joins the softmax scale
    const float sl2 = FP8 ? p.scale_log2 * __ldg(p.k_scale + g) : p.scale_log2;
    float m_ref = -INFINITY;  // raw score units
    float l = 0.f;
    bool ok = true;
    if (n_tiles > 0 && FP8) {
      // FP8 cache: this thread's query row of tile t, bf16 -> f16 in place (exact
      // for |q| < 65504), so that both MMA operands are f16.  Visiting chunk
      // c ^ (row & 7), the place of the row's logical chunk c, spreads a warp's
      // 32 rows over all shared-memory banks.
      ok = __all_sync(0xffffffffu, mbar_wait(q_full, 0, abort_flag, wait_limit));
      if (ok) {
#pragma unroll
        for (int h = 0; h < HALVES; ++h)
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint4* chunk = reinterpret_cast<uint4*>(sQ + t * QSTRIDE + h * kHalfBytes + row * 128 +
                                                    ((c ^ (row & 7)) << 4));
            uint4 v = *chunk;
            bf16x8_to_f16x8(v);
            *chunk = v;
          }
        fence_proxy_async_smem();
        mbar_arrive(q_conv);
      }
    }
    // One tile of the online softmax.  `masked`: some row of the warp must not
    // see some key of the tile (causal diagonal, end of the request); the mask
    // is applied to the registers, so other tiles never compare per element.
    auto softmax_tile = [&](int i, bool masked) -> bool {
      auto f = [](uint32_t bits) { return __uint_as_float(bits); };
      // the whole S row in registers: one round trip to tensor memory
      uint32_t sv[4][32];
      tmem_ld128(tS, sv);
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_wait_ld(sv[c]);
      if (QT) {
        // the shared S buffer is free for the other tile's QK
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);
      }
      if (masked) {
        const int kb = (kt0 + i) * kTileKeys;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (kb + 32 * c + e >= vis) sv[c][e] = 0xff800000u;  // -inf
      }
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int e = 0; e < 32; e += 2) mx[c] = max3(mx[c], f(sv[c][e]), f(sv[c][e + 1]));
      const float row_max = max3(mx[0], mx[1], fmaxf(mx[2], mx[3]));
      const float m_new = fmaxf(m_ref, row_max);
      float alpha = 1.f;
      bool rescale = false;
      if (m_ref == -INFINITY) {
        m_ref = m_new;  // nothing accumulated yet for this row (or only zeros)
      } else if ((m_new - m_ref) * sl2 > kRescaleLog2) {
        alpha = ex2((m_ref - m_new) * sl2);
        m_ref = m_new;
        rescale = true;
      }
      const float base = m_ref == -INFINITY ? 0.f : m_ref * sl2;
      // P = 2^(s*scale*log2e - base), packed in pairs (bf16, or f16 over an FP8 cache).
      // Queries in TMEM: f32x2 pairs for the scale-and-subtract and the sums (fewer
      // instructions per score); the P-over-S variants keep scalar arithmetic, whose
      // register allocation does not spill.
      uint64_t ls = f2_pack(0.f, 0.f);
      float ls0 = 0.f, ls1 = 0.f;
      const uint64_t sl2x2 = f2_pack(sl2, sl2), nbase2 = f2_pack(-base, -base);
      uint32_t pk[4][16];
      // two tiles: P(i) replaces P(i - 1) in this tile's tensor-memory columns once
      // PV(i - 1) has read it (complete by now as a rule: it was issued when this
      // tile's S was)
      bool waited = false;
      if (QT && i > 0) {
        if (!__all_sync(0xffffffffu,
                        mbar_wait(o_full + t, (i - 1) & 1, abort_flag, wait_limit, true)))
          return false;
        tc_fence_after();
        waited = true;
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float pa, pb;
          if constexpr (!QT) {
            pa = ex2(fmaf(f(sv[c][2 * e]), sl2, -base));
            pb = ex2(fmaf(f(sv[c][2 * e + 1]), sl2, -base));
            ls0 += pa;
            ls1 += pb;
          } else {
            float xa, xb;
            f2_unpack(f2_fma(f2_pack(f(sv[c][2 * e]), f(sv[c][2 * e + 1])), sl2x2, nbase2), xa, xb);
            pa = ex2(xa);
            pb = ex2(xb);
            ls = f2_add(ls, f2_pack(pa, pb));
          }
          pk[c][e] = FP8 ? pack_f16x2(pa, pb) : pack_bf16(pa, pb);
        }
      }
      // 128 keys as 64 columns of 2 (the tensor-memory A-operand layout), one store
      tmem_st64(tP, pk);
      if constexpr (QT) f2_unpack(ls, ls0, ls1);
      l = l * alpha + (ls0 + ls1);
      if (__any_sync(0xffffffffu, rescale)) {
        // O_t holds PV up to K tile i - 1; rescale it in place once that is complete
        if (!waited &&
            !__all_sync(0xffffffffu, mbar_wait(o_full + t, (i - 1) & 1, abort_flag, wait_limit)))
          return false;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + 32 * c, o);
          tmem_wait_ld(o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(tO + 32 * c, o);
        }
      }
      return true;
    };
    // A warp whose 32 rows hold no query (past the end of the chunk) only keeps
    // step with the barriers: its P rows feed only output rows nobody reads.
    const bool warp_live = __any_sync(0xffffffffu, row_valid);
    // One tile: before P of the last K tile n - 1 is signalled, PV(n - 2) must be
    // complete.  The S of tile n - 1 proves only PV(n - 3), and once P(n - 1) is
    // signalled PV(n - 1) may complete at any time; a later wait for PV(n - 2) could
    // then meet o_full at completion n, whose parity is that of n - 2, and wait for
    // a completion that never comes.  Confirmed here, o_full is at completion n - 1
    // or n when the epilogue waits for PV(n - 1), which one parity wait tells apart.
    auto last_pv_order = [&](int i) -> bool {
      if (!single || i != n_tiles - 1 || i == 0) return true;
      return __all_sync(0xffffffffu,
                        mbar_wait(o_full + t, (i - 1) & 1, abort_flag, wait_limit)) != 0;
    };
    // one K tile of softmax on S buffer sb (phase sph of its barriers)
    auto run_tile = [&](int i, int sb, uint32_t sph) -> bool {
      if (single) {
        tS = lane_base + 256 + 128 * sb;
        tP = lane_base + 128 + 64 * sb;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(s_full + sb, sph, abort_flag, wait_limit, true)))
        return false;
      if (!warp_live) {
        if (QT) {
          // release S; arrive for P(i) only after PV(i - 1), so that these
          // arrivals never count towards the previous P
          __syncwarp();
          if (lane == 0) mbar_arrive(s_free);
          if (i > 0 &&
              !__all_sync(0xffffffffu, mbar_wait(o_full + t, (i - 1) & 1, abort_flag, wait_limit)))
            return false;
        }
        if (!last_pv_order(i)) return false;
        mbar_arrive(p_full + sb);
        return true;
      }
      tc_fence_after();
      const bool masked = __any_sync(0xffffffffu, (kt0 + i + 1) * kTileKeys > vis);
      if (!softmax_tile(i, masked)) return false;
      tmem_wait_st();
      if (!last_pv_order(i)) return false;
      tc_fence_before();
      mbar_arrive(p_full + sb);
      return true;
    };
    if (single) {
      // S buffers alternate; unrolled by two so each buffer's address is fixed
      for (int i = 0; ok && i < n_tiles; i += 2) {
        const uint32_t sph = (i >> 1) & 1;
        ok = run_tile(i, 0, sph);
        if (ok && i + 1 < n_tiles) ok = run_tile(i + 1, 1, sph);
      }
    } else {
      for (int i = 0; ok && i < n_tiles; ++i) ok = run_tile(i, t, i & 1);
    }
    // order test (one tile): the last PV completes before this warp reaches the end
    // of the item
    if constexpr (SINGLE) {
      if (p.p_delay_ns > 0 && ok) __nanosleep(p.p_delay_ns);
    }
    if (!warp_live) ok = false;  // nothing to write
    // this row's O (fp32, D columns) in registers: every load issued, one wait
    auto load_o = [&](uint32_t (&o)[D / 32][32]) {
      if (n_tiles > 0) {
        tc_fence_after();
        if constexpr (D == 128) {
          tmem_ld128(tO, o);
        } else {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) tmem_ld32(tO + 32 * c, o[c]);
        }
#pragma unroll
        for (int c = 0; c < D / 32; ++c) tmem_wait_ld(o[c]);
      } else {
#pragma unroll
        for (int c = 0; c < D / 32; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e) o[c][e] = 0u;
      }
    };
    // PV complete up to tile n - 2 (two tiles: P(n - 1) was written after it; one
    // tile: confirmed before P(n - 1) was signalled), so o_full is at completion
    // n - 1 or n and a parity wait for PV(n - 1) is unambiguous
    if (ok && n_tiles > 0)
      ok = __all_sync(0xffffffffu,
                      mbar_wait(o_full + t, (n_tiles - 1) & 1, abort_flag, wait_limit));
    // Results leave through shared memory so that whole rows are stored: a thread
    // owns one row, and its own 16-byte pieces of it would put every warp store on 32
    // different lines.  The tile's query region is free (the commit of the tile's
    // last PV covers every earlier MMA).  Partials of a split piece: each warp stages
    // its 32 rows in a quarter of it, 16-byte chunk c of row-local r at
    // ((c & ~7) | ((c ^ r) & 7)), and copies rows out with consecutive lanes on
    // consecutive chunks.
    uint8_t* stage_w = sQ + t * QSTRIDE + quad * (QSTRIDE / 4);
    auto swz = [](int c, int r) { return (c & ~7) | ((c ^ r) & 7); };
    if (ok && slot >= 0) {
      // piece of a split item (or of a shared-prefix pass): O / l and log2(sum of exp)
      // of this key range, for every row that holds a query; fp32 rows go out in
      // passes of PCOLS columns (the staging quarter holds 32 rows of PCOLS floats)
      constexpr int PCOLS = (int)(QSTRIDE / 512) < D ? (int)(QSTRIDE / 512) : D;
      constexpr int PCH = PCOLS / 4;        // 16-byte chunks per row per pass
      constexpr int RPI = 32 / PCH;         // rows per warp instruction of the copy
      const float inv = l > 0.f ? (FP8 ? __ldg(p.v_scale + g) : 1.f) / l : 0.f;
      const int64_t prow0 = (int64_t)slot * kItemRows + t * kTileRows + quad * 32;
      uint32_t o[D / 32][32];
      load_o(o);
#pragma unroll
      for (int pass = 0; pass < D / PCOLS; ++pass) {
#pragma unroll
        for (int c = 0; c < PCH; ++c) {
          const int col = pass * PCOLS + 4 * c;
          const float4 v = make_float4(__uint_as_float(o[col / 32][col % 32]) * inv,
                                       __uint_as_float(o[col / 32][col % 32 + 1]) * inv,
                                       __uint_as_float(o[col / 32][col % 32 + 2]) * inv,
                                       __uint_as_float(o[col / 32][col % 32 + 3]) * inv);
          *reinterpret_cast<float4*>(stage_w + lane * (PCOLS * 4) + swz(c, lane) * 16) = v;
        }
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 32; k += RPI) {
          const int lr = k + lane / PCH, c = lane % PCH;
          const int qi_r = q0 + t * p.qpt + (quad * 32 + lr) / p.group;
          if (qi_r < q_len)
            *reinterpret_cast<float4*>(p.part_o + (prow0 + lr) * D + pass * PCOLS + 4 * c) =
                *reinterpret_cast<const float4*>(stage_w + lr * (PCOLS * 4) + swz(c, lr) * 16);
        }
        __syncwarp();
      }
      if (row_valid) p.part_lse[prow0 + lane] = l > 0.f ? m_ref * sl2 + log2f(l) : -INFINITY;
    } else if (!TMA_OUT && ok) {
      // a pass whose pieces mostly write partials: rows staged per warp, copied out
      constexpr int CH = D / 8;    // 16-byte chunks of a bf16 row
      constexpr int RPI = 32 / CH; // rows per warp instruction of the copy
      const float inv = l > 0.f ? (FP8 ? __ldg(p.v_scale + g) : 1.f) / l : 0.f;
      uint32_t o[D / 32][32];
      load_o(o);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          uint4 v;
          v.x = pack_bf16(__uint_as_float(o[c][e]) * inv, __uint_as_float(o[c][e + 1]) * inv);
          v.y = pack_bf16(__uint_as_float(o[c][e + 2]) * inv, __uint_as_float(o[c][e + 3]) * inv);
          v.z = pack_bf16(__uint_as_float(o[c][e + 4]) * inv, __uint_as_float(o[c][e + 5]) * inv);
          v.w = pack_bf16(__uint_as_float(o[c][e + 6]) * inv, __uint_as_float(o[c][e + 7]) * inv);
          *reinterpret_cast<uint4*>(stage_w + lane * (D * 2) + swz((32 * c + e) / 8, lane) * 16) = v;
        }
      }
      __syncwarp();
#pragma unroll
      for (int k = 0; k < 32; k += RPI) {
        const int lr = k + lane / CH, c = lane % CH;
        const int rr = quad * 32 + lr;
        const int qi_r = q0 + t * p.qpt + rr / p.group;
        if (qi_r < q_len)
          *reinterpret_cast<uint4*>(p.out + ((int64_t)(tok0 + qi_r) * p.q_heads + g * p.group +
                                             rr % p.group) * D + 8 * c) =
              *reinterpret_cast<const uint4*>(stage_w + lr * (D * 2) + swz(c, lr) * 16);
      }
      if (row_valid && p.lse)
        p.lse[(int64_t)(tok0 + qi) * p.q_heads + head] =
            l > 0.f ? (m_ref * sl2 + log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
    if (TMA_OUT && slot < 0) {
      // Final bf16 output, staged in the tile's query region in the layout of the
      // queries' TMA box (64-column panels of 128-byte rows, chunk c of row r at
      // c ^ (r & 7)).  A full query tile then leaves in two TMA stores issued by one
      // thread (the rows of one tile are qpt consecutive tokens x G heads, the box of
      // the output map); a tile with fewer queries than qpt is copied out a row per
      // D / 8 lanes, since a box would reach into the next request's rows.  The
      // tile's four warps agree at a barrier (an AND of their outcomes) before
      // staging, so a give-up anywhere leaves no warp waiting at the second one.
      constexpr int CH = D / 8;    // 16-byte chunks of a bf16 row
      constexpr int RPI = 32 / CH; // rows per warp instruction of the copy
      uint8_t* stage_t = sQ + t * QSTRIDE;
      const bool full = q0 + (t + 1) * p.qpt <= q_len;
      const bool go = full ? named_barrier_and(2 + t, 128, ok) : ok;
      if (go) {
        const float inv = l > 0.f ? (FP8 ? __ldg(p.v_scale + g) : 1.f) / l : 0.f;
        uint32_t o[D / 32][32];
        load_o(o);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 v;
            v.x = pack_bf16(__uint_as_float(o[c][e]) * inv, __uint_as_float(o[c][e + 1]) * inv);
            v.y = pack_bf16(__uint_as_float(o[c][e + 2]) * inv, __uint_as_float(o[c][e + 3]) * inv);
            v.z = pack_bf16(__uint_as_float(o[c][e + 4]) * inv, __uint_as_float(o[c][e + 5]) * inv);
            v.w = pack_bf16(__uint_as_float(o[c][e + 6]) * inv, __uint_as_float(o[c][e + 7]) * inv);
            const int ch = (32 * c + e) / 8;  // logical 16-byte chunk of the row
            *reinterpret_cast<uint4*>(stage_t + (ch >> 3) * kHalfBytes + row * 128 +
                                      (((ch & 7) ^ (row & 7)) << 4)) = v;
          }
        }
        if (full) {
          fence_proxy_async_smem();
          named_barrier(2 + t, 128);
          if (quad == 0 && lane == 0) {
#pragma unroll
            for (int h = 0; h < HALVES; ++h)
              tma_store_3d(&tm_o, stage_t + h * kHalfBytes, 64 * h, g * p.group,
                           tok0 + q0 + t * p.qpt);
            bulk_commit_group();
            bulk_wait_group_read0();  // the staging must be read before the CTA exits
          }
        } else {
          __syncwarp();
#pragma unroll
          for (int k = 0; k < 32; k += RPI) {
            const int rr = quad * 32 + k + lane / CH, c = lane % CH;
            const int qi_r = q0 + t * p.qpt + rr / p.group;
            if (qi_r < q_len)
              *reinterpret_cast<uint4*>(p.out + ((int64_t)(tok0 + qi_r) * p.q_heads + g * p.group +
                                                 rr % p.group) * D + 8 * c) =
                  *reinterpret_cast<const uint4*>(stage_t + (c >> 3) * kHalfBytes + rr * 128 +
                                                  (((c & 7) ^ (rr & 7)) << 4));
          }
        }
        if (row_valid && p.lse)
          p.lse[(int64_t)(tok0 + qi) * p.q_heads + head] =
              l > 0.f ? (m_ref * sl2 + log2f(l)) * 0.69314718055994531f : -INFINITY;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && *abort_flag) atomicOr(&g_device_error, 1);
}

// Combine the pieces of each split item: weights 2^(lse_j - max) on the pieces'
// normalised outputs.  One warp per row, each lane D/32 consecutive columns.
template <int D>
__global__ void __launch_bounds__(256) prefill_merge_kernel(const PrefillParams p) {
  constexpr int PER = D / 32;
  const int4 m0 = p.tab.merge[2 * blockIdx.x], m1 = p.tab.merge[2 * blockIdx.x + 1];
  const int req = m0.x, g = m0.y, q0 = m0.z, slot0 = m0.w, parts = m1.x;
  const int tok0 = __ldg(p.tab.q_offsets + req);
  const int q_len = __ldg(p.tab.q_offsets + req + 1) - tok0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int row = blockIdx.y * 8 + warp; row < kItemRows; row += 8 * gridDim.y) {
    const int t = row / kTileRows, r = row % kTileRows;
    const int qi = q0 + t * p.qpt + r / p.group;
    if (qi >= q_len) continue;
    const int head = g * p.group + r % p.group;
    float M = -INFINITY;
    for (int j = 0; j < parts; ++j)
      M = fmaxf(M, p.part_lse[(int64_t)(slot0 + j) * kItemRows + row]);
    const float Mb = M == -INFINITY ? 0.f : M;
    float acc[PER], L = 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] = 0.f;
    for (int j = 0; j < parts; ++j) {
      const int64_t prow = (int64_t)(slot0 + j) * kItemRows + row;
      const float w = ptx::ex2(p.part_lse[prow] - Mb);
      L += w;
      const float* po = p.part_o + prow * D + lane * PER;
#pragma unroll
      for (int e = 0; e < PER; e += 2) {
        const float2 x = *reinterpret_cast<const float2*>(po + e);
        acc[e] += w * x.x;
        acc[e + 1] += w * x.y;
      }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    __nv_bfloat16* orow = p.out + ((int64_t)(tok0 + qi) * p.q_heads + head) * D + lane * PER;
#pragma unroll
    for (int e = 0; e < PER; e += 2)
      *reinterpret_cast<uint32_t*>(orow + e) = pack_bf16(acc[e] * inv, acc[e + 1] * inv);
    if (p.lse && lane == 0)
      p.lse[(int64_t)(tok0 + qi) * p.q_heads + head] =
          L > 0.f ? (Mb + log2f(L)) * 0.69314718055994531f : -INFINITY;
  }
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

// bf16 maps are 128-byte swizzled (tensor-core operand layout); byte maps
// (E4M3 codes, staged for widening) are plain row-major.
bool encode(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims,
            const cuuint64_t* strides, const cuuint32_t* box, bool bytes = false) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint32_t elem[3] = {1, 1, 1};
  return fn(map, bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank,
            const_cast<void*>(base), dims, strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE,
            bytes ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, bool SINGLE, bool FP8, bool TMA_OUT>
int launch_items(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                 const CUtensorMap& tk3, const CUtensorMap& tv3, const CUtensorMap& to,
                 const PrefillParams& p, int n,
                 cudaStream_t stream) {
  constexpr size_t smem = prefill_smem_bytes<D, SINGLE, FP8>();
  if (cudaFuncSetAttribute(prefill_kernel<D, SINGLE, FP8, TMA_OUT>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return SEG_ATTN_ERR_CUDA;
  prefill_kernel<D, SINGLE, FP8, TMA_OUT><<<n, FP8 ? kThreadsFp8 : kThreads, smem, stream>>>(tq, tk, tv, tk3,
                                                                                  tv3, to, p);
  return cudaGetLastError() == cudaSuccess ? SEG_ATTN_OK : SEG_ATTN_ERR_CUDA;
}

template <int D, bool FP8>
int launch_prefill_d(const PrefillLaunch& a, cudaStream_t stream) {
  const seg_attn_table_desc& d = *a.desc;
  const int group = d.q_heads / d.kv_heads;
  CUtensorMap tq, tk, tv, tk3, tv3, to;
  {
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)d.q_heads, (cuuint64_t)d.total_q};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)d.q_heads * D * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)group, (cuuint32_t)d.queries_per_tile};
    if (!encode(&tq, a.q, 3, dims, strides, box)) return SEG_ATTN_ERR_CUDA;
    // the output has the queries' shape: full query tiles leave by TMA stores of the
    // same boxes (a pass that only writes partials has no output: no store is issued)
    if (!encode(&to, a.out ? a.out : a.q, 3, dims, strides, box)) return SEG_ATTN_ERR_CUDA;
  }
  {
    const int64_t rows = d.num_slots * d.kv_heads;
    const bool empty = rows == 0 || d.total_k == 0;
    // bf16: 64-column boxes (one swizzle panel); FP8: whole D-byte code rows
    constexpr int kElem = FP8 ? 1 : 2;
    constexpr cuuint32_t kBoxCols = FP8 ? D : 64;
    const cuuint64_t dims[2] = {(cuuint64_t)D, empty ? 1ull : (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)D * kElem};
    const cuuint32_t box[2] = {kBoxCols, 1};
    // with no keys no tile is ever loaded; the query buffer stands in as a valid address
    if (!encode(&tk, empty ? a.q : a.k_pool, 2, dims, strides, box, FP8)) return SEG_ATTN_ERR_CUDA;
    if (!encode(&tv, empty ? a.q : a.v_pool, 2, dims, strides, box, FP8)) return SEG_ATTN_ERR_CUDA;
    // the same pools as [slots][kv heads][d]: 128 consecutive slots of one head per box
    const cuuint64_t dims3[3] = {(cuuint64_t)D, (cuuint64_t)d.kv_heads,
                                 empty ? 1ull : (cuuint64_t)d.num_slots};
    const cuuint64_t strides3[2] = {(cuuint64_t)D * kElem, (cuuint64_t)d.kv_heads * D * kElem};
    const cuuint32_t box3[3] = {kBoxCols, 1, (cuuint32_t)kTileKeys};
    if (!encode(&tk3, empty ? a.q : a.k_pool, 3, dims3, strides3, box3, FP8))
      return SEG_ATTN_ERR_CUDA;
    if (!encode(&tv3, empty ? a.q : a.v_pool, 3, dims3, strides3, box3, FP8))
      return SEG_ATTN_ERR_CUDA;
  }
  PrefillParams p;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.lse = a.lse;
  p.tab = a.tab;
  p.scale_log2 = (float)((double)a.scale * 1.4426950408889634);
  p.q_heads = d.q_heads;
  p.kv_heads = d.kv_heads;
  p.group = group;
  p.qpt = d.queries_per_tile;
  p.causal = d.causal;
  p.part_o = a.part_o;
  p.part_lse = a.part_lse;
  p.k_scale = a.k_scale;
  p.v_scale = a.v_scale;
  p.wait_ns = g_stall_wait_ns.load();
  p.withhold_tile = g_stall_tile.load();
  p.p_delay_ns = g_order_delay_ns.load();
  // two-tile items first, then the single-tile items listed at the end.  A pass in
  // which some piece writes final rows runs the instantiation whose epilogue stores
  // full query tiles by TMA; a pass of partials only (every item split, or a pass
  // over shared prefixes) keeps the leaner epilogue, which measured faster there.
  const int n_single = d.num_single, n_two = d.num_work - d.num_single;
  const bool any_final = d.num_parts < d.num_work;
  auto launch = [&](auto single_tag, auto tma_tag, int base, int n) {
    p.work_base = base;
    return launch_items<D, decltype(single_tag)::value, FP8, decltype(tma_tag)::value>(
        tq, tk, tv, tk3, tv3, to, p, n, stream);
  };
  using T = std::true_type;
  using F = std::false_type;
  if (n_two > 0) {
    const int rc = any_final ? launch(F{}, T{}, 0, n_two) : launch(F{}, F{}, 0, n_two);
    if (rc != SEG_ATTN_OK) return rc;
  }
  if (n_single > 0) {
    const int rc = any_final ? launch(T{}, T{}, n_two, n_single) : launch(T{}, F{}, n_two, n_single);
    if (rc != SEG_ATTN_OK) return rc;
  }
  if (d.num_merge > 0) {
    prefill_merge_kernel<D><<<dim3(d.num_merge, 4), 256, 0, stream>>>(p);
    if (cudaGetLastError() != cudaSuccess) return SEG_ATTN_ERR_CUDA;
  }
  return SEG_ATTN_OK;
}

}  // namespace

int launch_prefill(const PrefillLaunch& a, cudaStream_t stream) {
  if (a.fp8)
    return a.desc->head_dim == 128 ? launch_prefill_d<128, true>(a, stream)
                                   : launch_prefill_d<64, true>(a, stream);
  return a.desc->head_dim == 128 ? launch_prefill_d<128, false>(a, stream)
                                 : launch_prefill_d<64, false>(a, stream);
}

namespace {

// Diagnostic: one warp waits, with the same bounded wait every kernel of this
// library uses, on an mbarrier that nothing ever arrives on.  The wait gives up
// after limit_ns and the grid records it in the device error word, as a stalled
// prefill or linear-attention kernel would.
__global__ void __launch_bounds__(32) wait_selftest_kernel(uint64_t limit_ns) {
  using namespace ptx;
  __shared__ uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncwarp();
  const bool done = mbar_wait(&bar, 0, &abort_flag, limit_ns);
  __syncwarp();
  if (threadIdx.x == 0 && (!done || abort_flag)) atomicOr(&g_device_error, 1);
}

}  // namespace

int set_order_test(int delay_ns) {
  g_order_delay_ns.store(delay_ns);
  return SEG_ATTN_OK;
}

int set_stall_test(int withhold_k_tile, int wait_us) {
  g_stall_tile.store(withhold_k_tile < 0 ? -1 : withhold_k_tile);
  g_stall_wait_ns.store((uint64_t)wait_us * 1000ull);
  return SEG_ATTN_OK;
}

int launch_wait_selftest(int wait_us, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>((uint64_t)wait_us * 1000ull);
  return cudaGetLastError() == cudaSuccess ? SEG_ATTN_OK : SEG_ATTN_ERR_CUDA;
}

int take_device_error(int* value) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess) return SEG_ATTN_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return SEG_ATTN_ERR_CUDA;
  *value = v;
  return SEG_ATTN_OK;
}

}  // namespace segattn
