// Internal declarations shared by the host entry points and the sm_100a kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "seg_attn.h"

namespace segattn {

constexpr int kTileKeys = 128;   // logical keys per prefill K/V tile
constexpr int kTileRows = 128;   // query rows (query x head) per prefill M-tile
constexpr int kTilesPerItem = 2; // M-tiles sharing each K/V tile in one prefill CTA
constexpr int kSmCount = 148;    // B200
constexpr int kItemRows = kTileRows * kTilesPerItem;  // query rows of one prefill item
constexpr int kMinPieceTiles = 8;       // shortest K range a split prefill piece gets
constexpr int kPieceOverheadTiles = 2;  // per-piece cost (prologue, epilogue) in K tiles
constexpr int kMaxSplit = 4;            // most pieces one prefill item is cut into

// Device views of the table arrays (device pointers into dev_table).
struct TableView {
  const int32_t* q_offsets;   // [B+1]
  const int32_t* k_lens;      // [B]
  const int32_t* seg_offsets; // [B+1]
  const int32_t* seg_start;   // [nseg]
  const int32_t* seg_kstart;  // [nseg]
  const int32_t* seg_len;     // [nseg]
  const int4* work;           // decode [num_work]; prefill [num_work][2]
  const int4* merge;          // prefill [num_merge][2]
  const int32_t* req_chunks;  // [B+1] (decode)
};

inline TableView make_view(const void* dev_table, const seg_attn_table_desc& d) {
  const int32_t* t = static_cast<const int32_t*>(dev_table);
  TableView v;
  v.q_offsets = t + d.off_q_offsets;
  v.k_lens = t + d.off_k_lens;
  v.seg_offsets = t + d.off_seg_offsets;
  v.seg_start = t + d.off_seg_start;
  v.seg_kstart = t + d.off_seg_kstart;
  v.seg_len = t + d.off_seg_len;
  v.work = reinterpret_cast<const int4*>(t + d.off_work);
  v.merge = reinterpret_cast<const int4*>(t + d.off_merge);
  v.req_chunks = t + d.off_req_chunks;
  return v;
}

struct PrefillLaunch {
  const void* q;
  const void* k_pool;
  const void* v_pool;
  void* out;
  float* lse;
  TableView tab;
  const seg_attn_table_desc* desc;
  float scale;
  float* part_o;    // [slots][kItemRows][D] fp32, normalised per piece (split items only)
  float* part_lse;  // [slots][kItemRows] fp32, log2 domain
};

struct DecodeLaunch {
  const void* q;
  const void* k_pool;
  const void* v_pool;
  void* out;
  float* lse;
  TableView tab;
  const seg_attn_table_desc* desc;
  float scale;
  float* part_o;    // [num_work][Hq][D] fp32, normalised per chunk
  float* part_lse;  // [num_work][Hq] fp32, log2 domain
  bool fp8;              // pools hold E4M3 codes
  const float* k_scale;  // [Hkv] device, FP8 only
  const float* v_scale;
};

// Each returns SEG_ATTN_OK or SEG_ATTN_ERR_CUDA (launch error).
int launch_prefill(const PrefillLaunch& a, cudaStream_t stream);
int launch_decode(const DecodeLaunch& a, cudaStream_t stream);

// Read and clear the device error words: a bounded wait that gave up (prefill)
// and a KV-append slot out of range.
int take_device_error(int* value);
int take_append_error(int* value);

// Workspace split of the decode call.
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline size_t prefill_part_o_bytes(int64_t slots, int head_dim) {
  return align_up((size_t)slots * kItemRows * head_dim * sizeof(float), 256);
}
inline size_t decode_part_o_bytes(const seg_attn_table_desc& d) {
  return align_up((size_t)d.num_work * d.q_heads * d.head_dim * sizeof(float), 256);
}

}  // namespace segattn
