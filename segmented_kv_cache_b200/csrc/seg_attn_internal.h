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
constexpr int kPieceOverheadTiles = 3;  // per-piece cost (prologue, epilogue) in K tiles (traced: ~12 k cycles)
constexpr int kMaxSplit = 4;            // most pieces one prefill item is cut into
constexpr int kMaxGroupSplit = 32;      // the same for a pass over a shared prefix
constexpr int kMinSharedKeys = 256;     // shortest prefix worth a pass of its own
// decode: key chunks are halved (down to 256 keys) until the grid has this many
// CTAs -- 4 waves at 2 CTAs per SM, so the last wave's tail stays short
constexpr int kDecodeTargetCtas = 8 * kSmCount;

// Device views of the table arrays (device pointers into dev_table).
struct TableView {
  const int32_t* q_offsets;   // [B+1]
  const int32_t* k_lens;      // [B]
  const int32_t* seg_offsets; // [B+1]
  const int32_t* seg_start;   // [nseg]
  const int32_t* seg_kstart;  // [nseg]
  const int32_t* seg_len;     // [nseg]
  const int4* work;           // decode [num_work]; prefill [num_work][4]
  const int4* merge;          // prefill [num_merge][2]
  const int32_t* req_chunks;  // [B+1] (decode)
};

// The pass over the shared prefixes is the prefill kernel run on a table of its
// own: one pseudo-request per group (its members' queries, non-causal, the
// prefix keys), every piece writing a partial.  This description of it points
// into the same table buffer.
inline seg_attn_table_desc group_pass_desc(const seg_attn_table_desc& d) {
  seg_attn_table_desc g = d;
  g.mode = SEG_ATTN_MODE_PREFILL;
  g.causal = 0;
  g.batch = d.num_groups;
  g.total_k = d.group_total_k;
  g.num_segments = d.num_group_segments;
  g.num_work = d.num_group_work;
  g.num_merge = 0;
  g.num_parts = d.num_group_parts;
  g.num_single = d.num_group_single;
  g.shared = 0;
  g.off_q_offsets = d.off_group_q_offsets;
  g.off_k_lens = d.off_group_k_lens;
  g.off_seg_offsets = d.off_group_seg_offsets;
  g.off_seg_start = d.off_group_seg_start;
  g.off_seg_kstart = d.off_group_seg_kstart;
  g.off_seg_len = d.off_group_seg_len;
  g.off_work = d.off_group_work;
  g.off_merge = 0;
  return g;
}

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
  bool fp8 = false;                // pools hold E4M3 codes
  const float* k_scale = nullptr;  // [Hkv] device, FP8 only
  const float* v_scale = nullptr;
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
int launch_wait_selftest(int wait_us, cudaStream_t stream);
// Stall test of the prefill kernel (seg_attn_stall_test).
int set_stall_test(int withhold_k_tile, int wait_us);
// Order test of the prefill kernel (seg_attn_order_test).
int set_order_test(int delay_ns);
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

// Byte offsets of the partial results in the workspace: the main pass's
// (prefill pieces [slot][kItemRows][D] + [slot][kItemRows], or decode chunks
// [chunk][Hq][D] + [chunk][Hq]), then the shared-prefix pass's pieces.
struct WorkspaceLayout {
  size_t main_o = 0, main_lse = 0, group_o = 0, group_lse = 0, total = 0;
};
inline WorkspaceLayout workspace_layout(const seg_attn_table_desc& d, bool decode_partials) {
  WorkspaceLayout w;
  size_t at = 0;
  if (d.mode == SEG_ATTN_MODE_PREFILL) {
    if (d.num_parts > 0) {
      at = prefill_part_o_bytes(d.num_parts, d.head_dim);
      w.main_lse = at;
      at += align_up((size_t)d.num_parts * kItemRows * sizeof(float), 256);
    }
  } else if (decode_partials || d.shared) {
    at = decode_part_o_bytes(d);
    w.main_lse = at;
    at += align_up((size_t)d.num_work * d.q_heads * sizeof(float), 256);
  }
  if (d.shared && d.num_group_parts > 0) {
    w.group_o = at;
    at += prefill_part_o_bytes(d.num_group_parts, d.head_dim);
    w.group_lse = at;
    at += align_up((size_t)d.num_group_parts * kItemRows * sizeof(float), 256);
  }
  w.total = at;
  return w;
}

// Merge of the shared-prefix partials with each request's own partials.
struct CascadeLaunch {
  const void* dev_table;
  const seg_attn_table_desc* desc;
  const float* main_o;
  const float* main_lse;
  const float* group_o;
  const float* group_lse;
  void* out;
  float* lse;
};
int launch_cascade_merge(const CascadeLaunch& a, cudaStream_t stream);

}  // namespace segattn
