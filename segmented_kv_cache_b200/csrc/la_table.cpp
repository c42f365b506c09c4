// Host side of segment linear attention: validates a batch and lays out its
// table (per-request rows and state slots, and the prefill chunk list).
#include <stdint.h>
#include <string.h>

#include <limits>
#include <unordered_set>
#include <vector>

#include "seg_la.h"
#include "seg_la_internal.h"

extern "C" int seg_la_build_table(int batch, const int32_t* q_lens, const int32_t* in_slot,
                                  const int32_t* out_slot, int64_t num_state_slots, int mode,
                                  int heads, int head_dim, void* host_out, size_t host_out_bytes,
                                  seg_la_table_desc* desc) {
  if (!desc) return SEG_ATTN_ERR_INVALID_ARG;
  memset(desc, 0, sizeof(*desc));
  if (batch < 0 || heads <= 0 || num_state_slots < 0 ||
      (mode != SEG_ATTN_MODE_PREFILL && mode != SEG_ATTN_MODE_DECODE))
    return SEG_ATTN_ERR_INVALID_ARG;
  if (batch > 0 && (!in_slot || !out_slot)) return SEG_ATTN_ERR_INVALID_ARG;
  if (batch > 0 && mode == SEG_ATTN_MODE_PREFILL && !q_lens) return SEG_ATTN_ERR_INVALID_ARG;
  if (head_dim != segla::kDim) return SEG_ATTN_ERR_UNSUPPORTED;
  const int64_t kI32Max = std::numeric_limits<int32_t>::max();
  if (num_state_slots * heads > kI32Max) return SEG_ATTN_ERR_UNSUPPORTED;

  std::unordered_set<int32_t> written;
  int64_t total_q = 0, n_chunks = 0;
  for (int r = 0; r < batch; ++r) {
    const int64_t q = q_lens ? q_lens[r] : 1;
    if (q < 0 || (mode == SEG_ATTN_MODE_DECODE && q != 1)) return SEG_ATTN_ERR_INVALID_ARG;
    if (in_slot[r] < -1 || in_slot[r] >= num_state_slots || out_slot[r] < -1 ||
        out_slot[r] >= num_state_slots)
      return SEG_ATTN_ERR_SEGMENT_OOB;
    if (out_slot[r] >= 0 && !written.insert(out_slot[r]).second)
      return SEG_ATTN_ERR_SEGMENT_OVERLAP;  // two requests write one slot
    total_q += q;
    n_chunks += (q + segla::kChunk - 1) / segla::kChunk;
  }
  for (int r = 0; r < batch; ++r)  // a slot read by one request and written by another
    if (in_slot[r] >= 0 && in_slot[r] != out_slot[r] && written.count(in_slot[r]))
      return SEG_ATTN_ERR_SEGMENT_OVERLAP;
  if (total_q > kI32Max || n_chunks * heads > kI32Max) return SEG_ATTN_ERR_UNSUPPORTED;

  int64_t n = 0;
  auto take = [&](int64_t count) {
    const int64_t at = n;
    n = (n + count + 3) / 4 * 4;  // 16-byte aligned arrays
    return at;
  };
  desc->off_q_offsets = take(batch + 1);
  desc->off_in_slot = take(batch);
  desc->off_out_slot = take(batch);
  const bool prefill = mode == SEG_ATTN_MODE_PREFILL;
  desc->off_req_chunks = take(prefill ? batch + 1 : 0);
  desc->off_chunks = take(prefill ? 4 * n_chunks : 0);
  desc->magic = SEG_LA_TABLE_MAGIC;
  desc->version = SEG_LA_TABLE_VERSION;
  desc->mode = mode;
  desc->batch = batch;
  desc->heads = heads;
  desc->head_dim = head_dim;
  desc->chunk_len = prefill ? segla::kChunk : 0;
  desc->num_chunks = prefill ? (int32_t)n_chunks : 0;
  desc->total_q = total_q;
  desc->num_state_slots = num_state_slots;
  desc->table_bytes = (uint64_t)n * sizeof(int32_t);
  desc->workspace_bytes = prefill ? segla::prefill_workspace(*desc).total : 0;

  if (!host_out) return SEG_ATTN_OK;
  if (host_out_bytes < desc->table_bytes) return SEG_ATTN_ERR_BUFFER_TOO_SMALL;
  if ((reinterpret_cast<uintptr_t>(host_out) & 15) != 0) return SEG_ATTN_ERR_INVALID_ARG;
  int32_t* t = static_cast<int32_t*>(host_out);
  memset(t, 0, desc->table_bytes);
  int32_t* q_off = t + desc->off_q_offsets;
  q_off[0] = 0;
  for (int r = 0; r < batch; ++r) {
    q_off[r + 1] = q_off[r] + (q_lens ? q_lens[r] : 1);
    t[desc->off_in_slot + r] = in_slot[r];
    t[desc->off_out_slot + r] = out_slot[r];
  }
  if (prefill) {
    int32_t* rc = t + desc->off_req_chunks;
    int32_t* ch = t + desc->off_chunks;
    int32_t c = 0;
    rc[0] = 0;
    for (int r = 0; r < batch; ++r) {
      for (int32_t t0 = 0, i = 0; t0 < q_lens[r]; t0 += segla::kChunk, ++i, ++c) {
        ch[4 * c + 0] = r;
        ch[4 * c + 1] = q_off[r] + t0;
        ch[4 * c + 2] = q_lens[r] - t0 < segla::kChunk ? q_lens[r] - t0 : segla::kChunk;
        ch[4 * c + 3] = i;
      }
      rc[r + 1] = c;
    }
  }
  return SEG_ATTN_OK;
}

extern "C" size_t seg_la_workspace_size(const seg_la_table_desc* desc) {
  if (!desc || desc->magic != SEG_LA_TABLE_MAGIC) return 0;
  return (size_t)desc->workspace_bytes;
}
