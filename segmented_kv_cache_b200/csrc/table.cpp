// Host side of the boundary: segment-table builder, validator and work
// planner (no device state is touched here).
//
// The segmentable KV cache (Flood README, "Introduction") stores each request
// as a few contiguous slot runs.  The builder flattens the per-request lists
// into CSR arrays, records each segment's logical start so the kernels can
// translate logical key j -> slot in O(1) per run, and plans the work:
//   prefill: one item per (request, kv head, pair of 128-row query tiles);
//            long items are cut into pieces along their K tiles when that
//            shortens the longest-first schedule on the 148 SMs (the pieces'
//            partial results are merged by a second kernel), then the pieces
//            are ordered longest first;
//   decode:  split-K chunks of logical keys (per-block partial attention with
//            a per-request reduction, FlashAccel article, "data layout
//            optimisation"), sized so the grid covers the 148 SMs many times.
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <array>
#include <functional>
#include <limits>
#include <numeric>
#include <queue>
#include <vector>

#include "seg_attn.h"
#include "seg_attn_internal.h"

namespace {

using segattn::align_up;

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

struct Layout {
  int64_t n = 0;  // int32 elements so far
  int64_t take(int64_t count) {
    int64_t at = n;
    n += count;
    n = (n + 3) / 4 * 4;  // every array starts 16-byte aligned
    return at;
  }
};

}  // namespace

extern "C" int seg_attn_build_table(int batch, const int32_t* q_lens, const int32_t* seg_counts,
                                    const int32_t* seg_starts, const int32_t* seg_lens,
                                    int64_t num_slots, int causal, int mode, int q_heads,
                                    int kv_heads, int head_dim, void* host_out,
                                    size_t host_out_bytes, seg_attn_table_desc* desc) {
  if (!desc) return SEG_ATTN_ERR_INVALID_ARG;
  memset(desc, 0, sizeof(*desc));
  if (batch < 0 || (mode != SEG_ATTN_MODE_PREFILL && mode != SEG_ATTN_MODE_DECODE) ||
      (causal != 0 && causal != 1) || num_slots < 0)
    return SEG_ATTN_ERR_INVALID_ARG;
  if (q_heads <= 0 || kv_heads <= 0 || q_heads % kv_heads != 0) return SEG_ATTN_ERR_INVALID_ARG;
  if (batch > 0 && !seg_counts) return SEG_ATTN_ERR_INVALID_ARG;
  if (batch > 0 && mode == SEG_ATTN_MODE_PREFILL && !q_lens) return SEG_ATTN_ERR_INVALID_ARG;
  const int group = q_heads / kv_heads;
  if (head_dim != 64 && head_dim != 128) return SEG_ATTN_ERR_UNSUPPORTED;
  if (!is_pow2(group)) return SEG_ATTN_ERR_UNSUPPORTED;
  if (mode == SEG_ATTN_MODE_PREFILL && group > segattn::kTileRows) return SEG_ATTN_ERR_UNSUPPORTED;
  if (mode == SEG_ATTN_MODE_DECODE && group > 8) return SEG_ATTN_ERR_UNSUPPORTED;
  // the K/V gather addresses pool rows (slot * kv_heads + head) with int32
  if (num_slots * (int64_t)kv_heads > (int64_t)std::numeric_limits<int32_t>::max())
    return SEG_ATTN_ERR_UNSUPPORTED;

  int64_t nseg = 0;
  for (int r = 0; r < batch; ++r) {
    if (seg_counts[r] < 0) return SEG_ATTN_ERR_INVALID_ARG;
    nseg += seg_counts[r];
  }
  if (nseg > std::numeric_limits<int32_t>::max()) return SEG_ATTN_ERR_UNSUPPORTED;
  if (nseg > 0 && (!seg_starts || !seg_lens)) return SEG_ATTN_ERR_INVALID_ARG;

  const int32_t kI32Max = std::numeric_limits<int32_t>::max();
  std::vector<int32_t> ql(batch), kl(batch);
  int64_t total_q = 0, total_k = 0;
  {
    int64_t s0 = 0;
    std::vector<std::pair<int64_t, int64_t>> runs;
    for (int r = 0; r < batch; ++r) {
      const int64_t q = q_lens ? q_lens[r] : 1;
      if (q < 0) return SEG_ATTN_ERR_INVALID_ARG;
      if (mode == SEG_ATTN_MODE_DECODE && q != 1) return SEG_ATTN_ERR_INVALID_ARG;
      int64_t k = 0;
      runs.clear();
      for (int s = 0; s < seg_counts[r]; ++s) {
        const int64_t st = seg_starts[s0 + s], ln = seg_lens[s0 + s];
        if (ln < 0) return SEG_ATTN_ERR_INVALID_ARG;
        if (st < 0 || st + ln > num_slots) return SEG_ATTN_ERR_SEGMENT_OOB;
        k += ln;
        if (ln > 0) runs.emplace_back(st, ln);
      }
      std::sort(runs.begin(), runs.end());
      for (size_t i = 1; i < runs.size(); ++i)
        if (runs[i].first < runs[i - 1].first + runs[i - 1].second)
          return SEG_ATTN_ERR_SEGMENT_OVERLAP;
      if (k > kI32Max) return SEG_ATTN_ERR_UNSUPPORTED;
      if (mode == SEG_ATTN_MODE_PREFILL && causal && q > k) return SEG_ATTN_ERR_QLEN_GT_KLEN;
      ql[r] = (int32_t)q;
      kl[r] = (int32_t)k;
      total_q += q;
      total_k += k;
      s0 += seg_counts[r];
    }
  }
  if (total_q > kI32Max) return SEG_ATTN_ERR_UNSUPPORTED;

  // ---- work plan
  std::vector<int4> work;                      // decode chunks
  std::vector<std::array<int32_t, 8>> pwork;   // prefill pieces
  std::vector<std::array<int32_t, 8>> pmerge;  // prefill items split over several pieces
  std::vector<int32_t> req_chunks;
  int32_t queries_per_tile = 0, chunk_len = 0, max_k_tiles = 0, part_slots = 0;
  if (mode == SEG_ATTN_MODE_PREFILL) {
    queries_per_tile = segattn::kTileRows / group;
    const int32_t span = queries_per_tile * segattn::kTilesPerItem;
    struct Item { int32_t r, g, q0, tiles; };
    std::vector<Item> items;
    for (int r = 0; r < batch; ++r) {
      const int64_t prior = (int64_t)kl[r] - ql[r];
      for (int32_t q0 = 0; q0 < ql[r]; q0 += span) {
        const int64_t q_end = std::min<int64_t>(ql[r], (int64_t)q0 + span);
        const int64_t visible = causal ? std::min<int64_t>(kl[r], prior + q_end) : kl[r];
        const int32_t tiles = (int32_t)((visible + segattn::kTileKeys - 1) / segattn::kTileKeys);
        for (int g = 0; g < kv_heads; ++g) items.push_back({r, g, q0, tiles});
        max_k_tiles = std::max(max_k_tiles, tiles);
      }
    }
    // Each CTA runs one piece (a contiguous range of an item's K tiles).  Pick how
    // far to split long items by simulating the longest-first assignment of pieces
    // to the SMs (what the block scheduler does with a grid in that order) and
    // keeping the factor with the shortest makespan; ties keep fewer splits.
    auto pieces_of = [](int32_t tiles, int f) {
      if (f <= 1 || tiles < 2 * segattn::kMinPieceTiles) return 1;
      return std::min(f, tiles / segattn::kMinPieceTiles);
    };
    auto makespan = [&](int f) {
      std::vector<int64_t> cost;
      for (const Item& it : items) {
        const int p = pieces_of(it.tiles, f);
        for (int j = 0; j < p; ++j)
          cost.push_back((int64_t)it.tiles * (j + 1) / p - (int64_t)it.tiles * j / p +
                         segattn::kPieceOverheadTiles);
      }
      std::sort(cost.begin(), cost.end(), std::greater<int64_t>());
      std::priority_queue<int64_t, std::vector<int64_t>, std::greater<int64_t>> sm;
      for (int i = 0; i < segattn::kSmCount; ++i) sm.push(0);
      int64_t span_max = 0;
      for (int64_t c : cost) {
        const int64_t t = sm.top() + c;
        sm.pop();
        sm.push(t);
        span_max = std::max(span_max, t);
      }
      return span_max;
    };
    int best_f = 1;
    int64_t best = makespan(1);
    for (int f = 2; f <= segattn::kMaxSplit; ++f) {
      const int64_t m = makespan(f);
      if (m * 100 < best * 98) {
        best = m;
        best_f = f;
      }
    }
    for (const Item& it : items) {
      const int p = pieces_of(it.tiles, best_f);
      const int32_t slot0 = p > 1 ? part_slots : -1;
      if (p > 1) {
        pmerge.push_back({it.r, it.g, it.q0, slot0, p, 0, 0, 0});
        part_slots += p;
      }
      for (int j = 0; j < p; ++j) {
        const int32_t kt0 = (int32_t)((int64_t)it.tiles * j / p);
        const int32_t kt1 = (int32_t)((int64_t)it.tiles * (j + 1) / p);
        pwork.push_back({it.r, it.g, it.q0, kt0, kt1, p > 1 ? slot0 + j : -1, 0, 0});
      }
    }
    // longest first; stable keeps (request, query tile, head, piece) order among equals
    std::stable_sort(pwork.begin(), pwork.end(),
                     [](const std::array<int32_t, 8>& a, const std::array<int32_t, 8>& b) {
                       return a[4] - a[3] > b[4] - b[3];
                     });
  } else {
    int64_t L = 2048;
    auto ctas = [&](int64_t len) {
      int64_t n = 0;
      for (int r = 0; r < batch; ++r) n += std::max<int64_t>(1, (kl[r] + len - 1) / len);
      return n * kv_heads;
    };
    while (L > 256 && ctas(L) < 4 * segattn::kSmCount) L /= 2;
    chunk_len = (int32_t)L;
    req_chunks.resize(batch + 1);
    req_chunks[0] = 0;
    for (int r = 0; r < batch; ++r) {
      const int32_t n = (int32_t)std::max<int64_t>(1, (kl[r] + L - 1) / L);
      for (int32_t c = 0; c < n; ++c) {
        const int32_t kb = (int32_t)(c * L);
        const int32_t ke = (int32_t)std::min<int64_t>(kl[r], (int64_t)(c + 1) * L);
        work.push_back(make_int4(r, kb, ke, n));
      }
      req_chunks[r + 1] = req_chunks[r] + n;
    }
  }
  const size_t n_work = mode == SEG_ATTN_MODE_PREFILL ? pwork.size() : work.size();
  if (n_work > (size_t)kI32Max) return SEG_ATTN_ERR_UNSUPPORTED;

  // ---- layout
  Layout lay;
  desc->off_q_offsets = lay.take(batch + 1);
  desc->off_k_lens = lay.take(batch);
  desc->off_seg_offsets = lay.take(batch + 1);
  desc->off_seg_start = lay.take(nseg);
  desc->off_seg_kstart = lay.take(nseg);
  desc->off_seg_len = lay.take(nseg);
  desc->off_work = lay.take((mode == SEG_ATTN_MODE_PREFILL ? 8 : 4) * (int64_t)n_work);
  desc->off_req_chunks = lay.take(mode == SEG_ATTN_MODE_DECODE ? batch + 1 : 0);
  desc->off_merge = lay.take(8 * (int64_t)pmerge.size());

  desc->magic = SEG_ATTN_TABLE_MAGIC;
  desc->version = SEG_ATTN_TABLE_VERSION;
  desc->mode = mode;
  desc->causal = causal;
  desc->batch = batch;
  desc->q_heads = q_heads;
  desc->kv_heads = kv_heads;
  desc->head_dim = head_dim;
  desc->num_slots = num_slots;
  desc->total_q = total_q;
  desc->total_k = total_k;
  desc->num_segments = (int32_t)nseg;
  desc->num_work = (int32_t)n_work;
  desc->num_merge = (int32_t)pmerge.size();
  desc->num_parts = part_slots;
  desc->queries_per_tile = queries_per_tile;
  desc->chunk_len = chunk_len;
  desc->max_k_tiles = max_k_tiles;
  desc->table_bytes = (uint64_t)lay.n * sizeof(int32_t);
  desc->workspace_bytes = 0;
  if (mode == SEG_ATTN_MODE_PREFILL && part_slots > 0)
    desc->workspace_bytes = segattn::prefill_part_o_bytes(part_slots, head_dim) +
                            align_up((size_t)part_slots * segattn::kItemRows * sizeof(float), 256);
  if (mode == SEG_ATTN_MODE_DECODE) {
    bool multi = false;
    for (int r = 0; r < batch; ++r) multi |= (req_chunks[r + 1] - req_chunks[r]) > 1;
    if (multi)
      desc->workspace_bytes = segattn::decode_part_o_bytes(*desc) +
                              align_up((size_t)desc->num_work * q_heads * sizeof(float), 256);
  }

  if (!host_out) return SEG_ATTN_OK;  // size query
  if (host_out_bytes < desc->table_bytes) return SEG_ATTN_ERR_BUFFER_TOO_SMALL;
  if ((reinterpret_cast<uintptr_t>(host_out) & 15) != 0) return SEG_ATTN_ERR_INVALID_ARG;

  int32_t* t = static_cast<int32_t*>(host_out);
  memset(t, 0, desc->table_bytes);
  int32_t* q_off = t + desc->off_q_offsets;
  int32_t* k_len = t + desc->off_k_lens;
  int32_t* s_off = t + desc->off_seg_offsets;
  int32_t* s_start = t + desc->off_seg_start;
  int32_t* s_kstart = t + desc->off_seg_kstart;
  int32_t* s_len = t + desc->off_seg_len;
  q_off[0] = 0;
  s_off[0] = 0;
  int64_t s0 = 0;
  for (int r = 0; r < batch; ++r) {
    q_off[r + 1] = q_off[r] + ql[r];
    k_len[r] = kl[r];
    s_off[r + 1] = (int32_t)(s0 + seg_counts[r]);
    int32_t logical = 0;
    for (int s = 0; s < seg_counts[r]; ++s) {
      s_start[s0 + s] = seg_starts[s0 + s];
      s_len[s0 + s] = seg_lens[s0 + s];
      s_kstart[s0 + s] = logical;
      logical += seg_lens[s0 + s];
    }
    s0 += seg_counts[r];
  }
  if (mode == SEG_ATTN_MODE_PREFILL) {
    for (size_t i = 0; i < pwork.size(); ++i)
      memcpy(t + desc->off_work + 8 * i, pwork[i].data(), 8 * sizeof(int32_t));
    for (size_t i = 0; i < pmerge.size(); ++i)
      memcpy(t + desc->off_merge + 8 * i, pmerge[i].data(), 8 * sizeof(int32_t));
  } else if (!work.empty()) {
    memcpy(t + desc->off_work, work.data(), work.size() * sizeof(int4));
  }
  if (mode == SEG_ATTN_MODE_DECODE)
    memcpy(t + desc->off_req_chunks, req_chunks.data(), req_chunks.size() * sizeof(int32_t));
  return SEG_ATTN_OK;
}

extern "C" size_t seg_attn_workspace_size(const seg_attn_table_desc* desc) {
  if (!desc || desc->magic != SEG_ATTN_TABLE_MAGIC) return 0;
  return (size_t)desc->workspace_bytes;
}

extern "C" const char* seg_attn_status_string(int status) {
  switch (status) {
    case SEG_ATTN_OK: return "ok";
    case SEG_ATTN_ERR_INVALID_ARG: return "invalid argument";
    case SEG_ATTN_ERR_SEGMENT_OOB: return "segment outside the slot pool";
    case SEG_ATTN_ERR_SEGMENT_OVERLAP: return "segments of one request overlap";
    case SEG_ATTN_ERR_QLEN_GT_KLEN: return "causal request has more queries than keys";
    case SEG_ATTN_ERR_WORKSPACE: return "workspace missing or too small";
    case SEG_ATTN_ERR_UNSUPPORTED: return "unsupported shape";
    case SEG_ATTN_ERR_CUDA: return "CUDA error";
    case SEG_ATTN_ERR_BUFFER_TOO_SMALL: return "output buffer too small";
    case SEG_ATTN_ERR_NO_SPACE: return "not enough free slots in the pool";
    default: return "unknown status";
  }
}

extern "C" int seg_attn_version(void) { return 100; }
