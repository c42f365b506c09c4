// Segment allocator for the shared token-slot pool (host only).
//
// Flood manages the KV cache with segmentable blocks instead of fixed pages so
// that each request's cache stays contiguous (Flood README, "Introduction").
// This allocator is that manager: every request ("sequence") owns a short list
// of contiguous slot runs.  Appending tokens first grows the sequence's last
// run in place when the slots right after it are free; whatever does not fit
// there goes to the smallest free run that holds all of it (best fit), or, when
// no single run is large enough, to the largest free runs in turn, so the
// sequence gets as few new segments as possible.  Releasing a sequence returns
// its runs to the free list and merges them with free neighbours.
//
// Free runs are kept twice: by start slot (to find neighbours) and by
// (length, start) (for best fit), both ordered, so every operation is
// O(log runs).  Not thread-safe: callers serialise calls on one pool.
#include <stdint.h>

#include <algorithm>
#include <limits>
#include <map>
#include <new>
#include <set>
#include <unordered_map>
#include <utility>
#include <vector>

#include "seg_attn.h"

struct seg_attn_pool {
  int64_t num_slots = 0;
  int64_t free_slots = 0;
  std::map<int64_t, int64_t> free_by_start;          // start -> length
  std::set<std::pair<int64_t, int64_t>> free_by_len;  // (length, start)
  std::unordered_map<int64_t, std::vector<std::pair<int32_t, int32_t>>> seqs;  // id -> runs

  void add_free(int64_t start, int64_t len) {
    // merge with the free run that ends at `start` and the one that begins at `start + len`
    auto next = free_by_start.lower_bound(start);
    if (next != free_by_start.begin()) {
      auto prev = std::prev(next);
      if (prev->first + prev->second == start) {
        free_by_len.erase({prev->second, prev->first});
        start = prev->first;
        len += prev->second;
        free_by_start.erase(prev);
      }
    }
    next = free_by_start.lower_bound(start + len);
    if (next != free_by_start.end() && next->first == start + len) {
      free_by_len.erase({next->second, next->first});
      len += next->second;
      free_by_start.erase(next);
    }
    free_by_start[start] = len;
    free_by_len.insert({len, start});
  }

  // take `len` slots from the front of the free run that starts at `start`
  void take_front(int64_t start, int64_t len) {
    auto it = free_by_start.find(start);
    const int64_t run = it->second;
    free_by_len.erase({run, start});
    free_by_start.erase(it);
    if (run > len) {
      free_by_start[start + len] = run - len;
      free_by_len.insert({run - len, start + len});
    }
  }
};

namespace {

void append_run(std::vector<std::pair<int32_t, int32_t>>& runs, int64_t start, int64_t len) {
  if (!runs.empty() && (int64_t)runs.back().first + runs.back().second == start)
    runs.back().second += (int32_t)len;  // contiguous with the last run: one segment
  else
    runs.push_back({(int32_t)start, (int32_t)len});
}

}  // namespace

extern "C" int seg_attn_pool_create(int64_t num_slots, seg_attn_pool** out) {
  if (!out || num_slots < 0 || num_slots > (int64_t)INT32_MAX) return SEG_ATTN_ERR_INVALID_ARG;
  *out = nullptr;
  seg_attn_pool* p = new (std::nothrow) seg_attn_pool();
  if (!p) return SEG_ATTN_ERR_NO_SPACE;
  p->num_slots = num_slots;
  if (num_slots > 0) p->add_free(0, num_slots);
  p->free_slots = num_slots;
  *out = p;
  return SEG_ATTN_OK;
}

extern "C" int seg_attn_pool_destroy(seg_attn_pool* pool) {
  delete pool;
  return SEG_ATTN_OK;
}

extern "C" int seg_attn_pool_append(seg_attn_pool* pool, int64_t seq, int64_t n_tokens,
                                    int32_t* new_slots) {
  if (!pool || n_tokens < 0) return SEG_ATTN_ERR_INVALID_ARG;
  if (n_tokens > pool->free_slots) return SEG_ATTN_ERR_NO_SPACE;
  auto& runs = pool->seqs[seq];  // creates the sequence on first use
  int64_t left = n_tokens, written = 0;
  auto emit = [&](int64_t start, int64_t len) {
    if (new_slots)
      for (int64_t i = 0; i < len; ++i) new_slots[written + i] = (int32_t)(start + i);
    written += len;
    append_run(runs, start, len);
  };
  // 1. grow the last run in place
  if (left > 0 && !runs.empty()) {
    const int64_t end = (int64_t)runs.back().first + runs.back().second;
    auto it = pool->free_by_start.find(end);
    if (it != pool->free_by_start.end()) {
      const int64_t take = std::min(left, it->second);
      pool->take_front(end, take);
      emit(end, take);
      left -= take;
    }
  }
  // 2. best fit for the rest, else the largest runs in turn
  while (left > 0) {
    auto fit = pool->free_by_len.lower_bound({left, std::numeric_limits<int64_t>::min()});
    int64_t start, take;
    if (fit != pool->free_by_len.end()) {
      start = fit->second;
      take = left;
    } else {
      auto largest = std::prev(pool->free_by_len.end());
      start = largest->second;
      take = largest->first;
    }
    pool->take_front(start, take);
    emit(start, take);
    left -= take;
  }
  pool->free_slots -= n_tokens;
  return SEG_ATTN_OK;
}

extern "C" int seg_attn_pool_release(seg_attn_pool* pool, int64_t seq) {
  if (!pool) return SEG_ATTN_ERR_INVALID_ARG;
  auto it = pool->seqs.find(seq);
  if (it == pool->seqs.end()) return SEG_ATTN_ERR_INVALID_ARG;
  for (const auto& r : it->second) {
    pool->add_free(r.first, r.second);
    pool->free_slots += r.second;
  }
  pool->seqs.erase(it);
  return SEG_ATTN_OK;
}

extern "C" int seg_attn_pool_segments(const seg_attn_pool* pool, int64_t seq, int32_t* starts,
                                      int32_t* lens, int capacity, int* count) {
  if (!pool || !count || capacity < 0) return SEG_ATTN_ERR_INVALID_ARG;
  auto it = pool->seqs.find(seq);
  if (it == pool->seqs.end()) return SEG_ATTN_ERR_INVALID_ARG;
  const int n = (int)it->second.size();
  *count = n;
  if (n > capacity) return SEG_ATTN_ERR_BUFFER_TOO_SMALL;
  if (n > 0 && (!starts || !lens)) return SEG_ATTN_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    starts[i] = it->second[i].first;
    lens[i] = it->second[i].second;
  }
  return SEG_ATTN_OK;
}

extern "C" int seg_attn_pool_get_stats(const seg_attn_pool* pool, seg_attn_pool_stats* out) {
  if (!pool || !out) return SEG_ATTN_ERR_INVALID_ARG;
  out->num_slots = pool->num_slots;
  out->free_slots = pool->free_slots;
  out->free_runs = (int64_t)pool->free_by_start.size();
  out->largest_free_run = pool->free_by_len.empty() ? 0 : pool->free_by_len.rbegin()->first;
  out->sequences = (int64_t)pool->seqs.size();
  int64_t segs = 0;
  for (const auto& kv : pool->seqs) segs += (int64_t)kv.second.size();
  out->segments = segs;
  return SEG_ATTN_OK;
}
