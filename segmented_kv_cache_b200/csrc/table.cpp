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
// With SEG_ATTN_SHARE_PREFIX (prefix caching, Flood README "Roadmap") it also
// finds requests whose leading keys sit in the same slots and plans one pass of
// the prefill kernel over each shared prefix with all the sharing requests'
// queries, the usual work over each request's remaining keys, and a merge.
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <cmath>
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
using Row8 = std::array<int32_t, 8>;
using Row4 = std::array<int32_t, 4>;
// prefill piece: request, kv head, first query, first K tile | end K tile, partial
// slot (-1: none), one-tile flag, end of the request's segments | first packed query
// row, queries and keys of the request, segment holding the piece's first key | pool
// slot of the piece's first key when its first K tile lies inside that segment (-1:
// it does not), three zero words
constexpr int kWorkInts = 16;
using Row16 = std::array<int32_t, kWorkInts>;

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

// A request's keys as a segment list (start, len) in logical order.
struct Segs {
  std::vector<int32_t> start, len;
  int64_t keys() const {
    int64_t k = 0;
    for (int32_t l : len) k += l;
    return k;
  }
};

// Leading logical keys that two segment lists map to the same slots.
int64_t common_prefix(const Segs& a, const Segs& b) {
  size_t ia = 0, ib = 0;
  int64_t oa = 0, ob = 0, n = 0;
  for (;;) {
    while (ia < a.len.size() && oa >= a.len[ia]) ++ia, oa = 0;
    while (ib < b.len.size() && ob >= b.len[ib]) ++ib, ob = 0;
    if (ia == a.len.size() || ib == b.len.size()) return n;
    if ((int64_t)a.start[ia] + oa != (int64_t)b.start[ib] + ob) return n;
    const int64_t step = std::min<int64_t>(a.len[ia] - oa, b.len[ib] - ob);
    n += step;
    oa += step;
    ob += step;
  }
}

// Keys [from, from + count) of a segment list, as a segment list.
Segs cut(const Segs& s, int64_t from, int64_t count) {
  Segs out;
  int64_t logical = 0;
  for (size_t i = 0; i < s.len.size() && count > 0; ++i) {
    const int64_t lo = std::max<int64_t>(from, logical), hi = logical + s.len[i];
    if (lo < hi) {
      const int64_t take = std::min(hi - lo, count);
      out.start.push_back((int32_t)(s.start[i] + (lo - logical)));
      out.len.push_back((int32_t)take);
      from = lo + take;
      count -= take;
    }
    logical = hi;
  }
  return out;
}

// One prefill item: (request, kv head, query tiles from q0) over `tiles` K tiles.
// `cascade` items write every piece as a partial for the shared-prefix merge;
// `single` items hold queries in their first 128-row query tile only.
struct PItem {
  int32_t r, g, q0, tiles;
  bool cascade, single;
};

struct Pieces {
  std::vector<Row16> work;      // two-tile pieces longest first, then single-tile ones
  std::vector<Row8> merge;      // split items that are not cascade items
  std::vector<int32_t> citem;   // per item: its index in `citems`, or -1
  int32_t slots = 0;            // partial-result slots
  int32_t single = 0;           // single-tile pieces (the tail of `work`)
};

// Cut items into pieces along their K tiles when that shortens the
// longest-first schedule on the SMs.  Each CTA runs one piece; the schedule is
// simulated by assigning pieces longest first to the least loaded SM (what the
// block scheduler does with a grid in that order) and the split factor with the
// shortest makespan wins (ties keep fewer splits).
void plan_pieces(const std::vector<PItem>& items, int max_split, std::vector<Row4>& citems,
                 Pieces& out) {
  auto pieces_of = [](int32_t tiles, int f) {
    if (f <= 1 || tiles < 2 * segattn::kMinPieceTiles) return 1;
    return std::min(f, tiles / segattn::kMinPieceTiles);
  };
  // Longest-first schedule of the pieces on the SMs (each piece costed at its K tiles
  // plus the per-piece start-up and epilogue), for a piece count per item.
  auto makespan = [&](const std::vector<int>& counts) {
    std::vector<int64_t> cost;
    for (size_t i = 0; i < items.size(); ++i) {
      const int64_t t = items[i].tiles;
      const int p = counts[i];
      for (int j = 0; j < p; ++j)
        cost.push_back(t * (j + 1) / p - t * j / p + segattn::kPieceOverheadTiles);
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
  // Candidate plans: every item cut into the same number of pieces f (1 .. max_split),
  // or every item cut into pieces of about L = (all K tiles) / (k waves x SMs) tiles,
  // k = 1 .. 8, so that items of different lengths end in pieces of one length that
  // fill whole waves.  Both respect the shortest piece and the most pieces per item.
  // The plan taken is the one with the fewest pieces among those whose simulated
  // makespan is within 2 % of the best.
  int64_t total_tiles = 0;
  for (const PItem& it : items) total_tiles += it.tiles;
  std::vector<std::vector<int>> cands;
  for (int f = 1; f <= max_split; ++f) {
    std::vector<int> c(items.size());
    for (size_t i = 0; i < items.size(); ++i) c[i] = pieces_of(items[i].tiles, f);
    cands.push_back(std::move(c));
  }
  for (int k = 1; k <= 8 && total_tiles > 0; ++k) {
    const double len = (double)total_tiles / ((double)k * segattn::kSmCount);
    std::vector<int> c(items.size());
    for (size_t i = 0; i < items.size(); ++i) {
      const int32_t t = items[i].tiles;
      if (t < 2 * segattn::kMinPieceTiles) {
        c[i] = 1;
        continue;
      }
      const int want = (int)std::lround((double)t / len);
      c[i] = std::max(1, std::min({want, max_split, (int)(t / segattn::kMinPieceTiles)}));
    }
    cands.push_back(std::move(c));
  }
  std::vector<int64_t> spans(cands.size()), npieces(cands.size(), 0);
  int64_t best_span = INT64_MAX;
  for (size_t j = 0; j < cands.size(); ++j) {
    spans[j] = makespan(cands[j]);
    for (int p : cands[j]) npieces[j] += p;
    best_span = std::min(best_span, spans[j]);
  }
  size_t pick = 0;
  for (size_t j = 0; j < cands.size(); ++j) {
    if (spans[j] * 100 > best_span * 102) continue;
    if (spans[pick] * 100 > best_span * 102 || npieces[j] < npieces[pick] ||
        (npieces[j] == npieces[pick] && spans[j] < spans[pick]))
      pick = j;
  }
  const std::vector<int>& counts = cands[pick];
  // The one-tile kernel runs a pass only when every item of it is single-tile: a
  // second launch for a few single-tile items would serialise behind the first
  // launch's tail (those items then run two-tile, their empty tile's softmax skipped).
  const bool all_single =
      std::all_of(items.begin(), items.end(), [](const PItem& it) { return it.single; });
  out.citem.assign(items.size(), -1);
  for (size_t i = 0; i < items.size(); ++i) {
    PItem it = items[i];
    it.single = all_single;
    const int p = counts[i];
    const bool slotted = p > 1 || it.cascade;
    const int32_t slot0 = slotted ? out.slots : -1;
    if (slotted) out.slots += p;
    if (it.cascade) {
      out.citem[i] = (int32_t)citems.size();
      citems.push_back({slot0, p, it.q0, 0});
    } else if (p > 1) {
      out.merge.push_back({it.r, it.g, it.q0, slot0, p, 0, 0, 0});
    }
    for (int j = 0; j < p; ++j) {
      const int32_t kt0 = (int32_t)((int64_t)it.tiles * j / p);
      const int32_t kt1 = (int32_t)((int64_t)it.tiles * (j + 1) / p);
      out.work.push_back({it.r, it.g, it.q0, kt0, kt1, slotted ? slot0 + j : -1,
                          it.single ? 1 : 0, 0, 0, 0, 0, 0, -1, 0, 0, 0});
      out.single += it.single ? 1 : 0;
    }
  }
  // Two-tile pieces, then single-tile pieces (word 6), each longest first in 16
  // length classes of the longest piece's 1/16; inside a class the pieces that read
  // the same keys (request, kv head, piece of the key range) are adjacent, ordered by
  // query block, so the CTAs running at one time share their K/V tiles through L2
  // instead of each streaming its own range from HBM.
  int32_t max_len = 1;
  for (const Row16& w : out.work) max_len = std::max(max_len, w[4] - w[3]);
  auto cls = [&](const Row16& w) { return (int64_t)(w[4] - w[3]) * 16 / max_len; };
  std::stable_sort(out.work.begin(), out.work.end(), [&](const Row16& a, const Row16& b) {
    if (a[6] != b[6]) return a[6] < b[6];
    if (cls(a) != cls(b)) return cls(a) > cls(b);
    if (a[0] != b[0]) return a[0] < b[0];  // request
    if (a[1] != b[1]) return a[1] < b[1];  // kv head
    if (a[3] != b[3]) return a[3] < b[3];  // first K tile of the piece
    return a[2] < b[2];                    // query block
  });
}

// Fill the per-request words of each piece from the arrays the kernel would
// otherwise read first (saves the dependent table loads at CTA start): end of
// the request's segments, first packed query row, queries, keys, and the
// segment that holds the piece's first key (the last segment whose logical
// start is <= that key, as the device's segment walk finds it).
void fill_request_words(std::vector<Row16>& work, const std::vector<int32_t>& q_off,
                        const std::vector<int32_t>& k_len, const std::vector<Segs>& lists,
                        const std::vector<int32_t>& seg_off) {
  for (Row16& w : work) {
    const int r = w[0];
    const int64_t first_key = (int64_t)w[3] * segattn::kTileKeys;
    int32_t seg = seg_off[r];
    const int32_t seg_end = seg_off[r + 1];
    int64_t kstart_next = seg < seg_end ? lists[r].len[0] : 0;  // logical start of seg + 1
    for (size_t i = 0; seg + 1 < seg_end && kstart_next <= first_key; ++i) {
      ++seg;
      kstart_next += lists[r].len[i + 1];
    }
    w[7] = seg_end;
    w[8] = q_off[r];
    w[9] = q_off[r + 1] - q_off[r];
    w[10] = k_len[r];
    w[11] = seg;
    // the first K tile in one segment: its slot (the producer loads it before
    // anything else of the CTA is set up)
    w[12] = -1;
    if (seg < seg_end && w[4] > w[3]) {
      const int32_t local = seg - seg_off[r];
      const int64_t ks = kstart_next - lists[r].len[local];
      if (first_key + segattn::kTileKeys <= kstart_next && first_key >= ks)
        w[12] = (int32_t)(lists[r].start[local] + (first_key - ks));
    }
  }
}

// Cut the batch into groups of consecutive requests that share a prefix.
// A group [j, i) shares P = min(common prefix of neighbours, cap of each
// member) keys; it saves, per kv head, the K tiles of P that its members would
// have read separately (once per 256-row item each) minus those read once per
// item of the group's packed queries.  Dynamic programme over group ends for
// the largest total saving; on ties the larger last group wins (fewer groups).
std::vector<int32_t> choose_groups(const std::vector<Segs>& segs, const std::vector<int32_t>& ql,
                                   const std::vector<int64_t>& cap, int64_t span,
                                   std::vector<int64_t>& shared_keys) {
  const int B = (int)segs.size();
  std::vector<int64_t> lcp(B, 0);
  for (int r = 1; r < B; ++r) lcp[r] = common_prefix(segs[r - 1], segs[r]);
  auto reads = [&](int64_t q) { return (q + span - 1) / span; };
  std::vector<int64_t> best(B + 1, 0);
  std::vector<int32_t> from(B + 1, 0);
  for (int i = 1; i <= B; ++i) {
    best[i] = best[i - 1];
    from[i] = i - 1;
    int64_t P = cap[i - 1], sum_q = ql[i - 1], sep = reads(ql[i - 1]);
    for (int j = i - 2; j >= 0; --j) {
      P = std::min({P, lcp[j + 1], cap[j]});
      if (P < segattn::kMinSharedKeys) break;
      sum_q += ql[j];
      sep += reads(ql[j]);
      const int64_t tiles = (P + segattn::kTileKeys - 1) / segattn::kTileKeys;
      const int64_t save = (sep - reads(sum_q)) * tiles;
      if (save > 0 && best[j] + save >= best[i]) {
        best[i] = best[j] + save;
        from[i] = j;
      }
    }
  }
  std::vector<int32_t> starts;  // first request of each group, then B
  for (int i = B; i > 0; i = from[i]) starts.push_back(from[i]);
  std::reverse(starts.begin(), starts.end());
  starts.push_back(B);
  shared_keys.assign(starts.size() - 1, 0);
  for (size_t p = 0; p + 1 < starts.size(); ++p) {
    const int j = starts[p], i = starts[p + 1];
    if (i - j < 2) continue;
    int64_t P = cap[j];
    for (int r = j + 1; r < i; ++r) P = std::min({P, lcp[r], cap[r]});
    shared_keys[p] = P;
  }
  return starts;
}

}  // namespace

extern "C" int seg_attn_build_table(int batch, const int32_t* q_lens, const int32_t* seg_counts,
                                    const int32_t* seg_starts, const int32_t* seg_lens,
                                    int64_t num_slots, int causal, int mode_flags, int q_heads,
                                    int kv_heads, int head_dim, void* host_out,
                                    size_t host_out_bytes, seg_attn_table_desc* desc) {
  if (!desc) return SEG_ATTN_ERR_INVALID_ARG;
  memset(desc, 0, sizeof(*desc));
  if ((mode_flags & ~(SEG_ATTN_SHARE_PREFIX | 0xff)) != 0) return SEG_ATTN_ERR_INVALID_ARG;
  const int mode = mode_flags & 0xff;
  const bool want_share = (mode_flags & SEG_ATTN_SHARE_PREFIX) != 0;
  if (batch < 0 || (mode != SEG_ATTN_MODE_PREFILL && mode != SEG_ATTN_MODE_DECODE) ||
      (causal != 0 && causal != 1) || num_slots < 0)
    return SEG_ATTN_ERR_INVALID_ARG;
  if (q_heads <= 0 || kv_heads <= 0 || q_heads % kv_heads != 0) return SEG_ATTN_ERR_INVALID_ARG;
  if (batch > 0 && !seg_counts) return SEG_ATTN_ERR_INVALID_ARG;
  if (batch > 0 && mode == SEG_ATTN_MODE_PREFILL && !q_lens) return SEG_ATTN_ERR_INVALID_ARG;
  const int group = q_heads / kv_heads;
  if (head_dim != 64 && head_dim != 128) return SEG_ATTN_ERR_UNSUPPORTED;
  if (!is_pow2(group)) return SEG_ATTN_ERR_UNSUPPORTED;
  // a prefill query tile packs whole groups; decode packs up to 8 heads per CTA and
  // covers a larger group with group / 8 sibling CTAs (and a shared-prefix decode
  // runs its prefix pass on the prefill kernel)
  if (group > segattn::kTileRows) return SEG_ATTN_ERR_UNSUPPORTED;
  // the K/V gather addresses pool rows (slot * kv_heads + head) with int32
  if (num_slots * (int64_t)kv_heads > (int64_t)std::numeric_limits<int32_t>::max())
    return SEG_ATTN_ERR_UNSUPPORTED;

  int64_t nseg_in = 0;
  for (int r = 0; r < batch; ++r) {
    if (seg_counts[r] < 0) return SEG_ATTN_ERR_INVALID_ARG;
    nseg_in += seg_counts[r];
  }
  if (nseg_in > std::numeric_limits<int32_t>::max()) return SEG_ATTN_ERR_UNSUPPORTED;
  if (nseg_in > 0 && (!seg_starts || !seg_lens)) return SEG_ATTN_ERR_INVALID_ARG;

  const int32_t kI32Max = std::numeric_limits<int32_t>::max();
  std::vector<int32_t> ql(batch), kl(batch);
  std::vector<Segs> segs(batch);
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
        segs[r].start.push_back((int32_t)st);
        segs[r].len.push_back((int32_t)ln);
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
  const int32_t qpt = segattn::kTileRows / group;  // queries per 128-row tile
  const int64_t span = (int64_t)qpt * segattn::kTilesPerItem;

  // ---- shared prefixes: groups of consecutive requests, each request's own keys
  std::vector<int32_t> gstart;   // first request of each group, then batch
  std::vector<int64_t> gkeys;    // shared keys of each group
  std::vector<int32_t> req_group(batch, -1);
  std::vector<int64_t> pre(batch, 0);  // keys request r takes from its group's prefix
  bool shared = false;
  if (want_share && batch > 1) {
    std::vector<int64_t> cap(batch);
    for (int r = 0; r < batch; ++r)
      cap[r] = (mode == SEG_ATTN_MODE_PREFILL && causal) ? (int64_t)kl[r] - ql[r] : kl[r];
    gstart = choose_groups(segs, ql, cap, span, gkeys);
    for (size_t p = 0; p + 1 < gstart.size(); ++p)
      for (int r = gstart[p]; r < gstart[p + 1]; ++r) {
        req_group[r] = (int32_t)p;
        pre[r] = gkeys[p];
        shared |= gkeys[p] > 0;
      }
  }
  // the arrays of the main pass describe each request's keys after its shared prefix
  std::vector<Segs> own(batch);
  std::vector<int32_t> okl(batch);
  for (int r = 0; r < batch; ++r) {
    own[r] = shared && pre[r] > 0 ? cut(segs[r], pre[r], (int64_t)kl[r] - pre[r]) : segs[r];
    okl[r] = (int32_t)(kl[r] - pre[r]);
  }
  int64_t nseg = 0;
  for (int r = 0; r < batch; ++r) nseg += (int64_t)own[r].len.size();
  auto in_shared_group = [&](int r) { return shared && pre[r] > 0; };

  // ---- work plan of the main pass
  std::vector<int4> work;  // decode chunks
  Pieces main_pieces, group_pieces;
  std::vector<Row4> citems;
  std::vector<int32_t> req_chunks, main_citem;  // main_citem: first cascade item of (r, q0 block)
  int32_t chunk_len = 0, max_k_tiles = 0;
  std::vector<int64_t> main_item_base(batch, -1);
  if (mode == SEG_ATTN_MODE_PREFILL) {
    std::vector<PItem> items;
    for (int r = 0; r < batch; ++r) {
      const int64_t prior = (int64_t)okl[r] - ql[r];
      main_item_base[r] = (int64_t)items.size();
      for (int32_t q0 = 0; q0 < ql[r]; q0 += (int32_t)span) {
        const int64_t q_end = std::min<int64_t>(ql[r], (int64_t)q0 + span);
        const int64_t visible = causal ? std::min<int64_t>(okl[r], prior + q_end) : okl[r];
        const int32_t tiles = (int32_t)((visible + segattn::kTileKeys - 1) / segattn::kTileKeys);
        const bool single = ql[r] - q0 <= qpt;
        for (int g = 0; g < kv_heads; ++g)
          items.push_back({r, g, q0, tiles, in_shared_group(r), single});
        max_k_tiles = std::max(max_k_tiles, tiles);
      }
    }
    plan_pieces(items, segattn::kMaxSplit, citems, main_pieces);
    main_citem = main_pieces.citem;
  } else {
    int64_t L = 4096;
    const int64_t slices = group > 8 ? group / 8 : 1;  // CTAs per (chunk, kv head)
    auto ctas = [&](int64_t len) {
      int64_t n = 0;
      for (int r = 0; r < batch; ++r) n += std::max<int64_t>(1, (okl[r] + len - 1) / len);
      return n * kv_heads * slices;
    };
    while (L > 256 && ctas(L) < segattn::kDecodeTargetCtas) L /= 2;
    chunk_len = (int32_t)L;
    req_chunks.resize(batch + 1);
    req_chunks[0] = 0;
    for (int r = 0; r < batch; ++r) {
      const int32_t n = (int32_t)std::max<int64_t>(1, (okl[r] + L - 1) / L);
      for (int32_t c = 0; c < n; ++c) {
        const int32_t kb = (int32_t)(c * L);
        const int32_t ke = (int32_t)std::min<int64_t>(okl[r], (int64_t)(c + 1) * L);
        // chunk count 0 marks a request whose result the cascade merge completes
        work.push_back(make_int4(r, kb, ke, in_shared_group(r) ? 0 : n));
      }
      req_chunks[r + 1] = req_chunks[r] + n;
    }
  }
  const size_t n_work = mode == SEG_ATTN_MODE_PREFILL ? main_pieces.work.size() : work.size();
  // decode launches n_work * (group / 8) CTAs along the grid's x dimension
  const size_t grid_x = n_work * (mode == SEG_ATTN_MODE_DECODE && group > 8 ? group / 8 : 1);
  if (grid_x > (size_t)kI32Max) return SEG_ATTN_ERR_UNSUPPORTED;

  // ---- shared-prefix pass and cascade rows
  std::vector<int32_t> gq_off, greq;      // per group: first query row, first request
  std::vector<Segs> gsegs;
  std::vector<int64_t> group_item_base;   // first item of each group's prefix pass
  std::vector<Row8> cascade;
  int64_t group_total_k = 0, ngseg = 0;
  if (shared) {
    const int ng = (int)gstart.size() - 1;
    gq_off.assign(ng + 1, 0);
    greq.assign(gstart.begin(), gstart.end());
    gsegs.resize(ng);
    group_item_base.assign(ng, -1);
    std::vector<int64_t> q_off(batch + 1, 0);
    for (int r = 0; r < batch; ++r) q_off[r + 1] = q_off[r] + ql[r];
    std::vector<PItem> items;
    for (int p = 0; p < ng; ++p) {
      gq_off[p] = (int32_t)q_off[gstart[p]];
      const int64_t gq = q_off[gstart[p + 1]] - q_off[gstart[p]];
      if (gkeys[p] > 0) {
        gsegs[p] = cut(segs[gstart[p]], 0, gkeys[p]);
        group_total_k += gkeys[p];
        group_item_base[p] = (int64_t)items.size();
        const int32_t tiles = (int32_t)((gkeys[p] + segattn::kTileKeys - 1) / segattn::kTileKeys);
        for (int32_t q0 = 0; q0 < gq; q0 += (int32_t)span)
          for (int g = 0; g < kv_heads; ++g) items.push_back({p, g, q0, tiles, true, gq - q0 <= qpt});
      }
      ngseg += (int64_t)gsegs[p].len.size();
    }
    gq_off[ng] = (int32_t)total_q;
    // the prefix passes are short and few: allow more pieces so they fill the SMs
    plan_pieces(items, segattn::kMaxGroupSplit, citems, group_pieces);
    if (group_pieces.work.size() > (size_t)kI32Max) return SEG_ATTN_ERR_UNSUPPORTED;
    // rows the cascade merge completes (citem of kv head g = the listed one + g)
    for (int r = 0; r < batch; ++r) {
      const int p = req_group[r];
      const bool pre_r = gkeys[p] > 0;
      if (mode == SEG_ATTN_MODE_DECODE) {
        if (!pre_r && req_chunks[r + 1] - req_chunks[r] == 1) continue;
        int32_t pc = -1, pl = 0;
        if (pre_r) {
          pl = (int32_t)(r - gstart[p]);
          pc = group_pieces.citem[group_item_base[p] + (pl / span) * kv_heads];
        }
        cascade.push_back({r, r, pc, pl, -1, 0, 0, 0});
      } else if (pre_r) {
        for (int32_t i = 0; i < ql[r]; ++i) {
          const int64_t row = q_off[r] + i;
          const int32_t pl = (int32_t)(row - gq_off[p]);
          const int32_t pc = group_pieces.citem[group_item_base[p] + (pl / span) * kv_heads];
          const int32_t sc = main_citem[main_item_base[r] + (i / span) * kv_heads];
          cascade.push_back({(int32_t)row, r, pc, pl, sc, i, 0, 0});
        }
      }
    }
    if (cascade.size() > (size_t)kI32Max) return SEG_ATTN_ERR_UNSUPPORTED;
  }

  // ---- layout
  Layout lay;
  desc->off_q_offsets = lay.take(batch + 1);
  desc->off_k_lens = lay.take(batch);
  desc->off_seg_offsets = lay.take(batch + 1);
  desc->off_seg_start = lay.take(nseg);
  desc->off_seg_kstart = lay.take(nseg);
  desc->off_seg_len = lay.take(nseg);
  desc->off_work = lay.take((mode == SEG_ATTN_MODE_PREFILL ? kWorkInts : 4) * (int64_t)n_work);
  desc->off_req_chunks = lay.take(mode == SEG_ATTN_MODE_DECODE ? batch + 1 : 0);
  desc->off_merge = lay.take(8 * (int64_t)main_pieces.merge.size());
  const int ng = shared ? (int)gstart.size() - 1 : 0;
  desc->off_group_req = lay.take(shared ? ng + 1 : 0);
  desc->off_group_q_offsets = lay.take(shared ? ng + 1 : 0);
  desc->off_group_k_lens = lay.take(ng);
  desc->off_group_seg_offsets = lay.take(shared ? ng + 1 : 0);
  desc->off_group_seg_start = lay.take(ngseg);
  desc->off_group_seg_kstart = lay.take(ngseg);
  desc->off_group_seg_len = lay.take(ngseg);
  desc->off_group_work = lay.take(kWorkInts * (int64_t)group_pieces.work.size());
  desc->off_citem = lay.take(4 * (int64_t)citems.size());
  desc->off_cascade = lay.take(8 * (int64_t)cascade.size());

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
  desc->num_merge = (int32_t)main_pieces.merge.size();
  desc->num_parts = main_pieces.slots;
  desc->shared = shared ? 1 : 0;
  desc->queries_per_tile = mode == SEG_ATTN_MODE_PREFILL || shared ? qpt : 0;
  desc->chunk_len = chunk_len;
  desc->max_k_tiles = max_k_tiles;
  desc->num_groups = ng;
  desc->num_group_segments = (int32_t)ngseg;
  desc->num_group_work = (int32_t)group_pieces.work.size();
  desc->num_group_parts = group_pieces.slots;
  desc->num_citems = (int32_t)citems.size();
  desc->num_cascade = (int32_t)cascade.size();
  desc->num_single = main_pieces.single;
  desc->num_group_single = group_pieces.single;
  desc->group_total_k = group_total_k;
  desc->table_bytes = (uint64_t)lay.n * sizeof(int32_t);
  desc->workspace_bytes = segattn::workspace_layout(*desc, [&] {
    if (mode != SEG_ATTN_MODE_DECODE) return false;
    for (int r = 0; r < batch; ++r)
      if (req_chunks[r + 1] - req_chunks[r] > 1) return true;
    return false;
  }()).total;

  if (!host_out) return SEG_ATTN_OK;  // size query
  if (host_out_bytes < desc->table_bytes) return SEG_ATTN_ERR_BUFFER_TOO_SMALL;
  if ((reinterpret_cast<uintptr_t>(host_out) & 15) != 0) return SEG_ATTN_ERR_INVALID_ARG;

  int32_t* t = static_cast<int32_t*>(host_out);
  memset(t, 0, desc->table_bytes);
  auto write_csr = [&](const std::vector<Segs>& lists, int32_t* s_off, int32_t* s_start,
                       int32_t* s_kstart, int32_t* s_len) {
    int32_t s0 = 0;
    s_off[0] = 0;
    for (size_t r = 0; r < lists.size(); ++r) {
      int32_t logical = 0;
      for (size_t s = 0; s < lists[r].len.size(); ++s, ++s0) {
        s_start[s0] = lists[r].start[s];
        s_len[s0] = lists[r].len[s];
        s_kstart[s0] = logical;
        logical += lists[r].len[s];
      }
      s_off[r + 1] = s0;
    }
  };
  int32_t* q_off = t + desc->off_q_offsets;
  int32_t* k_len = t + desc->off_k_lens;
  q_off[0] = 0;
  for (int r = 0; r < batch; ++r) {
    q_off[r + 1] = q_off[r] + ql[r];
    k_len[r] = okl[r];
  }
  write_csr(own, t + desc->off_seg_offsets, t + desc->off_seg_start, t + desc->off_seg_kstart,
            t + desc->off_seg_len);
  auto put_rows = [&](int64_t off, const auto& rows) {
    for (size_t i = 0; i < rows.size(); ++i)
      memcpy(t + off + rows[i].size() * i, rows[i].data(), rows[i].size() * sizeof(int32_t));
  };
  auto csr_offsets = [](const std::vector<Segs>& lists) {
    std::vector<int32_t> off(lists.size() + 1, 0);
    for (size_t r = 0; r < lists.size(); ++r) off[r + 1] = off[r] + (int32_t)lists[r].len.size();
    return off;
  };
  if (mode == SEG_ATTN_MODE_PREFILL) {
    std::vector<int32_t> qo(batch + 1, 0);
    for (int r = 0; r < batch; ++r) qo[r + 1] = qo[r] + ql[r];
    fill_request_words(main_pieces.work, qo, okl, own, csr_offsets(own));
    put_rows(desc->off_work, main_pieces.work);
    put_rows(desc->off_merge, main_pieces.merge);
  } else {
    if (!work.empty()) memcpy(t + desc->off_work, work.data(), work.size() * sizeof(int4));
    memcpy(t + desc->off_req_chunks, req_chunks.data(), req_chunks.size() * sizeof(int32_t));
  }
  if (shared) {
    memcpy(t + desc->off_group_req, greq.data(), greq.size() * sizeof(int32_t));
    memcpy(t + desc->off_group_q_offsets, gq_off.data(), gq_off.size() * sizeof(int32_t));
    for (int p = 0; p < ng; ++p) t[desc->off_group_k_lens + p] = (int32_t)gkeys[p];
    write_csr(gsegs, t + desc->off_group_seg_offsets, t + desc->off_group_seg_start,
              t + desc->off_group_seg_kstart, t + desc->off_group_seg_len);
    std::vector<int32_t> gk(ng);
    for (int p = 0; p < ng; ++p) gk[p] = (int32_t)gkeys[p];
    fill_request_words(group_pieces.work, gq_off, gk, gsegs, csr_offsets(gsegs));
    put_rows(desc->off_group_work, group_pieces.work);
    put_rows(desc->off_citem, citems);
    put_rows(desc->off_cascade, cascade);
  }
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
