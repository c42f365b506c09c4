/*
 * seg_attn.h -- C ABI of the B200 (sm_100a) SegmentAttention library.
 *
 * SegmentAttention is exact causal / variable-length / grouped-query softmax
 * attention over a *segmentable* KV cache (Flood README, "Introduction":
 * the cache is managed in segmentable blocks instead of paged blocks, which
 * keeps each request's cache contiguous; SegmentAttention is the attention
 * kernel written for that cache).  Each request's keys and values live in a
 * shared token-slot pool as a short list of contiguous runs (slot_start, len).
 * The same library serves chunked prefill (Flood README feature list: a chunk
 * of new queries attends to the prior context plus itself) and decode (one
 * query per request over its whole context; README "Kernels > Seg-attn",
 * batch 128, Q_len 1 rows).
 *
 * Math (per request r, query i, query head h):
 *   g = h / (q_heads / kv_heads)                      (contiguous GQA groups)
 *   logical key j of r lives in slot  seg_start[s] + (j - off_s), where
 *   off_s is the sum of the lengths listed before segment s (list order is
 *   logical order; slot order is irrelevant).
 *   causal: query i sees keys j <= (k_len - q_len) + i  (bottom-right aligned)
 *   s_j = scale * <q[i,h,:], K[slot(j), g, :]>
 *   out[i,h,:] = sum_j softmax(s)_j V[slot(j), g, :]
 *   lse[i,h]   = ln sum_j exp(s_j)                   (natural log, scale included)
 *   A query that sees no key gets out = 0 and lse = -inf.
 * Kernels use the online-softmax state (running max m_i, normaliser l_i) of
 * FlashAttention, described in the Ascend FlashAttention article, section
 * "bottleneck 2"; the decode split over key blocks with a per-request
 * reduction follows the per-block partial attention + per-request reduce of
 * the FlashAccel article, section "data layout optimisation".
 *
 * Conventions for every entry point:
 *   - The caller owns every buffer.  The library never allocates or frees
 *     memory and never synchronises the device.
 *   - Tensors are dense, row-major, 16-byte aligned:
 *       q, out   bf16 [total_q, q_heads, head_dim]   (requests packed in order)
 *       k_pool, v_pool  bf16 [num_slots, kv_heads, head_dim]
 *       lse      fp32 [total_q, q_heads]  (may be NULL)
 *   - The new tokens' K/V rows are already written into the pool: they are
 *     the last q_len logical keys of each request's segment list.
 *   - Supported shapes: head_dim in {64, 128}; q_heads % kv_heads == 0;
 *     group size q_heads/kv_heads a power of two <= 128 (prefill and decode).
 *   - Errors are returned synchronously as a negative seg_attn_status before
 *     anything is launched; nothing is launched on error.  A launch failure
 *     is reported as SEG_ATTN_ERR_CUDA.  Device code never traps.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 */
#ifndef SEG_ATTN_H_
#define SEG_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SEG_ATTN_OK = 0,
  SEG_ATTN_ERR_INVALID_ARG = -1,       /* bad pointer, size, shape or flag */
  SEG_ATTN_ERR_SEGMENT_OOB = -2,       /* a segment reaches outside [0, num_slots) */
  SEG_ATTN_ERR_SEGMENT_OVERLAP = -3,   /* two segments of one request share a slot */
  SEG_ATTN_ERR_QLEN_GT_KLEN = -4,      /* causal request with more queries than keys */
  SEG_ATTN_ERR_WORKSPACE = -5,         /* workspace missing or smaller than needed */
  SEG_ATTN_ERR_UNSUPPORTED = -6,       /* valid but outside the supported shapes */
  SEG_ATTN_ERR_CUDA = -7,              /* a CUDA runtime / driver call failed */
  SEG_ATTN_ERR_BUFFER_TOO_SMALL = -8,  /* output buffer smaller than needed */
  SEG_ATTN_ERR_NO_SPACE = -9           /* the slot pool has too few free slots */
} seg_attn_status;

enum { SEG_ATTN_MODE_PREFILL = 0, SEG_ATTN_MODE_DECODE = 1 };

/* OR-ed into the mode argument of seg_attn_build_table: plan shared prefixes
 * (see seg_attn_build_table). */
#define SEG_ATTN_SHARE_PREFIX 0x100

#define SEG_ATTN_TABLE_MAGIC 0x53454741u /* "SEGA" */
#define SEG_ATTN_TABLE_VERSION 5u

/*
 * Description of a built segment table.  Filled by seg_attn_build_table; the
 * caller passes it back unchanged to the compute calls.  Offsets count int32
 * elements from the start of the table buffer.
 */
typedef struct seg_attn_table_desc {
  uint32_t magic, version;
  int32_t mode, causal;
  int32_t batch, q_heads, kv_heads, head_dim;
  int64_t num_slots;
  int64_t total_q;         /* sum of q_lens = rows of q / out */
  int64_t total_k;         /* sum of k_lens */
  int32_t num_segments;
  int32_t num_work;        /* prefill: (request, kv head, query-tile pair, key range) items;
                              decode: chunks */
  int32_t queries_per_tile;/* prefill: 128 / group size */
  int32_t chunk_len;       /* decode: logical keys per split-K chunk */
  int32_t max_k_tiles;     /* prefill: largest number of 128-key tiles of one item */
  int32_t num_merge;       /* prefill: items whose key range was split over several CTAs */
  int32_t num_parts;       /* prefill: partial-result slots (split items, and every item of
                              a request in a shared-prefix group) */
  int32_t shared;          /* 1: a shared-prefix plan is present (fields below) */
  int64_t off_q_offsets;   /* [batch+1] packed query offset of each request */
  int64_t off_k_lens;      /* [batch]   keys of each request */
  int64_t off_seg_offsets; /* [batch+1] first segment of each request */
  int64_t off_seg_start;   /* [num_segments] first slot of each segment */
  int64_t off_seg_kstart;  /* [num_segments] logical index of each segment's first key */
  int64_t off_seg_len;     /* [num_segments] */
  int64_t off_work;        /* work items, 16-byte aligned: decode [num_work][4],
                              prefill [num_work][16] */
  int64_t off_req_chunks;  /* decode: [batch+1] first chunk of each request */
  int64_t off_merge;       /* prefill: [num_merge][8] split items and their partial slots */
  uint64_t table_bytes;    /* size of the table buffer */
  uint64_t workspace_bytes;/* device scratch the compute call needs (may be 0) */
  /* Shared-prefix plan (shared == 1).  Requests are cut into groups of
     consecutive requests; group p's members map their first P_p logical keys
     to the same slots.  The arrays above then describe each request's keys
     from P_p on (its suffix); the group arrays below describe the shared
     prefixes, one pseudo-request per group whose queries are all its
     members' queries.  A request that shares nothing is a group of its own
     with P = 0. */
  int32_t num_groups;
  int32_t num_group_segments;
  int32_t num_group_work;  /* prefill-kernel pieces over the shared prefixes */
  int32_t num_group_parts; /* partial-result slots of those pieces */
  int32_t num_citems;      /* items whose pieces write partials for the cascade merge */
  int32_t num_cascade;     /* output rows (prefill: tokens, decode: requests) merged by it */
  int32_t num_single;      /* prefill: the last num_single work items hold queries in their
                              first 128-row tile only (they run a one-tile kernel) */
  int32_t num_group_single;/* the same for the pieces of the shared-prefix pass */
  int64_t group_total_k;   /* sum of P_p */
  int64_t off_group_req;        /* [num_groups+1] first request of each group */
  int64_t off_group_q_offsets;  /* [num_groups+1] first query (packed row) of each group */
  int64_t off_group_k_lens;     /* [num_groups] P_p */
  int64_t off_group_seg_offsets;/* [num_groups+1] */
  int64_t off_group_seg_start;  /* [num_group_segments] */
  int64_t off_group_seg_kstart; /* [num_group_segments] */
  int64_t off_group_seg_len;    /* [num_group_segments] */
  int64_t off_group_work;       /* [num_group_work][16] */
  int64_t off_citem;            /* [num_citems][4] first slot, pieces, first query of the item */
  int64_t off_cascade;          /* [num_cascade][8] row, request, prefix item, row in group,
                                   suffix item, row in request */
} seg_attn_table_desc;

/*
 * seg_attn_build_table -- validate per-request segment lists and lay out the
 * table (CSR segment arrays + the kernel work list) in host memory.
 *
 *   batch                 number of requests (>= 0)
 *   q_lens [batch]        new queries per request (>= 0); NULL in decode mode
 *                         means 1 each; decode requires every q_len == 1
 *   seg_counts [batch]    segments per request (>= 0)
 *   seg_starts, seg_lens  [sum seg_counts] first slot and length (>= 0) of each
 *                         segment, requests back to back, logical order
 *   num_slots             pool rows; every segment must lie in [0, num_slots)
 *   causal                1 = bottom-right causal mask, 0 = none (decode
 *                         always sees every key of the request)
 *   mode                  SEG_ATTN_MODE_PREFILL or SEG_ATTN_MODE_DECODE, optionally
 *                         OR-ed with SEG_ATTN_SHARE_PREFIX
 *   q_heads, kv_heads, head_dim   shapes as above
 *   host_out, host_out_bytes      destination (any alignment >= 16 bytes);
 *                         pass host_out = NULL to only fill desc (size query)
 *   desc                  out: table description
 *
 * Segments of different requests may share slots (read-only prefix sharing);
 * segments of one request may not.
 *
 * SEG_ATTN_SHARE_PREFIX (prefix caching, Flood README "Roadmap"): the builder
 * finds, for each pair of neighbouring requests, how many leading logical keys
 * they map to the same slots, and cuts the batch into groups of consecutive
 * requests so that the number of K/V tiles read is smallest (a group's common
 * prefix is read once per 256 packed query rows instead of once per request;
 * prefixes shorter than 256 keys are not shared; a causal prefill prefix
 * stops where a member's new tokens begin).  The compute call then runs the
 * tensor-core prefill kernel over each shared prefix with all the group's
 * queries, the usual kernel over each request's remaining keys, and a merge of
 * the two partial results by their log-sum-exp; the results equal the
 * unshared computation up to fp32 rounding.  Callers that want sharing order
 * requests with common prefixes next to each other.  When no group shares
 * anything the table is the plain one (desc->shared = 0).
 * Returns SEG_ATTN_OK or a negative status;
 * on SEG_ATTN_ERR_BUFFER_TOO_SMALL desc->table_bytes holds the needed size.
 * Host only: touches no device state.  The caller copies table_bytes of
 * host_out to device memory (16-byte aligned) and passes that copy as
 * dev_table below.
 */
int seg_attn_build_table(int batch, const int32_t* q_lens, const int32_t* seg_counts,
                         const int32_t* seg_starts, const int32_t* seg_lens, int64_t num_slots,
                         int causal, int mode, int q_heads, int kv_heads, int head_dim,
                         void* host_out, size_t host_out_bytes, seg_attn_table_desc* desc);

/* Device workspace (bytes) the compute call for this table needs; 0 if none. */
size_t seg_attn_workspace_size(const seg_attn_table_desc* desc);

/*
 * seg_attn_prefill -- chunked-prefill attention (mode PREFILL table): a chunk
 * of new queries per request over its prior context plus itself (Flood README,
 * feature list: chunked prefill; the Q_len = K_len = 1024 rows of its
 * "Kernels > Seg-attn" table are the one-chunk case).  One sm_100a kernel
 * launch per pass (plus a merge kernel when long items are split): K/V tiles
 * of 128 logical keys are gathered from the pool with TMA, S = QK^T and
 * O += PV run on the tcgen05 tensor cores with accumulators in tensor memory,
 * the online softmax runs in registers.  Writes out (and lse if non-NULL) for
 * every row.
 *   softmax_scale  > 0 and finite (typically 1/sqrt(head_dim))
 *   workspace      device memory of at least seg_attn_workspace_size(desc)
 *                  bytes, 16-byte aligned, when that size is non-zero: the
 *                  planner splits the key range of long items over several
 *                  CTAs when that balances the grid, and their fp32 partials
 *                  are merged by a second kernel (contents are scratch)
 */
int seg_attn_prefill(const void* q, const void* k_pool, const void* v_pool, void* out, float* lse,
                     const void* dev_table, const seg_attn_table_desc* desc, float softmax_scale,
                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * seg_attn_decode -- one query per request over its whole context (mode
 * DECODE table; the Q_len = 1 rows of the Flood README "Kernels > Seg-attn"
 * table).  Split-K over chunks of logical keys, each chunk a partial attention
 * reduced per request afterwards (FlashAccel article, "data layout
 * optimisation"): one CTA per (chunk, kv head, slice of up to 8 query heads)
 * streams K/V with 128-bit loads, packs the slice's query heads so each K/V
 * byte fetched serves all of them, and keeps the softmax state in registers;
 * a second kernel merges the per-chunk partials by their log-sum-exp.
 * workspace: device memory of at least seg_attn_workspace_size(desc) bytes,
 * 16-byte aligned (contents are scratch).
 */
int seg_attn_decode(const void* q, const void* k_pool, const void* v_pool, void* out, float* lse,
                    const void* dev_table, const seg_attn_table_desc* desc, float softmax_scale,
                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * seg_attn_take_device_error -- read and clear the library's device error
 * word.  Kernels never trap; every wait on an mbarrier gives up after one
 * second, and a CTA that gave up drains its copies, frees its tensor memory,
 * returns, and sets bit 0 of this word (its output rows are then undefined);
 * seg_attn_kv_append sets bit 1 (value 2) for a slot out of range; a
 * segment linear attention prefill kernel (seg_la.h) that gave up sets bit 2
 * (value 4).  Synchronous: copies from the device (implicitly synchronises
 * the current device).  *value = 0 means no kernel gave up since the last call.
 */
int seg_attn_take_device_error(int* value);

/*
 * seg_attn_wait_selftest -- diagnostic (no counterpart on the source pages):
 * launches one warp on `stream` that waits, with the bounded wait every kernel
 * of this library uses, on an mbarrier nothing ever arrives on.  The wait gives
 * up after wait_us microseconds (1 .. 1000000) and sets bit 0 of the device
 * error word, which seg_attn_take_device_error then reports; the GPU context
 * stays usable.  For checking that a stalled kernel surfaces as an error
 * status instead of a hang.  wait_us out of range: SEG_ATTN_ERR_INVALID_ARG.
 */
int seg_attn_wait_selftest(int wait_us, void* stream);

/*
 * seg_attn_stall_test -- diagnostic (no counterpart on the source pages):
 * makes later prefill launches stall the way a copy that never lands would,
 * so that the kernel's give-up path can be exercised without a GPU fault.
 *   withhold_k_tile >= 0: the producer warp of every CTA whose piece has more
 *                  K tiles than that stops loading before that K tile; the
 *                  tensor-core and softmax warps then wait for it, give up
 *                  after wait_us, drain the copies and MMAs already issued,
 *                  free tensor memory and set bit 0 of the device error word
 *                  (the CTA's output rows are left unwritten).
 *   withhold_k_tile < 0: off (the default).
 *   wait_us        limit of every bounded wait of later prefill launches,
 *                  1 .. 1000000 (default 1000000, i.e. one second).
 * Host-side settings read at each launch (process-wide, not thread-safe with
 * concurrent prefill calls).  seg_attn_stall_test(-1, 1000000) restores the
 * defaults.  wait_us out of range: SEG_ATTN_ERR_INVALID_ARG.
 */
int seg_attn_stall_test(int withhold_k_tile, int wait_us);

/*
 * seg_attn_order_test -- diagnostic (no counterpart on the source pages): every
 * softmax warp of a one-query-tile item (a short chunk, a pass over shared
 * prefixes) in later prefill launches sleeps about delay_ns nanoseconds right
 * after it signals P of the item's last K tile, so the last P.V product has
 * completed before the warp waits for it at the end of the item -- the order a
 * slow warp meets there (an instruction-cache miss, a profiler's
 * instrumentation).  Results must not change and no wait may give up.
 *   delay_ns       0 .. 1000000; 0 is off (the default).
 * Host-side setting read at each launch (process-wide, not thread-safe with
 * concurrent prefill calls).  delay_ns out of range: SEG_ATTN_ERR_INVALID_ARG.
 */
int seg_attn_order_test(int delay_ns);

/*
 * seg_attn_decode_noalloc -- seg_attn_decode for callers that cannot allocate
 * device memory (no counterpart on the source pages; this is a library
 * convenience).  Typical callers: a plugin inside another runtime that owns
 * all device memory and offers no allocator, or a serving loop that must not
 * call cudaMalloc after start-up because it can synchronise the device.
 *
 * Same arguments and results as seg_attn_decode, minus the workspace: the
 * split-K scratch is a fixed 64 MiB device array inside the library, which
 * every GPU that loads the library keeps until the process exits.
 *   - Returns SEG_ATTN_ERR_WORKSPACE, launching nothing, when the table needs
 *     more than 64 MiB of scratch (seg_attn_workspace_size(desc) > 64 MiB).
 *   - All calls share the array and it keeps the last call's contents; no
 *     part of it needs to start at zero.  Calls that overlap on the GPU (other
 *     streams or host threads) race on it: order them, e.g. on one stream.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before starting any stream capture.  The address is remembered for the
 *     life of the process: after cudaDeviceReset (or anything else that
 *     destroys the device's primary context) the library's module is loaded
 *     again and the array may sit elsewhere, so do not call this entry point
 *     on that device again in the same process.
 *   - Calls no cudaMalloc, cudaFree or other allocating routine.
 */
int seg_attn_decode_noalloc(const void* q, const void* k_pool, const void* v_pool, void* out,
                            float* lse, const void* dev_table, const seg_attn_table_desc* desc,
                            float softmax_scale, void* stream);

/* ------------------------------------------------------------------------
 * Segment allocator (host) and KV append (device).
 *
 * The cache manager behind the tables: each sequence (request) owns a short
 * list of contiguous slot runs of the pool, as in Flood's segmentable KV cache
 * (Flood README, "Introduction": segmentable blocks instead of paged blocks,
 * for contiguity).  Appending n tokens to a sequence first grows its last run
 * in place when the slots right after it are free; the rest goes to the
 * smallest free run that holds all of it (ties: lowest start), or, when no
 * free run is large enough, to the largest free runs in turn (ties: highest
 * start) -- so a sequence keeps as few segments as possible.  Releasing a
 * sequence returns its runs to the free list, merged with free neighbours.
 * The pool object is host memory only; it is not thread-safe.
 * ---------------------------------------------------------------------- */
typedef struct seg_attn_pool seg_attn_pool;

typedef struct seg_attn_pool_stats {
  int64_t num_slots, free_slots;
  int64_t free_runs, largest_free_run;
  int64_t sequences, segments;
} seg_attn_pool_stats;

/* New pool of num_slots slots (0 <= num_slots <= INT32_MAX), all free. */
int seg_attn_pool_create(int64_t num_slots, seg_attn_pool** out);
int seg_attn_pool_destroy(seg_attn_pool* pool);

/*
 * Append n_tokens slots to sequence `seq` (created on first use).  On success
 * new_slots[i] (if non-NULL, [n_tokens]) is the slot of the i-th new token,
 * in logical order.  SEG_ATTN_ERR_NO_SPACE (pool unchanged) when fewer than
 * n_tokens slots are free.
 */
int seg_attn_pool_append(seg_attn_pool* pool, int64_t seq, int64_t n_tokens, int32_t* new_slots);

/* Return every slot of `seq` to the pool and forget the sequence. */
int seg_attn_pool_release(seg_attn_pool* pool, int64_t seq);

/*
 * Segment list of `seq` in logical order -- the (start, length) input of
 * seg_attn_build_table.  *count is always set; SEG_ATTN_ERR_BUFFER_TOO_SMALL
 * when it exceeds capacity.
 */
int seg_attn_pool_segments(const seg_attn_pool* pool, int64_t seq, int32_t* starts, int32_t* lens,
                           int capacity, int* count);

int seg_attn_pool_get_stats(const seg_attn_pool* pool, seg_attn_pool_stats* out);

/*
 * seg_attn_kv_append -- write the K/V rows of new tokens into their pool slots.
 *   k_new, v_new   bf16 [n_tokens, kv_heads, head_dim] (device, 16-byte aligned)
 *   slots          int32 [n_tokens] device array, slot of each token
 *   k_pool, v_pool bf16 [num_slots, kv_heads, head_dim] (device)
 * A slot outside [0, num_slots) is skipped and recorded in the device error
 * word (value 2, see seg_attn_take_device_error); nothing is written out of
 * bounds.  kv_heads * head_dim * 2 must be a multiple of 16 bytes.
 */
int seg_attn_kv_append(const void* k_new, const void* v_new, const int32_t* slots,
                       int64_t n_tokens, int kv_heads, int head_dim, void* k_pool, void* v_pool,
                       int64_t num_slots, void* stream);

/*
 * seg_attn_decode_fp8 -- seg_attn_decode over an FP8 KV cache (Flood README,
 * "Roadmap": segment attention especially with FP8 kvcache).
 *   k_pool, v_pool  uint8 E4M3 codes [num_slots, kv_heads, head_dim] (16-byte
 *                   aligned); the cached value is code * k_scale[g] (v_scale[g])
 *   k_scale, v_scale  device fp32 [kv_heads], per-kv-head dequantisation scales
 * Queries stay bf16 (used as f16 in the products: |q| must stay below 65504);
 * out / lse / table / workspace exactly as seg_attn_decode, shared-prefix
 * tables included (their prefix pass runs the FP8 prefill kernel).  Half the
 * HBM bytes of the bf16 cache.  Missing or misaligned scales return
 * SEG_ATTN_ERR_INVALID_ARG.
 */
int seg_attn_decode_fp8(const void* q, const void* k_pool, const void* v_pool, const float* k_scale,
                        const float* v_scale, void* out, float* lse, const void* dev_table,
                        const seg_attn_table_desc* desc, float softmax_scale, void* workspace,
                        size_t workspace_bytes, void* stream);

/*
 * seg_attn_prefill_fp8 -- seg_attn_prefill over an FP8 KV cache (Flood README,
 * "Roadmap": segment attention especially with FP8 kvcache), so chunked
 * prefill and decode can share one E4M3 cache.
 *   k_pool, v_pool  uint8 E4M3 codes [num_slots, kv_heads, head_dim] (16-byte
 *                   aligned); the cached value is code * k_scale[g] (v_scale[g])
 *   k_scale, v_scale  device fp32 [kv_heads], per-kv-head dequantisation scales
 * Computes exactly what seg_attn_prefill computes on the dequantised pools, up
 * to rounding: every product is f16 x f16 -> fp32 (codes widen exactly; queries
 * become f16, so |q| must stay below 65504 and values under 2^-14 lose bits;
 * P is f16).  out / lse / table / workspace exactly as seg_attn_prefill,
 * shared-prefix tables (SEG_ATTN_SHARE_PREFIX) included.  Missing or
 * misaligned scales return SEG_ATTN_ERR_INVALID_ARG.
 */
int seg_attn_prefill_fp8(const void* q, const void* k_pool, const void* v_pool,
                         const float* k_scale, const float* v_scale, void* out, float* lse,
                         const void* dev_table, const seg_attn_table_desc* desc,
                         float softmax_scale, void* workspace, size_t workspace_bytes,
                         void* stream);

/*
 * seg_attn_kv_append_fp8 -- quantise the bf16 K/V rows of new tokens to E4M3
 * (code = round-to-nearest-even(x / scale[g]), saturated to +-448) and write
 * them into their slots of FP8 pools.  Same slot rules as seg_attn_kv_append.
 */
int seg_attn_kv_append_fp8(const void* k_new, const void* v_new, const int32_t* slots,
                           int64_t n_tokens, int kv_heads, int head_dim, const float* k_scale,
                           const float* v_scale, void* k_pool, void* v_pool, int64_t num_slots,
                           void* stream);

/* Static English description of a status code (never NULL). */
const char* seg_attn_status_string(int status);

/* Library version as major*10000 + minor*100 + patch. */
int seg_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SEG_ATTN_H_ */
