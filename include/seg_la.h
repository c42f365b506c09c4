/*
 * seg_la.h -- C ABI of the B200 (sm_100a) segment linear attention library
 * (simple GLA), part of libsegattn.so.
 *
 * Flood ships a second kernel family next to SegmentAttention: segment linear
 * attention (Flood README, "News" 2025/09 and "Kernels > Seg-linear-attn"),
 * benchmarked with 16 heads, 16 kv heads and head_dim 128 against the simple
 * GLA kernels of flash-linear-attention.  Simple GLA keeps, per request and
 * head, one recurrent state S (d x d, key index i, value index j) and a scalar
 * log-decay g per token and head:
 *
 *   S <- exp(g[t,h]) * S + k[t,h,:]^T v[t,h,:]
 *   out[t,h,j] = scale * sum_i q[t,h,i] * S[i][j]
 *
 * The state of every request lives in one slot of a state pool (a request's
 * "segment" of the cache: its size does not grow with the sequence).  Prefill
 * processes a chunk of new tokens per request starting from the state in its
 * input slot and leaves the final state in its output slot; decode is the
 * one-token case.
 *
 * Conventions (as in seg_attn.h): the caller owns every buffer; the library
 * never allocates, frees or synchronises; errors are returned before anything
 * is launched; `stream` is a cudaStream_t passed as void*.
 *   q, k, v    bf16 [total_q, heads, head_dim]   (requests packed in order)
 *   g          fp32 [total_q, heads]             (log of the per-token decay)
 *   out        bf16 [total_q, heads, head_dim]
 *   state_pool fp32 [num_state_slots, heads, head_dim, head_dim], row-major
 *              in (i, j); read from in slots, written to out slots
 * Supported: head_dim 128; every pointer 16-byte aligned.
 */
#ifndef SEG_LA_H_
#define SEG_LA_H_

#include <stddef.h>
#include <stdint.h>

#include "seg_attn.h" /* status codes and mode values */

#ifdef __cplusplus
extern "C" {
#endif

#define SEG_LA_TABLE_MAGIC 0x53454c41u /* "SELA" */
#define SEG_LA_TABLE_VERSION 1u

/* Description of a built linear-attention table (offsets in int32 elements). */
typedef struct seg_la_table_desc {
  uint32_t magic, version;
  int32_t mode;            /* SEG_ATTN_MODE_PREFILL or SEG_ATTN_MODE_DECODE */
  int32_t batch, heads, head_dim;
  int32_t chunk_len;       /* prefill: tokens per chunk (128) */
  int32_t num_chunks;      /* prefill: chunks over all requests */
  int64_t total_q;
  int64_t num_state_slots;
  int64_t off_q_offsets;   /* [batch+1] first packed row of each request */
  int64_t off_in_slot;     /* [batch] state slot read (-1: zero state) */
  int64_t off_out_slot;    /* [batch] state slot written (-1: final state dropped) */
  int64_t off_req_chunks;  /* prefill: [batch+1] first chunk of each request */
  int64_t off_chunks;      /* prefill: [num_chunks][4] request, first packed row, tokens,
                              chunk index within the request */
  uint64_t table_bytes;
  uint64_t workspace_bytes;
} seg_la_table_desc;

/*
 * seg_la_build_table -- validate the batch and lay out the table in host memory.
 *   batch                requests (>= 0)
 *   q_lens [batch]       new tokens per request (>= 0); NULL in decode mode = 1 each;
 *                        decode requires 1
 *   in_slot, out_slot [batch]  state slots in [0, num_state_slots) or -1.  Output
 *                        slots must be distinct, and no request may read a slot
 *                        another request writes (a request may read and write
 *                        its own slot).
 *   mode                 SEG_ATTN_MODE_PREFILL or SEG_ATTN_MODE_DECODE
 *   heads, head_dim      head_dim must be 128
 *   host_out, host_out_bytes, desc   as seg_attn_build_table (host_out NULL =
 *                        size query); copy table_bytes of host_out to device
 *                        memory (16-byte aligned) and pass it as dev_table.
 */
int seg_la_build_table(int batch, const int32_t* q_lens, const int32_t* in_slot,
                       const int32_t* out_slot, int64_t num_state_slots, int mode, int heads,
                       int head_dim, void* host_out, size_t host_out_bytes,
                       seg_la_table_desc* desc);

/* Device workspace (bytes) the compute call for this table needs; 0 if none. */
size_t seg_la_workspace_size(const seg_la_table_desc* desc);

/*
 * seg_la_prefill -- chunked simple-GLA prefill.  Each request's tokens are cut
 * into chunks of 128; three sm_100a kernels run:
 *   1. per chunk (tcgen05): the chunk's contribution to the state,
 *      U = (K * exp(G_last - G))^T V, G the running sum of g inside the chunk;
 *   2. per request and head: the state entering every chunk, S_{c+1} =
 *      exp(G_last,c) S_c + U_c, from the input slot; the final state goes to
 *      the output slot;
 *   3. per chunk (tcgen05): out = scale * ((Q K^T . D) V + exp(G_t) Q S_c),
 *      D[t][s] = exp(G_t - G_s) for s <= t, else 0.
 * The products run on the tensor cores with bf16 operands (the state enters
 * them rounded to bf16) and fp32 accumulators; the state itself is carried in
 * fp32.  workspace: seg_la_workspace_size(desc) bytes, 16-byte aligned.
 */
int seg_la_prefill(const void* q, const void* k, const void* v, const float* g, void* out,
                   float* state_pool, const void* dev_table, const seg_la_table_desc* desc,
                   float scale, void* workspace, size_t workspace_bytes, void* stream);

/*
 * seg_la_decode -- one token per request: reads the state (fp32, 64 KiB per
 * head), applies the decay and the token's outer product, writes it back and
 * produces the output.  HBM-bound on the state; no workspace.
 */
int seg_la_decode(const void* q, const void* k, const void* v, const float* g, void* out,
                  float* state_pool, const void* dev_table, const seg_la_table_desc* desc,
                  float scale, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SEG_LA_H_ */
