// Internal declarations of segment linear attention (host entry points and kernels).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "seg_la.h"

namespace segla {

constexpr int kDim = 128;    // head_dim = state side
constexpr int kChunk = 128;  // prefill tokens per chunk (one 128-row MMA tile)

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Prefill workspace: per (chunk, head) the chunk's state contribution U (fp32
// d x d), the state entering the chunk as a bf16 d x d tile (the MMA operand of
// the third pass), and the chunk's total decay exp(G_last).
struct Workspace {
  size_t u = 0, s_in = 0, gamma = 0, total = 0;
};
inline Workspace prefill_workspace(const seg_la_table_desc& d) {
  Workspace w;
  const size_t units = (size_t)d.num_chunks * d.heads;
  w.u = 0;
  w.s_in = align_up(units * kDim * kDim * sizeof(float), 256);
  w.gamma = w.s_in + align_up(units * kDim * kDim * 2, 256);
  w.total = w.gamma + align_up(units * sizeof(float), 256);
  return w;
}

struct Table {
  const int32_t* q_offsets;   // [B+1]
  const int32_t* in_slot;     // [B]
  const int32_t* out_slot;    // [B]
  const int32_t* req_chunks;  // [B+1]
  const int4* chunks;         // [num_chunks]
};

inline Table make_table(const void* dev_table, const seg_la_table_desc& d) {
  const int32_t* t = static_cast<const int32_t*>(dev_table);
  Table v;
  v.q_offsets = t + d.off_q_offsets;
  v.in_slot = t + d.off_in_slot;
  v.out_slot = t + d.off_out_slot;
  v.req_chunks = t + d.off_req_chunks;
  v.chunks = reinterpret_cast<const int4*>(t + d.off_chunks);
  return v;
}

struct Launch {
  const void* q;
  const void* k;
  const void* v;
  const float* g;
  void* out;
  float* state_pool;
  Table tab;
  const seg_la_table_desc* desc;
  float scale;
  void* workspace;
};

// Each returns SEG_ATTN_OK or SEG_ATTN_ERR_CUDA.
int launch_la_prefill(const Launch& a, cudaStream_t stream);
int launch_la_decode(const Launch& a, cudaStream_t stream);
// Read and clear the device word set when a bounded wait of a prefill kernel gave up.
int take_la_error(int* value);

}  // namespace segla
