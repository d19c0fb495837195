// Internal launch interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "layout.h"

namespace pa {

// ---- KV scatter ------------------------------------------------------------
cudaError_t launch_write_kv(const void* k, const void* v, const int64_t* slot_mapping,
                            int64_t num_tokens, int row_vecs, void* k_cache, void* v_cache,
                            int64_t num_slots, int block_size, int64_t block_vecs, uint32_t* err,
                            int num_sms, cudaStream_t stream);

// ---- plan ------------------------------------------------------------------
void launch_plan(const int32_t* query_start_loc, const int32_t* seq_lens, int num_seqs,
                 long long num_q_tokens, int max_blocks_per_seq, int block_size,
                 int max_query_len, int max_seq_len, int causal, int num_kv_heads,
                 const int32_t* span_offsets, const int32_t* spans, int num_spans,
                 unsigned char* ws, const WorkspaceLayout& L, cudaStream_t stream);

// ---- split-KV decode -------------------------------------------------------
struct DecodeParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k_cache;
  const __nv_bfloat16* v_cache;
  const int32_t* block_tables;
  const int32_t* query_start_loc;
  const int32_t* seq_lens;
  int num_seqs;
  long long num_q_tokens;
  int max_blocks_per_seq;
  int max_query_len; // host hint, checked
  int max_seq_len;   // host hint, checked
  int num_q_heads;
  int num_kv_heads;
  int group;  // num_q_heads / num_kv_heads, <= 16
  long long num_blocks;
  long long block_stride;  // elements between consecutive cache blocks
  float scale_log2;  // scale * log2(e)
  int self_plan;     // 1: every CTA plans the decode work itself (num_seqs <= kSelfPlanMaxSeqs)
  uint16_t* out;     // elements of the kernel's type (bf16 or fp16)
  unsigned char* ws;
  WorkspaceLayout L;
};
// Persistent launch: one resident wave, num_sms from the device.
cudaError_t launch_decode(const DecodeParams& p, int head_dim, bool fp16, int num_sms,
                          cudaStream_t stream);

// ---- tcgen05 prefill ------------------------------------------------------
struct PrefillParams {
  const int32_t* block_tables;
  int max_blocks_per_seq;
  int num_q_heads;
  int num_kv_heads;
  int group;
  long long num_blocks;
  long long num_q_tokens;
  float scale_log2;
  int causal;
  const int32_t* span_offsets;  // full-attention spans (null: none)
  const int32_t* spans;
  int num_spans;
  uint16_t* out;  // [T, Hq, D] elements of the kernel's type (bf16 or fp16)
  unsigned char* ws;
  WorkspaceLayout L;
};
// Tensor maps are built by the host layer (they need the driver entry point).
cudaError_t launch_prefill(const PrefillParams& p, const CUtensorMap& q_map,
                           const CUtensorMap& k_map, const CUtensorMap& v_map, int head_dim,
                           bool fp16, int grid, cudaStream_t stream);

// ---- small-seq -------------------------------------------------------------
struct SmallSeqParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const int32_t* cu_seqlens_kv;
  int batch;
  int num_q_heads;
  int num_kv_heads;
  int group;
  int max_seqlen_kv;
  float scale_log2;
  uint16_t* out;  // elements of the kernel's type (bf16 or fp16)
  uint32_t* err;
  uint16_t* weights;  // optional [batch, Hq, weights_len] attention weights
  int weights_len;
};
cudaError_t launch_smallseq(const SmallSeqParams& p, int head_dim, bool fp16, int num_sms,
                            cudaStream_t stream);

// Backward of the small-seq attention from the forward's saved weights.
struct SmallSeqBwdParams {
  const uint16_t* q;        // [batch, Hq, D]
  const uint16_t* k;        // [total_kv, Hkv, D]
  const uint16_t* v;        // [total_kv, Hkv, D]
  const uint16_t* dout;     // [batch, Hq, D]
  const uint16_t* weights;  // [batch, Hq, weights_len]
  const int32_t* cu_seqlens_kv;
  int batch;
  int num_q_heads;
  int num_kv_heads;
  int group;
  int max_seqlen_kv;
  int weights_len;
  float scale;
  uint16_t* dq;  // [batch, Hq, D]
  uint16_t* dk;  // [total_kv, Hkv, D]
  uint16_t* dv;  // [total_kv, Hkv, D]
  uint32_t* err;
};
cudaError_t launch_smallseq_bwd(const SmallSeqBwdParams& p, int head_dim, bool fp16, int num_sms,
                                cudaStream_t stream);

}  // namespace pa
