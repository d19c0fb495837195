// Internal launch interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/pa.h"
#include "layout.h"

namespace pa {

// ---- host-side argument checks ---------------------------------------------
// Every host-visible check pa_attention_varlen makes, without launching or
// writing anything and without comparing a workspace size.  On PA_OK,
// *workspace_bytes is the workspace the call needs (0 when it has no rows, in
// which case *nothing_to_do is set and the pointers were not examined).
pa_status check_varlen_args(const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* block_tables, int32_t max_blocks_per_seq,
                            const int32_t* seq_lens, const int32_t* query_start_loc,
                            int32_t num_seqs, int64_t num_q_tokens, int32_t num_q_heads,
                            int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                            int64_t num_blocks, int32_t max_query_len, int32_t max_seq_len,
                            float scale, int32_t causal, const void* out, const void* workspace,
                            size_t* workspace_bytes, bool* nothing_to_do);

// ---- KV scatter ------------------------------------------------------------
// Cache destination of vector c of head h of slot s: (s / block_size) *
// block_vecs + (s % block_size) * slot_vecs + h * head_vecs + c (16-byte
// vectors; a head row holds 1 << dshift of them).
cudaError_t launch_write_kv(const void* k, const void* v, const int64_t* slot_mapping,
                            int64_t num_tokens, int row_vecs, void* k_cache, void* v_cache,
                            int64_t num_slots, int block_size, int64_t block_vecs,
                            int64_t slot_vecs, int64_t head_vecs, int dshift, uint32_t* err,
                            int num_sms, cudaStream_t stream);

// ---- plan ------------------------------------------------------------------
// What the plan needs to split the machine between the prefill and the decode
// kernel when they run side by side (sms = 0: they do not).
struct SplitShape {
  int sms;
  int num_q_heads, num_kv_heads, head_dim;
};
void launch_plan(const int32_t* query_start_loc, const int32_t* seq_lens, int num_seqs,
                 long long num_q_tokens, int max_blocks_per_seq, int block_size,
                 int max_query_len, int max_seq_len, int causal, long long num_counters,
                 const int32_t* span_offsets, const int32_t* spans, int num_spans,
                 unsigned char* ws, const WorkspaceLayout& L, const SplitShape& split,
                 cudaStream_t stream);

// ---- split-KV decode -------------------------------------------------------
// Score modifiers of a varlen call (soft-cap, ALiBi, additive mask), as the
// C ABI's pa_score_mods; kernels take a template flag when any is on.
struct ScoreMods {
  float softcap;        // > 0: s <- softcap * tanh(s / softcap)
  const float* alibi;   // [Hq] slopes or null
  const float* mask;    // additive fp32 mask or null
  long long mask_head, mask_tok, mask_len;
  bool any() const { return softcap > 0.f || alibi != nullptr || mask != nullptr; }
};

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
  int ppb_shift;     // log2(block_size / 16): a cache block holds 1 << ppb_shift 16-key pages
  int max_query_len; // host hint, checked
  int max_seq_len;   // host hint, checked
  int num_q_heads;
  int num_kv_heads;
  int group;   // num_q_heads / num_kv_heads, <= kMaxGroup
  int slices;  // warps per KV head: decode_slices(group)
  long long num_blocks;
  long long block_stride;  // elements between consecutive cache blocks
  long long c_slot, c_head;  // elements between slots of a block / KV heads of a slot
  long long q_tok, q_head;   // q strides (elements)
  long long o_tok, o_head;   // out strides (elements)
  float scale;       // softmax scale (used with modifiers)
  ScoreMods mods;
  float scale_log2;  // scale * log2(e)
  int self_plan;     // 1: every CTA plans the decode work itself (num_seqs <= kSelfPlanMaxSeqs)
  int split_sms;     // > 0: runs beside the prefill, on the plan's decode_sms of these SMs
  uint16_t* out;     // elements of the kernel's type (bf16 or fp16)
  unsigned char* ws;
  WorkspaceLayout L;
};
// Persistent launch: one resident wave, num_sms from the device.
cudaError_t launch_decode(const DecodeParams& p, int head_dim, bool fp16, int num_sms,
                          cudaStream_t stream);
// The same for slices > 1 (GQA groups of more than 16 query heads).
cudaError_t launch_decode_sliced(const DecodeParams& p, int head_dim, bool fp16, int num_sms,
                                 cudaStream_t stream);

// ---- tcgen05 prefill ------------------------------------------------------
struct PrefillParams {
  const int32_t* block_tables;
  int max_blocks_per_seq;
  int block_size;   // slots per cache block: 16 << ppb_shift
  int ppb_shift;    // log2(block_size / 16)
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
  int q_hnd;    // the q map's dims are (D, T, Hq) instead of (D, Hq, T)
  int kv_hnd;   // the cache maps' dims are (D, BS, Hkv, blocks) instead of (D, Hkv, BS, blocks)
  long long o_tok, o_head;  // out strides (elements)
  float scale;
  ScoreMods mods;
  uint16_t* out;  // elements of the kernel's type (bf16 or fp16)
  unsigned char* ws;
  WorkspaceLayout L;
  unsigned long long wait_limit_ns;  // bound of every mbarrier wait; 0: the 1 s default
  int split;  // 1: runs beside the decode kernel, on the plan's prefill_sms SMs
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
