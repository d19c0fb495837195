/*
 * pa.h — C ABI of the B200 (sm_100a) paged KV attention library (libpa.so).
 *
 * Operations, all asynchronous on the caller's CUDA stream:
 *
 *   pa_write_kv            scatter this step's K/V rows into a block-paged cache
 *   pa_attention_varlen    softmax attention of packed variable-length queries
 *                          over the paged cache (prefill, decode, chunked
 *                          prefill and any mix of them in one batch)
 *   pa_attention_smallseq  one query per batch entry over a handful (<= 16) of
 *                          contiguous keys
 *   pa_attention_smallseq_bwd  its gradients from the saved attention weights
 *   pa_attention_varlen_mods   varlen attention with score modifiers (soft-cap,
 *                          ALiBi, additive mask) and head-major layouts
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Element type: bfloat16 for every Q/K/V/cache/output tensor (passed as
 *    void*, 2 bytes per element), or fp16 where a call takes a pa_dtype (the
 *    _ex, _strided, _mods and small-seq _bwd forms); one type per call.
 *    Index tensors are int32 unless stated.
 *  - Layout (every entry point but the _mods / _strided ones, which take
 *    pa_strides): token-major ("NHD"), dense, innermost dimension last:
 *      q, out           [num_tokens, num_q_heads, head_dim]
 *      k, v (new rows)  [num_tokens, num_kv_heads, head_dim]
 *      k_cache, v_cache [num_blocks, block_size, num_kv_heads, head_dim]
 *  - Pointers are device pointers unless stated, 16-byte aligned.
 *  - The caller owns every buffer, including the workspace.  The library
 *    allocates no device memory and keeps no state between calls beyond a
 *    per-device table of attributes (SM count) and lazily-resolved driver
 *    entry points, with one exception: the PA_STATIC_SCRATCH_BYTES device
 *    array behind pa_attention_varlen_static, which every GPU that loads the
 *    library holds, and which carries that entry point's scratch (its
 *    split-KV arrival counters among it) from one call to the next.  Besides
 *    memory, each device gets one library-owned side stream and two events
 *    (created on the first varlen call with multi-query sequences made
 *    outside a stream capture; see pa_attention_varlen).
 *  - `stream` is a cudaStream_t passed as void*; NULL means the legacy default
 *    stream.  No call synchronises except pa_get_error.  Every call is
 *    ordered on `stream` as one unit: work a call runs on the side stream is
 *    forked from `stream` and joined back to it before the call returns.
 *  - `out` must not alias any input.
 *
 * Errors
 * ------
 *  Problems visible on the host (null pointers, non-positive sizes,
 *  num_q_heads % num_kv_heads != 0, unsupported head_dim or block_size,
 *  misaligned pointers, a workspace that is too small) are reported by the
 *  return value BEFORE anything is launched or written — the reject-before-
 *  write rule of TensorRT-LLM PR "CSA2 Vanilla sparse attention"
 *  (description, "rejected before anything is written").
 *  Problems only the device can see (a slot or block id outside the pool,
 *  inconsistent lengths, a query longer than its sequence, an exceeded length
 *  hint, a bounded wait that gave up) never fault: the kernel skips the
 *  offending row or reads zeros instead, and ORs a bit into a sticky 32-bit
 *  error word held in the first bytes of the workspace.  pa_get_error reads
 *  and clears it.
 */
#ifndef PA_H
#define PA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,  /* host-visible bad argument; nothing was launched */
  PA_ERR_UNSUPPORTED = 2,  /* valid request outside what this build supports */
  PA_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed */
  PA_ERR_DEVICE_INDEX = 4, /* pa_get_error: the device saw a bad index/length */
  PA_ERR_TIMEOUT = 5       /* pa_get_error: a bounded device wait gave up */
} pa_status;

/* Bits of the device error word (pa_get_error's *bits). */
#define PA_DEVERR_SLOT      0x1u  /* slot_mapping entry >= num_blocks*block_size */
#define PA_DEVERR_BLOCK     0x2u  /* block-table entry outside [0, num_blocks)   */
#define PA_DEVERR_LENGTHS   0x4u  /* query_start_loc / seq_lens / cu_seqlens bad */
#define PA_DEVERR_QLEN      0x8u  /* a sequence has more queries than keys       */
#define PA_DEVERR_HINT      0x10u /* a length exceeded max_query_len/max_seq_len */
#define PA_DEVERR_TIMEOUT   0x20u /* a bounded wait inside a kernel gave up      */
#define PA_DEVERR_SPANS     0x40u /* a full-attention span was malformed (unused) */

/* Bytes at the start of every workspace reserved for the error word. */
#define PA_ERROR_WORD_BYTES 256

/*
 * pa_write_kv — KV-cache write through slot_mapping.
 *
 * Defined by vllm-spyre PR #853 "Pytorch Native Attention on Spyre",
 * description, step 1: every new token's key/value row is written into the
 * paged cache at the slot slot_mapping names; slot s is block s / block_size,
 * offset s % block_size (the vLLM v1 convention).
 *
 *  k, v          [num_tokens, num_kv_heads, head_dim] bf16 (read)
 *  slot_mapping  [num_tokens] int64 (read).  slot < 0 marks a padding token:
 *                its row is skipped.  slot >= num_blocks*block_size: row
 *                skipped and PA_DEVERR_SLOT raised.
 *  k_cache, v_cache [num_blocks, block_size, num_kv_heads, head_dim] bf16,
 *                written in place; slots not named are left unchanged.
 *  workspace     NULL, or >= PA_ERROR_WORD_BYTES zero-initialised bytes whose
 *                error word receives PA_DEVERR_SLOT.
 * Two tokens naming the same slot is invalid input; the cache then holds one
 * of the candidate rows.  head_dim must be a multiple of 8.
 * The kernel lets the next kernel in the stream start early when that one is
 * launched with programmatic stream serialisation (the attention calls'
 * decode kernel is, and waits for this grid before reading any input); an
 * ordinary launch after it is not affected.  A successor from elsewhere
 * launched that way must itself wait (griddepcontrol.wait) before reading
 * the caches.
 */
pa_status pa_write_kv(const void* k, const void* v, const int64_t* slot_mapping,
                      int64_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                      void* k_cache, void* v_cache, int64_t num_blocks,
                      int32_t block_size, void* workspace, void* stream);

/*
 * pa_attention_varlen_workspace_size — bytes of workspace pa_attention_varlen
 * needs for these sizes (a function of the arguments only).  The workspace
 * must be zero-initialised once before its first use (the error word and the
 * split-KV arrival counters must start at zero); afterwards it can be reused
 * without clearing by consecutive calls on the same stream, whatever their
 * sizes (as long as it is large enough for each): the counters sit at a fixed
 * offset in a region used for nothing else, and every call leaves them at
 * zero.
 */
size_t pa_attention_varlen_workspace_size(int32_t num_seqs, int64_t num_q_tokens,
                                          int32_t num_q_heads, int32_t num_kv_heads,
                                          int32_t head_dim);

/*
 * pa_attention_varlen — paged softmax attention over packed varlen queries.
 *
 * Defined by vllm-spyre PR #853, description, steps 2-6 (keys of a sequence
 * reached through its block list; a boolean mask of padding validity and, for
 * prefill, causality; softmax attention per sequence; only real tokens
 * written) with grouped-query heads as the repeat_interleave expansion of the
 * same description, and causal alignment bottom-right as in vllm-omni
 * PR #9244 (kernel-semantics review).  For sequence s with
 * Lq = query_start_loc[s+1] - query_start_loc[s] queries and Lkv = seq_lens[s]
 * keys, query i (token query_start_loc[s] + i) and query head h see keys
 * j < Lkv, and with causal != 0 only j <= (Lkv - Lq) + i; they read KV head
 * h / (num_q_heads / num_kv_heads); key j lives in block
 * block_tables[s][j / block_size], offset j % block_size.
 *   out = softmax(scale * q . K^T over the visible keys) . V
 * A row with no visible key is written as zeros (TensorRT-LLM "CSA2 Vanilla
 * sparse attention", description: an empty selection gives zeros).
 * seq_lens counts every key of the sequence, this step's tokens included.
 * Sequences with Lq == 1 take the split-KV decode kernel; all others the
 * tensor-core prefill kernel; both may appear in one call.  When the prefill
 * kernel runs, the decode kernel runs beside it on the device's side stream
 * (forked from `stream` after the planning kernel, joined back before the
 * call returns), each on the share of the SMs the planning kernel picks for
 * this batch.  Inside a stream capture the fork and join are captured too,
 * once the side stream exists (the first such call outside a capture makes
 * it); until then, or while the side stream belongs to another open capture,
 * the two kernels run one after the other on `stream`.  Results are the same
 * either way up to rounding (the decode's split-KV partition follows the
 * share of SMs it gets).
 *
 *  q                [num_q_tokens, num_q_heads, head_dim] bf16
 *  k_cache, v_cache [num_blocks, block_size, num_kv_heads, head_dim] bf16
 *  block_tables     [num_seqs, max_blocks_per_seq] int32; entries past a
 *                   sequence's last needed block are never read
 *  seq_lens         [num_seqs] int32
 *  query_start_loc  [num_seqs + 1] int32, non-decreasing, starting at 0,
 *                   ending at <= num_q_tokens
 *  max_query_len    host hint: >= every Lq (1 means a pure decode batch, and
 *                   the prefill kernel is not launched).  A violated hint
 *                   raises PA_DEVERR_HINT.
 *  max_seq_len      host hint: >= every Lkv; checked like max_query_len.
 *  scale            multiplies q . k (usually 1/sqrt(head_dim)); finite, >= 0 (the
 *                   prefill takes its row maxima before scaling), else
 *                   PA_ERR_INVALID_ARG
 *  causal           0 or 1
 *  out              [num_q_tokens, num_q_heads, head_dim] bf16, written for
 *                   every token that belongs to a sequence
 *  workspace        device buffer of >= workspace_size bytes (see above)
 * Supported: head_dim in {64, 128}; block_size a multiple of 16, up to 512
 * (the kernels fetch and count keys in 16-slot pages; a block holds
 * block_size / 16 of them);
 * num_q_heads / num_kv_heads <= 128 (a decode warp serves up to 16 query heads
 * of a GQA group; larger groups are cut into 16-head slices, up to 8 warps
 * sharing the KV head's pages).
 */
pa_status pa_attention_varlen(const void* q, const void* k_cache, const void* v_cache,
                              const int32_t* block_tables, int32_t max_blocks_per_seq,
                              const int32_t* seq_lens, const int32_t* query_start_loc,
                              int32_t num_seqs, int64_t num_q_tokens,
                              int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                              int32_t block_size, int64_t num_blocks,
                              int32_t max_query_len, int32_t max_seq_len, float scale,
                              int32_t causal, void* out, void* workspace,
                              size_t workspace_bytes, void* stream);

/*
 * pa_attention_varlen_spans — pa_attention_varlen with piecewise block-causal
 * masking (full-attention blocks inside causal sequences).
 *
 * Defined by vllm-omni PR #9244 "Support piecewise block-causal attention for
 * full_attn_spans" (description: the shared segment plan).  A sequence's key
 * positions are split into full segments, listed as spans, and causal
 * segments (everything else).  With Lq queries and Lkv keys, query i sits at
 * key position p = (Lkv - Lq) + i.  If p lies in a span [start, end) the
 * query attends bidirectionally to keys 0 .. end-1 (the truncated prefix);
 * otherwise it attends to keys 0 .. p, as with causal == 1.  Single-query
 * (decode) sequences are unaffected: their one query sees every key either
 * way when spans end at or before Lkv.
 *
 *  span_offsets  [num_seqs + 1] int32: sequence s owns spans
 *                span_offsets[s] .. span_offsets[s+1]-1
 *  spans         [num_spans, 2] int32 (start, end) key positions, in
 *                increasing order per sequence; may be NULL if num_spans == 0
 *  num_spans     total spans
 * Every other argument is pa_attention_varlen's (there is no causal flag:
 * positions outside spans are causal).  A span that is empty, outside
 * [0, Lkv], or starts before the previous span of its sequence ends is
 * ignored and raises PA_DEVERR_SPANS; span_offsets that decrease or leave
 * [0, num_spans] make that sequence span-free and raise PA_DEVERR_SPANS.
 * The workspace is the same as pa_attention_varlen's.
 */
pa_status pa_attention_varlen_spans(const void* q, const void* k_cache, const void* v_cache,
                                    const int32_t* block_tables, int32_t max_blocks_per_seq,
                                    const int32_t* seq_lens, const int32_t* query_start_loc,
                                    int32_t num_seqs, int64_t num_q_tokens,
                                    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                    int32_t block_size, int64_t num_blocks,
                                    int32_t max_query_len, int32_t max_seq_len, float scale,
                                    const int32_t* span_offsets, const int32_t* spans,
                                    int32_t num_spans, void* out, void* workspace,
                                    size_t workspace_bytes, void* stream);

/*
 * Element type of q, k, v, the caches and out in the _ex entry points.
 */
typedef enum { PA_DTYPE_BF16 = 0, PA_DTYPE_FP16 = 1 } pa_dtype;

/*
 * pa_write_kv_ex — pa_write_kv with an explicit cache block stride and dtype.
 *
 * The cache layouts of vllm-spyre PR #853 "Pytorch Native Attention on
 * Spyre" (its code moves from separate K and V caches to one tensor shaped
 * (num_blocks, 2, block_size, Hkv, D)) differ only in the distance between
 * consecutive blocks: slot s of block b is row s of
 *     k_cache + b * block_stride   (and v_cache + b * block_stride),
 * each row [Hkv, D] contiguous.  Separate caches: block_stride =
 * block_size * Hkv * D (or 0, which means that).  One combined tensor KV:
 * k_cache = &KV[0][0], v_cache = &KV[0][1], block_stride = 2 * block_size *
 * Hkv * D.
 *  block_stride  elements; 0, or >= block_size * Hkv * D and a multiple of 8
 *  dtype         PA_DTYPE_BF16 or PA_DTYPE_FP16 (a bit copy either way)
 * Other arguments and errors as pa_write_kv.
 */
pa_status pa_write_kv_ex(const void* k, const void* v, const int64_t* slot_mapping,
                         int64_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                         void* k_cache, void* v_cache, int64_t num_blocks, int32_t block_size,
                         int64_t block_stride, int32_t dtype, void* workspace, void* stream);

/*
 * pa_attention_varlen_ex — the general varlen entry point: cache block stride
 * (see pa_write_kv_ex), element type, and optional full-attention spans
 * (span_offsets NULL: none, and causal applies; otherwise as
 * pa_attention_varlen_spans, and causal is ignored).  pa_attention_varlen and
 * pa_attention_varlen_spans are this call with block_stride 0, bf16.
 * The computation is the same in either element type: fp32 scores and
 * softmax, P rounded to the element type for P.V, out rounded to it.
 */
pa_status pa_attention_varlen_ex(const void* q, const void* k_cache, const void* v_cache,
                                 const int32_t* block_tables, int32_t max_blocks_per_seq,
                                 const int32_t* seq_lens, const int32_t* query_start_loc,
                                 int32_t num_seqs, int64_t num_q_tokens,
                                 int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                 int32_t block_size, int64_t num_blocks, int64_t block_stride,
                                 int32_t dtype, int32_t max_query_len, int32_t max_seq_len,
                                 float scale, int32_t causal, const int32_t* span_offsets,
                                 const int32_t* spans, int32_t num_spans, void* out,
                                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * pa_attention_varlen_static — pa_attention_varlen for callers that cannot
 * allocate device memory.  This is an addition of this library: the pages it
 * follows have no counterpart.
 *
 * Some callers may not call cudaMalloc: a host program that owns all device
 * memory through its own pool allocator and forbids other allocations, or a
 * latency-critical serving path where cudaMalloc/cudaFree would synchronise
 * the device.  This variant takes the same arguments as pa_attention_varlen
 * minus the workspace, runs the same kernels, and keeps its scratch in a
 * file-scope device array of PA_STATIC_SCRATCH_BYTES bytes that every GPU
 * loading the library holds until the process exits.  It allocates nothing.
 *
 *  - Sizes whose pa_attention_varlen_workspace_size() exceeds
 *    PA_STATIC_SCRATCH_BYTES return PA_ERR_UNSUPPORTED before any launch.
 *  - The first call on a device looks up the array's device address with
 *    that device current; make it before any stream capture.
 *  - All calls share the array, which keeps the last call's contents.  Each
 *    call rebuilds its plan lists and partial results; the split-KV arrival
 *    counters, the one part that must start at zero, sit in a region used for
 *    nothing else, zero when the module loads and returned to zero by every
 *    call (the merge that uses a counter resets it; the plan kernel, when it
 *    runs, zeroes them first).  Calls whose executions overlap on the GPU
 *    race on the array: issue them on one stream, one host thread at a time.
 *  - Bad arguments are reported as pa_attention_varlen reports them, before
 *    the size limit below is applied and before any CUDA call.
 *  - Device-side index errors are handled as in pa_attention_varlen but
 *    cannot be read back (there is no caller workspace for pa_get_error).
 */
#define PA_STATIC_SCRATCH_BYTES (32u << 20)
pa_status pa_attention_varlen_static(const void* q, const void* k_cache, const void* v_cache,
                                     const int32_t* block_tables, int32_t max_blocks_per_seq,
                                     const int32_t* seq_lens, const int32_t* query_start_loc,
                                     int32_t num_seqs, int64_t num_q_tokens,
                                     int32_t num_q_heads, int32_t num_kv_heads,
                                     int32_t head_dim, int32_t block_size, int64_t num_blocks,
                                     int32_t max_query_len, int32_t max_seq_len, float scale,
                                     int32_t causal, void* out, void* stream);

/*
 * Layouts: element strides of q, out and the paged caches (the innermost
 * head_dim elements of a row are always contiguous).  The HND / NHD layouts
 * of auto_round_kernel PR "Migrate CPU SDPA backend" (description: the public
 * sdpa() takes head-major or token-major tensors) are two settings of it:
 *   q / out NHD [T, H, D]: token = H*D, head = D
 *   q / out HND [H, T, D]: token = D,   head = T*D
 *   cache NHD [num_blocks, block_size, Hkv, D]: block = BS*Hkv*D, slot = Hkv*D, head = D
 *   cache HND [num_blocks, Hkv, block_size, D]: block = BS*Hkv*D, slot = D, head = BS*D
 * (padding between rows or blocks is allowed).  A pair (token, head) or
 * triple (block, slot, head) of zeros means the dense NHD layout.  Every
 * stride is a multiple of 8 elements; rows must not overlap: either
 * head >= D and token >= H*head (token-major) or token >= D and head >=
 * T*token (head-major); for the cache either head >= D and slot >=
 * Hkv*head, or slot >= D and head >= block_size*slot, and block >= the
 * extent of one block.  Anything else is PA_ERR_UNSUPPORTED.
 */
typedef struct pa_strides {
  int64_t q_token, q_head;
  int64_t out_token, out_head;
  int64_t cache_block, cache_slot, cache_head;
} pa_strides;

/*
 * Score modifiers (auto_round_kernel PR "Migrate CPU SDPA backend",
 * description: additive masks in the public sdpa(); ALiBi slopes and the
 * TANH30 soft-cap among the library's extensions).  With s = scale*<q, k_j>
 * for query token t (key position pos within its sequence) and head h:
 *   softcap > 0:   s <- softcap * tanh(s / softcap)      (TANH30: softcap = 30)
 *   alibi_slopes:  s <- s + alibi_slopes[h] * (j - pos)
 *   mask:          s <- s + mask[h * mask_head_stride + t * mask_token_stride + j]
 * in that order; causal / span / sequence-end masking then decides which
 * keys enter the softmax, and a row whose visible scores are all -inf gives
 * zeros.  alibi_slopes: NULL or [num_q_heads] fp32.  mask: NULL or fp32,
 * 16-byte aligned, entries finite or -inf; t is the packed query-token
 * index; the buffer must hold every (h, t) row a call addresses (the
 * library cannot check its extent, only the row length below);
 * mask_head_stride 0 shares one mask across heads; both strides are
 * multiples of 4; mask_len is the number of keys a mask row holds: a key at
 * or beyond it gets no mask value and raises PA_DEVERR_HINT.  With any
 * modifier on, scale must be > 0 (the kernels apply the modifiers to
 * unscaled scores), else PA_ERR_INVALID_ARG.
 */
typedef struct pa_score_mods {
  float softcap;
  const float* alibi_slopes;
  const float* mask;
  int64_t mask_head_stride;
  int64_t mask_token_stride;
  int64_t mask_len;
} pa_score_mods;

/*
 * pa_write_kv_strided — pa_write_kv_ex into caches of any layout above
 * (strides NULL: dense NHD).  k and v stay dense [num_tokens, Hkv, D].
 */
pa_status pa_write_kv_strided(const void* k, const void* v, const int64_t* slot_mapping,
                              int64_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                              void* k_cache, void* v_cache, int64_t num_blocks,
                              int32_t block_size, const pa_strides* strides, int32_t dtype,
                              void* workspace, void* stream);

/*
 * pa_attention_varlen_mods — pa_attention_varlen_ex with layouts (strides:
 * NULL = dense NHD everywhere; its cache_block replaces block_stride) and
 * score modifiers (mods: NULL or all off = none).  Other arguments, the
 * workspace and the errors as pa_attention_varlen_ex.
 */
pa_status pa_attention_varlen_mods(const void* q, const void* k_cache, const void* v_cache,
                                   const int32_t* block_tables, int32_t max_blocks_per_seq,
                                   const int32_t* seq_lens, const int32_t* query_start_loc,
                                   int32_t num_seqs, int64_t num_q_tokens, int32_t num_q_heads,
                                   int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                   int64_t num_blocks, int32_t dtype, int32_t max_query_len,
                                   int32_t max_seq_len, float scale, int32_t causal,
                                   const int32_t* span_offsets, const int32_t* spans,
                                   int32_t num_spans, const pa_strides* strides,
                                   const pa_score_mods* mods, void* out, void* workspace,
                                   size_t workspace_bytes, void* stream);

/*
 * pa_attention_smallseq — s_q = 1 cross attention over short contiguous KV.
 *
 * Defined by ROCm/TransformerEngine PR #461 "CK varlen cross attention for
 * small-seq", description: one query per batch entry, keys and values packed
 * THD with cu_seqlens_kv (entry b owns rows cu_seqlens_kv[b] ..
 * cu_seqlens_kv[b+1]-1), no causal mask, max_seqlen_kv <= 16; the batch is
 * the number of query tokens.  An empty entry gives zeros.
 *
 *  q, out   [batch, num_q_heads, head_dim] bf16
 *  k, v     [cu_seqlens_kv[batch], num_kv_heads, head_dim] bf16
 *  cu_seqlens_kv [batch + 1] int32, non-decreasing from 0
 *  max_seqlen_kv host hint, 0..16 (> 16: PA_ERR_UNSUPPORTED — use
 *           pa_attention_varlen); an entry longer than the hint raises
 *           PA_DEVERR_HINT and only its first max_seqlen_kv keys are used.
 *  workspace NULL or >= PA_ERROR_WORD_BYTES zero-initialised bytes (error word)
 * Supported: head_dim in {64, 128}.
 */
pa_status pa_attention_smallseq(const void* q, const void* k, const void* v,
                                const int32_t* cu_seqlens_kv, int32_t batch,
                                int32_t num_q_heads, int32_t num_kv_heads,
                                int32_t head_dim, int32_t max_seqlen_kv, float scale,
                                void* out, void* workspace, void* stream);

/*
 * pa_attention_smallseq_ex — pa_attention_smallseq with an element type and
 * the attention-weights output of ROCm/TransformerEngine PR #461
 * (description: the forward also returns the softmax weights, shaped
 * [batch, Hq, 1, max_seqlen_kv], in the q/k/v dtype, for the backward).
 *  dtype        PA_DTYPE_BF16 or PA_DTYPE_FP16 for q, k, v, out and weights
 *  weights      NULL, or [batch, Hq, weights_len] of dtype: entry b's weights
 *               in the first n_b slots (n_b its key count), zeros after
 *  weights_len  > 0 when weights is set; an entry with more keys raises
 *               PA_DEVERR_HINT and keeps its first weights_len weights
 * Other arguments as pa_attention_smallseq.
 */
pa_status pa_attention_smallseq_ex(const void* q, const void* k, const void* v,
                                   const int32_t* cu_seqlens_kv, int32_t batch,
                                   int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                   int32_t max_seqlen_kv, float scale, int32_t dtype, void* out,
                                   void* weights, int32_t weights_len, void* workspace,
                                   void* stream);

/*
 * pa_attention_smallseq_bwd — gradients of pa_attention_smallseq_ex.
 *
 * Defined by ROCm/TransformerEngine PR #461 (description: the small-seq
 * backward computes grad_V, grad_attn, the softmax backward and grad_Q /
 * grad_K, and reads the attention weights the forward wrote into the softmax
 * auxiliary buffer instead of recomputing them).  With P the saved weights of
 * query head h over its entry's n keys and dO its upstream gradient:
 *   dP_j = dO . v_j,  dS_j = P_j (dP_j - sum_k P_k dP_k),
 *   dQ = scale sum_j dS_j k_j,  dK_j = scale sum_h dS_hj q_h,
 *   dV_j = sum_h P_hj dO_h  (sums over h run over the query heads of the
 *   KV head that owns key j).
 *
 *  q, dout, dq    [batch, num_q_heads, head_dim] of dtype
 *  k, v, dk, dv   [cu_seqlens_kv[batch], num_kv_heads, head_dim] of dtype
 *  weights        [batch, num_q_heads, weights_len] of dtype, as written by
 *                 pa_attention_smallseq_ex (2-byte aligned)
 *  weights_len    > 0; an entry with more keys than min(weights_len,
 *                 max_seqlen_kv) raises PA_DEVERR_HINT and only its first
 *                 keys are used (the others' dk/dv rows are left unwritten)
 *  max_seqlen_kv  0..16, num_q_heads / num_kv_heads <= 16 (else
 *                 PA_ERR_UNSUPPORTED)
 *  workspace      NULL or the error word, as for the forward
 * Every dq row is written (zeros for an entry with no keys); every dk/dv row
 * of a key that belongs to some entry is written once.  Outputs must not
 * alias inputs.  Supported: head_dim in {64, 128}.
 */
pa_status pa_attention_smallseq_bwd(const void* q, const void* k, const void* v,
                                    const void* dout, const void* weights, int32_t weights_len,
                                    const int32_t* cu_seqlens_kv, int32_t batch,
                                    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                    int32_t max_seqlen_kv, float scale, int32_t dtype, void* dq,
                                    void* dk, void* dv, void* workspace, void* stream);

/*
 * pa_get_error — synchronise `stream`, read the workspace's error word into
 * *bits (may be NULL), clear it, and map it to a status: PA_OK when zero,
 * PA_ERR_TIMEOUT when PA_DEVERR_TIMEOUT is set, PA_ERR_DEVICE_INDEX otherwise.
 */
pa_status pa_get_error(void* workspace, void* stream, uint32_t* bits);

/* Static description of a status code. */
const char* pa_status_string(pa_status status);

/* Library version string, e.g. "pa 0.1 sm_100a". */
const char* pa_version(void);

/*
 * pa_set_wait_limit_ns — a test hook for the failure path of the tensor-core
 * prefill (an addition of this library: the pages it follows have no
 * counterpart).  Every wait of that kernel on one of its own pipeline
 * barriers is bounded in wall time; after the limit it raises
 * PA_DEVERR_TIMEOUT in the workspace's error word, lets the copies and MMAs
 * it already issued land, releases its tensor memory and exits (its rows are
 * left unwritten), so a lost arrival never hangs the GPU.  The default limit,
 * one second, is far beyond any legitimate wait.  This call sets the limit
 * for prefill launches made from now on, process-wide; ns = 0 restores the
 * default.  A short limit makes ordinary waits give up, which is how a test
 * reaches the timeout path; production code has no reason to call it.
 */
void pa_set_wait_limit_ns(uint64_t ns);

#ifdef __cplusplus
}
#endif

#endif /* PA_H */
