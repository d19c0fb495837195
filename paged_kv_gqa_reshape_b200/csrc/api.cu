// C ABI (include/pa.h): argument checks, workspace layout, launches.
//
// Every host-visible problem is rejected before anything is launched or
// written (the reject-before-write rule of TensorRT-LLM PR "CSA2 Vanilla
// sparse attention", description).  The library allocates no device memory;
// its only state is a per-device SM count and the lazily resolved driver
// entry point used to encode TMA tensor maps — apart from the fixed device
// array of pa_attention_varlen_static (api_static.cu), which every GPU that
// loads the library holds and which keeps that entry point's scratch.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "../../include/pa.h"
#include "kernels.h"
#include "layout.h"

namespace {

using pa::WorkspaceLayout;

constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices];
std::mutex g_mu;

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_sm_count[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    g_sm_count[dev] = n;
  }
  return g_sm_count[dev];
}

// Per-device resources for running a call's decode kernel beside its prefill
// kernel: a side stream (non-blocking) and the two events that fork it from
// and join it back to the caller's stream.  Created by the first call that
// can use them outside a stream capture; the mutex keeps each call's
// record / wait pairs together when several host threads share a device.
// Inside a capture the fork and join are recorded as graph dependencies (the
// side stream joins the capture), so a replay runs the two kernels side by
// side as an eager call does, with the same results.
struct SideStream {
  std::mutex mu;
  bool tried = false;
  bool ok = false;
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
SideStream g_side[kMaxDevices];

// The current device's side stream, or nullptr (the call then launches the
// two kernels one after the other on the caller's stream): no device,
// creation failed, the caller's stream is being captured before the side
// stream exists (creating it inside a capture is avoided), or the side stream
// is already part of a different, still open capture.
SideStream* side_stream(cudaStream_t caller) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  unsigned long long cap_id = 0;
  if (cudaStreamGetCaptureInfo(caller, &cap, &cap_id) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  SideStream* s = &g_side[dev];
  std::lock_guard<std::mutex> lock(s->mu);
  if (s->tried && s->ok) {
    cudaStreamCaptureStatus side_cap = cudaStreamCaptureStatusNone;
    unsigned long long side_id = 0;
    if (cudaStreamGetCaptureInfo(s->stream, &side_cap, &side_id) != cudaSuccess) {
      (void)cudaGetLastError();
      return nullptr;
    }
    if (side_cap != cudaStreamCaptureStatusNone &&
        (cap != cudaStreamCaptureStatusActive || side_id != cap_id))
      return nullptr;
    return s;
  }
  if (cap != cudaStreamCaptureStatusNone) return nullptr;
  if (!s->tried) {
    s->tried = true;
    s->ok = cudaStreamCreateWithFlags(&s->stream, cudaStreamNonBlocking) == cudaSuccess &&
            cudaEventCreateWithFlags(&s->fork, cudaEventDisableTiming) == cudaSuccess &&
            cudaEventCreateWithFlags(&s->join, cudaEventDisableTiming) == cudaSuccess;
    if (!s->ok) (void)cudaGetLastError();
  }
  return s->ok ? s : nullptr;
}

bool log_enabled() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("PA_LOG");
    v = (e && *e && strcmp(e, "0") != 0) ? 1 : 0;
  }
  return v == 1;
}

// Bound of the prefill kernel's mbarrier waits for launches from now on
// (0: the kernel's 1 s default); set only through pa_set_wait_limit_ns.
std::atomic<unsigned long long> g_wait_limit_ns{0};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---- cuTensorMapEncodeTiled through the runtime's driver entry point ------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// bf16 or fp16 tensor map with a 128-byte swizzle; dims/strides innermost first.
bool make_map(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims,
              const cuuint64_t* strides_bytes, const cuuint32_t* box, bool fp16) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint32_t estride[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                  (cuuint32_t)rank, const_cast<void*>(base),
                  dims, strides_bytes, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Element strides of q, out and the caches after defaults and checks.
struct Strides {
  int64_t qt, qh, ot, oh;  // q / out: token, head
  int64_t cb, cs, ch;      // cache: block, slot, head
  bool q_hnd, kv_hnd;      // head-major q; head-major cache rows within a block
};

// A (token, head) pair for T tokens of H heads of D elements: (0, 0) is dense
// NHD; otherwise token-major (head >= D, token >= H*head) or head-major
// (token >= D, head >= T*token), every stride a positive multiple of 8.
pa_status resolve_rows(int64_t tok, int64_t head, int64_t T, int64_t H, int64_t D, int64_t* rt,
                       int64_t* rh, bool* hnd) {
  if (tok == 0 && head == 0) {
    *rt = H * D;
    *rh = D;
    *hnd = false;
    return PA_OK;
  }
  if (tok <= 0 || head <= 0 || tok % 8 || head % 8) return PA_ERR_INVALID_ARG;
  if (head >= D && tok >= H * head) {
    *hnd = false;
  } else if (tok >= D && head >= T * tok) {
    *hnd = true;
  } else {
    return PA_ERR_UNSUPPORTED;
  }
  *rt = tok;
  *rh = head;
  return PA_OK;
}

// Cache strides: slot and head 0 mean dense [Hkv, D] rows per slot, with
// block 0 meaning BS*Hkv*D; otherwise slot-major (head >= D, slot >=
// Hkv*head) or head-major (slot >= D, head >= BS*slot) rows, and a block
// stride covering one block's rows.
pa_status resolve_cache(const pa_strides* st, int64_t BS, int64_t Hkv, int64_t D, Strides* r) {
  int64_t cb = st ? st->cache_block : 0, cs = st ? st->cache_slot : 0,
          ch = st ? st->cache_head : 0;
  if (cs == 0 && ch == 0) {
    cs = Hkv * D;
    ch = D;
    r->kv_hnd = false;
    if (cb == 0) cb = BS * Hkv * D;
  } else {
    if (cs <= 0 || ch <= 0 || cs % 8 || ch % 8) return PA_ERR_INVALID_ARG;
    if (ch >= D && cs >= Hkv * ch) {
      r->kv_hnd = false;
    } else if (cs >= D && ch >= BS * cs) {
      r->kv_hnd = true;
    } else {
      return PA_ERR_UNSUPPORTED;
    }
  }
  const int64_t extent = r->kv_hnd ? Hkv * ch : BS * cs;
  if (cb < extent || cb % 8) return PA_ERR_INVALID_ARG;
  r->cb = cb;
  r->cs = cs;
  r->ch = ch;
  return PA_OK;
}

pa_status resolve_strides(const pa_strides* st, int64_t T, int64_t Hq, int64_t Hkv, int64_t D,
                          int64_t BS, Strides* r) {
  bool o_hnd = false;
  pa_status e = resolve_rows(st ? st->q_token : 0, st ? st->q_head : 0, T, Hq, D, &r->qt, &r->qh,
                             &r->q_hnd);
  if (e != PA_OK) return e;
  e = resolve_rows(st ? st->out_token : 0, st ? st->out_head : 0, T, Hq, D, &r->ot, &r->oh, &o_hnd);
  if (e != PA_OK) return e;
  return resolve_cache(st, BS, Hkv, D, r);
}

// Score modifiers after checks (mods NULL or all off: none).
pa_status resolve_mods(const pa_score_mods* m, pa::ScoreMods* r) {
  *r = pa::ScoreMods{};
  if (!m) return PA_OK;
  if (!(m->softcap >= 0.f) || !isfinite(m->softcap)) return PA_ERR_INVALID_ARG;
  if (m->alibi_slopes && (reinterpret_cast<uintptr_t>(m->alibi_slopes) & 3u))
    return PA_ERR_INVALID_ARG;
  if (m->mask && (!aligned16(m->mask) || m->mask_head_stride < 0 || m->mask_token_stride < 0 ||
                  m->mask_head_stride % 4 || m->mask_token_stride % 4 || m->mask_len <= 0))
    return PA_ERR_INVALID_ARG;
  r->softcap = m->softcap;
  r->alibi = m->alibi_slopes;
  r->mask = m->mask;
  r->mask_head = m->mask ? m->mask_head_stride : 0;
  r->mask_tok = m->mask ? m->mask_token_stride : 0;
  r->mask_len = m->mask ? m->mask_len : 0;
  return PA_OK;
}

}  // namespace

extern "C" {

const char* pa_status_string(pa_status s) {
  switch (s) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG: bad argument (nothing was launched)";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED: request outside this build's support";
    case PA_ERR_CUDA: return "PA_ERR_CUDA: a CUDA call failed";
    case PA_ERR_DEVICE_INDEX: return "PA_ERR_DEVICE_INDEX: the device saw a bad index or length";
    case PA_ERR_TIMEOUT: return "PA_ERR_TIMEOUT: a bounded device wait gave up";
  }
  return "pa: unknown status";
}

const char* pa_version(void) { return "pa 0.1 sm_100a"; }

void pa_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns.store(ns, std::memory_order_relaxed); }

pa_status pa_write_kv(const void* k, const void* v, const int64_t* slot_mapping,
                      int64_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                      void* k_cache, void* v_cache, int64_t num_blocks, int32_t block_size,
                      void* workspace, void* stream) {
  return pa_write_kv_ex(k, v, slot_mapping, num_tokens, num_kv_heads, head_dim, k_cache, v_cache,
                        num_blocks, block_size, 0, PA_DTYPE_BF16, workspace, stream);
}

pa_status pa_write_kv_ex(const void* k, const void* v, const int64_t* slot_mapping,
                         int64_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                         void* k_cache, void* v_cache, int64_t num_blocks, int32_t block_size,
                         int64_t block_stride, int32_t dtype, void* workspace, void* stream) {
  if (block_stride < 0) return PA_ERR_INVALID_ARG;
  pa_strides st{};
  st.cache_block = block_stride;
  return pa_write_kv_strided(k, v, slot_mapping, num_tokens, num_kv_heads, head_dim, k_cache,
                             v_cache, num_blocks, block_size, &st, dtype, workspace, stream);
}

pa_status pa_write_kv_strided(const void* k, const void* v, const int64_t* slot_mapping,
                              int64_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                              void* k_cache, void* v_cache, int64_t num_blocks,
                              int32_t block_size, const pa_strides* strides, int32_t dtype,
                              void* workspace, void* stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || head_dim % 8 != 0 ||
      num_blocks <= 0 || block_size <= 0)
    return PA_ERR_INVALID_ARG;
  if (dtype != PA_DTYPE_BF16 && dtype != PA_DTYPE_FP16) return PA_ERR_INVALID_ARG;
  Strides sd{};
  pa_status rs = resolve_cache(strides, block_size, num_kv_heads, head_dim, &sd);
  if (rs != PA_OK) return rs;
  int dshift = 0;
  while ((1 << dshift) < head_dim / 8) ++dshift;
  const bool dense = sd.cs == (int64_t)num_kv_heads * head_dim && sd.ch == head_dim;
  if (!dense && (1 << dshift) != head_dim / 8) return PA_ERR_UNSUPPORTED;
  if (num_tokens == 0) return PA_OK;
  if (!k || !v || !slot_mapping || !k_cache || !v_cache) return PA_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache) ||
      (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
    return PA_ERR_INVALID_ARG;
  const int row_vecs = num_kv_heads * head_dim / 8;
  uint32_t* err = workspace ? static_cast<uint32_t*>(workspace) : nullptr;
  cudaError_t e = pa::launch_write_kv(k, v, slot_mapping, num_tokens, row_vecs, k_cache, v_cache,
                                      num_blocks * (int64_t)block_size, block_size, sd.cb / 8,
                                      sd.cs / 8, sd.ch / 8, dshift, err, sm_count(),
                                      static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

size_t pa_attention_varlen_workspace_size(int32_t num_seqs, int64_t num_q_tokens,
                                          int32_t num_q_heads, int32_t num_kv_heads,
                                          int32_t head_dim) {
  if (num_seqs < 0 || num_q_tokens < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0)
    return 0;
  return pa::make_layout(num_seqs, num_q_tokens, num_q_heads, num_kv_heads, head_dim).total;
}

namespace {

// Every host-visible check of a varlen call, in order; nothing is launched or
// written.  On PA_OK, *sd, *mods and *L hold the resolved strides, modifiers
// and workspace layout.  *nothing_to_do is set when the call has no rows (the
// pointers are then not examined).  The workspace size is not compared here.
pa_status varlen_checks(const void* q, const void* k_cache, const void* v_cache,
                        const int32_t* block_tables, int32_t max_blocks_per_seq,
                        const int32_t* seq_lens, const int32_t* query_start_loc,
                        int32_t num_seqs, int64_t num_q_tokens, int32_t num_q_heads,
                        int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                        int64_t num_blocks, const pa_strides* strides, int32_t dtype,
                        int32_t max_query_len, int32_t max_seq_len, float scale, int32_t causal,
                        const int32_t* span_offsets, const int32_t* spans, int32_t num_spans,
                        const pa_score_mods* score_mods, const void* out, const void* workspace,
                        Strides* sd, pa::ScoreMods* mods, WorkspaceLayout* L,
                        bool* nothing_to_do) {
  *nothing_to_do = false;
  if (dtype != PA_DTYPE_BF16 && dtype != PA_DTYPE_FP16) return PA_ERR_INVALID_ARG;
  if (num_seqs < 0 || num_q_tokens < 0 || num_q_tokens > 0x7fffffffll || num_q_heads <= 0 ||
      num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0 || max_blocks_per_seq <= 0 ||
      num_blocks <= 0 || num_blocks > 0x7fffffffll || max_query_len < 0 || max_seq_len < 0 ||
      (causal != 0 && causal != 1) || !isfinite(scale) || scale < 0.f)
    return PA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (block_size < pa::kPageKeys || block_size > pa::kMaxBlockSize ||
      (block_size & (block_size - 1)) != 0)
    return PA_ERR_UNSUPPORTED;
  if (num_q_heads / num_kv_heads > pa::kMaxGroup) return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0 || num_q_tokens == 0) {
    *nothing_to_do = true;
    return PA_OK;
  }
  if (!q || !k_cache || !v_cache || !block_tables || !seq_lens || !query_start_loc || !out ||
      !workspace)
    return PA_ERR_INVALID_ARG;
  if (span_offsets && (num_spans < 0 || (num_spans > 0 && !spans) ||
                       (reinterpret_cast<uintptr_t>(span_offsets) & 3u) ||
                       (reinterpret_cast<uintptr_t>(spans) & 3u)))
    return PA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
      !aligned16(workspace) || (reinterpret_cast<uintptr_t>(block_tables) & 3u) ||
      (reinterpret_cast<uintptr_t>(seq_lens) & 3u) ||
      (reinterpret_cast<uintptr_t>(query_start_loc) & 3u))
    return PA_ERR_INVALID_ARG;
  pa_status rs = resolve_strides(strides, num_q_tokens, num_q_heads, num_kv_heads, head_dim,
                                 block_size, sd);
  if (rs != PA_OK) return rs;
  rs = resolve_mods(score_mods, mods);
  if (rs != PA_OK) return rs;
  if (mods->any() && !(scale > 0.f)) return PA_ERR_INVALID_ARG;
  *L = pa::make_layout(num_seqs, num_q_tokens, num_q_heads, num_kv_heads, head_dim);
  return PA_OK;
}

// pa_attention_varlen and pa_attention_varlen_spans (span_offsets non-null)
pa_status attention_varlen_impl(const void* q, const void* k_cache, const void* v_cache,
                                const int32_t* block_tables, int32_t max_blocks_per_seq,
                                const int32_t* seq_lens, const int32_t* query_start_loc,
                                int32_t num_seqs, int64_t num_q_tokens, int32_t num_q_heads,
                                int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                int64_t num_blocks, const pa_strides* strides, int32_t dtype,
                                int32_t max_query_len, int32_t max_seq_len,
                                float scale, int32_t causal, const int32_t* span_offsets,
                                const int32_t* spans, int32_t num_spans,
                                const pa_score_mods* score_mods, void* out,
                                void* workspace, size_t workspace_bytes, void* stream) {
  // ---- host-visible checks (nothing launched yet) ----
  Strides sd{};
  pa::ScoreMods mods{};
  WorkspaceLayout L{};
  bool nothing = false;
  pa_status rs = varlen_checks(q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                               query_start_loc, num_seqs, num_q_tokens, num_q_heads, num_kv_heads,
                               head_dim, block_size, num_blocks, strides, dtype, max_query_len,
                               max_seq_len, scale, causal, span_offsets, spans, num_spans,
                               score_mods, out, workspace, &sd, &mods, &L, &nothing);
  if (rs != PA_OK || nothing) return rs;
  if (workspace_bytes < L.total) return PA_ERR_INVALID_ARG;
  const bool fp16 = dtype == PA_DTYPE_FP16;
  const int group = num_q_heads / num_kv_heads;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  const int nsm = sm_count();
  const float scale_log2 = scale * 1.4426950408889634f;
  const bool run_prefill = max_query_len > 1;

  CUtensorMap q_map, k_map, v_map;
  if (run_prefill) {
    // dimensions ordered by increasing stride: (D, head, token) for a
    // token-major q, (D, token, head) for a head-major one; the kernel
    // swaps its coordinates to match (likewise slot and head of the cache)
    const cuuint32_t box_q[3] = {64, sd.q_hnd ? (cuuint32_t)pa::kPrefillTileM : 1u,
                                 sd.q_hnd ? 1u : (cuuint32_t)pa::kPrefillTileM};
    const cuuint64_t dq[3] = {(cuuint64_t)head_dim,
                              (cuuint64_t)(sd.q_hnd ? num_q_tokens : num_q_heads),
                              (cuuint64_t)(sd.q_hnd ? num_q_heads : num_q_tokens)};
    const cuuint64_t sq[2] = {(cuuint64_t)(sd.q_hnd ? sd.qt : sd.qh) * 2,
                              (cuuint64_t)(sd.q_hnd ? sd.qh : sd.qt) * 2};
    const cuuint32_t box_kv[4] = {64, sd.kv_hnd ? (cuuint32_t)pa::kPageKeys : 1u,
                                  sd.kv_hnd ? 1u : (cuuint32_t)pa::kPageKeys, 1};
    const cuuint64_t dkv[4] = {(cuuint64_t)head_dim,
                               (cuuint64_t)(sd.kv_hnd ? block_size : num_kv_heads),
                               (cuuint64_t)(sd.kv_hnd ? num_kv_heads : block_size),
                               (cuuint64_t)num_blocks};
    const cuuint64_t skv[3] = {(cuuint64_t)(sd.kv_hnd ? sd.cs : sd.ch) * 2,
                               (cuuint64_t)(sd.kv_hnd ? sd.ch : sd.cs) * 2,
                               (cuuint64_t)sd.cb * 2};
    if (!make_map(&q_map, q, 3, dq, sq, box_q, fp16) ||
        !make_map(&k_map, k_cache, 4, dkv, skv, box_kv, fp16) ||
        !make_map(&v_map, v_cache, 4, dkv, skv, box_kv, fp16))
      return PA_ERR_CUDA;
  }

  // decode CTAs compute their page ranges themselves for up to
  // kSelfPlanMaxSeqs sequences whose arrival counters fit the fixed counter
  // region (kept zero between calls); beyond that the plan kernel writes the
  // prefix and zeroes the counters
  const bool self_plan =
      num_seqs <= pa::kSelfPlanMaxSeqs &&
      pa::counter_slots_needed(num_seqs, num_q_heads, num_kv_heads) <= pa::kFixedCounterSlots;
  // A call with multi-query sequences runs its decode kernel on a side stream
  // beside the prefill kernel, each on the share of the SMs the plan kernel
  // picks (the prefill is tensor-bound and the decode HBM-bound, so the two
  // overlap); the side stream forks from the caller's stream after the plan
  // and joins it again before the call returns.
  SideStream* side = run_prefill ? side_stream(st) : nullptr;
  std::unique_lock<std::mutex> side_lock;
  if (side) side_lock = std::unique_lock<std::mutex>(side->mu);
  pa::SplitShape split{};
  if (side) split = pa::SplitShape{nsm, num_q_heads, num_kv_heads, head_dim};
  cudaError_t e = cudaSuccess;
  if (run_prefill || !self_plan) {
    pa::launch_plan(query_start_loc, seq_lens, num_seqs, num_q_tokens, max_blocks_per_seq,
                    block_size, max_query_len, max_seq_len, causal,
                    pa::counter_slots_needed(num_seqs, num_q_heads, num_kv_heads), span_offsets,
                    spans, num_spans, ws, L, split, st);
    e = cudaGetLastError();
    if (e != cudaSuccess) return PA_ERR_CUDA;
  }
  cudaStream_t dec_st = st;
  if (side) {
    if (cudaEventRecord(side->fork, st) != cudaSuccess ||
        cudaStreamWaitEvent(side->stream, side->fork, 0) != cudaSuccess)
      return PA_ERR_CUDA;
    dec_st = side->stream;
  }

  if (run_prefill) {
    pa::PrefillParams pp{};
    pp.block_tables = block_tables;
    pp.max_blocks_per_seq = max_blocks_per_seq;
    pp.block_size = block_size;
    pp.ppb_shift = pa::log2_pages_per_block(block_size);
    pp.num_q_heads = num_q_heads;
    pp.num_kv_heads = num_kv_heads;
    pp.group = group;
    pp.num_blocks = num_blocks;
    pp.num_q_tokens = num_q_tokens;
    pp.scale_log2 = scale_log2;
    pp.causal = causal;
    pp.span_offsets = span_offsets;
    pp.spans = spans;
    pp.num_spans = num_spans;
    pp.q_hnd = sd.q_hnd ? 1 : 0;
    pp.kv_hnd = sd.kv_hnd ? 1 : 0;
    pp.o_tok = sd.ot;
    pp.o_head = sd.oh;
    pp.scale = scale;
    pp.mods = mods;
    pp.out = static_cast<uint16_t*>(out);
    pp.ws = ws;
    pp.L = L;
    pp.wait_limit_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
    pp.split = side ? 1 : 0;
    e = pa::launch_prefill(pp, q_map, k_map, v_map, head_dim, fp16, nsm, st);
  }

  pa::DecodeParams dp{};
  dp.q = static_cast<const __nv_bfloat16*>(q);
  dp.k_cache = static_cast<const __nv_bfloat16*>(k_cache);
  dp.v_cache = static_cast<const __nv_bfloat16*>(v_cache);
  dp.block_tables = block_tables;
  dp.query_start_loc = query_start_loc;
  dp.seq_lens = seq_lens;
  dp.num_seqs = num_seqs;
  dp.num_q_tokens = num_q_tokens;
  dp.max_query_len = max_query_len;
  dp.max_blocks_per_seq = max_blocks_per_seq;
  dp.ppb_shift = pa::log2_pages_per_block(block_size);
  dp.max_seq_len = max_seq_len;
  dp.self_plan = self_plan ? 1 : 0;
  dp.split_sms = side ? nsm : 0;
  dp.num_q_heads = num_q_heads;
  dp.num_kv_heads = num_kv_heads;
  dp.group = group;
  dp.slices = pa::decode_slices(group);
  dp.num_blocks = num_blocks;
  dp.block_stride = sd.cb;
  dp.c_slot = sd.cs;
  dp.c_head = sd.ch;
  dp.q_tok = sd.qt;
  dp.q_head = sd.qh;
  dp.o_tok = sd.ot;
  dp.o_head = sd.oh;
  dp.scale = scale;
  dp.mods = mods;
  dp.scale_log2 = scale_log2;
  dp.out = static_cast<uint16_t*>(out);
  dp.ws = ws;
  dp.L = L;
  const cudaError_t e_dec = e == cudaSuccess ? pa::launch_decode(dp, head_dim, fp16, nsm, dec_st) : e;
  if (side) {
    // join even after a failed launch, so the caller's stream never runs ahead
    // of work queued on the side stream
    const bool joined = cudaEventRecord(side->join, side->stream) == cudaSuccess &&
                        cudaStreamWaitEvent(st, side->join, 0) == cudaSuccess;
    if (!joined && e_dec == cudaSuccess) return PA_ERR_CUDA;
  }
  e = e_dec;
  if (log_enabled())
    fprintf(stderr, "[pa] varlen S=%d T=%lld Hq=%d Hkv=%d D=%d prefill=%d sms=%d\n", num_seqs,
            (long long)num_q_tokens, num_q_heads, num_kv_heads, head_dim, (int)run_prefill, nsm);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace

}  // extern "C"

namespace pa {

pa_status check_varlen_args(const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* block_tables, int32_t max_blocks_per_seq,
                            const int32_t* seq_lens, const int32_t* query_start_loc,
                            int32_t num_seqs, int64_t num_q_tokens, int32_t num_q_heads,
                            int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                            int64_t num_blocks, int32_t max_query_len, int32_t max_seq_len,
                            float scale, int32_t causal, const void* out, const void* workspace,
                            size_t* workspace_bytes, bool* nothing_to_do) {
  Strides sd{};
  ScoreMods mods{};
  WorkspaceLayout L{};
  const pa_status rs = varlen_checks(
      q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens, query_start_loc, num_seqs,
      num_q_tokens, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, nullptr,
      PA_DTYPE_BF16, max_query_len, max_seq_len, scale, causal, nullptr, nullptr, 0, nullptr, out,
      workspace, &sd, &mods, &L, nothing_to_do);
  *workspace_bytes = (rs == PA_OK && !*nothing_to_do) ? L.total : 0;
  return rs;
}

}  // namespace pa

extern "C" {

pa_status pa_attention_varlen(const void* q, const void* k_cache, const void* v_cache,
                              const int32_t* block_tables, int32_t max_blocks_per_seq,
                              const int32_t* seq_lens, const int32_t* query_start_loc,
                              int32_t num_seqs, int64_t num_q_tokens, int32_t num_q_heads,
                              int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                              int64_t num_blocks, int32_t max_query_len, int32_t max_seq_len,
                              float scale, int32_t causal, void* out, void* workspace,
                              size_t workspace_bytes, void* stream) {
  return attention_varlen_impl(q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                               query_start_loc, num_seqs, num_q_tokens, num_q_heads, num_kv_heads,
                               head_dim, block_size, num_blocks, nullptr, PA_DTYPE_BF16,
                               max_query_len, max_seq_len, scale, causal, nullptr, nullptr, 0,
                               nullptr, out, workspace, workspace_bytes, stream);
}

pa_status pa_attention_varlen_spans(const void* q, const void* k_cache, const void* v_cache,
                                    const int32_t* block_tables, int32_t max_blocks_per_seq,
                                    const int32_t* seq_lens, const int32_t* query_start_loc,
                                    int32_t num_seqs, int64_t num_q_tokens, int32_t num_q_heads,
                                    int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                    int64_t num_blocks, int32_t max_query_len, int32_t max_seq_len,
                                    float scale, const int32_t* span_offsets, const int32_t* spans,
                                    int32_t num_spans, void* out, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  if (!span_offsets && num_seqs > 0) return PA_ERR_INVALID_ARG;
  return attention_varlen_impl(q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                               query_start_loc, num_seqs, num_q_tokens, num_q_heads, num_kv_heads,
                               head_dim, block_size, num_blocks, nullptr, PA_DTYPE_BF16,
                               max_query_len, max_seq_len, scale, 1, span_offsets, spans,
                               num_spans, nullptr, out, workspace, workspace_bytes, stream);
}

pa_status pa_attention_varlen_ex(const void* q, const void* k_cache, const void* v_cache,
                                 const int32_t* block_tables, int32_t max_blocks_per_seq,
                                 const int32_t* seq_lens, const int32_t* query_start_loc,
                                 int32_t num_seqs, int64_t num_q_tokens, int32_t num_q_heads,
                                 int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                 int64_t num_blocks, int64_t block_stride, int32_t dtype,
                                 int32_t max_query_len, int32_t max_seq_len, float scale,
                                 int32_t causal, const int32_t* span_offsets, const int32_t* spans,
                                 int32_t num_spans, void* out, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  if (block_stride < 0) return PA_ERR_INVALID_ARG;
  pa_strides st{};
  st.cache_block = block_stride;
  return attention_varlen_impl(q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                               query_start_loc, num_seqs, num_q_tokens, num_q_heads, num_kv_heads,
                               head_dim, block_size, num_blocks, &st, dtype, max_query_len,
                               max_seq_len, scale, span_offsets ? 1 : causal, span_offsets, spans,
                               num_spans, nullptr, out, workspace, workspace_bytes, stream);
}

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
                                   size_t workspace_bytes, void* stream) {
  return attention_varlen_impl(q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                               query_start_loc, num_seqs, num_q_tokens, num_q_heads, num_kv_heads,
                               head_dim, block_size, num_blocks, strides, dtype, max_query_len,
                               max_seq_len, scale, span_offsets ? 1 : causal, span_offsets, spans,
                               num_spans, mods, out, workspace, workspace_bytes, stream);
}

pa_status pa_attention_smallseq(const void* q, const void* k, const void* v,
                                const int32_t* cu_seqlens_kv, int32_t batch, int32_t num_q_heads,
                                int32_t num_kv_heads, int32_t head_dim, int32_t max_seqlen_kv,
                                float scale, void* out, void* workspace, void* stream) {
  return pa_attention_smallseq_ex(q, k, v, cu_seqlens_kv, batch, num_q_heads, num_kv_heads,
                                  head_dim, max_seqlen_kv, scale, PA_DTYPE_BF16, out, nullptr, 0,
                                  workspace, stream);
}

pa_status pa_attention_smallseq_ex(const void* q, const void* k, const void* v,
                                   const int32_t* cu_seqlens_kv, int32_t batch,
                                   int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                   int32_t max_seqlen_kv, float scale, int32_t dtype, void* out,
                                   void* weights, int32_t weights_len, void* workspace,
                                   void* stream) {
  if (dtype != PA_DTYPE_BF16 && dtype != PA_DTYPE_FP16) return PA_ERR_INVALID_ARG;
  if (weights && (weights_len <= 0 || (reinterpret_cast<uintptr_t>(weights) & 1u)))
    return PA_ERR_INVALID_ARG;
  if (batch < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0 ||
      max_seqlen_kv < 0 || !isfinite(scale))
    return PA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (max_seqlen_kv > 16) return PA_ERR_UNSUPPORTED;
  if (batch == 0) return PA_OK;
  if (!q || !k || !v || !cu_seqlens_kv || !out) return PA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens_kv) & 3u) || (workspace && !aligned16(workspace)))
    return PA_ERR_INVALID_ARG;
  pa::SmallSeqParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.cu_seqlens_kv = cu_seqlens_kv;
  p.batch = batch;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.group = num_q_heads / num_kv_heads;
  p.max_seqlen_kv = max_seqlen_kv;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.out = static_cast<uint16_t*>(out);
  p.err = static_cast<uint32_t*>(workspace);
  p.weights = static_cast<uint16_t*>(weights);
  p.weights_len = weights ? weights_len : 0;
  cudaError_t e = pa::launch_smallseq(p, head_dim, dtype == PA_DTYPE_FP16, sm_count(),
                                      static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_attention_smallseq_bwd(const void* q, const void* k, const void* v,
                                    const void* dout, const void* weights, int32_t weights_len,
                                    const int32_t* cu_seqlens_kv, int32_t batch,
                                    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                    int32_t max_seqlen_kv, float scale, int32_t dtype, void* dq,
                                    void* dk, void* dv, void* workspace, void* stream) {
  if (dtype != PA_DTYPE_BF16 && dtype != PA_DTYPE_FP16) return PA_ERR_INVALID_ARG;
  if (batch < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0 ||
      max_seqlen_kv < 0 || weights_len <= 0 || !isfinite(scale))
    return PA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (max_seqlen_kv > 16 || num_q_heads / num_kv_heads > 16) return PA_ERR_UNSUPPORTED;
  if (batch == 0) return PA_OK;
  if (!q || !k || !v || !dout || !weights || !cu_seqlens_kv || !dq || !dk || !dv)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || (reinterpret_cast<uintptr_t>(weights) & 1u) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens_kv) & 3u) || (workspace && !aligned16(workspace)))
    return PA_ERR_INVALID_ARG;
  pa::SmallSeqBwdParams p{};
  p.q = static_cast<const uint16_t*>(q);
  p.k = static_cast<const uint16_t*>(k);
  p.v = static_cast<const uint16_t*>(v);
  p.dout = static_cast<const uint16_t*>(dout);
  p.weights = static_cast<const uint16_t*>(weights);
  p.cu_seqlens_kv = cu_seqlens_kv;
  p.batch = batch;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.group = num_q_heads / num_kv_heads;
  p.max_seqlen_kv = max_seqlen_kv;
  p.weights_len = weights_len;
  p.scale = scale;
  p.dq = static_cast<uint16_t*>(dq);
  p.dk = static_cast<uint16_t*>(dk);
  p.dv = static_cast<uint16_t*>(dv);
  p.err = static_cast<uint32_t*>(workspace);
  cudaError_t e = pa::launch_smallseq_bwd(p, head_dim, dtype == PA_DTYPE_FP16, sm_count(),
                                          static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_get_error(void* workspace, void* stream, uint32_t* bits) {
  if (bits) *bits = 0;
  if (!workspace) return PA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, workspace, sizeof word, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return PA_ERR_CUDA;
  if (cudaMemsetAsync(workspace, 0, sizeof word, st) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return PA_ERR_CUDA;
  if (bits) *bits = word;
  if (word == 0) return PA_OK;
  return (word & PA_DEVERR_TIMEOUT) ? PA_ERR_TIMEOUT : PA_ERR_DEVICE_INDEX;
}

}  // extern "C"
