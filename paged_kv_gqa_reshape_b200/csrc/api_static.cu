// pa_attention_varlen_static: paged varlen attention for callers that cannot
// allocate device memory.
//
// Some callers may not call cudaMalloc at all: a host program that owns every
// byte of device memory through its own pool allocator and forbids any other
// allocation, or a latency-critical serving path where cudaMalloc/cudaFree
// would synchronise the device.  Such callers still pass their inputs and
// outputs, but cannot hand over a workspace.  This entry point runs exactly
// the same kernels as pa_attention_varlen, with the workspace placed in a
// file-scope device array of PA_STATIC_SCRATCH_BYTES bytes instead.
//
// Properties the caller must know:
//  - Every GPU that loads this library holds the array until the process
//    exits, whether or not this entry point is ever called.
//  - The first call on a device looks up the array's device address
//    (cudaGetSymbolAddress) with that device current, and caches it; make that
//    first call before any stream capture.
//  - All calls share the one array, which keeps the last call's contents.
//    What a call needs at zero is its split-KV arrival counters: they sit in
//    a region of the array that only ever holds counters, which starts at
//    zero (a __device__ array is zero-initialised when the module loads) and
//    is returned to zero by every merge that uses a counter; when the plan
//    kernel runs (any batch with a multi-query sequence, or too many
//    sequences for the decode CTAs to plan for themselves) it also zeroes
//    them.  The plan lists and partial results are rebuilt by each call.
//    Calls whose executions overlap on the GPU (different streams, or
//    different host threads) race on the array and must not be issued.
//  - Device-side index errors are handled as in pa_attention_varlen (rows
//    skipped, reads zero-filled) but cannot be read back: the error word lives
//    in the shared array, which nothing reads.
//  - Bad arguments are reported exactly as pa_attention_varlen reports them;
//    then sizes whose workspace would exceed PA_STATIC_SCRATCH_BYTES are
//    rejected with PA_ERR_UNSUPPORTED.  Both happen before anything is
//    launched or written.
// Nothing here calls cudaMalloc, cudaFree or any allocating library routine.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/pa.h"
#include "kernels.h"

namespace {

constexpr int kMaxDevices = 64;

// The scratch area: one copy per device that loads the library.
static __device__ __align__(256) unsigned char g_pa_static_scratch[PA_STATIC_SCRATCH_BYTES];

void* g_scratch_addr[kMaxDevices];  // device address of the array, per device
std::mutex g_scratch_mu;

// Device address of the current device's copy of the array (looked up once
// per device; the array's name in host code is only a host-side stand-in).
pa_status scratch_address(void** addr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_pa_static_scratch) != cudaSuccess || p == nullptr)
      return PA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *addr = g_scratch_addr[dev];
  return PA_OK;
}

}  // namespace

extern "C" pa_status pa_attention_varlen_static(
    const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
    int32_t max_blocks_per_seq, const int32_t* seq_lens, const int32_t* query_start_loc,
    int32_t num_seqs, int64_t num_q_tokens, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t block_size, int64_t num_blocks, int32_t max_query_len,
    int32_t max_seq_len, float scale, int32_t causal, void* out, void* stream) {
  // The arguments are checked first, with the array's alignment standing in
  // for the workspace pointer (the array is 256-byte aligned, so that check
  // passes for it), so that a bad call is reported before any CUDA call.
  const void* aligned_stand_in = reinterpret_cast<const void*>(uintptr_t(256));
  size_t need = 0;
  bool nothing = false;
  pa_status st = pa::check_varlen_args(
      q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens, query_start_loc, num_seqs,
      num_q_tokens, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, max_query_len,
      max_seq_len, scale, causal, out, aligned_stand_in, &need, &nothing);
  if (st != PA_OK || nothing) return st;
  if (need > (size_t)PA_STATIC_SCRATCH_BYTES) return PA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != PA_OK) return st;
  return pa_attention_varlen(q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                             query_start_loc, num_seqs, num_q_tokens, num_q_heads, num_kv_heads,
                             head_dim, block_size, num_blocks, max_query_len, max_seq_len, scale,
                             causal, out, scratch, (size_t)PA_STATIC_SCRATCH_BYTES, stream);
}
