// KV-cache write through slot_mapping (the cache-update step of vllm-spyre
// PR #853 "Pytorch Native Attention on Spyre", description, step 1).
//
// One warp per token: it reads the token's K and V rows (num_kv_heads *
// head_dim elements each, contiguous) with 16-byte loads and stores them to
// slot slot_mapping[t] of the caches: a dense NHD cache holds the slot's
// [Hkv, D] row contiguously; other layouts (HND: each head's D elements of
// the slot at their own stride) take the per-head destination.  Pure
// bandwidth: every byte is read once and written once.  A negative slot marks
// a padding token (skipped); a slot beyond the pool is skipped and reported.
#include "common.cuh"
#include "kernels.h"

namespace pa {

__global__ void __launch_bounds__(256) write_kv_kernel(const uint4* __restrict__ k,
                                                       const uint4* __restrict__ v,
                                                       const int64_t* __restrict__ slot_mapping,
                                                       long long num_tokens, int row_vecs,
                                                       uint4* __restrict__ k_cache,
                                                       uint4* __restrict__ v_cache,
                                                       long long num_slots, int block_size,
                                                       long long block_vecs, long long slot_vecs,
                                                       long long head_vecs, int dshift,
                                                       uint32_t* err) {
  // dense rows ([Hkv, D] contiguous per slot): vector idx of the token row
  // lands at vector idx of the slot row
  const bool dense = head_vecs == (1ll << dshift) && slot_vecs == row_vecs;
  // the attention call that follows reads the caches only after this grid has
  // completed (griddep_wait); its planning may overlap this scatter
  griddep_launch_dependents();
  // Launched with programmatic stream serialisation: when the previous kernel
  // lets this one start early (the decode kernel does, so that the next
  // step's scatter is resident before it ends), wait here, before touching
  // any input or the caches, until it has completed and its writes are
  // visible (it may still be reading the cache rows this grid overwrites).
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long t = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
       t < num_tokens; t += warps) {
    const long long slot = slot_mapping[t];
    if (slot < 0) continue;
    if (slot >= num_slots) {
      if (lane == 0) raise_error(err, PA_DEVERR_SLOT);
      continue;
    }
    const uint4* ks = k + t * row_vecs;
    const uint4* vs = v + t * row_vecs;
    // block slot / block_size, row slot % block_size (blocks block_vecs apart)
    const long long at = (slot / block_size) * block_vecs + (slot % block_size) * slot_vecs;
    uint4* kd = k_cache + at;
    uint4* vd = v_cache + at;
    // vector idx = head * (D / 8) + c of the token row goes to head * head_vecs + c
    auto dst = [&](int idx) -> long long {
      return dense ? idx : (long long)(idx >> dshift) * head_vecs + (idx & ((1 << dshift) - 1));
    };
    // issue all loads of this lane before its stores (row_vecs <= 32 * 8 here)
    constexpr int kMaxPerLane = 8;
    uint4 kr[kMaxPerLane], vr[kMaxPerLane];
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
      const int idx = i * 32 + lane;
      if (idx < row_vecs) {
        kr[i] = __ldcs(ks + idx);
        vr[i] = __ldcs(vs + idx);
      }
    }
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
      const int idx = i * 32 + lane;
      if (idx < row_vecs) {
        kd[dst(idx)] = kr[i];
        vd[dst(idx)] = vr[i];
      }
    }
    // rows wider than 32 * 8 vectors (Hkv * D > 2048) continue here
    for (int idx = kMaxPerLane * 32 + lane; idx < row_vecs; idx += 32) {
      kd[dst(idx)] = __ldcs(ks + idx);
      vd[dst(idx)] = __ldcs(vs + idx);
    }
  }
}

cudaError_t launch_write_kv(const void* k, const void* v, const int64_t* slot_mapping,
                            int64_t num_tokens, int row_vecs, void* k_cache, void* v_cache,
                            int64_t num_slots, int block_size, int64_t block_vecs,
                            int64_t slot_vecs, int64_t head_vecs, int dshift, uint32_t* err,
                            int num_sms, cudaStream_t stream) {
  if (num_tokens <= 0) return cudaSuccess;
  const int threads = 256;
  const long long warps_needed = num_tokens;
  long long blocks = (warps_needed + (threads / 32) - 1) / (threads / 32);
  const long long cap = (long long)num_sms * 8;  // 8 resident 256-thread CTAs per SM
  if (blocks > cap) blocks = cap;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, write_kv_kernel, static_cast<const uint4*>(k),
                            static_cast<const uint4*>(v), slot_mapping, (long long)num_tokens,
                            row_vecs, static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache),
                            (long long)num_slots, block_size, (long long)block_vecs,
                            (long long)slot_vecs, (long long)head_vecs, dshift, err);
}

}  // namespace pa
