// Split-KV decode attention over the paged cache (single-query sequences).
//
// Work item = (sequence, key chunk, KV head).  One CTA of 4 warps owns an
// item; its warps take the chunk's 16-key pages round-robin.  The query rows
// of the KV head's whole GQA group (g = Hq/Hkv <= 16 heads of the one decode
// token) form the M = 16 rows of an m16n8k16 bf16 tile, so each K/V page is
// read from HBM once for all g heads (the repeat_interleave expansion of
// vllm-spyre PR #853 "Pytorch Native Attention on Spyre" is never
// materialised).  Decode is HBM-bound: the contraction is ~g FLOP per byte,
// so the legacy mma.sync path keeps up with the 16-key pages and tcgen05's
// minimum M of 64 would buy nothing.
//
// Memory path: every warp streams its pages through a private NSTAGE-deep
// ring of cp.async 16-byte copies (XOR-swizzled rows, conflict-free ldmatrix),
// and its producer runs ahead across item boundaries, so the ring never
// drains between items.  Keys past the sequence end are zero-filled instead
// of read; a block id outside the pool is reported and read as zeros.
//
// Per page: S = Q.K^T (fp32), masked, online softmax in the log2 domain
// (scale folded with log2 e), P rounded to bf16, O += P.V.  At item end the
// four warps' (max, sum, O) states are merged through shared memory.  A
// sequence with one chunk writes bf16 output directly; otherwise the chunk
// writes a normalised fp32 partial plus its log2-sum-exp, and the last CTA to
// finish a (sequence, KV head) merges all chunks (arrival counter + fences),
// so no separate combine launch is needed.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "layout.h"

namespace pa {



template <int D, int NSTAGE>
struct DecodeShape {
  static constexpr int kChunks = D / 8;               // 16-byte chunks per row
  static constexpr int kPageElems = kPageKeys * D;    // one page of one KV head
  static constexpr int kWarpStageBytes = 2 * kPageElems * 2;  // K + V
  static constexpr int kRingBytes = kDecodeWarps * NSTAGE * kWarpStageBytes;
  static __host__ __device__ constexpr int combine_bytes(int g) {
    return kDecodeWarps * g * (2 + D) * 4;
  }
  static __host__ __device__ constexpr int smem_bytes(int g) {
    return kRingBytes + combine_bytes(g);
  }
};

namespace {

// The item a producer or consumer is working on.
struct Item {
  int seq;
  int kvh;
  int chunk;
  int first_key;  // first key of the chunk
  int n_keys;     // keys in the chunk
  int n_pages;
  int kv_len;
};

__device__ __forceinline__ Item load_item(int item, const int2* pairs, const SeqInfo* info,
                                          int num_kv_heads) {
  Item it;
  int2 pr = pairs[item / num_kv_heads];
  it.seq = pr.x;
  it.chunk = pr.y;
  it.kvh = item % num_kv_heads;
  SeqInfo si = info[pr.x];
  it.kv_len = si.kv_len;
  it.first_key = pr.y * si.chunk_len;
  it.n_keys = max(0, min(si.chunk_len, si.kv_len - it.first_key));
  it.n_pages = (it.n_keys + kPageKeys - 1) / kPageKeys;
  return it;
}

}  // namespace

template <int D, int NSTAGE>
__global__ void __launch_bounds__(kDecodeWarps * 32, 2) decode_kernel(DecodeParams p) {
  using Shape = DecodeShape<D, NSTAGE>;
  constexpr int CH = Shape::kChunks;
  constexpr int KSTEPS = D / 16;
  constexpr int NT = D / 8;  // output n-tiles of 8 columns

  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int g = p.group;
  const int Hkv = p.num_kv_heads;

  unsigned char* ws = p.ws;
  uint32_t* err = reinterpret_cast<uint32_t*>(ws + p.L.err);
  const PlanHeader* hdr = reinterpret_cast<const PlanHeader*>(ws + p.L.header);
  const SeqInfo* info = reinterpret_cast<const SeqInfo*>(ws + p.L.seq_info);
  const int2* pairs = reinterpret_cast<const int2*>(ws + p.L.pairs);
  int32_t* counters = reinterpret_cast<int32_t*>(ws + p.L.counters);
  float* lse_buf = reinterpret_cast<float*>(ws + p.L.lse);
  float* part_buf = reinterpret_cast<float*>(ws + p.L.partial);

  const int num_items = hdr->num_decode_pairs * Hkv;

  __nv_bfloat16* ring =
      reinterpret_cast<__nv_bfloat16*>(smem) + (size_t)warp * NSTAGE * 2 * Shape::kPageElems;
  float* comb_m = reinterpret_cast<float*>(smem + Shape::kRingBytes);
  float* comb_l = comb_m + kDecodeWarps * g;
  float* comb_o = comb_l + kDecodeWarps * g;
  __shared__ int s_last;

  const size_t row_stride = (size_t)Hkv * D;  // elements between consecutive slots

  // ---------------- producer: this warp's page stream ----------------------
  int p_item = blockIdx.x;
  int p_page = warp;
  Item pit;
  if (p_item < num_items) pit = load_item(p_item, pairs, info, Hkv);
  auto p_skip_empty = [&]() {
    while (p_item < num_items && p_page >= pit.n_pages) {
      p_item += gridDim.x;
      p_page = warp;
      if (p_item < num_items) pit = load_item(p_item, pairs, info, Hkv);
    }
  };
  p_skip_empty();

  auto issue = [&](int slot) {
    if (p_item < num_items) {
      const int key0 = pit.first_key + p_page * kPageKeys;
      const int32_t* table = p.block_tables + (size_t)pit.seq * p.max_blocks_per_seq;
      const long long block = table[key0 / kPageKeys];
      const bool block_ok = block >= 0 && block < p.num_blocks;
      if (!block_ok && lane == 0) raise_error(err, PA_DEVERR_BLOCK);
      const long long safe_block = block_ok ? block : 0;
      __nv_bfloat16* kdst = ring + slot * 2 * Shape::kPageElems;
      __nv_bfloat16* vdst = kdst + Shape::kPageElems;
      const size_t base = ((size_t)safe_block * kPageKeys * Hkv + pit.kvh) * D;
#pragma unroll
      for (int i = 0; i < kPageKeys * CH / 32; ++i) {
        const int idx = i * 32 + lane;
        const int r = idx / CH, c = idx % CH;
        const bool ok = block_ok && (key0 + r < pit.kv_len);
        const size_t src = base + (size_t)r * row_stride + c * 8;
        const int dst = r * D + ((c ^ (r & 7)) * 8);
        cp_async_16(smem_u32(kdst + dst), p.k_cache + (ok ? src : 0), ok);
        cp_async_16(smem_u32(vdst + dst), p.v_cache + (ok ? src : 0), ok);
      }
      p_page += kDecodeWarps;
      p_skip_empty();
    }
    cp_async_commit();
  };

#pragma unroll
  for (int s = 0; s < NSTAGE; ++s) issue(s);
  int c_slot = 0;

  const int gr = lane >> 2;  // fragment row (head within the group)
  const int tq = lane & 3;   // fragment column pair

  for (int c_item = blockIdx.x; c_item < num_items; c_item += gridDim.x) {
    const Item it = load_item(c_item, pairs, info, Hkv);
    const SeqInfo si = info[it.seq];
    const int tok = si.q_start;

    // Q fragments (A operand) for the group's rows; rows >= g are zero.
    uint32_t qa[KSTEPS][4];
    {
      const uint32_t* q32 = reinterpret_cast<const uint32_t*>(p.q);
      const size_t row0 = ((size_t)tok * p.num_q_heads + (size_t)it.kvh * g + gr) * D;
      const size_t row1 = row0 + (size_t)8 * D;
#pragma unroll
      for (int ks = 0; ks < KSTEPS; ++ks) {
        const int col = ks * 16 + tq * 2;
        qa[ks][0] = gr < g ? q32[(row0 + col) / 2] : 0u;
        qa[ks][1] = gr + 8 < g ? q32[(row1 + col) / 2] : 0u;
        qa[ks][2] = gr < g ? q32[(row0 + col + 8) / 2] : 0u;
        qa[ks][3] = gr + 8 < g ? q32[(row1 + col + 8) / 2] : 0u;
      }
    }

    float o[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

    for (int pg = warp; pg < it.n_pages; pg += kDecodeWarps) {
      cp_async_wait<NSTAGE - 1>();
      __syncwarp();
      const __nv_bfloat16* ks_ = ring + c_slot * 2 * Shape::kPageElems;
      const __nv_bfloat16* vs_ = ks_ + Shape::kPageElems;
      const uint32_t kbase = smem_u32(ks_), vbase = smem_u32(vs_);

      // ---- S = Q . K^T for 16 keys (two n-tiles of 8) ----
      float s[2][4];
#pragma unroll
      for (int n = 0; n < 2; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
      {
        const int mi = lane >> 3, rr = lane & 7;
        const int key = (mi >> 1) * 8 + rr;
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks) {
          const int chunk = ks * 2 + (mi & 1);
          const uint32_t addr = kbase + (key * D + ((chunk ^ (key & 7)) * 8)) * 2;
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4(addr, b0, b1, b2, b3);
          mma_bf16_16816(s[0], qa[ks], b0, b1);
          mma_bf16_16816(s[1], qa[ks], b2, b3);
        }
      }
      // ---- mask + online softmax (log2 domain) ----
      const int key0 = it.first_key + pg * kPageKeys;
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int n = 0; n < 2; ++n) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = key0 + n * 8 + tq * 2 + (e & 1);
          float v = s[n][e] * p.scale_log2;
          if (key >= it.kv_len) v = -INFINITY;
          s[n][e] = v;
        }
        mx0 = fmaxf(mx0, fmaxf(s[n][0], s[n][1]));
        mx1 = fmaxf(mx1, fmaxf(s[n][2], s[n][3]));
      }
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      const float base0 = mn0 == -INFINITY ? 0.f : mn0;
      const float base1 = mn1 == -INFINITY ? 0.f : mn1;
      const float a0 = fast_exp2(m0 - base0), a1 = fast_exp2(m1 - base1);
      m0 = mn0;
      m1 = mn1;
      float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
      for (int n = 0; n < 2; ++n) {
        s[n][0] = fast_exp2(s[n][0] - base0);
        s[n][1] = fast_exp2(s[n][1] - base0);
        s[n][2] = fast_exp2(s[n][2] - base1);
        s[n][3] = fast_exp2(s[n][3] - base1);
        rs0 += s[n][0] + s[n][1];
        rs1 += s[n][2] + s[n][3];
      }
      l0 = l0 * a0 + rs0;
      l1 = l1 * a1 + rs1;
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        o[n][0] *= a0;
        o[n][1] *= a0;
        o[n][2] *= a1;
        o[n][3] *= a1;
      }
      uint32_t pa[4];
      pa[0] = pack_bf16x2(s[0][0], s[0][1]);
      pa[1] = pack_bf16x2(s[0][2], s[0][3]);
      pa[2] = pack_bf16x2(s[1][0], s[1][1]);
      pa[3] = pack_bf16x2(s[1][2], s[1][3]);
      // ---- O += P . V ----
      {
        const int mi = lane >> 3, rr = lane & 7;
        const int key = (mi & 1) * 8 + rr;
#pragma unroll
        for (int dp = 0; dp < D / 16; ++dp) {
          const int chunk = dp * 2 + (mi >> 1);
          const uint32_t addr = vbase + (key * D + ((chunk ^ (key & 7)) * 8)) * 2;
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4_trans(addr, b0, b1, b2, b3);
          mma_bf16_16816(o[2 * dp], pa, b0, b1);
          mma_bf16_16816(o[2 * dp + 1], pa, b2, b3);
        }
      }
      __syncwarp();
      issue(c_slot);  // refill the slot just consumed (may belong to a later item)
      c_slot = (c_slot + 1 == NSTAGE) ? 0 : c_slot + 1;
    }

    // ---- merge the four warps' states ----
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    if (tq == 0) {
      if (gr < g) {
        comb_m[warp * g + gr] = m0;
        comb_l[warp * g + gr] = l0;
      }
      if (gr + 8 < g) {
        comb_m[warp * g + gr + 8] = m1;
        comb_l[warp * g + gr + 8] = l1;
      }
    }
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int d = n * 8 + tq * 2;
      if (gr < g) {
        comb_o[(warp * g + gr) * D + d] = o[n][0];
        comb_o[(warp * g + gr) * D + d + 1] = o[n][1];
      }
      if (gr + 8 < g) {
        comb_o[(warp * g + gr + 8) * D + d] = o[n][2];
        comb_o[(warp * g + gr + 8) * D + d + 1] = o[n][3];
      }
    }
    __syncthreads();

    const int n_chunks = si.n_chunks;
    const int pair = si.pair_base + it.chunk;
    for (int e = threadIdx.x; e < g * (D / 8); e += blockDim.x) {
      const int r = e / (D / 8);
      const int d0 = (e % (D / 8)) * 8;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kDecodeWarps; ++w) M = fmaxf(M, comb_m[w * g + r]);
      float f[kDecodeWarps];
      float Lsum = 0.f;
#pragma unroll
      for (int w = 0; w < kDecodeWarps; ++w) {
        const float mw = comb_m[w * g + r];
        f[w] = (mw == -INFINITY) ? 0.f : fast_exp2(mw - M);
        Lsum += comb_l[w * g + r] * f[w];
      }
      const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
      float acc[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float a = 0.f;
#pragma unroll
        for (int w = 0; w < kDecodeWarps; ++w) a += comb_o[(w * g + r) * D + d0 + j] * f[w];
        acc[j] = a * inv;
      }
      const int head = it.kvh * g + r;
      if (n_chunks <= 1) {
        uint4 v;
        v.x = pack_bf16x2(acc[0], acc[1]);
        v.y = pack_bf16x2(acc[2], acc[3]);
        v.z = pack_bf16x2(acc[4], acc[5]);
        v.w = pack_bf16x2(acc[6], acc[7]);
        *reinterpret_cast<uint4*>(p.out + ((size_t)tok * p.num_q_heads + head) * D + d0) = v;
      } else {
        float* dst = part_buf + ((size_t)pair * p.num_q_heads + head) * D + d0;
        *reinterpret_cast<float4*>(dst) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        *reinterpret_cast<float4*>(dst + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
        if (d0 == 0)
          lse_buf[(size_t)pair * p.num_q_heads + head] =
              Lsum > 0.f ? M + log2f(Lsum) : -INFINITY;
      }
    }

    if (n_chunks > 1) {
      // split-KV merge by the last CTA to finish this (sequence, KV head)
      __threadfence();
      __syncthreads();
      if (threadIdx.x == 0) {
        const int old = atomicAdd(&counters[it.seq * Hkv + it.kvh], 1);
        s_last = (old == n_chunks - 1);
      }
      __syncthreads();
      if (s_last) {
        __threadfence();
        const int pb = si.pair_base;
        for (int e = threadIdx.x; e < g * (D / 8); e += blockDim.x) {
          const int r = e / (D / 8);
          const int d0 = (e % (D / 8)) * 8;
          const int head = it.kvh * g + r;
          float M = -INFINITY;
          for (int c = 0; c < n_chunks; ++c)
            M = fmaxf(M, __ldcg(lse_buf + (size_t)(pb + c) * p.num_q_heads + head));
          float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          float wsum = 0.f;
          if (M != -INFINITY) {
            for (int c = 0; c < n_chunks; ++c) {
              const float lc = __ldcg(lse_buf + (size_t)(pb + c) * p.num_q_heads + head);
              const float w = (lc == -INFINITY) ? 0.f : fast_exp2(lc - M);
              wsum += w;
              const float* src = part_buf + ((size_t)(pb + c) * p.num_q_heads + head) * D + d0;
              const float4 x0 = __ldcg(reinterpret_cast<const float4*>(src));
              const float4 x1 = __ldcg(reinterpret_cast<const float4*>(src + 4));
              acc[0] += w * x0.x;
              acc[1] += w * x0.y;
              acc[2] += w * x0.z;
              acc[3] += w * x0.w;
              acc[4] += w * x1.x;
              acc[5] += w * x1.y;
              acc[6] += w * x1.z;
              acc[7] += w * x1.w;
            }
          }
          const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
          uint4 v;
          v.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
          v.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
          v.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
          v.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
          *reinterpret_cast<uint4*>(p.out + ((size_t)tok * p.num_q_heads + head) * D + d0) = v;
        }
      }
    }
    __syncthreads();  // the combine area is rewritten by the next item
  }
  cp_async_wait<0>();
}

template <int D, int NSTAGE>
static cudaError_t launch_decode_t(const DecodeParams& p, int grid, cudaStream_t stream) {
  using Shape = DecodeShape<D, NSTAGE>;
  const int smem = Shape::smem_bytes(p.group);
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, NSTAGE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  decode_kernel<D, NSTAGE><<<grid, kDecodeWarps * 32, smem, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeParams& p, int head_dim, int grid, cudaStream_t stream) {
  if (head_dim == 128) return launch_decode_t<128, 2>(p, grid, stream);
  return launch_decode_t<64, 3>(p, grid, stream);
}

}  // namespace pa
