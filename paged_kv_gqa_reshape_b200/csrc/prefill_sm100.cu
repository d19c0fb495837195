// Paged prefill / chunked-prefill attention on the 5th-generation tensor cores.
//
// Computes, for every query row of every multi-query sequence, the masked
// softmax attention of vllm-spyre PR #853 "Pytorch Native Attention on Spyre"
// (description, steps 2-6) with bottom-right causal alignment (vllm-omni
// PR #9244, kernel-semantics review: query i of Sq sees key j iff
// j <= (Skv - Sq) + i), GQA head sharing, and zeros for a row with no visible
// key.  The pages' own kernels (Spyre's fused-head matmul with a block-
// diagonal mask, BestLA's CPU tiles) are prior art; this is a flash-style
// kernel written for sm_100a:
//
//  * persistent grid, one CTA per SM, walking the plan's tile list (128 query
//    rows of one head per work item, most expensive first);
//  * warp 0 (one lane): TMA producer.  Q tile via a 3-D map over
//    [tokens, Hq, D]; each 128-key K/V tile as eight 16-key pages fetched
//    through the block table with a 4-D map over [blocks, 16, Hkv, D]
//    (a page past the sequence end, or a bad block id, is fetched at an
//    out-of-range coordinate, i.e. as zeros).  128-byte swizzle, no
//    multicast.  NS-deep K and V rings;
//  * warp 1 (one lane): tcgen05.mma issuer.  S = Q.K^T into one of two TMEM
//    buffers (M = 128, N = 128, K = 16 per instruction), O += P.V into a TMEM
//    accumulator (B = V read MN-major straight from the TMA layout);
//    completion reported through tcgen05.commit -> mbarrier;
//  * warps 2-5: softmax, one thread per query row (= TMEM lane).  tcgen05.ld
//    of the S row, scale folded with log2 e, mask only on tiles that cross
//    the diagonal or the sequence end, online softmax in fp32 with lazy
//    rescaling (O in TMEM is rescaled only when the running max grows by
//    more than 2^8), P rounded to bf16 into a swizzled SMEM tile that is the
//    A operand of the P.V MMA; final O / l -> bf16 -> global.
// Every mbarrier wait is bounded in time; a CTA that gives up raises
// PA_DEVERR_TIMEOUT, lets in-flight copies land, frees its TMEM and exits.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "layout.h"

namespace pa {

namespace {

constexpr int kThreads = 192;  // 6 warps
constexpr int BM = kPrefillTileM;
constexpr int BN = kPrefillTileN;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale when max grows by > 2^8

template <int D, int NS>
struct PrefillSmem {
  static constexpr int kQBytes = BM * D * 2;
  static constexpr int kKVBytes = BN * D * 2;  // one K or V tile
  static constexpr int kPBytes = BM * BN * 2;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kQBytes;
  static constexpr int kVOff = kKOff + NS * kKVBytes;
  static constexpr int kPOff = kVOff + NS * kKVBytes;
  static constexpr int kBarOff = kPOff + kPBytes;
  // barriers: q_full, q_empty, k_full[NS], k_empty[NS], v_full[NS], v_empty[NS],
  //           s_full[2], p_full, o_done
  static constexpr int kNumBars = 2 + 4 * NS + 2 + 2;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 64;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024 B
};

struct Work {
  int seq, head, row0, rows, q_start, q_len, kv_len, n;
};

__device__ __forceinline__ Work decode_work(int w, const int2* tiles, const SeqInfo* info,
                                            int num_q_heads, int causal) {
  Work k;
  const int2 t = tiles[w / num_q_heads];
  k.head = w % num_q_heads;
  k.seq = t.x;
  k.row0 = t.y;
  const SeqInfo si = info[t.x];
  k.q_start = si.q_start;
  k.q_len = si.q_len;
  k.kv_len = si.kv_len;
  k.rows = min(BM, si.q_len - t.y);
  int vis = si.kv_len;
  if (causal) vis = max(0, min(si.kv_len, si.kv_len - si.q_len + t.y + k.rows));
  k.n = (vis + BN - 1) / BN;
  return k;
}

}  // namespace

template <int D, int NS>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(PrefillParams p, const __grid_constant__ CUtensorMap q_map,
                   const __grid_constant__ CUtensorMap k_map,
                   const __grid_constant__ CUtensorMap v_map) {
  using SM = PrefillSmem<D, NS>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBarOff);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;
  uint64_t* k_empty = k_full + NS;
  uint64_t* v_full = k_empty + NS;
  uint64_t* v_empty = v_full + NS;
  uint64_t* s_full = v_empty + NS;  // [2]
  uint64_t* p_full = s_full + 2;
  uint64_t* o_done = p_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SM::kMiscOff + 4);

  const uint32_t q_s = smem_u32(smem + SM::kQOff);
  const uint32_t k_s = smem_u32(smem + SM::kKOff);
  const uint32_t v_s = smem_u32(smem + SM::kVOff);
  const uint32_t p_s = smem_u32(smem + SM::kPOff);

  unsigned char* ws = p.ws;
  uint32_t* err = reinterpret_cast<uint32_t*>(ws + p.L.err);
  const PlanHeader* hdr = reinterpret_cast<const PlanHeader*>(ws + p.L.header);
  const SeqInfo* info = reinterpret_cast<const SeqInfo*>(ws + p.L.seq_info);
  const int2* tiles = reinterpret_cast<const int2*>(ws + p.L.tiles);
  const int num_work = hdr->num_prefill_tiles * p.num_q_heads;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(k_full + i, 1);
      mbar_init(k_empty + i, 1);
      mbar_init(v_full + i, 1);
      mbar_init(v_empty + i, 1);
    }
    mbar_init(s_full + 0, 1);
    mbar_init(s_full + 1, 1);
    mbar_init(p_full, 4 * 32);
    mbar_init(o_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_s0 = tmem;          // S buffers: columns [0, 256)
  const uint32_t tmem_o = tmem + 2 * BN;  // O: columns [256, 256 + D)

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      prefetch_tma_desc(&q_map);
      prefetch_tma_desc(&k_map);
      prefetch_tma_desc(&v_map);
      int kv_it = 0, tcount = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < num_work && ok; w += gridDim.x) {
        const Work wk = decode_work(w, tiles, info, p.num_q_heads, p.causal);
        if (wk.n == 0) continue;
        const int kvh = wk.head / p.group;
        if (tcount > 0) ok = mbar_wait_bounded(q_empty, (tcount - 1) & 1, abort_flag, err);
        if (!ok) break;
        mbar_arrive_expect_tx(q_full, SM::kQBytes);
#pragma unroll
        for (int dh = 0; dh < D / 64; ++dh)
          tma_load_3d(q_s + dh * (BM * 128), &q_map, q_full, dh * 64, wk.head,
                      wk.q_start + wk.row0);
        const int32_t* table = p.block_tables + (size_t)wk.seq * p.max_blocks_per_seq;
        for (int j = 0; j < wk.n && ok; ++j, ++kv_it) {
          const int st = kv_it % NS, round = kv_it / NS;
          int blk[BN / kPageKeys];
#pragma unroll
          for (int pg = 0; pg < BN / kPageKeys; ++pg) {
            const int key0 = j * BN + pg * kPageKeys;
            int b = (int)p.num_blocks;  // out of range => zero fill
            if (key0 < wk.kv_len) {
              const int t = table[key0 / kPageKeys];
              if (t >= 0 && t < p.num_blocks)
                b = t;
              else
                raise_error(err, PA_DEVERR_BLOCK);
            }
            blk[pg] = b;
          }
          if (round > 0) ok = mbar_wait_bounded(k_empty + st, (round - 1) & 1, abort_flag, err);
          if (!ok) break;
          mbar_arrive_expect_tx(k_full + st, SM::kKVBytes);
#pragma unroll
          for (int pg = 0; pg < BN / kPageKeys; ++pg)
#pragma unroll
            for (int dh = 0; dh < D / 64; ++dh)
              tma_load_4d(k_s + st * SM::kKVBytes + dh * (BN * 128) + pg * (kPageKeys * 128),
                          &k_map, k_full + st, dh * 64, kvh, 0, blk[pg]);
          if (round > 0) ok = mbar_wait_bounded(v_empty + st, (round - 1) & 1, abort_flag, err);
          if (!ok) break;
          mbar_arrive_expect_tx(v_full + st, SM::kKVBytes);
#pragma unroll
          for (int pg = 0; pg < BN / kPageKeys; ++pg)
#pragma unroll
            for (int dh = 0; dh < D / 64; ++dh)
              tma_load_4d(v_s + st * SM::kKVBytes + dh * (BN * 128) + pg * (kPageKeys * 128),
                          &v_map, v_full + st, dh * 64, kvh, 0, blk[pg]);
        }
        ++tcount;
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer --------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc_s = instr_desc_bf16(BM, BN, 0);
      constexpr uint32_t idesc_o = instr_desc_bf16(BM, D, 1);
      int kv_it = 0, s_it = 0, tcount = 0;
      bool ok = true;
      auto issue_s = [&](int sidx, int stage) {
        const uint32_t d_tmem = tmem_s0 + (sidx & 1) * BN;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
          const uint64_t a = smem_desc_sw128(q_s + off, 16, 1024);
          const uint64_t b = smem_desc_sw128(k_s + stage * SM::kKVBytes + off, 16, 1024);
          tc_mma(d_tmem, a, b, idesc_s, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_o = [&](int stage, bool accumulate) {
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t a =
              smem_desc_sw128(p_s + (kk >> 2) * (BM * 128) + (kk & 3) * 32, 16, 1024);
          const uint64_t b = smem_desc_sw128(v_s + stage * SM::kKVBytes + kk * (16 * 128),
                                             BN * 128, 1024);
          tc_mma(tmem_o, a, b, idesc_o, (accumulate || kk > 0) ? 1u : 0u);
        }
      };
      for (int w = blockIdx.x; w < num_work && ok; w += gridDim.x) {
        const Work wk = decode_work(w, tiles, info, p.num_q_heads, p.causal);
        if (wk.n == 0) continue;
        ok = mbar_wait_bounded(q_full, tcount & 1, abort_flag, err);
        if (!ok) break;
        tc_fence_after();
        {
          const int st = kv_it % NS;
          ok = mbar_wait_bounded(k_full + st, (kv_it / NS) & 1, abort_flag, err);
          if (!ok) break;
          tc_fence_after();
          issue_s(s_it, st);
          tc_commit(s_full + (s_it & 1));
          tc_commit(k_empty + st);
          if (wk.n == 1) tc_commit(q_empty);
        }
        for (int j = 0; j < wk.n && ok; ++j) {
          const int cur = s_it + j;
          if (j + 1 < wk.n) {
            const int kvn = kv_it + j + 1, st = kvn % NS;
            ok = mbar_wait_bounded(k_full + st, (kvn / NS) & 1, abort_flag, err);
            if (!ok) break;
            tc_fence_after();
            issue_s(cur + 1, st);
            tc_commit(s_full + ((cur + 1) & 1));
            tc_commit(k_empty + st);
            if (j + 2 == wk.n) tc_commit(q_empty);  // last S of the tile issued
          }
          ok = mbar_wait_bounded(p_full, cur & 1, abort_flag, err);
          if (!ok) break;
          const int kvc = kv_it + j, st = kvc % NS;
          ok = mbar_wait_bounded(v_full + st, (kvc / NS) & 1, abort_flag, err);
          if (!ok) break;
          tc_fence_after();
          issue_o(st, j > 0);
          tc_commit(o_done);
          tc_commit(v_empty + st);
        }
        kv_it += wk.n;
        s_it += wk.n;
        ++tcount;
      }
    }
  } else {
    // ------------------------------ softmax warps -----------------------------
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    int s_it = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < num_work && ok; w += gridDim.x) {
      const Work wk = decode_work(w, tiles, info, p.num_q_heads, p.causal);
      const bool row_ok = r < wk.rows;
      __nv_bfloat16* orow =
          p.out + ((size_t)(wk.q_start + wk.row0 + r) * p.num_q_heads + wk.head) * D;
      if (wk.n == 0) {
        if (row_ok) {
#pragma unroll
          for (int c = 0; c < D / 8; ++c)
            reinterpret_cast<uint4*>(orow)[c] = make_uint4(0, 0, 0, 0);
        }
        continue;
      }
      // last key this row may see (inclusive); below 0 means none
      int limit = wk.kv_len - 1;
      if (p.causal) limit = min(limit, wk.kv_len - wk.q_len + wk.row0 + r);
      float m_use = -INFINITY, l = 0.f;
      for (int j = 0; j < wk.n; ++j) {
        const int cur = s_it + j;
        ok = mbar_wait_bounded(s_full + (cur & 1), (cur >> 1) & 1, abort_flag, err);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        uint32_t sv[BN];
        {
          const uint32_t base = tmem_s0 + (cur & 1) * BN + lane_base;
          tmem_ld32(base + 0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
          tmem_ld32(base + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
          tmem_ld32(base + 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[64]));
          tmem_ld32(base + 96, *reinterpret_cast<uint32_t(*)[32]>(&sv[96]));
          tmem_ld_wait();
        }
        float s[BN];
        const int key0 = j * BN;
        float m_tile = -INFINITY;
        if (key0 + BN - 1 > limit) {
#pragma unroll
          for (int c = 0; c < BN; ++c) {
            const float v = __uint_as_float(sv[c]) * p.scale_log2;
            s[c] = (key0 + c <= limit) ? v : -INFINITY;
            m_tile = fmaxf(m_tile, s[c]);
          }
        } else {
#pragma unroll
          for (int c = 0; c < BN; ++c) {
            s[c] = __uint_as_float(sv[c]) * p.scale_log2;
            m_tile = fmaxf(m_tile, s[c]);
          }
        }
        const float m_old = m_use;
        const bool grow = m_tile > m_old + kRescaleThreshold || (m_old == -INFINITY && m_tile > -INFINITY);
        if (grow) m_use = m_tile;
        const float base = (m_use == -INFINITY) ? 0.f : m_use;
        const bool rescale_o = grow && m_old != -INFINITY && j > 0;
        const float alpha = (grow && m_old != -INFINITY) ? fast_exp2(m_old - m_use) : 1.f;
        float rowsum = 0.f;
        uint32_t pk[BN / 2];
#pragma unroll
        for (int c = 0; c < BN; c += 2) {
          const float p0 = fast_exp2(s[c] - base);
          const float p1 = fast_exp2(s[c + 1] - base);
          rowsum += p0 + p1;
          pk[c / 2] = pack_bf16x2(p0, p1);
        }
        l = l * alpha + rowsum;

        // P buffer free and O stable once the previous P.V has completed
        if (cur > 0) {
          ok = mbar_wait_bounded(o_done, (cur - 1) & 1, abort_flag, err);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
        }
        if (__any_sync(0xffffffffu, rescale_o)) {
          const float f = rescale_o ? alpha : 1.f;
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t ov[32];
            tmem_ld32(tmem_o + lane_base + c0, ov);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * f);
            tmem_st32(tmem_o + lane_base + c0, ov);
          }
          tmem_st_wait();
        }
        // P row -> swizzled K-major SMEM tile (A operand of O += P.V)
        {
          const uint32_t row_base = p_s + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
          for (int kc = 0; kc < BN / 8; ++kc) {
            const uint32_t addr =
                row_base + (kc >> 3) * (BM * 128) + (((kc & 7) ^ (r & 7)) << 4);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                         "r"(pk[kc * 4 + 0]), "r"(pk[kc * 4 + 1]), "r"(pk[kc * 4 + 2]),
                         "r"(pk[kc * 4 + 3])
                         : "memory");
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(p_full);
      }
      if (!ok) break;
      // epilogue: O / l -> bf16 -> global
      const int last = s_it + wk.n - 1;
      ok = mbar_wait_bounded(o_done, last & 1, abort_flag, err);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t ov[32];
        tmem_ld32(tmem_o + lane_base + c0, ov);
        tmem_ld_wait();
        if (row_ok) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(ov[i + 0]) * inv, __uint_as_float(ov[i + 1]) * inv);
            v.y = pack_bf16x2(__uint_as_float(ov[i + 2]) * inv, __uint_as_float(ov[i + 3]) * inv);
            v.z = pack_bf16x2(__uint_as_float(ov[i + 4]) * inv, __uint_as_float(ov[i + 5]) * inv);
            v.w = pack_bf16x2(__uint_as_float(ov[i + 6]) * inv, __uint_as_float(ov[i + 7]) * inv);
            *reinterpret_cast<uint4*>(orow + c0 + i) = v;
          }
        }
      }
      tc_fence_before();
      s_it += wk.n;
    }
  }

  __syncthreads();
  if (*abort_flag) {
    // give in-flight TMA copies and MMAs time to land before TMEM is freed
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 20000000ull) __nanosleep(1000);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, int NS>
static cudaError_t launch_prefill_t(const PrefillParams& p, const CUtensorMap& q_map,
                                    const CUtensorMap& k_map, const CUtensorMap& v_map, int grid,
                                    cudaStream_t stream) {
  using SM = PrefillSmem<D, NS>;
  cudaError_t e = cudaFuncSetAttribute(prefill_kernel<D, NS>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kAlloc);
  if (e != cudaSuccess) return e;
  prefill_kernel<D, NS><<<grid, kThreads, SM::kAlloc, stream>>>(p, q_map, k_map, v_map);
  return cudaGetLastError();
}

cudaError_t launch_prefill(const PrefillParams& p, const CUtensorMap& q_map,
                           const CUtensorMap& k_map, const CUtensorMap& v_map, int head_dim,
                           int grid, cudaStream_t stream) {
  if (head_dim == 128) return launch_prefill_t<128, 2>(p, q_map, k_map, v_map, grid, stream);
  return launch_prefill_t<64, 4>(p, q_map, k_map, v_map, grid, stream);
}

}  // namespace pa
