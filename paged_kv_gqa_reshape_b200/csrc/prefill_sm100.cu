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
//  * persistent grid, one CTA per SM, walking the plan's work list; a work
//    item is 256 query rows of one head, split into two 128-row tiles A and B
//    that share every K/V tile;
//  * warp 0 (one lane): TMA producer.  Q tiles via a 3-D map over
//    [tokens, Hq, D]; each 128-key K/V tile as eight 16-key pages fetched
//    through the block table with a 4-D map over [blocks, block_size, Hkv,
//    D] (a block of 16k slots holds k pages)
//    (a page past the sequence end, or a bad block id, is fetched at an
//    out-of-range coordinate, i.e. as zeros).  128-byte swizzle, no
//    multicast.  K and V tiles go through one ring (4 slots for D = 128,
//    10 for D = 64) in the order K0 V0 K1 V1 ...;
//  * warp 1 (one lane): tcgen05.mma issuer.  Per KV tile j it issues
//    PV_A(j), S_A(j+1), PV_B(j), S_B(j+1): S = Q.K^T into the tile's TMEM
//    S buffer (M = 128, N = 128, K = 16 per instruction) and O += P.V into
//    the tile's TMEM accumulator, with A = P read from TMEM and B = V read
//    MN-major straight from the TMA layout.  S_x(j+1) overwrites the columns
//    that hold P_x(j), so it is issued once P_x(j).V has completed.  While one
//    tile's softmax runs, the tensor core works on the other tile;
//    completion is reported through tcgen05.commit -> mbarrier;
//  * warps 2-5 / 6-9: softmax of tile A / B, one thread per query row
//    (= TMEM lane).  The 128 scores of the row come into registers once,
//    the mask is applied only on tiles that cross the diagonal or the
//    sequence end, online softmax in fp32 (3-input max, scale folded into a
//    packed-pair FFMA, packed row sums) with lazy rescaling (O in TMEM is
//    rescaled only when the running max grows by more than 2^8), P rounded
//    to bf16 and written back over the first 64 columns of S (two keys per
//    column), the A operand of the P.V MMA; final O / l -> bf16 -> global.
// TMEM: S_A, S_B, O_A, O_B (4 x 128 columns for D = 128); P_x inside S_x.
// SMEM: Q_A, Q_B and the K/V ring (224 KB for D = 128).
// Every mbarrier wait is bounded in time; a CTA that gives up raises
// PA_DEVERR_TIMEOUT, lets in-flight copies land, frees its TMEM and exits.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "layout.h"
#include "spans.cuh"

namespace pa {

namespace {

constexpr int kWarps = 10;  // 0 producer, 1 MMA, 2-5 softmax A, 6-9 softmax B
constexpr int kThreads = kWarps * 32;
constexpr int BM = kPrefillTileM;
constexpr int BN = kPrefillTileN;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale when max grows by > 2^8

template <int D>
struct PrefillSmem {
  static constexpr int kQBytes = BM * D * 2;   // one 128-row Q tile
  static constexpr int kKVBytes = BN * D * 2;  // one K or V tile
  static constexpr int kRing = D == 128 ? 4 : 10;  // K/V slots (measured: 4 as fast as 5)
  static constexpr int kQOff = 0;              // Q_A, Q_B
  static constexpr int kRingOff = kQOff + 2 * kQBytes;
  static constexpr int kBarOff = kRingOff + kRing * kKVBytes;
  // barriers: q_full, q_empty, slot_full[kRing], slot_empty[kRing], s_full[2],
  //           p_full[2], o_done[2], item_full[kItemRing], item_empty[kItemRing]
  static constexpr int kItemRing = 4;  // work-item indices in flight to the consumers
  static constexpr int kNumBars = 2 + 2 * kRing + 6 + 2 * kItemRing;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 64;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024 B
};

struct Work {
  int seq, head, row0, q_start, q_len, kv_len;
  int rows[2];  // query rows of tile A / B in this item (B may have none)
  int n[2];     // KV tiles tile A / B must visit
  int nmax;
};

// work item w: sequence, rows, and the KV tiles of its two 128-row tiles (as
// the plan kernel counted them: causal, full-attention spans or all keys)
__device__ __forceinline__ Work decode_work(int w, const int2* tiles, const int2* tile_n,
                                            const SeqInfo* info, int num_q_heads) {
  Work k;
  const int2 t = tiles[w / num_q_heads];
  const int2 tn = tile_n[w / num_q_heads];
  k.head = w % num_q_heads;
  k.seq = t.x;
  k.row0 = t.y;
  const SeqInfo si = info[t.x];
  k.q_start = si.q_start;
  k.q_len = si.q_len;
  k.kv_len = si.kv_len;
  k.rows[0] = min(BM, si.q_len - t.y);
  k.rows[1] = max(0, min(BM, si.q_len - t.y - BM));
  k.n[0] = tn.x;
  k.n[1] = tn.y;
  k.nmax = max(k.n[0], k.n[1]);
  return k;
}

}  // namespace

// Element offset of out row (token t, head h): dense [T, Hq, D] unless STRIDED.
template <int D, bool STRIDED>
__device__ __forceinline__ size_t out_offset(const PrefillParams& p, int t, int h) {
  if constexpr (STRIDED) return (size_t)t * p.o_tok + (size_t)h * p.o_head;
  return ((size_t)t * p.num_q_heads + h) * D;
}

// PG: cache blocks of more than 16 slots (block_size = 16 << p.ppb_shift), so
// a 16-key page sits at a slot offset inside its block; 16-slot blocks take the
// plain path, in which a page is a whole block.
template <int D, bool H, bool MODS, bool STRIDED, bool PG>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(PrefillParams p, const __grid_constant__ CUtensorMap q_map,
                   const __grid_constant__ CUtensorMap k_map,
                   const __grid_constant__ CUtensorMap v_map) {
  using SM = PrefillSmem<D>;
  constexpr int kRing = SM::kRing;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBarOff);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* slot_full = bars + 2;
  uint64_t* slot_empty = slot_full + kRing;
  uint64_t* s_full = slot_empty + kRing;  // [2]: tile A, tile B
  uint64_t* p_full = s_full + 2;          // [2]
  uint64_t* o_done = p_full + 2;          // [2]
  uint64_t* item_full = o_done + 2;       // [kItemRing]: index published
  uint64_t* item_empty = item_full + SM::kItemRing;  // [kItemRing]: read by every consumer
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SM::kMiscOff + 4);
  volatile int* s_item = reinterpret_cast<volatile int*>(smem + SM::kMiscOff + 8);  // [kItemRing]

  const uint32_t q_s = smem_u32(smem + SM::kQOff);
  const uint32_t ring_s = smem_u32(smem + SM::kRingOff);

  unsigned char* ws = p.ws;
  uint32_t* err = reinterpret_cast<uint32_t*>(ws + p.L.err);
  const PlanHeader* hdr = reinterpret_cast<const PlanHeader*>(ws + p.L.header);
  const SeqInfo* info = reinterpret_cast<const SeqInfo*>(ws + p.L.seq_info);
  const int2* tiles = reinterpret_cast<const int2*>(ws + p.L.tiles);
  const int2* tile_n = reinterpret_cast<const int2*>(ws + p.L.tile_n);
  const int num_work = hdr->num_prefill_tiles * p.num_q_heads;
  const uint64_t wlim = p.wait_limit_ns ? p.wait_limit_ns : kWaitLimitNs;
  // Beside the decode kernel only the plan's share of the CTAs (one per SM)
  // takes work: the others are handed no item and leave, freeing their SMs.
  const int ctas = p.split ? min((int)gridDim.x, max(1, hdr->prefill_sms)) : (int)gridDim.x;
  // Work distribution: the first item of a CTA is blockIdx.x; later ones are
  // taken from a counter (sorted by descending cost, so the longest go first),
  // so SMs that run faster take more items.  The producer publishes each item
  // index in a small ring; the MMA thread and the softmax warps read it (-1:
  // no more work).
  int* next_item = const_cast<int*>(&hdr->prefill_next);
  auto read_item = [&](int k, bool& ok) -> int {
    const int slot = k % SM::kItemRing;
    ok = ok && mbar_wait_bounded(item_full + slot, (uint32_t)((k / SM::kItemRing) & 1), abort_flag,
                                 err, wlim);
    return ok ? s_item[slot] : -1;
  };

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < kRing; ++i) {
      mbar_init(slot_full + i, 1);
      mbar_init(slot_empty + i, 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(s_full + x, 1);
      mbar_init(p_full + x, 4 * 32);
      mbar_init(o_done + x, 1);
    }
    for (int i = 0; i < SM::kItemRing; ++i) {
      mbar_init(item_full + i, 1);
      mbar_init(item_empty + i, 1 + 8);  // the MMA thread and the 8 softmax warps
    }
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
  // S_A, S_B: columns [0, 128), [128, 256); O_A, O_B: [256, 256 + D), [256 + D, 256 + 2D).
  // P_x (bf16, two keys per 32-bit column) overwrites the first 64 columns of
  // S_x once the softmax holds those scores in registers.
  auto tmem_s = [&](int x) { return tmem + (uint32_t)(x * BN); };
  auto tmem_o = [&](int x) { return tmem + (uint32_t)(2 * BN + x * D); };

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      prefetch_tma_desc(&q_map);
      prefetch_tma_desc(&k_map);
      prefetch_tma_desc(&v_map);
      long long ld = 0;  // K/V tiles loaded so far (slot = ld % kRing)
      int tcount = 0;
      bool ok = true;
      // head-major q / cache swap two tensor-map coordinates (strided
      // instantiation only; the dense one keeps token-major order)
      const bool q_hnd = STRIDED && p.q_hnd != 0, kv_hnd = STRIDED && p.kv_hnd != 0;
      for (int k = 0; ok; ++k) {
        int w = k == 0 ? ((int)blockIdx.x < ctas ? (int)blockIdx.x : num_work)
                       : ctas + atomicAdd(next_item, 1);
        if (w >= num_work) w = -1;
        const int slot = k % SM::kItemRing;
        if (k >= SM::kItemRing)
          ok = mbar_wait_bounded(item_empty + slot, (uint32_t)((k / SM::kItemRing - 1) & 1),
                                 abort_flag, err, wlim);
        if (!ok) break;
        s_item[slot] = w;
        mbar_arrive(item_full + slot);
        if (w < 0) break;
        const Work wk = decode_work(w, tiles, tile_n, info, p.num_q_heads);
        if (wk.nmax == 0) continue;
        const int kvh = wk.head / p.group;
        const int kv_c1 = kv_hnd ? 0 : kvh, kv_c2 = kv_hnd ? kvh : 0;  // (head, slot) or (slot, head)
        if (tcount > 0) ok = mbar_wait_bounded(q_empty, (tcount - 1) & 1, abort_flag, err, wlim);
        if (!ok) break;
        mbar_arrive_expect_tx(q_full, 2 * SM::kQBytes);
#pragma unroll
        for (int x = 0; x < 2; ++x)
#pragma unroll
          for (int dh = 0; dh < D / 64; ++dh)
            tma_load_3d(q_s + x * SM::kQBytes + dh * (BM * 128), &q_map, q_full, dh * 64,
                        q_hnd ? wk.q_start + wk.row0 + x * BM : wk.head,
                        q_hnd ? wk.head : wk.q_start + wk.row0 + x * BM);
        const int32_t* table = p.block_tables + (size_t)wk.seq * p.max_blocks_per_seq;
        for (int j = 0; j < wk.nmax && ok; ++j) {
          // page pg (16 keys) of the tile: block blk, and with PG slots
          // [slot, slot + 16) of it
          int blk[BN / kPageKeys];
          [[maybe_unused]] int slot[BN / kPageKeys];
#pragma unroll
          for (int pg = 0; pg < BN / kPageKeys; ++pg) {
            const int key0 = j * BN + pg * kPageKeys;
            int b = (int)p.num_blocks;  // out of range => zero fill
            if (key0 < wk.kv_len) {
              const int t = PG ? table[key0 >> (p.ppb_shift + 4)] : table[key0 / kPageKeys];
              if (t >= 0 && t < p.num_blocks)
                b = t;
              else
                raise_error(err, PA_DEVERR_BLOCK);
            }
            blk[pg] = b;
            if constexpr (PG) slot[pg] = key0 & (p.block_size - 1);
          }
#pragma unroll
          for (int kv = 0; kv < 2; ++kv, ++ld) {  // K_j, then V_j
            const int st = (int)(ld % kRing);
            const long long round = ld / kRing;
            if (round > 0) ok = mbar_wait_bounded(slot_empty + st, (round - 1) & 1, abort_flag, err, wlim);
            if (!ok) break;
            mbar_arrive_expect_tx(slot_full + st, SM::kKVBytes);
            const void* map = kv == 0 ? (const void*)&k_map : (const void*)&v_map;
#pragma unroll
            for (int pg = 0; pg < BN / kPageKeys; ++pg)
#pragma unroll
              for (int dh = 0; dh < D / 64; ++dh) {  // coordinates (d, head, slot) or (d, slot, head)
                const uint32_t dst = ring_s + st * SM::kKVBytes + dh * (BN * 128) + pg * (kPageKeys * 128);
                if constexpr (PG)
                  tma_load_4d(dst, map, slot_full + st, dh * 64, kv_hnd ? slot[pg] : kvh,
                              kv_hnd ? kvh : slot[pg], blk[pg]);
                else
                  tma_load_4d(dst, map, slot_full + st, dh * 64, kv_c1, kv_c2, blk[pg]);
              }
          }
        }
        ++tcount;
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer --------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc_s = instr_desc_f16kind(BM, BN, 0, H);
      constexpr uint32_t idesc_o = instr_desc_f16kind(BM, D, 1, H);
      long long ld = 0;   // K/V tiles consumed (mirrors the producer)
      int tcount = 0;
      int s_it[2] = {0, 0}, pv_it[2] = {0, 0};
      bool ok = true;
      auto wait_tile = [&](long long idx) {
        return mbar_wait_bounded(slot_full + (int)(idx % kRing), (uint32_t)((idx / kRing) & 1),
                                 abort_flag, err, wlim);
      };
      auto issue_s = [&](int x, long long kidx) {
        const uint32_t kb = ring_s + (int)(kidx % kRing) * SM::kKVBytes;
        const uint32_t qb = q_s + x * SM::kQBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
          tc_mma(tmem_s(x), smem_desc_sw128(qb + off, 16, 1024), smem_desc_sw128(kb + off, 16, 1024),
                 idesc_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(s_full + x);
        ++s_it[x];
      };
      auto issue_pv = [&](int x, long long vidx, bool accumulate) {
        const uint32_t vb = ring_s + (int)(vidx % kRing) * SM::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          // A = P from TMEM: keys 16kk..16kk+15 are columns 8kk..8kk+7 of P_x
          const uint64_t b = smem_desc_sw128(vb + kk * (16 * 128), BN * 128, 1024);
          tc_mma_ts(tmem_o(x), tmem_s(x) + 8 * kk, b, idesc_o, (accumulate || kk > 0) ? 1u : 0u);
        }
        tc_commit(o_done + x);
        ++pv_it[x];
      };
      for (int k = 0; ok; ++k) {
        const int w = read_item(k, ok);
        mbar_arrive(item_empty + k % SM::kItemRing);
        if (w < 0) break;
        const Work wk = decode_work(w, tiles, tile_n, info, p.num_q_heads);
        if (wk.nmax == 0) continue;
        ok = mbar_wait_bounded(q_full, tcount & 1, abort_flag, err, wlim);
        if (!ok) break;
        tc_fence_after();
        const long long base = ld;  // K_j = base + 2j, V_j = base + 2j + 1
        ok = wait_tile(base);
        if (!ok) break;
        tc_fence_after();
        // S_x(0) overwrites the columns the previous item's last P_x occupied:
        // let that P_x.V finish first (MMAs on different accumulators are
        // not ordered by their issue)
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          if (wk.n[x] == 0) continue;
          if (pv_it[x] > 0) {
            ok = mbar_wait_bounded(o_done + x, (pv_it[x] - 1) & 1, abort_flag, err, wlim);
            if (!ok) break;
            tc_fence_after();
          }
          issue_s(x, base);
        }
        if (!ok) break;
        tc_commit(slot_empty + (int)(base % kRing));  // K_0 read by both S MMAs
        if (wk.nmax == 1) tc_commit(q_empty);
        for (int j = 0; j < wk.nmax && ok; ++j) {
          const long long kn = base + 2 * (j + 1), vj = base + 2 * j + 1;
          if constexpr (MODS) {
            // the modifiers' longer softmax leaves V_j and K_{j+1} landed long
            // before P_x(j) is ready: check both first, off the P -> P.V -> S
            // chain (in the plain kernel this order measured slower)
            ok = wait_tile(vj);
            if (ok && j + 1 < wk.nmax) ok = wait_tile(kn);
            if (!ok) break;
          }
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            if (j >= wk.n[x]) continue;
            ok = mbar_wait_bounded(p_full + x, pv_it[x] & 1, abort_flag, err, wlim);
            if (!MODS && ok) ok = wait_tile(vj);
            if (!ok) break;
            tc_fence_after();
            issue_pv(x, vj, j > 0);
            if (j + 1 < wk.n[x]) {
              // S_x(j+1) overwrites the columns P_x(j) occupies: let P_x(j).V finish
              ok = mbar_wait_bounded(o_done + x, (pv_it[x] - 1) & 1, abort_flag, err, wlim);
              if (!MODS && ok) ok = wait_tile(kn);
              if (!ok) break;
              tc_fence_after();
              issue_s(x, kn);
            }
          }
          if (!ok) break;
          tc_commit(slot_empty + (int)(vj % kRing));            // V_j done
          if (j + 1 < wk.nmax) tc_commit(slot_empty + (int)(kn % kRing));  // K_{j+1} done
          if (j + 2 == wk.nmax) tc_commit(q_empty);             // last S MMAs issued
        }
        ld = base + 2 * wk.nmax;
        ++tcount;
      }
    }
  } else {
    // ------------------------- softmax warps (tile x) --------------------------
    const int x = (warp - 2) >> 2;  // 0: tile A (warps 2-5), 1: tile B (warps 6-9)
    const int quarter = warp & 3;   // TMEM lanes this warp may access
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t s_col = tmem_s(x) + lane_base;
    const uint32_t o_col = tmem_o(x) + lane_base;
    int it = 0;  // S tiles of this query tile consumed so far (phase counter)
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int w = read_item(k, ok);
      ok = __all_sync(0xffffffffu, ok);
      __syncwarp();
      if (lane == 0) mbar_arrive(item_empty + k % SM::kItemRing);
      if (!ok || w < 0) break;
      const Work wk = decode_work(w, tiles, tile_n, info, p.num_q_heads);
      const int rows = wk.rows[x], n = wk.n[x];
      const int qrow = wk.row0 + x * BM + r;  // query index within the sequence
      const bool row_ok = r < rows;
      if (n == 0) {
        if (row_ok) {
          uint16_t* orow = p.out + out_offset<D, STRIDED>(p, wk.q_start + qrow, wk.head);
#pragma unroll
          for (int c = 0; c < D / 8; ++c) reinterpret_cast<uint4*>(orow)[c] = make_uint4(0, 0, 0, 0);
        }
        continue;
      }
      // last key this row may see (inclusive); below 0 means none
      int limit = wk.kv_len - 1;
      const int pos = wk.kv_len - wk.q_len + qrow;  // the row's key position
      if (p.span_offsets) {
        const SpanList sl = span_list(p.span_offsets, p.spans, p.num_spans, wk.seq, wk.kv_len);
        limit = span_visible(sl, pos, pos, nullptr) - 1;
      } else if (p.causal) {
        limit = min(limit, pos);
      }
      // score modifiers of this row (head wk.head, query token q_start + qrow)
      float slope = 0.f;
      const float* mrow = nullptr;
      if constexpr (MODS) {
        if (p.mods.alibi) slope = __ldg(p.mods.alibi + wk.head);
        if (p.mods.mask && row_ok)
          mrow = p.mods.mask + (size_t)wk.head * p.mods.mask_head +
                 (size_t)(wk.q_start + qrow) * p.mods.mask_tok;
      }
      float m_use = -INFINITY, l = 0.f;
      for (int j = 0; j < n; ++j) {
        const int cur = it + j;
        // S_x(j) has landed.  P_x(j-1).V was issued before S_x(j) by the same
        // thread, so waiting for it here (P buffer free, O stable) costs nothing
        // and lets P be stored as it is computed.
        ok = mbar_wait_bounded(s_full + x, cur & 1, abort_flag, err, wlim);
        if (ok && cur > 0) ok = mbar_wait_bounded(o_done + x, (cur - 1) & 1, abort_flag, err, wlim);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        // The row's 128 raw scores come into registers with four TMEM loads and
        // one wait; the max and the exponentials both work from those registers.
        // The scale is applied after the max (scale_log2 >= 0, so the max
        // commutes with it) and in the exponent's FFMA.  Reductions use
        // independent partials (short trees, not 128-long dependency chains).
        const int key0 = j * BN;
        const bool masked_tile = key0 + BN - 1 > limit;
        const int valid = limit - key0 + 1;  // keys [0, valid) of this tile are visible
        uint32_t sv[BN];
#pragma unroll
        for (int c = 0; c < BN; c += 32)
          tmem_ld32(s_col + c, *reinterpret_cast<uint32_t(*)[32]>(&sv[c]));
        tmem_ld_wait();
        if constexpr (MODS) {
          // The modifiers act in raw-score units, so the plain path's scaling
          // (after the max, in the exponent) still applies: raw <- (cap /
          // scale) tanh(raw scale / cap), then + (slope (j - pos) + mask) /
          // scale.  One uniform branch per modifier; keys past `valid` get
          // -inf below, so their mask values are not read.
          if (p.mods.softcap > 0.f) {
            const float a1 = p.scale / p.mods.softcap, capr = p.mods.softcap / p.scale;
            // When |x| = |raw| a1 < 1/4 for all of the warp's scores, (c / scale)
            // tanh(x) = raw (1 - x^2/3 + 2x^4/15 - 17x^6/315) (Taylor series;
            // the first term left out, 62x^9/2835, is 3e-7 relative at 1/4),
            // on packed pairs with no SFU operation.  Otherwise tanh on the SFU.
            float mabs = 0.f;
#pragma unroll
            for (int c = 0; c < BN; c += 2)
              mabs = fmax3(mabs, fabsf(__uint_as_float(sv[c])), fabsf(__uint_as_float(sv[c + 1])));
            if (__all_sync(0xffffffffu, mabs * a1 < 0.25f)) {
              const float y1 = a1 * a1;
              const uint64_t k1 = f2_pack(-y1 / 3.f, -y1 / 3.f),
                             k2 = f2_pack(2.f * y1 * y1 / 15.f, 2.f * y1 * y1 / 15.f),
                             k3 = f2_pack(-17.f * y1 * y1 * y1 / 315.f, -17.f * y1 * y1 * y1 / 315.f),
                             one = f2_pack(1.f, 1.f);
#pragma unroll
              for (int c = 0; c < BN; c += 2) {
                const uint64_t r = f2_pack(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1]));
                const uint64_t y = f2_mul(r, r);
                const uint64_t t = f2_mul(r, f2_fma(f2_fma(f2_fma(k3, y, k2), y, k1), y, one));
                sv[c] = __float_as_uint(f2_lo(t));
                sv[c + 1] = __float_as_uint(f2_hi(t));
              }
            } else {
#pragma unroll
              for (int c = 0; c < BN; ++c)
                sv[c] = __float_as_uint(capr * tanh_sfu(__uint_as_float(sv[c]) * a1));
            }
          }
          if (slope != 0.f) {
            // + slope' (key0 - pos + c), slope' = slope / scale, on fp32 pairs
            // The bias of pair c is carried in one of four running pairs
            // (advanced by 8 keys per use) rather than rebuilt from c.
            const float sr = slope / p.scale;
            const float b0 = sr * (float)(key0 - pos);
            const uint64_t step8 = f2_pack(8.f * sr, 8.f * sr);
            uint64_t bias[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
              bias[i] = f2_pack(fmaf(sr, (float)(2 * i), b0), fmaf(sr, (float)(2 * i + 1), b0));
#pragma unroll
            for (int c = 0; c < BN; c += 2) {
              uint64_t& b = bias[(c / 2) % 4];
              const uint64_t v = f2_add(f2_pack(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), b);
              b = f2_add(b, step8);
              sv[c] = __float_as_uint(f2_lo(v));
              sv[c + 1] = __float_as_uint(f2_hi(v));
            }
          }
          if (mrow) {
            const int vis = masked_tile ? max(0, min(valid, BN)) : BN;
            const long long left = p.mods.mask_len - key0;
            const int mlim = (int)max(0ll, min((long long)vis, left));  // keys with a mask value
            if (mlim < vis) raise_error(err, PA_DEVERR_HINT);
            const float is = 1.f / p.scale;
            const uint64_t is2 = f2_pack(is, is);
#pragma unroll
            for (int c = 0; c < BN; c += 4) {
              float4 mv = make_float4(0.f, 0.f, 0.f, 0.f);
              if (c + 4 <= mlim) {
                mv = __ldg(reinterpret_cast<const float4*>(mrow + key0 + c));
              } else if (c < mlim) {
                mv.x = __ldg(mrow + key0 + c);
                if (c + 1 < mlim) mv.y = __ldg(mrow + key0 + c + 1);
                if (c + 2 < mlim) mv.z = __ldg(mrow + key0 + c + 2);
              }
              const uint64_t v0 = f2_fma(f2_pack(mv.x, mv.y), is2,
                                         f2_pack(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])));
              const uint64_t v1 = f2_fma(f2_pack(mv.z, mv.w), is2,
                                         f2_pack(__uint_as_float(sv[c + 2]), __uint_as_float(sv[c + 3])));
              sv[c] = __float_as_uint(f2_lo(v0));
              sv[c + 1] = __float_as_uint(f2_hi(v0));
              sv[c + 2] = __float_as_uint(f2_lo(v1));
              sv[c + 3] = __float_as_uint(f2_hi(v1));
            }
          }
        }
        // Tiles crossing the diagonal or the sequence end set hidden keys to
        // -inf once; the others skip every per-key test.  A masked tile is
        // scaled here, before the -inf goes in, and then runs with unit scale
        // below: with scale 0 the product -inf * 0 would be NaN, whereas
        // scaling first gives 0 for every visible key (a uniform softmax)
        // and keeps the hidden ones at -inf.
        float tile_scale = p.scale_log2;
        if (masked_tile) {
          tile_scale = 1.f;
#pragma unroll
          for (int c = 0; c < BN; ++c)
            sv[c] = __float_as_uint(c >= valid ? -INFINITY : __uint_as_float(sv[c]) * p.scale_log2);
        }
        constexpr int NP = 4;
        float mp[NP];
#pragma unroll
        for (int i = 0; i < NP; ++i) mp[i] = -INFINITY;
#pragma unroll
        for (int c = 0; c < BN; c += 2)
          mp[(c / 2) % NP] = fmax3(mp[(c / 2) % NP], __uint_as_float(sv[c]), __uint_as_float(sv[c + 1]));
#pragma unroll
        for (int wdt = NP / 2; wdt >= 1; wdt >>= 1)
#pragma unroll
          for (int i = 0; i < wdt; ++i) mp[i] = fmaxf(mp[i], mp[i + wdt]);
        // tile_scale >= 0, so the max commutes with it; on an unmasked tile
        // every score is finite, so scale 0 gives 0 here, not NaN
        const float m_tile = mp[0] * tile_scale;
        const float m_old = m_use;
        const bool grow =
            m_tile > m_old + kRescaleThreshold || (m_old == -INFINITY && m_tile > -INFINITY);
        if (grow) m_use = m_tile;
        const float base = (m_use == -INFINITY) ? 0.f : m_use;
        const bool rescale_o = grow && m_old != -INFINITY && j > 0;
        const float alpha = (grow && m_old != -INFINITY) ? fast_exp2(m_old - m_use) : 1.f;
        // p = 2^(scale_log2 * s - base), rounded to bf16 and written to TMEM as
        // the A operand of O += P.V.  Scaling and row sums run on packed fp32
        // pairs; the exponentials on the SFU.
        const uint64_t scale2 = f2_pack(tile_scale, tile_scale);
        const uint64_t nbase2 = f2_pack(-base, -base);
        uint64_t rs2[NP / 2];
#pragma unroll
        for (int i = 0; i < NP / 2; ++i) rs2[i] = 0;
#pragma unroll
        for (int h = 0; h < BN; h += 32) {
          // 32 scores -> 16 packed bf16 pairs over S columns [h/2, h/2 + 16),
          // whose scores are already in registers
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int c = h + 2 * e;
            const uint64_t xx = f2_fma(f2_pack(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])),
                                       scale2, nbase2);
            const uint64_t pp = f2_pack(fast_exp2(f2_lo(xx)), fast_exp2(f2_hi(xx)));
            rs2[e % (NP / 2)] = f2_add(rs2[e % (NP / 2)], pp);
            pk[e] = epack<H>(f2_lo(pp), f2_hi(pp));
          }
          tmem_st16(s_col + h / 2, pk);
        }
#pragma unroll
        for (int i = 1; i < NP / 2; ++i) rs2[0] = f2_add(rs2[0], rs2[i]);
        float rs[1] = {f2_lo(rs2[0]) + f2_hi(rs2[0])};
        l = l * alpha + rs[0];
        // O *= alpha where the running max moved (rare: lazy threshold); done
        // after P so the scores' registers are free.  PV(j-1) has completed.
        if (__any_sync(0xffffffffu, rescale_o)) {
          const float f = rescale_o ? alpha : 1.f;
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t ov[32];
            tmem_ld32(o_col + c0, ov);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * f);
            tmem_st32(o_col + c0, ov);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_full + x);
      }
      if (!ok) break;
      // epilogue: O / l -> bf16 -> global
      const int last = it + n - 1;
      ok = mbar_wait_bounded(o_done + x, last & 1, abort_flag, err, wlim);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      uint16_t* orow = p.out + out_offset<D, STRIDED>(p, wk.q_start + qrow, wk.head);
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t ov[32];
        tmem_ld32(o_col + c0, ov);
        tmem_ld_wait();
        if (row_ok) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint4 v;
            v.x = epack<H>(__uint_as_float(ov[i + 0]) * inv, __uint_as_float(ov[i + 1]) * inv);
            v.y = epack<H>(__uint_as_float(ov[i + 2]) * inv, __uint_as_float(ov[i + 3]) * inv);
            v.z = epack<H>(__uint_as_float(ov[i + 4]) * inv, __uint_as_float(ov[i + 5]) * inv);
            v.w = epack<H>(__uint_as_float(ov[i + 6]) * inv, __uint_as_float(ov[i + 7]) * inv);
            *reinterpret_cast<uint4*>(orow + c0 + i) = v;
          }
        }
      }
      tc_fence_before();
      it += n;
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

template <int D, bool H, bool MODS, bool STRIDED, bool PG>
static cudaError_t launch_prefill_b(const PrefillParams& p, const CUtensorMap& q_map,
                                    const CUtensorMap& k_map, const CUtensorMap& v_map, int grid,
                                    cudaStream_t stream) {
  using SM = PrefillSmem<D>;
  auto kernel = prefill_kernel<D, H, MODS, STRIDED, PG>;
  cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kAlloc);
  if (e != cudaSuccess) return e;
  kernel<<<grid, kThreads, SM::kAlloc, stream>>>(p, q_map, k_map, v_map);
  return cudaGetLastError();
}

template <int D, bool H, bool MODS, bool STRIDED>
static cudaError_t launch_prefill_m(const PrefillParams& p, const CUtensorMap& q_map,
                                    const CUtensorMap& k_map, const CUtensorMap& v_map, int grid,
                                    cudaStream_t stream) {
  return p.ppb_shift > 0
             ? launch_prefill_b<D, H, MODS, STRIDED, true>(p, q_map, k_map, v_map, grid, stream)
             : launch_prefill_b<D, H, MODS, STRIDED, false>(p, q_map, k_map, v_map, grid, stream);
}

template <int D, bool H>
static cudaError_t launch_prefill_t(const PrefillParams& p, const CUtensorMap& q_map,
                                    const CUtensorMap& k_map, const CUtensorMap& v_map, int grid,
                                    cudaStream_t stream) {
  const bool strided = p.q_hnd || p.kv_hnd || p.o_tok != (long long)p.num_q_heads * D ||
                       p.o_head != D;
  if (p.mods.any())
    return strided ? launch_prefill_m<D, H, true, true>(p, q_map, k_map, v_map, grid, stream)
                   : launch_prefill_m<D, H, true, false>(p, q_map, k_map, v_map, grid, stream);
  return strided ? launch_prefill_m<D, H, false, true>(p, q_map, k_map, v_map, grid, stream)
                 : launch_prefill_m<D, H, false, false>(p, q_map, k_map, v_map, grid, stream);
}

cudaError_t launch_prefill(const PrefillParams& p, const CUtensorMap& q_map,
                           const CUtensorMap& k_map, const CUtensorMap& v_map, int head_dim,
                           bool fp16, int grid, cudaStream_t stream) {
  if (head_dim == 128)
    return fp16 ? launch_prefill_t<128, true>(p, q_map, k_map, v_map, grid, stream)
                : launch_prefill_t<128, false>(p, q_map, k_map, v_map, grid, stream);
  return fp16 ? launch_prefill_t<64, true>(p, q_map, k_map, v_map, grid, stream)
              : launch_prefill_t<64, false>(p, q_map, k_map, v_map, grid, stream);
}

}  // namespace pa
