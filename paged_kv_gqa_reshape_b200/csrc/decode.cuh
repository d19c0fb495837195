// Split-KV decode attention over the paged cache (single-query sequences):
// the kernel template and its launch, instantiated by decode.cu (GQA groups
// of up to 16 query heads) and decode_sliced.cu (larger groups).
//
// Work split: the pages (16 keys) of all single-query sequences are laid end
// to end and cut into gridDim.x / groups equal contiguous ranges, one per
// resident CTA and group of HPC KV heads, so every CTA streams the same
// number of pages (+-1) whatever the length mix; a sequence cut by a range
// boundary is finished by a split-KV merge.  (The per-page ranges replace
// fixed-size work items, whose last item set the finish time.)  Warp w of a
// CTA computes KV head (group * HPC + w); its query heads' GQA group is
// served by one pass over the pages, so the repeat_interleave expansion of
// vllm-spyre PR #853 "Pytorch Native Attention on Spyre" is never
// materialised.
//
// Memory path: each 16-slot page is copied by the whole CTA as the
// contiguous rows it is in HBM (slot r holds [Hkv, D]), through an
// NSTAGE-deep shared-memory ring of cp.async 16-byte copies (rows
// XOR-swizzled for conflict-free ldmatrix).  The copies run NSTAGE pages
// ahead across sequence boundaries; one barrier per page publishes the page
// that landed and frees the one before it.  Keys past the sequence end are
// zero-filled instead of read; a block id outside the pool is reported and
// read as zeros.
//
// Per page each warp computes S^T = K . Q^T with mma.sync m16n8k16: the
// page's 16 keys are the M rows and the group's query heads the N columns
// (8 per n-tile), so a GQA group of 8 fills the tile exactly.  The online
// softmax runs per head column in the log2 domain (scale folded with log2 e);
// P^T is rounded to bf16 and turned into the B operand of O^T += V^T . P^T
// with movmatrix.  Decode moves ~g FLOP per byte, so it is HBM-bound: the
// legacy mma path keeps up and tcgen05's M >= 64 would buy nothing.
//
// Planning: with up to kSelfPlanMaxSeqs sequences every CTA computes the
// page prefix itself from query_start_loc / seq_lens (one pass + a block scan
// into shared memory), so a pure decode batch needs no plan launch; beyond
// that it reads the prefix the plan kernel wrote.
//
// Output: a sequence inside one range writes bf16 directly.  Otherwise each
// range's segment writes its normalised fp32 partial and log2-sum-exp per head
// into slot (range + sequence), and the last warp to finish a (sequence, KV
// head) merges the segments (arrival counter + fences, reset after use).
#pragma once

#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "layout.h"

namespace pa {

template <int D, int HPC, int NSTAGE>
struct DecodeShape {
  static constexpr int kChunks = D / 8;                     // 16-byte chunks per row
  static constexpr int kHeadPage = kPageKeys * D;           // one head's page (elements)
  static constexpr int kTensorStage = HPC * kHeadPage;      // K (or V) of one stage
  static constexpr int kStageBytes = 2 * kTensorStage * 2;  // K + V
  static constexpr int kRingBytes = NSTAGE * kStageBytes;
  static constexpr int kPlanBytes = (2 * kSelfPlanMaxSeqs + 1) * 4;
  static constexpr int smem_bytes(bool self_plan) {
    return kRingBytes + (self_plan ? kPlanBytes : 0);
  }
};

namespace {

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

}  // namespace

template <int D, int HPC, int NSTAGE, int NGT, bool H, bool MODS, int SL>
__global__ void __launch_bounds__(HPC * 32, 8 / HPC) decode_kernel(DecodeParams p) {
  using Shape = DecodeShape<D, HPC, NSTAGE>;
  constexpr int CH = Shape::kChunks;
  constexpr int KSTEPS = D / 16;  // k-steps of S^T = K . Q^T and m-tiles of O^T
  constexpr int NT = HPC * 32;    // threads per CTA
  constexpr unsigned FULL = 0xffffffffu;

  extern __shared__ __align__(128) unsigned char smem[];
  // Launched with programmatic stream serialisation: when the previous
  // kernel lets this one start early (the cache scatter does), the CTAs are
  // resident before it ends and wait here, before reading any input, until
  // it has completed and its writes are visible.
  griddep_wait();
  // The next kernel on the stream, if launched the same way (the next step's
  // cache scatter is), may become resident now; it waits for this grid to
  // complete before it touches anything.
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int tid = threadIdx.x;
  const int g = p.group;
  const int Hkv = p.num_kv_heads;
  // SL warps share a KV head when its GQA group is larger than one warp's 16
  // query heads (SL a power of two dividing HPC; 1 for groups up to 16)
  static_assert(HPC % SL == 0, "the slices of a KV head tile the CTA's warps");
  constexpr int hpc = HPC / SL;  // KV heads per CTA
  constexpr int hpc_shift = hpc == 8 ? 3 : hpc == 4 ? 2 : hpc == 2 ? 1 : 0;
  const int groups = Hkv / hpc;
  const int S = p.num_seqs;
  const int hg = blockIdx.x % groups;           // KV-head group of this CTA
  const long long c = blockIdx.x / groups;      // page range of this CTA
  // page ranges per group: one per CTA of the grid, or, beside the prefill,
  // the plan's share of the grid (the other CTAs leave at once)
  long long G = gridDim.x / groups;
  if (p.split_sms > 0) {
    const PlanHeader* hdr = reinterpret_cast<const PlanHeader*>(p.ws + p.L.header);
    G = max(1ll, G * min(hdr->decode_sms, p.split_sms) / p.split_sms);
    if (c >= G) return;
  }
  const int kvl = warp / SL;                    // this warp's KV head within the CTA
  const int slice = warp - kvl * SL;            // and its slice of the GQA group
  const int kvh = hg * hpc + kvl;               // this warp's KV head
  const int head0 = kvh * g + slice * 16;       // its first query head
  const int gw = min(g - slice * 16, NGT * 8);  // its query heads (none if <= 0)

  unsigned char* ws = p.ws;
  uint32_t* err = reinterpret_cast<uint32_t*>(ws + p.L.err);
  const SeqInfo* info = reinterpret_cast<const SeqInfo*>(ws + p.L.seq_info);
  const int32_t* g_pfx = reinterpret_cast<const int32_t*>(ws + p.L.page_pfx);
  int32_t* counters = reinterpret_cast<int32_t*>(ws + p.L.counters);
  float* lse_buf = reinterpret_cast<float*>(ws + p.L.lse);
  float* part_buf = reinterpret_cast<float*>(ws + p.L.partial);

  __nv_bfloat16* ring = reinterpret_cast<__nv_bfloat16*>(smem);
  // with an additive mask, each ring stage also holds the page's 16 mask
  // values of every query head of the CTA (copied with the page's K/V)
  constexpr int kMaskHeads = HPC * NGT * 8;
  constexpr int kMaskStage = MODS ? kMaskHeads * kPageKeys : 0;  // floats per stage
  float* mring = reinterpret_cast<float*>(smem + Shape::kRingBytes);
  [[maybe_unused]] const bool mask_shared = MODS && p.mods.mask_head == 0;
  int* s_pg = reinterpret_cast<int*>(smem + Shape::kRingBytes + NSTAGE * kMaskStage * 4);  // [S + 1] page prefix
  int* s_kv = s_pg + kSelfPlanMaxSeqs + 1;                       // [S] decode kv_len or -1
  __shared__ uint32_t s_err;
  __shared__ int s_scan[HPC];
  __shared__ int s_carry;

  // ------------------------------- plan ------------------------------------
  if (p.self_plan) {
    if (tid == 0) {
      s_err = 0;
      s_carry = 0;
    }
    __syncthreads();
    const long long reach = ((long long)p.max_blocks_per_seq << p.ppb_shift) * kPageKeys;
    uint32_t e = 0;
    for (int s = tid; s < S; s += NT) {
      const long long qs = p.query_start_loc[s], qe = p.query_start_loc[s + 1];
      long long kv = p.seq_lens[s];
      const bool bad_q = qs < 0 || qe < qs || qe > p.num_q_tokens;
      if (bad_q) e |= PA_DEVERR_LENGTHS;
      if (kv < 0) {
        e |= PA_DEVERR_LENGTHS;
        kv = 0;
      }
      if (kv > reach) {
        e |= PA_DEVERR_LENGTHS;
        kv = reach;
      }
      if (!bad_q && (qe - qs > p.max_query_len || kv > p.max_seq_len)) e |= PA_DEVERR_HINT;
      const bool dec = !bad_q && qe - qs == 1;
      if (dec && kv == 0) e |= PA_DEVERR_QLEN;
      s_kv[s] = dec ? (int)kv : -1;
    }
    if (e) atomicOr(&s_err, e);
    __syncthreads();
    for (int base = 0; base < S; base += NT) {
      const int s = base + tid;
      const int n = (s < S && s_kv[s] > 0) ? (s_kv[s] + kPageKeys - 1) / kPageKeys : 0;
      int x = n;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(FULL, x, o);
        if (lane >= o) x += y;
      }
      if (lane == 31) s_scan[warp] = x;
      __syncthreads();
      int before = s_carry;
      for (int w = 0; w < warp; ++w) before += s_scan[w];
      if (s < S) s_pg[s] = before + x - n;
      __syncthreads();
      if (tid == 0) {
        int tot = 0;
        for (int w = 0; w < HPC; ++w) tot += s_scan[w];
        s_carry += tot;
      }
      __syncthreads();
    }
    if (tid == 0) s_pg[S] = s_carry;
    __syncthreads();
    if (blockIdx.x == 0 && tid == 0 && s_err) atomicOr(err, s_err);
  }
  auto pfx = [&](int s) -> long long { return p.self_plan ? s_pg[s] : __ldg(g_pfx + s); };
  auto seq_kv = [&](int s) -> int { return p.self_plan ? s_kv[s] : info[s].kv_len; };
  auto seq_q = [&](int s) -> int { return p.self_plan ? p.query_start_loc[s] : info[s].q_start; };
  auto is_decode = [&](int s) -> bool { return p.self_plan ? s_kv[s] >= 0 : info[s].q_len == 1; };

  const long long P = pfx(S);

  // single-query sequences with no key: zero output rows (spread over the ranges)
  for (long long s = c; s < S; s += G) {
    if (is_decode((int)s) && seq_kv((int)s) == 0) {
      uint16_t* o0 = p.out + (size_t)seq_q((int)s) * p.o_tok + (size_t)head0 * p.o_head;
      for (int i = lane; i < gw * D; i += 32)
        o0[(size_t)(i / D) * p.o_head + i % D] = 0;  // +0 in both element types
    }
  }
  if (P == 0) return;

  // min(G, P) ranges, so that every range holds at least one page and every
  // range counted by a sequence's merge really produces a partial
  const long long R = G < P ? G : P;
  if (c >= R) return;
  const long long b0 = c * P / R, b1 = (c + 1) * P / R;  // this CTA's pages [b0, b1)
  // range holding page x: the largest c' with c' * P / R <= x
  auto range_of = [&](long long x) -> long long { return ((x + 1) * R - 1) / P; };
  // the sequence holding page x: the last s with pfx(s) <= x
  auto seq_of = [&](long long x) -> int {
    int lo = 0, hi = S - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pfx(mid) <= x)
        lo = mid;
      else
        hi = mid - 1;
    }
    return lo;
  };
  if (b0 >= b1) return;

  // ---------------- producer: pages [x_p, b1) in order ----------------------
  long long x_p = b0;
  int seq_p = seq_of(b0);
  long long p_first = pfx(seq_p), p_end = pfx(seq_p + 1);
  int p_kv = seq_kv(seq_p);
  [[maybe_unused]] int p_tok = MODS ? seq_q(seq_p) : 0;  // the sequence's query token
  long long x = b0;  // consumer position
  // Each K/V page is read once per call: streaming it evict-first keeps the
  // lines that are read again (the partials a split-KV merge reads back, q,
  // the tables) in L2 while the stream passes through.
  const uint64_t kv_policy = policy_evict_first();
  auto issue_page = [&]() {
    const int stage = (int)((x_p - b0) % NSTAGE);
    const int page = (int)(x_p - p_first);  // 16-key page of the sequence
    const int key0 = page * kPageKeys;
    // the page is slots [16 (page % ppb), +16) of block page / ppb, ppb = 1 << ppb_shift
    const int ppb_shift = p.ppb_shift;
    const long long block = p.block_tables[(size_t)seq_p * p.max_blocks_per_seq + (page >> ppb_shift)];
    const bool block_ok = block >= 0 && block < p.num_blocks;
    if (!block_ok && tid == 0) raise_error(err, PA_DEVERR_BLOCK);
    const size_t base = (size_t)(block_ok ? block : 0) * p.block_stride +
                        (size_t)((page & ((1 << ppb_shift) - 1)) * kPageKeys) * p.c_slot +
                        (size_t)hg * hpc * p.c_head;
    if constexpr (MODS) {
      if (p.mods.mask) {
        // the page's mask values: 16 keys (4 chunks of 4) for each query-head
        // slot (warp w's local head hl) of the CTA, or once when every head
        // shares the mask (head stride 0: one copy, not one identical
        // request per head to the same L2 line); keys past the sequence
        // end or the mask row read nothing and are zero-filled
        float* mdst = mring + (size_t)stage * kMaskStage;
        const long long lim = min((long long)p_kv, p.mods.mask_len);
        const int mask_slots = mask_shared ? 1 : kMaskHeads;
        for (int ci = tid; ci < mask_slots * 4; ci += NT) {
          const int hs = ci >> 2, q4 = ci & 3;
          const int w = hs / (NGT * 8), hl = hs - w * (NGT * 8);  // warp w's local head hl
          const int wsl = w % SL, wh0 = (hg * hpc + w / SL) * g + wsl * 16;
          const int k = key0 + 4 * q4;
          const int nb = (hl < g - wsl * 16) ? (int)max(0ll, min(4ll, lim - k)) * 4 : 0;
          const float* src = p.mods.mask + (size_t)(wh0 + hl) * p.mods.mask_head +
                             (size_t)p_tok * p.mods.mask_tok + k;
          cp_async_16n(smem_u32(mdst + hs * kPageKeys + 4 * q4), nb ? src : p.mods.mask, nb);
        }
        if (tid == 0 && min((long long)p_kv, (long long)key0 + kPageKeys) > p.mods.mask_len)
          raise_error(err, PA_DEVERR_HINT);
      }
    }
    __nv_bfloat16* kdst = ring + (size_t)stage * 2 * Shape::kTensorStage;
    __nv_bfloat16* vdst = kdst + Shape::kTensorStage;
    // the page's rows of the CTA's hpc KV heads: 16 * hpc * CH chunks of 16 B
    static_assert(CH == 8 || CH == 16, "head_dim 64 or 128");
    constexpr int kChShift = CH == 16 ? 4 : 3;
#pragma unroll
    for (int i = 0; i < CH / 2; ++i) {
      const int ci = i * NT + tid;  // chunk index within the page's K (or V) rows
      if (ci >= (kPageKeys * CH) << hpc_shift) break;
      const int r = ci >> (hpc_shift + kChShift);
      const int rem = ci & ((CH << hpc_shift) - 1);
      const int h = rem >> kChShift, cc = rem & (CH - 1);
      const bool ok = block_ok && (key0 + r < p_kv);
      const size_t src = base + (size_t)r * p.c_slot + (size_t)h * p.c_head + cc * 8;
      const int dst = (h * kPageKeys + r) * D + ((cc ^ (r & 7)) * 8);
      cp_async_16_hint(smem_u32(kdst + dst), p.k_cache + (ok ? src : 0), ok, kv_policy);
      cp_async_16_hint(smem_u32(vdst + dst), p.v_cache + (ok ? src : 0), ok, kv_policy);
    }
    cp_async_commit();
    ++x_p;
    if (x_p < b1 && x_p >= p_end) {  // next sequence with pages
      do {
        ++seq_p;
      } while (pfx(seq_p + 1) <= x_p);
      p_first = pfx(seq_p);
      p_end = pfx(seq_p + 1);
      p_kv = seq_kv(seq_p);
      if constexpr (MODS) p_tok = seq_q(seq_p);
    }
  };
  auto fill = [&]() {
    while (x_p - x < NSTAGE && x_p < b1) issue_page();
  };
  fill();

  const int gq = lane >> 2;  // fragment group: key row of S^T / d row of O^T / head of B
  const int tq = lane & 3;   // fragment column pair: heads 2tq, 2tq+1
  const uint32_t* q32 = reinterpret_cast<const uint32_t*>(p.q);

  int seq = seq_of(b0);
  while (x < b1) {
    const long long seg_first = pfx(seq), seg_last = pfx(seq + 1);
    const long long seg_end = seg_last < b1 ? seg_last : b1;
    const int seg_kv = seq_kv(seq);
    const int seg_q = seq_q(seq);
    const long long c_first = range_of(seg_first), c_last = range_of(seg_last - 1);
    const int n_chunks = (int)(c_last - c_first + 1);
    const int pair_base = (int)c_first + seq;

    // Q^T as the B operand (k = d, n = head): heads nt*8 + gq of the group
    uint32_t qb[NGT][KSTEPS][2];
#pragma unroll
    for (int nt = 0; nt < NGT; ++nt) {
      const int hl = nt * 8 + gq;
      const bool hv = hl < gw;
      const size_t row = (size_t)seg_q * p.q_tok + (size_t)(head0 + (hv ? hl : 0)) * p.q_head;
#pragma unroll
      for (int ks = 0; ks < KSTEPS; ++ks) {
        qb[nt][ks][0] = hv ? q32[(row + ks * 16 + 2 * tq) / 2] : 0u;
        qb[nt][ks][1] = hv ? q32[(row + ks * 16 + 2 * tq + 8) / 2] : 0u;
      }
    }
    float o[NGT][KSTEPS][4];
    float m[NGT][2], l[NGT][2];
#pragma unroll
    for (int nt = 0; nt < NGT; ++nt) {
      m[nt][0] = m[nt][1] = -INFINITY;
      l[nt][0] = l[nt][1] = 0.f;
#pragma unroll
      for (int mt = 0; mt < KSTEPS; ++mt) o[nt][mt][0] = o[nt][mt][1] = o[nt][mt][2] = o[nt][mt][3] = 0.f;
    }

    // ALiBi slopes (log2 units) of this lane's heads, two per n-tile
    [[maybe_unused]] float msl[NGT][2];
    if constexpr (MODS) {
#pragma unroll
      for (int nt = 0; nt < NGT; ++nt) {
        const int hl0 = nt * 8 + 2 * tq;
#pragma unroll
        for (int j = 0; j < 2; ++j)
          msl[nt][j] = (p.mods.alibi && hl0 + j < gw) ? __ldg(p.mods.alibi + head0 + hl0 + j) * kLog2e
                                                      : 0.f;
      }
    }

    for (; x < seg_end; ++x) {
      cp_async_wait_dyn((int)(x_p - x - 1));  // my copies of page x have landed
      __syncthreads();  // everyone's have, and page x-1's stage is free
      fill();
      const __nv_bfloat16* kst =
          ring + (size_t)((x - b0) % NSTAGE) * 2 * Shape::kTensorStage + kvl * Shape::kHeadPage;
      const uint32_t kbase = smem_u32(kst), vbase = smem_u32(kst + Shape::kTensorStage);
      const int mi = lane >> 3, rr = lane & 7;

      // ---- S^T = K . Q^T : 16 keys x 8 heads per n-tile ----
      float sc[NGT][4];
#pragma unroll
      for (int nt = 0; nt < NGT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
      {
        const int key = (mi & 1) * 8 + rr;
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks) {
          const int chunk = ks * 2 + (mi >> 1);
          uint32_t a[4];
          ldmatrix_x4(kbase + (key * D + ((chunk ^ (key & 7)) * 8)) * 2, a[0], a[1], a[2], a[3]);
#pragma unroll
          for (int nt = 0; nt < NGT; ++nt) mma_16816<H>(sc[nt], a, qb[nt][ks][0], qb[nt][ks][1]);
        }
      }
      // ---- mask, online softmax per head column ----
      const int key0 = (int)(x - seg_first) * kPageKeys;
      const bool ok0 = key0 + gq < seg_kv, ok1 = key0 + gq + 8 < seg_kv;
      uint32_t pb[NGT][2];
#pragma unroll
      for (int nt = 0; nt < NGT; ++nt) {
        float s0, s1, s2, s3;
        if constexpr (MODS) {
          // soft-cap, ALiBi, additive mask on scale * s, in log2 units; the
          // query sits at key position seg_kv - 1
          const float cap = p.mods.softcap;
          const float a1 = cap > 0.f ? p.scale / cap : p.scale_log2, a2 = cap * kLog2e;
          auto mod = [&](float raw, float slope2, float mv, int key) {
            const float x = raw * a1;
            const float t = cap > 0.f ? a2 * tanh_sfu(x) : x;
            return fmaf(slope2, (float)(key - (seg_kv - 1)), t) + mv;
          };
          // this page's mask values (log2 units) from the ring stage
          float mv[4] = {0.f, 0.f, 0.f, 0.f};
          if (p.mods.mask) {
            const int hstride = mask_shared ? 0 : kPageKeys;  // floats between head slots
            const float* mst = mring + (size_t)((x - b0) % NSTAGE) * kMaskStage +
                               (size_t)(warp * NGT * 8 + nt * 8 + 2 * tq) * hstride + gq;
            mv[0] = mst[0] * kLog2e;
            mv[1] = mst[hstride] * kLog2e;
            mv[2] = mst[8] * kLog2e;
            mv[3] = mst[hstride + 8] * kLog2e;
          }
          s0 = ok0 ? mod(sc[nt][0], msl[nt][0], mv[0], key0 + gq) : -INFINITY;
          s1 = ok0 ? mod(sc[nt][1], msl[nt][1], mv[1], key0 + gq) : -INFINITY;
          s2 = ok1 ? mod(sc[nt][2], msl[nt][0], mv[2], key0 + gq + 8) : -INFINITY;
          s3 = ok1 ? mod(sc[nt][3], msl[nt][1], mv[3], key0 + gq + 8) : -INFINITY;
        } else {
          s0 = ok0 ? sc[nt][0] * p.scale_log2 : -INFINITY;
          s1 = ok0 ? sc[nt][1] * p.scale_log2 : -INFINITY;
          s2 = ok1 ? sc[nt][2] * p.scale_log2 : -INFINITY;
          s3 = ok1 ? sc[nt][3] * p.scale_log2 : -INFINITY;
        }
        float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
        for (int o2 = 4; o2 < 32; o2 <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(FULL, mx0, o2));
          mx1 = fmaxf(mx1, __shfl_xor_sync(FULL, mx1, o2));
        }
        const float mn0 = fmaxf(m[nt][0], mx0), mn1 = fmaxf(m[nt][1], mx1);
        const float base0 = mn0 == -INFINITY ? 0.f : mn0;
        const float base1 = mn1 == -INFINITY ? 0.f : mn1;
        const float a0 = fast_exp2(m[nt][0] - base0), a1 = fast_exp2(m[nt][1] - base1);
        m[nt][0] = mn0;
        m[nt][1] = mn1;
        s0 = fast_exp2(s0 - base0);
        s1 = fast_exp2(s1 - base1);
        s2 = fast_exp2(s2 - base0);
        s3 = fast_exp2(s3 - base1);
        l[nt][0] = l[nt][0] * a0 + s0 + s2;
        l[nt][1] = l[nt][1] * a1 + s1 + s3;
#pragma unroll
        for (int mt = 0; mt < KSTEPS; ++mt) {
          o[nt][mt][0] *= a0;
          o[nt][mt][1] *= a1;
          o[nt][mt][2] *= a0;
          o[nt][mt][3] *= a1;
        }
        pb[nt][0] = movmatrix_trans(epack<H>(s0, s1));  // keys 0-7
        pb[nt][1] = movmatrix_trans(epack<H>(s2, s3));  // keys 8-15
      }
      // ---- O^T += V^T . P^T : 16 d rows x 8 heads per m-tile ----
      {
        const int key = (mi >> 1) * 8 + rr;
#pragma unroll
        for (int mt = 0; mt < KSTEPS; ++mt) {
          const int chunk = mt * 2 + (mi & 1);
          uint32_t a[4];
          ldmatrix_x4_trans(vbase + (key * D + ((chunk ^ (key & 7)) * 8)) * 2, a[0], a[1], a[2],
                            a[3]);
#pragma unroll
          for (int nt = 0; nt < NGT; ++nt) mma_16816<H>(o[nt][mt], a, pb[nt][0], pb[nt][1]);
        }
      }
    }

    // ---- finish this warp's KV head of the segment ----
#pragma unroll
    for (int nt = 0; nt < NGT; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int o2 = 4; o2 < 32; o2 <<= 1) l[nt][j] += __shfl_xor_sync(FULL, l[nt][j], o2);

    if (n_chunks <= 1) {
#pragma unroll
      for (int nt = 0; nt < NGT; ++nt)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int hl = nt * 8 + 2 * tq + j;
          if (hl < gw) {
            const float inv = l[nt][j] > 0.f ? 1.f / l[nt][j] : 0.f;
            uint16_t* orow = p.out + (size_t)seg_q * p.o_tok + (size_t)(head0 + hl) * p.o_head;
#pragma unroll
            for (int mt = 0; mt < KSTEPS; ++mt) {
              orow[mt * 16 + gq] = ebits<H>(o[nt][mt][j] * inv);
              orow[mt * 16 + gq + 8] = ebits<H>(o[nt][mt][2 + j] * inv);
            }
          }
        }
    } else {
      const int pair = (int)c + seq;  // partial slot of (range c, sequence seq)
#pragma unroll
      for (int nt = 0; nt < NGT; ++nt)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int hl = nt * 8 + 2 * tq + j;
          if (hl < gw) {
            const float inv = l[nt][j] > 0.f ? 1.f / l[nt][j] : 0.f;
            float* dst = part_buf + ((size_t)pair * p.num_q_heads + head0 + hl) * D;
#pragma unroll
            for (int mt = 0; mt < KSTEPS; ++mt) {
              dst[mt * 16 + gq] = o[nt][mt][j] * inv;
              dst[mt * 16 + gq + 8] = o[nt][mt][2 + j] * inv;
            }
            if (gq == 0)
              lse_buf[(size_t)pair * p.num_q_heads + head0 + hl] =
                  l[nt][j] > 0.f ? m[nt][j] + log2f(l[nt][j]) : -INFINITY;
          }
        }
      __threadfence();
      __syncwarp();
      int old = 0;
      // one arrival counter per (sequence, KV head, slice)
      int32_t* counter = &counters[((size_t)seq * Hkv + kvh) * SL + slice];
      if (lane == 0) old = atomicAdd(counter, 1);
      old = __shfl_sync(FULL, old, 0);
      if (old == n_chunks - 1) {
        // last chunk of this (sequence, KV head) to finish: merge all of them.
        // out = sum_c 2^(lse_c - M) O_c / sum_c 2^(lse_c - M), M = max_c lse_c.
        // Loads are issued in batches so that a merge costs a few dependent
        // global round trips rather than two per chunk and head.
        __threadfence();
        const int pb0 = pair_base;
        const int nhc = gw * n_chunks;  // (head, chunk) pairs, head-major
        constexpr int kFast = 24;
        if (nhc <= kFast) {
          // One round of loads: lane i holds pair i's log-sum-exp, and every
          // lane this lane's 4 d-values of every pair's partial.
          float lse_mine = -INFINITY;
          if (lane < nhc)
            lse_mine = __ldcg(lse_buf + (size_t)(pb0 + lane % n_chunks) * p.num_q_heads + head0 +
                              lane / n_chunks);
          float4 xv[kFast];
#pragma unroll
          for (int i = 0; i < kFast; ++i) {
            xv[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i < nhc && lane * 4 < D)
              xv[i] = __ldcg(reinterpret_cast<const float4*>(
                  part_buf + ((size_t)(pb0 + i % n_chunks) * p.num_q_heads + head0 + i / n_chunks) * D +
                  lane * 4));
          }
          // per-head max and weight sum over the head's lanes [h*nc, h*nc + nc)
          const int seg0 = (lane / n_chunks) * n_chunks;
          float M = -INFINITY;
          for (int j = 0; j < n_chunks; ++j)
            M = fmaxf(M, __shfl_sync(FULL, lse_mine, (seg0 + j) & 31));
          const float w_mine =
              (lane < nhc && lse_mine != -INFINITY && M != -INFINITY) ? fast_exp2(lse_mine - M) : 0.f;
          float wsum = 0.f;
          for (int j = 0; j < n_chunks; ++j) wsum += __shfl_sync(FULL, w_mine, (seg0 + j) & 31);
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int i = 0; i < kFast; ++i) {
            if (i < nhc) {
              const float w = __shfl_sync(FULL, w_mine, i);
              const float ws = __shfl_sync(FULL, wsum, i);
              acc.x += w * xv[i].x;
              acc.y += w * xv[i].y;
              acc.z += w * xv[i].z;
              acc.w += w * xv[i].w;
              if (i % n_chunks == n_chunks - 1) {  // the head's last chunk: write it
                if (lane * 4 < D) {
                  const float inv = ws > 0.f ? 1.f / ws : 0.f;
                  uint2 v;
                  v.x = epack<H>(acc.x * inv, acc.y * inv);
                  v.y = epack<H>(acc.z * inv, acc.w * inv);
                  *reinterpret_cast<uint2*>(p.out + (size_t)seg_q * p.o_tok +
                                            (size_t)(head0 + i / n_chunks) * p.o_head + lane * 4) = v;
                }
                acc = make_float4(0.f, 0.f, 0.f, 0.f);
              }
            }
          }
        } else {
        // larger merges: per head, loads batched four chunks at a time
        const bool one_pass = gw * n_chunks <= 32;
        float lse_mine = -INFINITY;
        if (one_pass && lane < gw * n_chunks)
          lse_mine = __ldcg(lse_buf + (size_t)(pb0 + lane % n_chunks) * p.num_q_heads + head0 +
                            lane / n_chunks);
        for (int hl = 0; hl < gw; ++hl) {
          const int head = head0 + hl;
          // lane c (c < n_chunks, per pass of 32) holds chunk c's weight
          float M = -INFINITY;
          for (int c0 = 0; c0 < n_chunks; c0 += 32) {
            const float lc = one_pass ? __shfl_sync(FULL, lse_mine, (hl * n_chunks + lane) & 31)
                             : (c0 + lane < n_chunks
                                    ? __ldcg(lse_buf + (size_t)(pb0 + c0 + lane) * p.num_q_heads + head)
                                    : -INFINITY);
            M = fmaxf(M, lane < n_chunks - c0 ? lc : -INFINITY);
          }
#pragma unroll
          for (int o2 = 16; o2 > 0; o2 >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL, M, o2));
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
          float wsum = 0.f;
          if (M != -INFINITY) {
            for (int c0 = 0; c0 < n_chunks; c0 += 32) {
              float lc = one_pass ? __shfl_sync(FULL, lse_mine, (hl * n_chunks + lane) & 31)
                         : (c0 + lane < n_chunks
                                ? __ldcg(lse_buf + (size_t)(pb0 + c0 + lane) * p.num_q_heads + head)
                                : -INFINITY);
              if (lane >= n_chunks - c0) lc = -INFINITY;
              const float w_mine = (lc == -INFINITY) ? 0.f : fast_exp2(lc - M);
              const int nc = min(32, n_chunks - c0);
              for (int cb = 0; cb < nc; cb += 4) {
                float4 xv[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                  xv[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                  if (cb + u < nc && lane * 4 < D)
                    xv[u] = __ldcg(reinterpret_cast<const float4*>(
                        part_buf + ((size_t)(pb0 + c0 + cb + u) * p.num_q_heads + head) * D + lane * 4));
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                  const float w = __shfl_sync(FULL, w_mine, (cb + u) & 31);
                  if (cb + u < nc) {
                    wsum += w;
                    acc.x += w * xv[u].x;
                    acc.y += w * xv[u].y;
                    acc.z += w * xv[u].z;
                    acc.w += w * xv[u].w;
                  }
                }
              }
            }
          }
          if (lane * 4 < D) {
            const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
            uint2 v;
            v.x = epack<H>(acc.x * inv, acc.y * inv);
            v.y = epack<H>(acc.z * inv, acc.w * inv);
            *reinterpret_cast<uint2*>(p.out + (size_t)seg_q * p.o_tok + (size_t)head * p.o_head +
                                      lane * 4) = v;
          }
        }
        }
        if (lane == 0) *counter = 0;  // ready for the next call
      }
    }


    // ---- next sequence with pages ----
    if (x < b1) {
      do {
        ++seq;
      } while (pfx(seq + 1) <= x);
    }
  }
  cp_async_wait<0>();
}

// Warps per CTA: slices warps per KV head times the largest number of KV
// heads (a power of two, at most 8 / slices) that divides num_kv_heads.
inline int warps_per_cta(int num_kv_heads, int slices) {
  for (int h = 8 / slices; h > 1; h >>= 1)
    if (num_kv_heads % h == 0) return h * slices;
  return slices;
}

template <int D, int HPC, int NSTAGE, int NGT, bool H, bool MODS, int SL>
cudaError_t launch_t(const DecodeParams& p, int num_sms, cudaStream_t stream) {
  using Shape = DecodeShape<D, HPC, NSTAGE>;
  auto kernel = decode_kernel<D, HPC, NSTAGE, NGT, H, MODS, SL>;
  const int smem =
      Shape::smem_bytes(p.self_plan != 0) + (MODS ? NSTAGE * HPC * NGT * 8 * kPageKeys * 4 : 0);
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, HPC * 32, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  // one resident wave; each KV-head group gets the same number of page ranges,
  // and there are never more ranges per group than the partial slots allow
  const int groups = p.num_kv_heads / (HPC / SL);
  long long ranges = (long long)per_sm * num_sms / groups;
  const long long cap = (kDecodeMaxWarps + p.num_kv_heads - 1) / p.num_kv_heads;
  if (ranges > cap) ranges = cap;
  if (ranges < 1) ranges = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(ranges * groups));
  cfg.blockDim = dim3(HPC * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, p);
}

}  // namespace pa
