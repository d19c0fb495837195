// s_q = 1 cross attention over at most 16 contiguous keys per batch entry —
// the small-seq case of ROCm/TransformerEngine PR #461 "CK varlen cross
// attention for small-seq" (description: one query per entry, THD keys with
// cu_seqlens_kv, no causal mask, s_kv <= 16), written for B200.
//
// Work item = (entry, query head), one warp at a time.  The grid is one
// resident wave of persistent warps (three 256-thread CTAs per SM); warp w
// takes items w, w + W, w + 2W, ... (W = all warps), so at any moment the
// warps cover a contiguous run of entries and DRAM sees whole [s_kv, H, D]
// key blocks, and no time goes to retiring and launching short-lived CTAs.
// Each item's K and V rows (16-byte loads, up to 16 keys) are all issued
// before any arithmetic, and the next item's cu_seqlens bounds are loaded
// while the current item computes.  The math runs over the smallest power of
// two of key passes covering the entry, as straight-line code, so the shuffle
// trees of all passes overlap (a branch per pass serialised them: 76 % -> 85 %
// of the copy bandwidth).  (Holding a second item's rows in registers instead
// halves the resident warps and measured at half the bandwidth; staging whole
// entries through a shared-memory ring with bulk copies left the per-entry
// math of 16 warps per SM as the bound.)
//
// Within an item a key row of head_dim bf16 is covered by D/8 lanes holding
// 16 bytes each (32/(D/8) keys per pass: 2 for D = 128).  Dot products reduce
// with xor-shuffles inside a key's lane group; the softmax over <= 16 scores
// stays in registers (log2 domain, scale folded with log2 e); an empty entry
// writes zeros.  The work is pure bandwidth: 2 FLOP per byte.
#include <math.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace pa {

namespace {

template <int D>
struct SmallSeqItem {
  static constexpr int LPK = D / 8;        // lanes per key row
  static constexpr int KPP = 32 / LPK;     // keys per pass
  static constexpr int PASSES = 16 / KPP;  // passes for the 16-key maximum
  static_assert(PASSES <= LPK, "one lane per pass in each key group");
  uint4 q;
  uint4 k[PASSES], v[PASSES];
  int n;  // keys of the entry (clamped)
};

}  // namespace

template <int D, bool H>
__global__ void __launch_bounds__(256, 3) smallseq_kernel(SmallSeqParams p) {
  using It = SmallSeqItem<D>;
  constexpr int LPK = It::LPK, KPP = It::KPP, PASSES = It::PASSES;
  const int lane = threadIdx.x & 31;
  const int sub = lane / LPK, l = lane % LPK;
  const long long total = (long long)p.batch * p.num_q_heads;
  const long long W = (long long)gridDim.x * (blockDim.x >> 5);
  long long item = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);

  // cu_seqlens bounds of an item (the first link of the load chain)
  auto bounds = [&](long long it, int& start, int& n) {
    start = 0;
    n = 0;
    if (it < total) {
      const int b = (int)(it / p.num_q_heads);
      start = p.cu_seqlens_kv[b];
      n = p.cu_seqlens_kv[b + 1] - start;
    }
  };
  // issue every load of an item whose bounds are known
  auto load = [&](long long it, int start, int n, It& x) {
    x.n = 0;
    if (it >= total) return;
    const int b = (int)(it / p.num_q_heads);
    const int h = (int)(it - (long long)b * p.num_q_heads);
    if (start < 0 || n < 0) {
      if (lane == 0) raise_error(p.err, PA_DEVERR_LENGTHS);
      n = 0;
    }
    if (n > p.max_seqlen_kv) {
      if (lane == 0) raise_error(p.err, PA_DEVERR_HINT);
      n = p.max_seqlen_kv;
    }
    x.n = n;
    const int kvh = h / p.group;
    x.q = __ldcs(reinterpret_cast<const uint4*>(p.q + ((size_t)b * p.num_q_heads + h) * D) + l);
#pragma unroll
    for (int pp = 0; pp < PASSES; ++pp) {
      const int j = pp * KPP + sub;
      if (j < n) {
        const size_t row = ((size_t)(start + j) * p.num_kv_heads + kvh) * D;
        x.k[pp] = __ldcs(reinterpret_cast<const uint4*>(p.k + row) + l);
        x.v[pp] = __ldcs(reinterpret_cast<const uint4*>(p.v + row) + l);
      } else {
        x.k[pp] = make_uint4(0, 0, 0, 0);
        x.v[pp] = make_uint4(0, 0, 0, 0);
      }
    }
  };

  It cur;
  int s1, n1;
  bounds(item, s1, n1);

  for (; item < total; item += W) {
    load(item, s1, n1, cur);
    bounds(item + W, s1, n1);  // the next item's bounds load overlaps this item

    // ---- compute the current item ----
    const int b = (int)(item / p.num_q_heads);
    const int h = (int)(item - (long long)b * p.num_q_heads);
    float qf[8];
    {
      const uint32_t w[4] = {cur.q.x, cur.q.y, cur.q.z, cur.q.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        qf[2 * i] = elo<H>(w[i]) * p.scale_log2;
        qf[2 * i + 1] = ehi<H>(w[i]) * p.scale_log2;
      }
    }
    // NP passes of KPP keys, straight-line (the shuffle trees of all passes
    // overlap); NP is the smallest power of two covering the entry's keys
    float sum = 0.f, acc[8];
    float pwv[PASSES];  // unnormalised weight of this lane's key in each pass
#pragma unroll
    for (int pp = 0; pp < PASSES; ++pp) pwv[pp] = 0.f;
    auto attend = [&](auto np_tag) {
      constexpr int NP = decltype(np_tag)::value;
      float sc[NP];
#pragma unroll
      for (int pp = 0; pp < NP; ++pp) {
        const uint32_t w[4] = {cur.k[pp].x, cur.k[pp].y, cur.k[pp].z, cur.k[pp].w};
        float dot = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          dot = fmaf(qf[2 * i], elo<H>(w[i]), dot);
          dot = fmaf(qf[2 * i + 1], ehi<H>(w[i]), dot);
        }
        sc[pp] = dot;
      }
#pragma unroll
      for (int o = LPK / 2; o >= 1; o >>= 1)
#pragma unroll
        for (int pp = 0; pp < NP; ++pp) sc[pp] += __shfl_xor_sync(0xffffffffu, sc[pp], o);
      float m = -INFINITY;
#pragma unroll
      for (int pp = 0; pp < NP; ++pp) {
        if (pp * KPP + sub >= cur.n) sc[pp] = -INFINITY;
        m = fmaxf(m, sc[pp]);
      }
#pragma unroll
      for (int o = LPK; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
      for (int pp = 0; pp < NP; ++pp) {
        const float pw = (sc[pp] == -INFINITY) ? 0.f : fast_exp2(sc[pp] - m);
        sum += pw;
        pwv[pp] = pw;
        const uint32_t w[4] = {cur.v[pp].x, cur.v[pp].y, cur.v[pp].z, cur.v[pp].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[2 * i] = fmaf(pw, elo<H>(w[i]), acc[2 * i]);
          acc[2 * i + 1] = fmaf(pw, ehi<H>(w[i]), acc[2 * i + 1]);
        }
      }
    };
    const int npass = (cur.n + KPP - 1) / KPP;
    if (npass <= 1)
      attend(std::integral_constant<int, 1>{});
    else if (npass <= 2)
      attend(std::integral_constant<int, 2>{});
    else if (PASSES <= 4 || npass <= 4)
      attend(std::integral_constant<int, (PASSES < 4 ? PASSES : 4)>{});
    else
      attend(std::integral_constant<int, PASSES>{});
#pragma unroll
    for (int o = LPK; o < 32; o <<= 1) {
      sum += __shfl_xor_sync(0xffffffffu, sum, o);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
    }
    if (p.weights) {
      // attention weights [batch, Hq, weights_len]: the entry's softmax, then zeros
      const float winv = sum > 0.f ? 1.f / sum : 0.f;
      uint16_t* wrow = p.weights + ((size_t)b * p.num_q_heads + h) * p.weights_len;
      if (cur.n > p.weights_len && lane == 0) raise_error(p.err, PA_DEVERR_HINT);
      // lane t writes weight t (one coalesced row store).  Key t is pass
      // t / KPP of key group t % KPP, whose lanes all hold its weight: lane
      // pp of each group (PASSES <= LPK) offers its pass-pp weight, and one
      // shuffle brings key t's to lane t (lanes past the last pass read 0).
      float mine = 0.f;
#pragma unroll
      for (int pp = 0; pp < PASSES; ++pp)
        if (l == pp) mine = pwv[pp];
      const float wt = __shfl_sync(0xffffffffu, mine, (lane % KPP) * LPK + lane / KPP);
      for (int t = lane; t < p.weights_len; t += 32)  // written once, not read back here
        __stcs(reinterpret_cast<unsigned short*>(wrow + t),
               (t < cur.n && t == lane) ? ebits<H>(wt * winv) : (unsigned short)0);
    }
    if (sub == 0) {
      const float inv = sum > 0.f ? 1.f / sum : 0.f;  // an empty entry writes zeros
      uint4 ov;
      ov.x = epack<H>(acc[0] * inv, acc[1] * inv);
      ov.y = epack<H>(acc[2] * inv, acc[3] * inv);
      ov.z = epack<H>(acc[4] * inv, acc[5] * inv);
      ov.w = epack<H>(acc[6] * inv, acc[7] * inv);
      __stcs(reinterpret_cast<uint4*>(p.out + ((size_t)b * p.num_q_heads + h) * D) + l, ov);
    }
  }
}

cudaError_t launch_smallseq(const SmallSeqParams& p, int head_dim, bool fp16, int num_sms,
                            cudaStream_t stream) {
  const long long warps = (long long)p.batch * p.num_q_heads;
  if (warps == 0) return cudaSuccess;
  const int threads = 256;
  auto kernel = head_dim == 128 ? (fp16 ? smallseq_kernel<128, true> : smallseq_kernel<128, false>)
                                 : (fp16 ? smallseq_kernel<64, true> : smallseq_kernel<64, false>);
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, 0);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  long long blocks = (long long)per_sm * num_sms;  // one resident wave of persistent warps
  const long long needed = (warps + 7) / 8;
  if (blocks > needed) blocks = needed;
  kernel<<<(unsigned)blocks, threads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace pa
