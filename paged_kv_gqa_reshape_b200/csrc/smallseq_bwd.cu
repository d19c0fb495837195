// Backward of the s_q = 1 small-seq attention — ROCm/TransformerEngine PR
// #461 "CK varlen cross attention for small-seq" (description: grad_V,
// grad_attn, the softmax backward and grad_Q / grad_K, reading the attention
// weights the forward saved instead of recomputing the softmax).
//
// For one entry, query head h and its KV head, with saved weights p_j, keys
// k_j, values v_j (j < n), query q and upstream gradient dO:
//     dP_j = <dO, v_j>                        grad_attn
//     dS_j = p_j (dP_j - sum_k p_k dP_k)      softmax backward
//     dQ   = scale * sum_j dS_j k_j           grad_Q
//     dK_j = scale * sum_h dS_hj q_h          grad_K (over the query heads
//     dV_j = sum_h p_hj dO_h                  grad_V  sharing the KV head)
//
// Work item = (entry, KV head), one warp, persistent warps as in the forward
// (so each K/V row's gradient is written by exactly one warp, no atomics).
// K and V rows go to per-warp shared-memory buffers by cp.async (no
// registers held while in flight); each buffer takes the next item's rows as
// soon as this item has used its own, so the next item's loads overlap this
// item's compute, and the next item's key range is read ahead too.
// Phase A1 walks the group's query heads with the V slices (dP, the softmax
// backward; p and dS go to shared memory), phase A2 with the K slices (the
// dQ rows), phase B walks the key passes and sums the heads' contributions
// to each key's dK and dV row.  Lanes cover a key row
// of D elements with D/8 lanes of 16 bytes, as in the forward; the passes are
// straight-line over the smallest power of two covering the entry.
#include <math.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace pa {

namespace {

constexpr int kBwdWarps = 8;
constexpr int kBwdMaxGroup = 16;
constexpr int kBwdMaxKeys = 16;
constexpr int kBwdBlocksPerSm = 2;

// dynamic shared memory of one warp: K and V rows, then p and dS
constexpr int smallseq_bwd_warp_bytes(int d) {
  return 2 * kBwdMaxKeys * d * 2 + 2 * kBwdMaxGroup * kBwdMaxKeys * 4;
}

}  // namespace

template <int D, bool H>
__global__ void __launch_bounds__(kBwdWarps * 32, kBwdBlocksPerSm)
    smallseq_bwd_kernel(SmallSeqBwdParams p) {
  constexpr int LPK = D / 8;        // lanes per key row (16 bytes each)
  constexpr int KPP = 32 / LPK;     // keys per pass
  constexpr int PASSES = kBwdMaxKeys / KPP;
  constexpr unsigned FULL = 0xffffffffu;
  // per warp, in dynamic shared memory: the item's K and V rows (16-byte
  // slice t of the item at index t, so a pass of 32 lanes reads 512
  // contiguous bytes), then p and dS per (head, key)
  extern __shared__ __align__(16) uint4 smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane / LPK, l = lane % LPK;
  const int g = p.group;
  const long long total = (long long)p.batch * p.num_kv_heads;
  const long long W = (long long)gridDim.x * (blockDim.x >> 5);
  uint4* sk = smem + (size_t)warp * (smallseq_bwd_warp_bytes(D) / 16);
  uint4* sv = sk + kBwdMaxKeys * LPK;
  float (*sp)[kBwdMaxKeys] = reinterpret_cast<float (*)[kBwdMaxKeys]>(sv + kBwdMaxKeys * LPK);
  float (*sds)[kBwdMaxKeys] = sp + kBwdMaxGroup;
  const int nmax = min(p.max_seqlen_kv, p.weights_len);

  auto bounds = [&](long long it, int& st, int& cnt) {
    st = 0;
    cnt = 0;
    if (it < total) {
      const int bb = (int)(it / p.num_kv_heads);
      st = p.cu_seqlens_kv[bb];
      cnt = p.cu_seqlens_kv[bb + 1] - st;
    }
  };
  // keys of an item that are used (the same clamping the item applies below)
  auto used = [&](int st, int cnt) { return (st < 0 || cnt < 0) ? 0 : min(cnt, nmax); };
  // start an item's K or V rows into this warp's buffer as one cp.async
  // group: every lane copies exactly the slices it reads later, so its own
  // wait makes them visible
  auto copy_rows = [&](uint4* buf, const uint16_t* src, long long it, int st, int cnt) {
    const int nn = it < total ? used(st, cnt) : 0;
    const int kvh_it = (int)(it % p.num_kv_heads);
    for (int t = lane; t < nn * LPK; t += 32) {
      const size_t row = ((size_t)(st + t / LPK) * p.num_kv_heads + kvh_it) * D;
      cp_async_16(smem_u32(buf + t), reinterpret_cast<const uint4*>(src + row) + t % LPK, true);
    }
    cp_async_commit();
  };
  // cp.async groups in flight at the top of every item: [V of the item,
  // K of the item]; V is read (wait <= 1 pending) before phase A1, K before
  // phase A2, and each buffer takes the next item's rows once this lane has
  // used its own, so the next item's loads overlap this item's compute

  // start an item's q, dO and weight rows towards L1 (one lane per 128-byte line)
  auto prefetch_rows = [&](long long it) {
    if (it >= total) return;
    const int bb = (int)(it / p.num_kv_heads);
    const int h0 = (int)(it - (long long)bb * p.num_kv_heads) * g;
    for (int hl = sub; hl < g; hl += KPP) {
      const size_t qrow = ((size_t)bb * p.num_q_heads + h0 + hl) * D;
      if ((l & 7) == 0) {
        prefetch_l1(p.q + qrow + l * 8);
        prefetch_l1(p.dout + qrow + l * 8);
      }
      if (l == 0) prefetch_l1(p.weights + ((size_t)bb * p.num_q_heads + h0 + hl) * p.weights_len);
    }
  };

  long long item = (long long)blockIdx.x * (blockDim.x >> 5) + warp;
  int s1, n1;
  bounds(item, s1, n1);
  prefetch_rows(item);
  copy_rows(sv, p.v, item, s1, n1);
  copy_rows(sk, p.k, item, s1, n1);
  for (; item < total; item += W) {
    const int b = (int)(item / p.num_kv_heads);
    const int kvh = (int)(item - (long long)b * p.num_kv_heads);
    const int start = s1;
    int n = n1;
    bounds(item + W, s1, n1);  // the next item's range arrives while this one computes
    if (start < 0 || n < 0) {
      if (lane == 0) raise_error(p.err, PA_DEVERR_LENGTHS);
      n = 0;
    }
    if (n > nmax) {
      if (lane == 0) raise_error(p.err, PA_DEVERR_HINT);
      n = nmax;
    }
    const int head0 = kvh * g;
    if (n == 0) {  // no key: the output is zero for every query, so is dQ
      for (int i = lane; i < g * (D / 8); i += 32)
        reinterpret_cast<uint4*>(p.dq + ((size_t)b * p.num_q_heads + head0) * D)[i] =
            make_uint4(0, 0, 0, 0);
      cp_async_wait<0>();
      copy_rows(sv, p.v, item + W, s1, n1);
      copy_rows(sk, p.k, item + W, s1, n1);
      prefetch_rows(item + W);
      continue;
    }
    // the group's q, dO and weight rows are re-read per head and per key
    // pass: they depend only on the item, so the next item's rows are
    // started towards L1 now (this item's were started one item ago)
    prefetch_rows(item + W);

    auto run = [&](auto np_tag) {
      constexpr int NP = decltype(np_tag)::value;
      constexpr int R = LPK / NP;  // lanes left holding the same pass (NP <= LPK / 2)
      // this lane's 16-byte slices of its keys' V rows
      cp_async_wait<1>();
      uint4 vr[NP];
#pragma unroll
      for (int pp = 0; pp < NP; ++pp)
        vr[pp] = (pp * KPP + sub < n) ? sv[pp * 32 + lane] : make_uint4(0, 0, 0, 0);
      // ---- phase A1 (V): per query head, dP and dS into shared memory ----
      for (int hl = 0; hl < g; ++hl) {
        const size_t qrow = ((size_t)b * p.num_q_heads + head0 + hl) * D;
        const uint4 dov = *(reinterpret_cast<const uint4*>(p.dout + qrow) + l);
        const uint16_t* wrow = p.weights + ((size_t)b * p.num_q_heads + head0 + hl) * p.weights_len;
        const uint32_t dw[4] = {dov.x, dov.y, dov.z, dov.w};
        float dp[NP];
#pragma unroll
        for (int pp = 0; pp < NP; ++pp) {
          const uint32_t vw[4] = {vr[pp].x, vr[pp].y, vr[pp].z, vr[pp].w};
          float dot = 0.f;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            dot = fmaf(elo<H>(dw[i]), elo<H>(vw[i]), dot);
            dot = fmaf(ehi<H>(dw[i]), ehi<H>(vw[i]), dot);
          }
          dp[pp] = dot;
        }
        // reduce-scatter over the LPK lanes of a key group: each level sends
        // half of the remaining passes to the partner and keeps the other
        // half, so lane l ends with pass l / R summed over the group
#pragma unroll
        for (int h = NP / 2, o = LPK / 2; h >= 1; h >>= 1, o >>= 1) {
          const bool up = (l & o) != 0;
#pragma unroll
          for (int i = 0; i < h; ++i) {
            const float send = up ? dp[i] : dp[i + h];
            const float keep = up ? dp[i + h] : dp[i];
            dp[i] = keep + __shfl_xor_sync(FULL, send, o);
          }
        }
#pragma unroll
        for (int o = R / 2; o >= 1; o >>= 1) dp[0] += __shfl_xor_sync(FULL, dp[0], o);
        const int jo = (l / R) * KPP + sub;  // the key whose dP this lane holds
        float pw = 0.f;
        if (jo < n) {
          const uint16_t wb = wrow[jo];
          pw = H ? __half2float(__ushort_as_half(wb)) : __uint_as_float((uint32_t)wb << 16);
        }
        // sum_k p_k dP_k, one lane per key
        float pdp = (l % R == 0) ? pw * dp[0] : 0.f;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) pdp += __shfl_xor_sync(FULL, pdp, o);
        if (l % R == 0) {
          sp[hl][jo] = pw;
          sds[hl][jo] = p.scale * pw * (dp[0] - pdp);  // dS, times scale
        }
      }
      __syncwarp();
      // this lane's V slices have been used: the buffer takes the next item's V
      copy_rows(sv, p.v, item + W, s1, n1);
      // ---- phase A2 (K, from shared memory): per query head, the dQ row ----
      cp_async_wait<1>();
      uint4 kr[NP];
#pragma unroll
      for (int pp = 0; pp < NP; ++pp)
        kr[pp] = (pp * KPP + sub < n) ? sk[pp * 32 + lane] : make_uint4(0, 0, 0, 0);
      for (int hl = 0; hl < g; ++hl) {
        float dq[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) dq[i] = 0.f;
#pragma unroll
        for (int pp = 0; pp < NP; ++pp) {
          const float ds = sds[hl][pp * KPP + sub];
          const uint32_t kw[4] = {kr[pp].x, kr[pp].y, kr[pp].z, kr[pp].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            dq[2 * i] = fmaf(ds, elo<H>(kw[i]), dq[2 * i]);
            dq[2 * i + 1] = fmaf(ds, ehi<H>(kw[i]), dq[2 * i + 1]);
          }
        }
        // reduce-scatter over the KPP key groups: lane ends with E of the 8
        // elements of its slice, at element offset base, summed over all keys
        constexpr int E = 8 / KPP;
        int base = 0;
#pragma unroll
        for (int h = 4, o = 16; h >= E; h >>= 1, o >>= 1) {
          const bool up = (lane & o) != 0;
#pragma unroll
          for (int i = 0; i < h; ++i) {
            const float send = up ? dq[i] : dq[i + h];
            const float keep = up ? dq[i + h] : dq[i];
            dq[i] = keep + __shfl_xor_sync(FULL, send, o);
          }
          base += up ? h : 0;
        }
        uint16_t* dst = p.dq + ((size_t)b * p.num_q_heads + head0 + hl) * D + l * 8 + base;
        if constexpr (E == 4) {
          *reinterpret_cast<uint2*>(dst) = make_uint2(epack<H>(dq[0], dq[1]), epack<H>(dq[2], dq[3]));
        } else {
          *reinterpret_cast<uint32_t*>(dst) = epack<H>(dq[0], dq[1]);
        }
      }
      // this lane's K slices have been used (so read): the buffer takes the
      // next item's K while phase B runs
      copy_rows(sk, p.k, item + W, s1, n1);
      __syncwarp();
      // ---- phase B: per key, dK and dV over the group's query heads ----
      auto store_kv = [&](int j, const float (&dk)[8], const float (&dv)[8]) {
        const size_t row = ((size_t)(start + j) * p.num_kv_heads + kvh) * D;
        uint4 ko, vo;
        ko.x = epack<H>(dk[0], dk[1]);
        ko.y = epack<H>(dk[2], dk[3]);
        ko.z = epack<H>(dk[4], dk[5]);
        ko.w = epack<H>(dk[6], dk[7]);
        vo.x = epack<H>(dv[0], dv[1]);
        vo.y = epack<H>(dv[2], dv[3]);
        vo.z = epack<H>(dv[4], dv[5]);
        vo.w = epack<H>(dv[6], dv[7]);
        *(reinterpret_cast<uint4*>(p.dk + row) + l) = ko;
        *(reinterpret_cast<uint4*>(p.dv + row) + l) = vo;
      };
      if (g == 1) {  // one query head per KV head: q and dO widened once
        const size_t qrow = ((size_t)b * p.num_q_heads + head0) * D;
        const uint4 qv = *(reinterpret_cast<const uint4*>(p.q + qrow) + l);
        const uint4 dov = *(reinterpret_cast<const uint4*>(p.dout + qrow) + l);
        const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
        const uint32_t dw[4] = {dov.x, dov.y, dov.z, dov.w};
        float qf[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          qf[2 * i] = elo<H>(qw[i]);
          qf[2 * i + 1] = ehi<H>(qw[i]);
        }
#pragma unroll
        for (int pp = 0; pp < NP; ++pp) {
          const int j = pp * KPP + sub;
          if (j < n) {
            const float ds = sds[0][j];
            const uint32_t pb = ebits<H>(sp[0][j]);  // the saved 16-bit weight, exactly
            const uint32_t p2 = pb | (pb << 16);
            const size_t row = ((size_t)(start + j) * p.num_kv_heads + kvh) * D;
            uint4 ko, vo;
            ko.x = epack<H>(ds * qf[0], ds * qf[1]);
            ko.y = epack<H>(ds * qf[2], ds * qf[3]);
            ko.z = epack<H>(ds * qf[4], ds * qf[5]);
            ko.w = epack<H>(ds * qf[6], ds * qf[7]);
            // dV = p dO: a product of two 16-bit values is exact in fp32, so
            // the packed 16-bit multiply rounds it exactly as fp32 would
            vo.x = emul2<H>(p2, dw[0]);
            vo.y = emul2<H>(p2, dw[1]);
            vo.z = emul2<H>(p2, dw[2]);
            vo.w = emul2<H>(p2, dw[3]);
            *(reinterpret_cast<uint4*>(p.dk + row) + l) = ko;
            *(reinterpret_cast<uint4*>(p.dv + row) + l) = vo;
          }
        }
      } else {
#pragma unroll
        for (int pp = 0; pp < NP; ++pp) {
          const int j = pp * KPP + sub;
          if (j < n) {
            float dk[8], dv[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) dk[i] = dv[i] = 0.f;
            for (int hl = 0; hl < g; ++hl) {
              const size_t qrow = ((size_t)b * p.num_q_heads + head0 + hl) * D;
              const uint4 qv = *(reinterpret_cast<const uint4*>(p.q + qrow) + l);
              const uint4 dov = *(reinterpret_cast<const uint4*>(p.dout + qrow) + l);
              const float pw = sp[hl][j], ds = sds[hl][j];
              const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
              const uint32_t dw[4] = {dov.x, dov.y, dov.z, dov.w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                dk[2 * i] = fmaf(ds, elo<H>(qw[i]), dk[2 * i]);
                dk[2 * i + 1] = fmaf(ds, ehi<H>(qw[i]), dk[2 * i + 1]);
                dv[2 * i] = fmaf(pw, elo<H>(dw[i]), dv[2 * i]);
                dv[2 * i + 1] = fmaf(pw, ehi<H>(dw[i]), dv[2 * i + 1]);
              }
            }
            store_kv(j, dk, dv);
          }
        }
      }
      __syncwarp();
    };
    const int npass = (n + KPP - 1) / KPP;
    if (npass <= 1)
      run(std::integral_constant<int, 1>{});
    else if (npass <= 2)
      run(std::integral_constant<int, 2>{});
    else if (PASSES <= 4 || npass <= 4)
      run(std::integral_constant<int, (PASSES < 4 ? PASSES : 4)>{});
    else
      run(std::integral_constant<int, PASSES>{});
  }
}

cudaError_t launch_smallseq_bwd(const SmallSeqBwdParams& p, int head_dim, bool fp16,
                                int num_sms, cudaStream_t stream) {
  const long long items = (long long)p.batch * p.num_kv_heads;
  if (items == 0) return cudaSuccess;
  auto kernel = head_dim == 128
                    ? (fp16 ? smallseq_bwd_kernel<128, true> : smallseq_bwd_kernel<128, false>)
                    : (fp16 ? smallseq_bwd_kernel<64, true> : smallseq_bwd_kernel<64, false>);
  const int smem = kBwdWarps * smallseq_bwd_warp_bytes(head_dim);
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kBwdWarps * 32, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  long long blocks = (long long)per_sm * num_sms;  // one resident wave of persistent warps
  const long long needed = (items + kBwdWarps - 1) / kBwdWarps;
  if (blocks > needed) blocks = needed;
  kernel<<<(unsigned)blocks, kBwdWarps * 32, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace pa
