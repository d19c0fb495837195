// s_q = 1 cross attention over at most 16 contiguous keys per batch entry —
// the small-seq case of ROCm/TransformerEngine PR #461 "CK varlen cross
// attention for small-seq" (description: one query per entry, THD keys with
// cu_seqlens_kv, no causal mask, s_kv <= 16), written for B200.
//
// One warp per (entry, query head).  A key row of head_dim bf16 is covered by
// D/8 lanes holding 16 bytes each, so a warp takes 32/(D/8) keys per pass
// (2 for D = 128).  All of the entry's K and V rows for this head are loaded
// before any arithmetic (up to 16 keys => 8 passes of 16-byte loads in flight
// per lane), which is what keeps HBM busy: the work is pure bandwidth (2 FLOP
// per byte).  Dot products reduce with xor-shuffles inside a key's lane group;
// the softmax over <= 16 scores stays in registers (log2 domain, scale folded
// with log2 e); an empty entry writes zeros.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace pa {

template <int D>
__global__ void __launch_bounds__(256) smallseq_kernel(SmallSeqParams p) {
  constexpr int LPK = D / 8;        // lanes per key row
  constexpr int KPP = 32 / LPK;     // keys per pass
  constexpr int PASSES = 16 / KPP;  // passes for the 16-key maximum
  const int lane = threadIdx.x & 31;
  const long long wid = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (wid >= (long long)p.batch * p.num_q_heads) return;
  const int b = (int)(wid / p.num_q_heads);
  const int h = (int)(wid % p.num_q_heads);
  const int kvh = h / p.group;
  const int sub = lane / LPK, l = lane % LPK;

  const int start = p.cu_seqlens_kv[b];
  int n = p.cu_seqlens_kv[b + 1] - start;
  if (start < 0 || n < 0) {
    if (lane == 0) raise_error(p.err, PA_DEVERR_LENGTHS);
    n = 0;
  }
  if (n > p.max_seqlen_kv) {
    if (lane == 0) raise_error(p.err, PA_DEVERR_HINT);
    n = p.max_seqlen_kv;
  }

  const uint4 qv = __ldcs(reinterpret_cast<const uint4*>(p.q + ((size_t)b * p.num_q_heads + h) * D) + l);
  float qf[8];
  {
    const uint32_t w[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      qf[2 * i] = bf16lo(w[i]) * p.scale_log2;
      qf[2 * i + 1] = bf16hi(w[i]) * p.scale_log2;
    }
  }

  uint4 kr[PASSES], vr[PASSES];
#pragma unroll
  for (int pp = 0; pp < PASSES; ++pp) {
    const int j = pp * KPP + sub;
    if (j < n) {
      const size_t row = ((size_t)(start + j) * p.num_kv_heads + kvh) * D;
      kr[pp] = __ldcs(reinterpret_cast<const uint4*>(p.k + row) + l);
      vr[pp] = __ldcs(reinterpret_cast<const uint4*>(p.v + row) + l);
    } else {
      kr[pp] = make_uint4(0, 0, 0, 0);
      vr[pp] = make_uint4(0, 0, 0, 0);
    }
  }

  float s[PASSES];
  float m = -INFINITY;
#pragma unroll
  for (int pp = 0; pp < PASSES; ++pp) {
    const uint32_t w[4] = {kr[pp].x, kr[pp].y, kr[pp].z, kr[pp].w};
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      dot = fmaf(qf[2 * i], bf16lo(w[i]), dot);
      dot = fmaf(qf[2 * i + 1], bf16hi(w[i]), dot);
    }
#pragma unroll
    for (int o = LPK / 2; o >= 1; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    s[pp] = (pp * KPP + sub < n) ? dot : -INFINITY;
    m = fmaxf(m, s[pp]);
  }
#pragma unroll
  for (int o = LPK; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));

  float sum = 0.f, acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
  for (int pp = 0; pp < PASSES; ++pp) {
    const float pw = (s[pp] == -INFINITY) ? 0.f : fast_exp2(s[pp] - m);
    sum += pw;
    const uint32_t w[4] = {vr[pp].x, vr[pp].y, vr[pp].z, vr[pp].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] = fmaf(pw, bf16lo(w[i]), acc[2 * i]);
      acc[2 * i + 1] = fmaf(pw, bf16hi(w[i]), acc[2 * i + 1]);
    }
  }
#pragma unroll
  for (int o = LPK; o < 32; o <<= 1) {
    sum += __shfl_xor_sync(0xffffffffu, sum, o);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
  }
  if (sub == 0) {
    const float inv = sum > 0.f ? 1.f / sum : 0.f;
    uint4 ov;
    ov.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    ov.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
    ov.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
    ov.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
    __stcs(reinterpret_cast<uint4*>(p.out + ((size_t)b * p.num_q_heads + h) * D) + l, ov);
  }
}

cudaError_t launch_smallseq(const SmallSeqParams& p, int head_dim, cudaStream_t stream) {
  const long long warps = (long long)p.batch * p.num_q_heads;
  if (warps == 0) return cudaSuccess;
  const int threads = 256;
  const long long blocks = (warps + 7) / 8;
  if (blocks > 0x7fffffffll) return cudaErrorInvalidConfiguration;
  if (head_dim == 128)
    smallseq_kernel<128><<<(unsigned)blocks, threads, 0, stream>>>(p);
  else
    smallseq_kernel<64><<<(unsigned)blocks, threads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace pa
