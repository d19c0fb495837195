// Split-KV decode attention for GQA groups of more than 16 query heads (MQA
// included): each KV head's group is cut into 16-head slices, one warp per
// slice, and the warps of a KV head share its pages in shared memory (one
// copy of K and V per KV head, however large the group).  The kernel is the
// one in decode.cuh, instantiated here with SL = 2, 4 or 8 slices per KV head
// (the group of repeat_interleave'd query heads of vllm-spyre PR #853
// "Pytorch Native Attention on Spyre", description, for any group size).
#include "decode.cuh"

namespace pa {

namespace {

template <int D, int NSTAGE, bool H, bool MODS>
cudaError_t launch_sliced_t(const DecodeParams& p, int num_sms, cudaStream_t stream) {
  const int warps = warps_per_cta(p.num_kv_heads, p.slices);
  switch (p.slices) {
    case 2:
      if (warps == 8) return launch_t<D, 8, NSTAGE, 2, H, MODS, 2>(p, num_sms, stream);
      if (warps == 4) return launch_t<D, 4, NSTAGE, 2, H, MODS, 2>(p, num_sms, stream);
      return launch_t<D, 2, NSTAGE, 2, H, MODS, 2>(p, num_sms, stream);
    case 4:
      if (warps == 8) return launch_t<D, 8, NSTAGE, 2, H, MODS, 4>(p, num_sms, stream);
      return launch_t<D, 4, NSTAGE, 2, H, MODS, 4>(p, num_sms, stream);
    default:
      return launch_t<D, 8, NSTAGE, 2, H, MODS, 8>(p, num_sms, stream);
  }
}

template <bool H, bool MODS>
cudaError_t launch_sliced_d(const DecodeParams& p, int head_dim, int num_sms,
                            cudaStream_t stream) {
  if (head_dim == 128) return launch_sliced_t<128, 3, H, MODS>(p, num_sms, stream);
  return launch_sliced_t<64, MODS ? 4 : 6, H, MODS>(p, num_sms, stream);
}

}  // namespace

cudaError_t launch_decode_sliced(const DecodeParams& p, int head_dim, bool fp16, int num_sms,
                                 cudaStream_t stream) {
  if (p.mods.any())
    return fp16 ? launch_sliced_d<true, true>(p, head_dim, num_sms, stream)
                : launch_sliced_d<false, true>(p, head_dim, num_sms, stream);
  return fp16 ? launch_sliced_d<true, false>(p, head_dim, num_sms, stream)
              : launch_sliced_d<false, false>(p, head_dim, num_sms, stream);
}

}  // namespace pa
