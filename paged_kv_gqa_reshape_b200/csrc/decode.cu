// Split-KV decode attention: launches for GQA groups of up to 16 query heads
// (one warp per KV head); decode_sliced.cu covers larger groups.  The kernel
// and its design notes are in decode.cuh.
#include "decode.cuh"

namespace pa {

namespace {

template <int D, int NSTAGE, int NGT, bool H, bool MODS>
cudaError_t launch_hpc(const DecodeParams& p, int hpc, int num_sms, cudaStream_t stream) {
  switch (hpc) {
    case 8: return launch_t<D, 8, NSTAGE, NGT, H, MODS, 1>(p, num_sms, stream);
    case 4: return launch_t<D, 4, NSTAGE, NGT, H, MODS, 1>(p, num_sms, stream);
    case 2: return launch_t<D, 2, NSTAGE, NGT, H, MODS, 1>(p, num_sms, stream);
    default: return launch_t<D, 1, NSTAGE, NGT, H, MODS, 1>(p, num_sms, stream);
  }
}

template <bool H, bool MODS>
cudaError_t launch_decode_t(const DecodeParams& p, int head_dim, int num_sms,
                            cudaStream_t stream) {
  const int hpc = warps_per_cta(p.num_kv_heads, p.slices);
  if (head_dim == 128) {
    if (p.group <= 8) return launch_hpc<128, 3, 1, H, MODS>(p, hpc, num_sms, stream);
    return launch_hpc<128, 3, 2, H, MODS>(p, hpc, num_sms, stream);
  }
  // head_dim 64 with modifiers: 4 stages, so the mask stages fit beside the ring
  constexpr int kStages64 = MODS ? 4 : 6;
  if (p.group <= 8) return launch_hpc<64, kStages64, 1, H, MODS>(p, hpc, num_sms, stream);
  return launch_hpc<64, kStages64, 2, H, MODS>(p, hpc, num_sms, stream);
}

}  // namespace

cudaError_t launch_decode(const DecodeParams& p, int head_dim, bool fp16, int num_sms,
                          cudaStream_t stream) {
  if (p.slices > 1) return launch_decode_sliced(p, head_dim, fp16, num_sms, stream);
  if (p.mods.any())
    return fp16 ? launch_decode_t<true, true>(p, head_dim, num_sms, stream)
                : launch_decode_t<false, true>(p, head_dim, num_sms, stream);
  return fp16 ? launch_decode_t<true, false>(p, head_dim, num_sms, stream)
              : launch_decode_t<false, false>(p, head_dim, num_sms, stream);
}

}  // namespace pa
