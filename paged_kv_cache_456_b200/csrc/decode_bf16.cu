// decode_bf16.cu -- decode kernel instances with bf16 elements.
// Ring depth and warps per CTA are chosen per shape so that two or more CTAs
// fit in an SM's shared memory with several tiles in flight per warp.
#include "decode_kernel.cuh"

namespace pa {

template <int D, int G, int DEPTH, int WARPS>
static bool fill(DecodeKernelInfo* info) {
  info->fn = reinterpret_cast<const void*>(&paged_decode_kernel<__nv_bfloat16, D, G, DEPTH, WARPS>);
  info->merge_fn = reinterpret_cast<const void*>(&paged_decode_merge_kernel<__nv_bfloat16, D, G>);
  info->warps = WARPS;
  info->depth = DEPTH;
  info->warp_bytes = DecodeCfg<__nv_bfloat16, D, G, DEPTH, WARPS>::WARP_BYTES;
  return true;
}

// Build-time overrides for tuning sweeps of the head_dim 128 instances.
#ifndef PA_BF16_128_DEPTH
#define PA_BF16_128_DEPTH 2
#endif
#ifndef PA_BF16_128_DEPTH_G8
#define PA_BF16_128_DEPTH_G8 2
#endif
#ifndef PA_BF16_128_WARPS
#define PA_BF16_128_WARPS 4
#endif

bool decode_kernel_bf16(int head_dim, int group, DecodeKernelInfo* info) {
  constexpr int kD = PA_BF16_128_DEPTH, kD8 = PA_BF16_128_DEPTH_G8, kW = PA_BF16_128_WARPS;
  switch (head_dim * 100 + group) {
    case 6401: return fill<64, 1, 4, 4>(info);
    case 6402: return fill<64, 2, 4, 4>(info);
    case 6404: return fill<64, 4, 4, 4>(info);
    case 6408: return fill<64, 8, 4, 4>(info);
    case 12801: return fill<128, 1, kD, kW>(info);
    case 12802: return fill<128, 2, kD, kW>(info);
    case 12804: return fill<128, 4, kD, kW>(info);
    case 12808: return fill<128, 8, kD8, kW>(info);
    default: return false;
  }
}

}  // namespace pa
