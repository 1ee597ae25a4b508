// decode_f32.cu -- decode kernel instances with f32 elements.
// Ring depth and warps per CTA are chosen per shape so that two or more CTAs
// fit in an SM's shared memory with several tiles in flight per warp.
#include "decode_kernel.cuh"
#include "merge_kernel.cuh"

namespace pa {

template <int D, int G, int HS, int DEPTH, int WARPS, int MIN_CTAS = 1>
static bool fill(DecodeKernelInfo* info) {
  info->fn = reinterpret_cast<const void*>(&paged_decode_kernel<float, D, G, HS, DEPTH, WARPS, MIN_CTAS>);
  info->merge_fn = reinterpret_cast<const void*>(&paged_decode_merge_kernel<float, D, G>);
  info->warps = WARPS;
  info->workers = WARPS / HS;
  info->depth = DEPTH;
  info->cta_bytes = DecodeCfg<float, D, G / HS, G, HS, DEPTH, WARPS>::CTA_BYTES;
  info->tma = false;
  info->rows_per_item = 1;
  return true;
}

bool decode_kernel_f32(int head_dim, int group, DecodeKernelInfo* info) {
  switch (head_dim * 100 + group) {
    case 6401: return fill<64, 1, 1, 3, 4, 3>(info);
    case 6402: return fill<64, 2, 1, 3, 4>(info);
    case 6404: return fill<64, 4, 1, 3, 4>(info);
    case 6408: return fill<64, 8, 2, 2, 4>(info);
    case 12801: return fill<128, 1, 1, 2, 2>(info);
    case 12802: return fill<128, 2, 1, 2, 2>(info);
    case 12804: return fill<128, 4, 1, 2, 2>(info);
    case 12808: return fill<128, 8, 2, 2, 2>(info);
    default: return false;
  }
}

}  // namespace pa
