// decode_bf16.cu -- decode kernel instances with bf16 elements.
// Ring depth, warps per CTA and head split are chosen per shape so that three
// CTAs (12 warps) fit an SM's registers and shared memory.  A group of 8 query
// heads runs on the tensor cores, one warp per KV head (or, built with
// PA_G8_MMA=0, on the CUDA cores split over two warps that share one ring).
#include "decode_kernel.cuh"
#include "merge_kernel.cuh"

namespace pa {

template <int D, int G, int HS, int DEPTH, int WARPS, int MIN_CTAS = 1, bool MMA = false,
          int NR = 1>
static bool fill(DecodeKernelInfo* info) {
  info->fn = reinterpret_cast<const void*>(
      &paged_decode_kernel<__nv_bfloat16, D, G, HS, DEPTH, WARPS, MIN_CTAS, MMA, NR>);
  info->merge_fn =
      reinterpret_cast<const void*>(&paged_decode_merge_kernel<__nv_bfloat16, D, NR * G, G>);
  info->warps = WARPS;
  info->workers = WARPS / HS;
  info->depth = DEPTH;
  info->cta_bytes = DecodeCfg<__nv_bfloat16, D, G / HS, G, HS, DEPTH, WARPS, MMA, NR>::CTA_BYTES;
  info->tma = MMA;
  info->rows_per_item = NR;
  return true;
}

// Build-time overrides for tuning sweeps of the head_dim 128 instances.
#ifndef PA_BF16_128_DEPTH
#define PA_BF16_128_DEPTH 2
#endif
#ifndef PA_BF16_128_DEPTH_G8
#define PA_BF16_128_DEPTH_G8 3
#endif
#ifndef PA_BF16_128_WARPS
#define PA_BF16_128_WARPS 4
#endif
#ifndef PA_BF16_128_MINCTAS_G8
#define PA_BF16_128_MINCTAS_G8 3
#endif
// Groups of 8 query heads per KV head run on the tensor cores (1) or on the
// CUDA cores with the heads split over two warps (0).
#ifndef PA_G8_MMA
#define PA_G8_MMA 1
#endif
#ifndef PA_MMA_DEPTH
#define PA_MMA_DEPTH 3
#endif
#ifndef PA_MMA_WARPS
#define PA_MMA_WARPS 2
#endif
#ifndef PA_MMA_MINCTAS
#define PA_MMA_MINCTAS 3
#endif

// Several query tokens per sequence with 8 heads per KV head: the
// tensor-core kernel with groups of PA_PREFILL_ROWS query rows per item (they
// share every K/V tile of the group's longest prefix).
#ifndef PA_PREFILL_ROWS
#define PA_PREFILL_ROWS 2
#endif
#ifndef PA_PREFILL_DEPTH
#define PA_PREFILL_DEPTH 2
#endif

bool prefill_kernel_bf16(int head_dim, int group, DecodeKernelInfo* info) {
  if (!PA_G8_MMA || group != 8 || PA_PREFILL_ROWS < 2) return false;
  switch (head_dim) {
    case 64:
      return fill<64, 8, 1, PA_PREFILL_DEPTH, PA_MMA_WARPS, PA_MMA_MINCTAS, true, PA_PREFILL_ROWS>(info);
    case 128:
      return fill<128, 8, 1, PA_PREFILL_DEPTH, PA_MMA_WARPS, PA_MMA_MINCTAS, true, PA_PREFILL_ROWS>(info);
    default: return false;
  }
}

bool decode_kernel_bf16(int head_dim, int group, DecodeKernelInfo* info) {
  constexpr int kD = PA_BF16_128_DEPTH, kD8 = PA_BF16_128_DEPTH_G8, kW = PA_BF16_128_WARPS;
  switch (head_dim * 100 + group) {
    case 6401: return fill<64, 1, 1, 4, 4, 3>(info);
    case 6402: return fill<64, 2, 1, 4, 4, 3>(info);
    case 6404: return fill<64, 4, 1, 4, 4, 3>(info);
    case 6408:
      if (PA_G8_MMA) return fill<64, 8, 1, PA_MMA_DEPTH, PA_MMA_WARPS, PA_MMA_MINCTAS, true>(info);
      return fill<64, 8, 2, 4, 4, 3>(info);
    case 12801: return fill<128, 1, 1, kD, kW, 3>(info);
    case 12802: return fill<128, 2, 1, kD, kW, 3>(info);
    case 12804: return fill<128, 4, 1, kD, kW, 3>(info);
    case 12808:
      if (PA_G8_MMA) return fill<128, 8, 1, PA_MMA_DEPTH, PA_MMA_WARPS, PA_MMA_MINCTAS, true>(info);
      return fill<128, 8, 2, kD8, kW, PA_BF16_128_MINCTAS_G8>(info);
    default: return false;
  }
}

}  // namespace pa
