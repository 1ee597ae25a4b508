// cache_ops.cu -- the two cache-maintenance kernels around decode.
//
// Slot write ("reshape_and_cache"): each step's new key/value rows go to the
// cache slot slot_mapping[t] (the cache "grows ... as the model generates new
// tokens": "vLLM Solved the Wrong Bottleneck...", section "Paged Attention").
// Block copy-on-write ("copy_blocks"): a shared block that must diverge is
// copied whole to a fresh block (day-9 post, section "Idea 1: PagedAttention").
//
// Both are pure byte copies, bandwidth-bound and tiny next to decode: 16-byte
// vector loads and stores, consecutive threads on consecutive 16-byte chunks
// of a row (coalesced), a grid-stride loop sized to the SM count.  Indices
// read from device memory are range-checked before any address is formed;
// a bad one skips its item and sets a bit in err_flag.
#include <cstdint>
#include <cuda_runtime.h>

#include "pa_internal.h"

namespace pa {

__global__ void __launch_bounds__(256)
reshape_and_cache_kernel(const uint4* __restrict__ key, const uint4* __restrict__ value,
                         uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                         const int64_t* __restrict__ slot_mapping, int num_tokens,
                         int num_kv_heads, int chunks_per_row, int block_size,
                         long long num_slots, int32_t* err_flag) {
  const long long per_token = static_cast<long long>(num_kv_heads) * chunks_per_row;
  const long long total = per_token * num_tokens;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long t = i / per_token;
    const long long rem = i - t * per_token;
    const long long slot = slot_mapping[t];
    if (slot < 0) continue;  // padding token
    if (slot >= num_slots) {
      if (rem == 0 && err_flag) atomicOr(err_flag, kErrSlot);
      continue;
    }
    const long long h = rem / chunks_per_row;
    const long long c = rem - h * chunks_per_row;
    const long long blk = slot / block_size;
    const long long off = slot - blk * block_size;
    const long long dst = ((blk * num_kv_heads + h) * block_size + off) * chunks_per_row + c;
    k_cache[dst] = key[i];
    v_cache[dst] = value[i];
  }
}

__global__ void __launch_bounds__(256)
copy_blocks_kernel(uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                   const int32_t* __restrict__ block_mapping, int num_pairs,
                   long long chunks_per_block, int num_blocks, int32_t* err_flag) {
  for (int p = blockIdx.y; p < num_pairs; p += gridDim.y) {
    const int src = block_mapping[2 * p];
    const int dst = block_mapping[2 * p + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks || src == dst) {
      if (blockIdx.x == 0 && threadIdx.x == 0 && err_flag) atomicOr(err_flag, kErrPair);
      continue;
    }
    const uint4* ks = k_cache + static_cast<long long>(src) * chunks_per_block;
    const uint4* vs = v_cache + static_cast<long long>(src) * chunks_per_block;
    uint4* kd = k_cache + static_cast<long long>(dst) * chunks_per_block;
    uint4* vd = v_cache + static_cast<long long>(dst) * chunks_per_block;
    for (long long c = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
         c < chunks_per_block; c += static_cast<long long>(gridDim.x) * blockDim.x) {
      const uint4 a = ks[c];
      const uint4 b = vs[c];
      kd[c] = a;
      vd[c] = b;
    }
  }
}

cudaError_t launch_reshape_and_cache(const void* key, const void* value, void* k_cache,
                                     void* v_cache, const int64_t* slot_mapping, int num_tokens,
                                     int num_kv_heads, int row_bytes, int block_size,
                                     long long num_slots, int32_t* err_flag, int num_sms,
                                     cudaStream_t stream) {
  const int chunks_per_row = row_bytes / 16;
  const long long total = static_cast<long long>(num_tokens) * num_kv_heads * chunks_per_row;
  const long long want = (total + 255) / 256;
  const int grid = static_cast<int>(want < 8LL * num_sms ? want : 8LL * num_sms);
  reshape_and_cache_kernel<<<grid, 256, 0, stream>>>(
      static_cast<const uint4*>(key), static_cast<const uint4*>(value),
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), slot_mapping, num_tokens,
      num_kv_heads, chunks_per_row, block_size, num_slots, err_flag);
  return cudaGetLastError();
}

cudaError_t launch_copy_blocks(void* k_cache, void* v_cache, const int32_t* block_mapping,
                               int num_pairs, long long block_bytes, int num_blocks,
                               int32_t* err_flag, int num_sms, cudaStream_t stream) {
  const long long chunks = block_bytes / 16;
  long long gx = (chunks + 255) / 256;
  if (gx > 64) gx = 64;
  const int gy = num_pairs < 65535 ? num_pairs : 65535;
  (void)num_sms;
  copy_blocks_kernel<<<dim3(static_cast<unsigned>(gx), gy), 256, 0, stream>>>(
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), block_mapping, num_pairs,
      chunks, num_blocks, err_flag);
  return cudaGetLastError();
}

}  // namespace pa
