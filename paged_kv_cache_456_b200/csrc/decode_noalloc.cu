// decode_noalloc.cu -- pa_decode_noalloc: decode attention whose scratch
// memory lives in a fixed array inside the library, so the caller never has
// to allocate a workspace.
//
// Who needs this: code that must not allocate device memory once it is
// running -- for instance an engine whose memory pool has already claimed
// the device for its KV cache, or a step loop that cannot accept the device
// synchronisation that cudaMalloc/cudaFree may cause -- and callers that
// simply have no allocator to hand (a C caller holding only raw pointers).
//
// The scratch is one file-scope __device__ array of PA_NOALLOC_SCRATCH_BYTES.
// Every GPU that loads this library holds that much memory until the process
// exits.  Host code must not pass the array's name to a kernel: on the host
// the name is only a stand-in, not a device address.  Its device address is
// looked up once per device with cudaGetSymbolAddress (see scratch_for) and
// that pointer is what the launch receives.
//
// Every call shares the one array and it keeps whatever the last call left
// there.  The part that must start at zero (the merge-pass header and the
// per-(sequence, KV head) piece counters) is cleared with cudaMemsetAsync on the caller's stream
// before each launch.  Calls whose work can overlap on the GPU (different
// streams, no ordering between them) race on the array.
#include <cmath>
#include <cstdint>
#include <initializer_list>
#include <mutex>

#include <cuda_runtime.h>

#include "paged_attention.h"
#include "pa_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[PA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up on
// the first call made with that device current.
pa_status scratch_for(void** ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return PA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *ptr = g_scratch_ptr[dev];
  return PA_OK;
}

}  // namespace

extern "C" pa_status pa_decode_noalloc(void* out, const void* q, const void* k_cache,
                                       const void* v_cache, const int32_t* block_tables,
                                       const int32_t* context_lens, int num_seqs,
                                       int num_q_heads, int num_kv_heads, int head_dim,
                                       int block_size, int max_blocks_per_seq, int num_blocks,
                                       int max_context_len, float scale, int partition_size,
                                       pa_dtype dtype, int32_t* err_flag, void* stream) {
  if (num_seqs == 0)
    return pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs,
                     num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                     num_blocks, max_context_len, scale, partition_size, dtype, nullptr, 0,
                     err_flag, stream);
  // the arguments pa_decode would reject are rejected here too, before the
  // memset below is enqueued, so a bad call leaves the stream untouched
  if (num_seqs < 0 || max_blocks_per_seq <= 0 || num_blocks <= 0 || block_size <= 0 ||
      !std::isfinite(scale) || !out || !q || !k_cache || !v_cache || !block_tables ||
      !context_lens)
    return PA_ERR_INVALID_ARG;
  for (const void* p : {static_cast<const void*>(out), q, k_cache, v_cache})
    if (reinterpret_cast<uintptr_t>(p) & 15u) return PA_ERR_INVALID_ARG;
  if (block_size != 16) return PA_ERR_UNSUPPORTED;
  size_t need = 0;
  pa_status st = pa_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                          max_context_len, partition_size, dtype, &need);
  if (st != PA_OK) return st;
  if (need > static_cast<size_t>(PA_NOALLOC_SCRATCH_BYTES)) return PA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if ((st = scratch_for(&scratch)) != PA_OK) return st;
  // the fields that must begin at zero sit at the start of the scratch
  const size_t zero = pa::decode_zero_prefix_bytes(num_seqs, num_kv_heads);
  if (cudaMemsetAsync(scratch, 0, zero, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return PA_ERR_CUDA;
  return pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs, num_q_heads,
                   num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
                   max_context_len, scale, partition_size, dtype, scratch,
                   static_cast<size_t>(PA_NOALLOC_SCRATCH_BYTES), err_flag, stream);
}
