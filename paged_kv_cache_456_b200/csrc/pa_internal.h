// pa_internal.h -- definitions shared by the library's translation units
// (not part of the public ABI, which is include/paged_attention.h).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda.h>  // CUtensorMap (a plain 128-byte descriptor; no driver call here)
#include <cuda_runtime.h>

namespace pa {

constexpr int kBlockSize = 16;            // token slots per KV block
constexpr float kRescaleThreshold = 8.f;  // log2 growth of the running max before o is rescaled

constexpr int kErrBlockId = 1;
constexpr int kErrContextLen = 2;
constexpr int kErrSlot = 4;
constexpr int kErrPair = 8;
constexpr int kErrTimeout = 16;
constexpr int kErrQuery = 32;
constexpr int kErrGroup = 64;

// Work schedule: the last 1/kTailDiv of the tiles is handed out at run time
// in chunks of kChunkTiles (0 = everything static).
#ifndef PA_TAIL_DIV
#define PA_TAIL_DIV 0
#endif
#ifndef PA_CHUNK_TILES
#define PA_CHUNK_TILES 2
#endif
constexpr int kTailDiv = PA_TAIL_DIV;
constexpr int kChunkTiles = PA_CHUNK_TILES;

__host__ __device__ inline long long chunk_tiles(int part_blocks) {
  return part_blocks > 0 && part_blocks < kChunkTiles ? part_blocks : kChunkTiles;
}
// tiles of the claimed tail; only used when every worker can get a chunk
__host__ __device__ inline long long tail_tiles(long long W, long long workers) {
  constexpr int div = kTailDiv > 0 ? kTailDiv : 1;
  return (kTailDiv > 0 && W / div >= workers) ? W / div : 0;
}

struct DecodeArgs {
  void* out;
  const void* q;
  const void* key;    // fused append: [num_seqs][num_kv_heads][head_dim] newest token of each
  const void* value;  // sequence (position context_lens[s] - 1), or null for plain decode
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_tables;
  const int32_t* context_lens;
  int num_seqs;
  int num_q_heads;
  int num_kv_heads;
  int max_blocks_per_seq;
  int num_blocks;
  int len_cap;       // longest valid context: min(max_context_len, max_blocks_per_seq * 16)
  int part_blocks;   // most blocks one partial covers (0 = balanced share)
  float scale_log2;  // scale * log2(e)
  int* counters;     // [num_seqs * num_kv_heads * 2] pieces finished per (item, head half),
                     // zero between calls
  int* heavy;        // [8]: items of many pieces listed for the merge pass, merge CTAs
                     // done, tail chunks claimed, decode workers done, items of few
                     // pieces listed (all zero between calls)
  int* heavy_list;   // [num_seqs * num_kv_heads] int4 records {seq * Hkv + kv head, first
                     // range, pieces, first piece's slot} of many-piece items
  int* light_list;   // the same for items of few pieces
  float* ws_o;       // [2 * ranges][G][head_dim] unnormalised partial outputs
  float2* ws_ml;     // [2 * ranges][G] (running max, sum) of each partial; sum < 0 = poisoned
  int32_t* err_flag;
  // several query tokens per sequence (null for decode): the kernel's
  // "sequences" are then the num_seqs query rows, each attending causally;
  // query_start[num_table_rows + 1] maps them to the block-table rows
  const int32_t* query_start;
  int num_table_rows;
  int num_query_rows;  // rows of q and out (several query tokens per sequence)
  // shared-prefix decode (all null otherwise): per sequence the number of
  // leading blocks the shared-prefix pass attended to (> 0; 0 or less: none),
  // and that pass's state per (sequence, query head): the unnormalised output
  // and (running max in log2 units, sum of weights).  The kernel then attends
  // to the remaining blocks only, starting from that state.
  const int32_t* pre_blocks;  // [num_seqs]
  const float* pre_o;         // [num_seqs][num_q_heads][head_dim]
  const float2* pre_ml;       // [num_seqs][num_q_heads]
  // tensor-core path only: the caches as 2-D tensors [num_blocks * Hkv * 16][head_dim]
  // read in boxes of 16 rows x 128 bytes with the 128-byte swizzle
  CUtensorMap tm_k;
  CUtensorMap tm_v;
};

// CUDA-core path: a split (seq, kv head) whose pieces x G exceed this is merged
// by the separate merge pass instead of by the warp of the decode kernel that
// finishes its last piece.  0 (the default, measured faster since the merge
// pass takes one warp per item): every split goes to the merge pass, and the
// decode kernel needs no fence or counter per piece.
#ifndef PA_FUSE_MAX_VALUES
#define PA_FUSE_MAX_VALUES 0
#endif
constexpr int kFuseMaxValues = PA_FUSE_MAX_VALUES;
constexpr int kMergeThreads = 256;
// Merge pass: an item of at most this many pieces is merged by one warp (all
// its heads); items with more pieces get a whole CTA per head.
constexpr int kWarpMergeMaxPieces = 8;

struct DecodeKernelInfo {
  const void* fn;   // the __global__ function
  const void* merge_fn;  // the merge pass for the same element type / shape
  int warps;        // warps per CTA
  int workers;      // work streams per CTA (warps / head split)
  int depth;        // ring slots per worker
  int cta_bytes;    // dynamic shared memory per CTA, without the per-sequence arrays
  bool tma;         // reads tiles through the tm_k / tm_v tensor maps
  int rows_per_item;  // query rows an item groups (several query tokens per sequence)
};

bool decode_kernel_bf16(int head_dim, int group, DecodeKernelInfo* info);
// The kernel for several query tokens per sequence when it differs from the
// decode one (false: use decode_kernel_*).
bool prefill_kernel_bf16(int head_dim, int group, DecodeKernelInfo* info);

// Bytes at the start of a decode workspace that must be zero when a call
// begins (the merge-pass header and the piece counters).
size_t decode_zero_prefix_bytes(int num_seqs, int num_kv_heads);
bool decode_kernel_f32(int head_dim, int group, DecodeKernelInfo* info);

// The shared-prefix pass of deduplicated decode (shared_prefix.cu).
struct SharedPrefixLaunch {
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_tables;
  const int32_t* context_lens;
  const int32_t* group_seqs;    // [num_listed] member sequences, group by group
  const int32_t* group_start;   // [num_groups + 1] offsets into group_seqs
  const int32_t* group_blocks;  // [num_groups] leading blocks the members share
  int num_groups;
  int num_listed;
  int num_seqs;
  int num_q_heads;
  int num_kv_heads;
  int head_dim;
  int max_blocks_per_seq;
  int num_blocks;
  int len_cap;
  float scale_log2;
  void* workspace;              // shared_prefix_workspace_bytes(...) bytes, zero on first use
  int32_t* err_flag;
  const CUtensorMap* tm_k;      // the caches' tensor maps (tensor-core pass)
  const CUtensorMap* tm_v;
  // outputs for the decode kernel (inside the workspace)
  int32_t* pre_blocks;
  float* pre_o;
  float2* pre_ml;
};
// Bytes of the pass's workspace region; 0 if the shape is unsupported.
size_t shared_prefix_workspace_bytes(int num_seqs, int num_listed, int num_q_heads,
                                     int head_dim, int max_blocks_per_seq);
// Fills pre_blocks / pre_o / pre_ml of `l` from its workspace and launches the
// pass; returns cudaSuccess or the launch error.
cudaError_t launch_shared_prefix(SharedPrefixLaunch& l, int num_sms, cudaStream_t stream);

// A cache as the 2-D bf16 tensor [num_blocks * num_kv_heads * 16][head_dim],
// read in boxes of 16 rows x 64 elements with the 128-byte swizzle (abi.cu).
bool encode_cache_map(CUtensorMap* map, const void* base, long long rows, int head_dim);
// The prefill output [rows][num_q_heads][head_dim] bf16 as a 3-D tensor
// (head_dim, query heads, rows) with boxes of 64 x group x 128/group, 128-byte
// swizzle: the tensor-core kernel's epilogue stores a column tile through it.
bool encode_prefill_out_map(CUtensorMap* map, void* out, int num_query_rows, int num_q_heads,
                            int head_dim, int group);

// ---- tensor-core attention of many query columns (tc_attention.cu) ----------
// Several query tokens per sequence: one column per (query row, query head),
// 128 columns per MMA tile, on the tcgen05 tensor cores (bf16).
struct TcPrefillLaunch {
  const void* q;
  void* out;
  const int32_t* block_tables;
  const int32_t* context_lens;
  const int32_t* query_start;
  int num_seqs;        // block-table rows
  int num_query_rows;  // rows of q and out
  int num_q_heads;
  int num_kv_heads;
  int head_dim;
  int max_blocks_per_seq;
  int num_blocks;
  int len_cap;
  float scale_log2;
  void* workspace;     // tc_prefill_workspace_bytes(...) bytes (no zeroing needed)
  int32_t* err_flag;
  const CUtensorMap* tm_k;
  const CUtensorMap* tm_v;
  const CUtensorMap* tm_out;  // the output for the epilogue's tensor stores (null: plain stores)
};
bool tc_prefill_supported(int head_dim, int group);
size_t tc_prefill_workspace_bytes(int num_seqs, int num_query_tokens, int num_q_heads,
                                  int num_kv_heads);
int tc_launch_smem(int head_dim);
constexpr int kTcWarps = 10;
cudaError_t launch_tc_prefill(const TcPrefillLaunch& l, int num_sms, cudaStream_t stream);

// The shared-prefix pass on the tcgen05 tensor cores: (member, query head)
// columns of a group, 128 per tile, over ranges of the group's shared blocks.
struct TcSharedLaunch {
  const void* q;
  const int32_t* block_tables;
  const int32_t* context_lens;
  const int32_t* group_seqs;
  const int32_t* group_start;
  const int32_t* group_blocks;
  int num_groups;
  int num_listed;
  int num_seqs;
  int num_q_heads;
  int num_kv_heads;
  int head_dim;
  int max_blocks_per_seq;
  int num_blocks;
  int len_cap;
  int max_ranges;      // ranges the partial arrays hold per column
  float scale_log2;
  int* unit_start;     // [num_groups + 1]
  int4* units;         // [max_units][2] work-unit records
  int max_units;
  int* group_ranges;   // [num_groups] ranges of each group's shared blocks (plan kernel)
  int* claim;          // [num_seqs], zeroed before the pass
  float2* part_ml;
  float* part_o;
  float2* pre_ml;
  float* pre_o;
  int32_t* err_flag;
  const CUtensorMap* tm_k;
  const CUtensorMap* tm_v;
};
bool tc_shared_prefix_supported(int head_dim, int group);
cudaError_t launch_tc_shared_prefix(const TcSharedLaunch& l, int num_sms, cudaStream_t stream);

}  // namespace pa
