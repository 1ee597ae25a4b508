// abi.cu -- the extern "C" entry points of libpa.so (include/paged_attention.h):
// argument validation on the host, launch planning, launches.  No entry point
// allocates memory or synchronises; everything after validation is
// asynchronous on the caller's stream.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "paged_attention.h"
#include "pa_internal.h"

namespace pa {
cudaError_t launch_reshape_and_cache(const void* key, const void* value, void* k_cache,
                                     void* v_cache, const int64_t* slot_mapping, int num_tokens,
                                     int num_kv_heads, int row_bytes, int block_size,
                                     long long num_slots, int32_t* err_flag, int num_sms,
                                     cudaStream_t stream);
cudaError_t launch_copy_blocks(void* k_cache, void* v_cache, const int32_t* block_mapping,
                               int num_pairs, long long block_bytes, int num_blocks,
                               int32_t* err_flag, int num_sms, cudaStream_t stream);
}  // namespace pa

static_assert(pa::kErrBlockId == PA_ERRBIT_BLOCK_ID, "error bit mismatch");
static_assert(pa::kErrContextLen == PA_ERRBIT_CONTEXT_LEN, "error bit mismatch");
static_assert(pa::kErrSlot == PA_ERRBIT_SLOT, "error bit mismatch");
static_assert(pa::kErrPair == PA_ERRBIT_PAIR, "error bit mismatch");
static_assert(pa::kErrTimeout == PA_ERRBIT_TIMEOUT, "error bit mismatch");
static_assert(pa::kErrQuery == PA_ERRBIT_QUERY, "error bit mismatch");
static_assert(pa::kErrGroup == PA_ERRBIT_GROUP, "error bit mismatch");

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int sms = 0;
  int smem_optin = 0;
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
// (device, kernel, dynamic smem) -> resident CTAs per SM
std::map<std::tuple<int, const void*, size_t>, int> g_occupancy;
// (device, kernel) -> the dynamic smem limit set on it so far; it only grows,
// so every size met before stays launchable
std::map<std::pair<int, const void*>, size_t> g_smem_limit;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elem_bytes(pa_dtype dt) { return dt == PA_BF16 ? 2 : 4; }

bool valid_dtype(pa_dtype dt) { return dt == PA_F32 || dt == PA_BF16; }

pa_status device_info(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess)
      return PA_ERR_CUDA;
    d.ready = true;
  }
  *out = d;
  return PA_OK;
}

struct DecodePlan {
  pa::DecodeKernelInfo kernel{};
  int grid = 0;
  size_t smem = 0;
  long long ranges = 0;      // most ranges the device can form
  int sms = 0;
  // workspace layout; everything before zero_bytes must be zero on entry
  size_t heavy_off = 0;      // [8] ints: merge-pass counts, merge CTAs done, chunks, workers done
  size_t list_off = 0;       // 2 x [S*Hkv] int4 records: items for the merge pass (many, few pieces)
  size_t counters_off = 0;   // [S*Hkv*2] ints
  size_t zero_bytes = 0;
  size_t o_off = 0;
  size_t ml_off = 0;
  size_t ws_bytes = 0;
};

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

pa_status encode_cache_map(CUtensorMap* map, const void* base, long long rows, int head_dim) {
  return pa::encode_cache_map(map, base, rows, head_dim) ? PA_OK : PA_ERR_CUDA;
}

pa_status occupancy(const pa::DecodeKernelInfo& k, size_t smem, int* occ) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  size_t& limit = g_smem_limit[std::make_pair(dev, k.fn)];
  if (smem > limit) {
    if (cudaFuncSetAttribute(k.fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess ||
        cudaFuncSetAttribute(k.fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess) {
      cudaGetLastError();  // leave no launch-time error behind for the caller
      return PA_ERR_CUDA;
    }
    limit = smem;
  }
  const auto key = std::make_tuple(dev, k.fn, smem);
  auto it = g_occupancy.find(key);
  if (it != g_occupancy.end()) {
    *occ = it->second;
    return PA_OK;
  }
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(occ, k.fn, k.warps * 32, smem) != cudaSuccess) {
    cudaGetLastError();
    return PA_ERR_CUDA;
  }
  g_occupancy[key] = *occ;
  return PA_OK;
}

// Shape checks shared by the decode entry points (no device needed).
pa_status check_decode_shape(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                             int max_context_len, int partition_size, pa_dtype dtype) {
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
      max_context_len < 0 || partition_size < 0 || !valid_dtype(dtype))
    return PA_ERR_INVALID_ARG;
  if (num_q_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
  if (partition_size % pa::kBlockSize != 0) return PA_ERR_INVALID_ARG;
  const int group = num_q_heads / num_kv_heads;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (group != 1 && group != 2 && group != 4 && group != 8) return PA_ERR_UNSUPPORTED;
  if (num_kv_heads > 0xffff) return PA_ERR_UNSUPPORTED;
  return PA_OK;
}

// table_rows >= 0: several query tokens per sequence; num_seqs counts query
// rows and the kernel also keeps their table rows and query_start on chip.
pa_status make_plan(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                    int max_context_len, int partition_size, pa_dtype dtype, DecodePlan* p,
                    int table_rows = -1) {
  pa_status st = check_decode_shape(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                    max_context_len, partition_size, dtype);
  if (st != PA_OK) return st;
  const int group = num_q_heads / num_kv_heads;
  // several query tokens per sequence: bf16 groups of 8 heads have their own
  // kernel (groups of query rows per item); everything else shares decode's
  bool found = table_rows >= 0 && dtype == PA_BF16 &&
               pa::prefill_kernel_bf16(head_dim, group, &p->kernel);
  if (!found)
    found = dtype == PA_BF16 ? pa::decode_kernel_bf16(head_dim, group, &p->kernel)
                             : pa::decode_kernel_f32(head_dim, group, &p->kernel);
  if (!found) return PA_ERR_UNSUPPORTED;
  const int columns = group * p->kernel.rows_per_item;  // partial columns per item
  // tiles: must fit the kernel's 32-bit tile counter
  const long long blocks_max = (static_cast<long long>(max_context_len) + pa::kBlockSize - 1) /
                               pa::kBlockSize;
  const long long tiles_max = static_cast<long long>(num_seqs) * num_kv_heads * blocks_max;
  if (tiles_max >= (1LL << 31)) return PA_ERR_UNSUPPORTED;

  DeviceInfo dev;
  if ((st = device_info(&dev)) != PA_OK) return st;
  size_t seq_ints = 2 * static_cast<size_t>(num_seqs) + 1;  // item starts, lengths
  if (table_rows >= 0) {
    seq_ints += static_cast<size_t>(num_seqs) + table_rows + 1;  // table rows, query_start
    if (p->kernel.rows_per_item > 1)
      seq_ints += static_cast<size_t>(num_seqs) + table_rows + 1;  // group rows, group starts
  }
  const size_t seq_bytes = round_up(seq_ints * sizeof(int), 16);
  p->smem = static_cast<size_t>(p->kernel.cta_bytes) + seq_bytes;
  if (p->smem > static_cast<size_t>(dev.smem_optin)) return PA_ERR_UNSUPPORTED;
  int occ = 0;
  if ((st = occupancy(p->kernel, p->smem, &occ)) != PA_OK) return st;
  if (occ < 1) return PA_ERR_UNSUPPORTED;
  const long long resident = static_cast<long long>(dev.sms) * occ;
  const long long by_work = (tiles_max + p->kernel.workers - 1) / p->kernel.workers;
  p->grid = static_cast<int>(by_work < resident ? (by_work > 0 ? by_work : 1) : resident);
  const long long workers = static_cast<long long>(p->grid) * p->kernel.workers;
  // static ranges (at most) plus tail chunks (at most), as the kernel cuts them
  long long ranges = workers;
  if (partition_size > 0) {
    const long long per = workers * (partition_size / pa::kBlockSize);
    const long long rounds = (tiles_max + per - 1) / per;
    ranges = workers * (rounds > 1 ? rounds : 1);
  }
  if (ranges > tiles_max) ranges = tiles_max > 0 ? tiles_max : 1;
  const long long cs = pa::chunk_tiles(partition_size / pa::kBlockSize);
  ranges += (pa::tail_tiles(tiles_max, workers) + cs - 1) / cs + 1;
  p->ranges = ranges;
  p->sms = dev.sms;
  const size_t slots = 2 * static_cast<size_t>(ranges);
  const size_t items = static_cast<size_t>(num_seqs) * num_kv_heads;
  // zero-on-entry fields first: the merge pass's count/done pair, the piece counters
  p->heavy_off = 0;
  p->counters_off = 8 * sizeof(int);
  p->zero_bytes = pa::decode_zero_prefix_bytes(num_seqs, num_kv_heads);
  p->list_off = round_up(p->zero_bytes, 16);  // (int4 records)
  p->o_off = round_up(p->list_off + 2 * items * 4 * sizeof(int), 256);
  p->ml_off = round_up(p->o_off + slots * columns * head_dim * sizeof(float), 256);
  p->ws_bytes = round_up(p->ml_off + slots * columns * 2 * sizeof(float), 256);
  return PA_OK;
}

}  // namespace

// A cache as the 2-D bf16 tensor [rows][head_dim] read by the tensor-core
// paths in boxes of 16 rows x 64 elements (128 bytes) with the 128-byte
// swizzle.  The encoder is a host-side driver routine, looked up once.
bool pa::encode_cache_map(CUtensorMap* map, const void* base, long long rows, int head_dim) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
      if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                           &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn) {
        cudaGetLastError();
        return false;
      }
      encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
  }
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(head_dim) * 2};
  const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(pa::kBlockSize)};
  const cuuint32_t elem_strides[2] = {1, 1};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
                            dims, strides, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool pa::encode_prefill_out_map(CUtensorMap* map, void* out, int num_query_rows,
                                int num_q_heads, int head_dim, int group) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
      if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                           &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn) {
        cudaGetLastError();
        return false;
      }
      encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
  }
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(num_q_heads),
                              static_cast<cuuint64_t>(num_query_rows)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * 2,
                                 static_cast<cuuint64_t>(num_q_heads) * head_dim * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(group), static_cast<cuuint32_t>(128 / group)};
  const cuuint32_t elem_strides[3] = {1, 1, 1};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, out, dims, strides, box,
                            elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

size_t pa::decode_zero_prefix_bytes(int num_seqs, int num_kv_heads) {
  return 8 * sizeof(int) + 2 * static_cast<size_t>(num_seqs) * num_kv_heads * sizeof(int);
}

extern "C" {

const char* pa_status_str(pa_status status) {
  switch (status) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
    case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE";
    case PA_ERR_CUDA: return "PA_ERR_CUDA";
  }
  return "PA_ERR_UNKNOWN";
}

pa_status pa_decode_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                   int max_context_len, int partition_size, pa_dtype dtype,
                                   size_t* bytes) {
  if (!bytes) return PA_ERR_INVALID_ARG;
  DecodePlan p;
  const pa_status st = make_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                                 partition_size, dtype, &p);
  if (st != PA_OK) return st;
  *bytes = p.ws_bytes;
  return PA_OK;
}

// Items of a call with several query tokens per sequence: one per query
// row, or -- with the grouping kernel -- at most ceil((T + (NR-1) R) / NR)
// groups of NR rows (sum over sequences of ceil(Q_s / NR)).
static int prefill_items(int num_seqs, int num_query_tokens, int num_q_heads, int num_kv_heads,
                  int head_dim, pa_dtype dtype) {
  pa::DecodeKernelInfo k{};
  if (dtype != PA_BF16 || num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0 ||
      !pa::prefill_kernel_bf16(head_dim, num_q_heads / num_kv_heads, &k) || k.rows_per_item <= 1)
    return num_query_tokens;
  const long long nr = k.rows_per_item;
  const long long items = (num_query_tokens + (nr - 1) * static_cast<long long>(num_seqs) + nr - 1) / nr;
  return static_cast<int>(items < num_query_tokens ? items : num_query_tokens);
}

// Several query tokens per sequence go to the tcgen05 kernel (bf16 caches)
// unless the library is built with PA_PREFILL_TC=0; fp32 caches always take
// the decode kernel with query rows as items.
#ifndef PA_PREFILL_TC
#define PA_PREFILL_TC 1
#endif
// (the tensor-core kernel numbers its pairs of 128-column tiles in 16 bits)
static bool prefill_on_tensor_cores(int num_query_tokens, int num_q_heads, int num_kv_heads,
                                    int head_dim, pa_dtype dtype) {
  return PA_PREFILL_TC && dtype == PA_BF16 && num_kv_heads > 0 && num_q_heads > 0 &&
         num_q_heads % num_kv_heads == 0 &&
         static_cast<long long>(num_query_tokens) * (num_q_heads / num_kv_heads) < (1LL << 24) &&
         pa::tc_prefill_supported(head_dim, num_q_heads / num_kv_heads);
}

pa_status pa_prefill_workspace_size(int num_seqs, int num_query_tokens, int num_q_heads,
                                    int num_kv_heads, int head_dim, int max_context_len,
                                    int partition_size, pa_dtype dtype, size_t* bytes) {
  if (!bytes || num_seqs < 0 || num_query_tokens < 0) return PA_ERR_INVALID_ARG;
  if (prefill_on_tensor_cores(num_query_tokens, num_q_heads, num_kv_heads, head_dim, dtype)) {
    const pa_status st = check_decode_shape(num_query_tokens, num_q_heads, num_kv_heads, head_dim,
                                            max_context_len, partition_size, dtype);
    if (st != PA_OK) return st;
    *bytes = round_up(pa::tc_prefill_workspace_bytes(num_seqs, num_query_tokens, num_q_heads,
                                                     num_kv_heads),
                      256);
    return PA_OK;
  }
  DecodePlan p;
  const int items = prefill_items(num_seqs, num_query_tokens, num_q_heads, num_kv_heads,
                                  head_dim, dtype);
  const pa_status st = make_plan(items, num_q_heads, num_kv_heads, head_dim, max_context_len,
                                 partition_size, dtype, &p, num_seqs > 0 ? num_seqs : 1);
  if (st != PA_OK) return st;
  *bytes = p.ws_bytes;
  return PA_OK;
}

pa_status pa_decode_workspace_init(void* workspace, size_t bytes, void* stream) {
  if (!workspace && bytes) return PA_ERR_INVALID_ARG;
  if (!bytes) return PA_OK;
  return cudaMemsetAsync(workspace, 0, bytes, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? PA_OK
             : PA_ERR_CUDA;
}

pa_status pa_decode_launch_config(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                  int max_context_len, int partition_size, pa_dtype dtype,
                                  int* grid, int* warps_per_cta, int* pipeline_depth,
                                  int* smem_bytes) {
  DecodePlan p;
  const pa_status st = make_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                                 partition_size, dtype, &p);
  if (st != PA_OK) return st;
  if (grid) *grid = p.grid;
  if (warps_per_cta) *warps_per_cta = p.kernel.warps;
  if (pipeline_depth) *pipeline_depth = p.kernel.depth;
  if (smem_bytes) *smem_bytes = static_cast<int>(p.smem);
  return PA_OK;
}

pa_status pa_prefill_launch_config(int num_seqs, int num_query_tokens, int num_q_heads,
                                   int num_kv_heads, int head_dim, int max_context_len,
                                   int partition_size, pa_dtype dtype, int* grid,
                                   int* warps_per_cta, int* pipeline_depth, int* smem_bytes) {
  if (num_seqs < 0 || num_query_tokens < 0) return PA_ERR_INVALID_ARG;
  if (prefill_on_tensor_cores(num_query_tokens, num_q_heads, num_kv_heads, head_dim, dtype)) {
    pa_status st = check_decode_shape(num_query_tokens, num_q_heads, num_kv_heads, head_dim,
                                      max_context_len, partition_size, dtype);
    if (st != PA_OK) return st;
    DeviceInfo dev;
    if ((st = device_info(&dev)) != PA_OK) return st;
    if (grid) *grid = dev.sms;
    if (warps_per_cta) *warps_per_cta = pa::kTcWarps;
    if (pipeline_depth) *pipeline_depth = 3;
    if (smem_bytes) *smem_bytes = pa::tc_launch_smem(head_dim);
    return PA_OK;
  }
  DecodePlan p;
  const int items = prefill_items(num_seqs, num_query_tokens, num_q_heads, num_kv_heads,
                                  head_dim, dtype);
  const pa_status st = make_plan(items, num_q_heads, num_kv_heads, head_dim, max_context_len,
                                 partition_size, dtype, &p, num_seqs > 0 ? num_seqs : 1);
  if (st != PA_OK) return st;
  if (grid) *grid = p.grid;
  if (warps_per_cta) *warps_per_cta = p.kernel.warps;
  if (pipeline_depth) *pipeline_depth = p.kernel.depth;
  if (smem_bytes) *smem_bytes = static_cast<int>(p.smem);
  return PA_OK;
}

namespace {

// pa_decode and pa_decode_append: key/value null = plain decode.
// query_start non-null: num_seqs counts query rows of table_rows sequences.
pa_status decode_impl(void* out, const void* q, const void* key, const void* value,
                      const void* k_cache, const void* v_cache, const int32_t* block_tables,
                      const int32_t* context_lens, int num_seqs, int num_q_heads,
                      int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                      int num_blocks, int max_context_len, float scale, int partition_size,
                      pa_dtype dtype, void* workspace, size_t workspace_bytes,
                      int32_t* err_flag, void* stream, const int32_t* query_start = nullptr,
                      int table_rows = -1, int query_rows = 0,
                      const pa::SharedPrefixLaunch* pre = nullptr) {
  pa_status st = check_decode_shape(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                    max_context_len, partition_size, dtype);
  if (st != PA_OK) return st;
  if (max_blocks_per_seq <= 0 || num_blocks <= 0 || block_size <= 0 || !std::isfinite(scale))
    return PA_ERR_INVALID_ARG;
  if (block_size != pa::kBlockSize) return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID_ARG;
  if (query_start && table_rows <= 0) return PA_ERR_INVALID_ARG;
  if (static_cast<long long>(num_seqs) * num_kv_heads * max_blocks_per_seq >= (1LL << 31))
    return PA_ERR_UNSUPPORTED;
  DecodePlan p;
  if ((st = make_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                      partition_size, dtype, &p, query_start ? table_rows : -1)) != PA_OK)
    return st;
  if (!workspace || workspace_bytes < p.ws_bytes || !aligned16(workspace))
    return PA_ERR_WORKSPACE;

  pa::DecodeArgs args;
  args.out = out;
  args.q = q;
  args.key = key;
  args.value = value;
  args.k_cache = k_cache;
  args.v_cache = v_cache;
  args.block_tables = block_tables;
  args.context_lens = context_lens;
  args.num_seqs = num_seqs;
  args.num_q_heads = num_q_heads;
  args.num_kv_heads = num_kv_heads;
  args.max_blocks_per_seq = max_blocks_per_seq;
  args.num_blocks = num_blocks;
  const long long cap = static_cast<long long>(max_blocks_per_seq) * pa::kBlockSize;
  args.len_cap = static_cast<int>(max_context_len < cap ? max_context_len : cap);
  args.part_blocks = partition_size / pa::kBlockSize;
  args.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  char* ws = static_cast<char*>(workspace);
  args.counters = reinterpret_cast<int*>(ws + p.counters_off);
  args.heavy = reinterpret_cast<int*>(ws + p.heavy_off);
  args.heavy_list = reinterpret_cast<int*>(ws + p.list_off);
  args.light_list = args.heavy_list + 4 * static_cast<size_t>(num_seqs) * num_kv_heads;
  args.ws_o = reinterpret_cast<float*>(ws + p.o_off);
  args.ws_ml = reinterpret_cast<float2*>(ws + p.ml_off);
  args.err_flag = err_flag;
  args.query_start = query_start;
  args.num_table_rows = query_start ? table_rows : num_seqs;
  args.num_query_rows = query_start ? query_rows : num_seqs;
  args.pre_blocks = pre ? pre->pre_blocks : nullptr;
  args.pre_o = pre ? pre->pre_o : nullptr;
  args.pre_ml = pre ? pre->pre_ml : nullptr;
  if (p.kernel.tma) {
    // tile coordinates are 32-bit: row (block * Hkv + kv head) * 16 of the 2-D view
    const long long rows = static_cast<long long>(num_blocks) * num_kv_heads * pa::kBlockSize;
    if (rows >= (1LL << 31)) return PA_ERR_UNSUPPORTED;
    if ((st = encode_cache_map(&args.tm_k, k_cache, rows, head_dim)) != PA_OK ||
        (st = encode_cache_map(&args.tm_v, v_cache, rows, head_dim)) != PA_OK)
      return st;
  }

  void* params[] = {&args};
  cudaStream_t st_ = static_cast<cudaStream_t>(stream);
  if (cudaLaunchKernel(p.kernel.fn, dim3(p.grid), dim3(p.kernel.warps * 32), params, p.smem,
                       st_) != cudaSuccess) {
    cudaGetLastError();  // a refused launch is reported here, not left for the caller
    return PA_ERR_CUDA;
  }
  // merge pass for the split items, launched behind the decode kernel with
  // programmatic dependent launch (it waits for the decode grid)
  int workers = p.grid * p.kernel.workers;
  void* mparams[] = {&args, &workers};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * p.sms);
  cfg.blockDim = dim3(pa::kMergeThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st_;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelExC(&cfg, p.kernel.merge_fn, mparams) != cudaSuccess) {
    cudaGetLastError();
    return PA_ERR_CUDA;
  }
  return PA_OK;
}

}  // namespace

pa_status pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
                    int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                    int max_blocks_per_seq, int num_blocks, int max_context_len, float scale,
                    int partition_size, pa_dtype dtype, void* workspace, size_t workspace_bytes,
                    int32_t* err_flag, void* stream) {
  return decode_impl(out, q, nullptr, nullptr, k_cache, v_cache, block_tables, context_lens,
                     num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                     max_blocks_per_seq, num_blocks, max_context_len, scale, partition_size,
                     dtype, workspace, workspace_bytes, err_flag, stream);
}

pa_status pa_decode_append(void* out, const void* q, const void* key, const void* value,
                           void* k_cache, void* v_cache, const int32_t* block_tables,
                           const int32_t* context_lens, int num_seqs, int num_q_heads,
                           int num_kv_heads, int head_dim, int block_size,
                           int max_blocks_per_seq, int num_blocks, int max_context_len,
                           float scale, int partition_size, pa_dtype dtype, void* workspace,
                           size_t workspace_bytes, int32_t* err_flag, void* stream) {
  if (num_seqs > 0 && (!key || !value || !aligned16(key) || !aligned16(value)))
    return PA_ERR_INVALID_ARG;
  return decode_impl(out, q, key, value, k_cache, v_cache, block_tables, context_lens, num_seqs,
                     num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                     num_blocks, max_context_len, scale, partition_size, dtype, workspace,
                     workspace_bytes, err_flag, stream);
}

pa_status pa_prefill(void* out, const void* q, const void* k_cache, const void* v_cache,
                     const int32_t* block_tables, const int32_t* context_lens,
                     const int32_t* query_start, int num_seqs, int num_query_tokens,
                     int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                     int max_blocks_per_seq, int num_blocks, int max_context_len, float scale,
                     int partition_size, pa_dtype dtype, void* workspace,
                     size_t workspace_bytes, int32_t* err_flag, void* stream) {
  if (num_seqs < 0 || num_query_tokens < 0) return PA_ERR_INVALID_ARG;
  if (num_query_tokens == 0) return PA_OK;
  if (num_seqs == 0 || !query_start) return PA_ERR_INVALID_ARG;
  if (prefill_on_tensor_cores(num_query_tokens, num_q_heads, num_kv_heads, head_dim, dtype)) {
    pa_status st = check_decode_shape(num_query_tokens, num_q_heads, num_kv_heads, head_dim,
                                      max_context_len, partition_size, dtype);
    if (st != PA_OK) return st;
    if (max_blocks_per_seq <= 0 || num_blocks <= 0 || block_size <= 0 || !std::isfinite(scale))
      return PA_ERR_INVALID_ARG;
    if (block_size != pa::kBlockSize) return PA_ERR_UNSUPPORTED;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
      return PA_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
      return PA_ERR_INVALID_ARG;
    const long long rows = static_cast<long long>(num_blocks) * num_kv_heads * pa::kBlockSize;
    if (rows + pa::kBlockSize >= (1LL << 31)) return PA_ERR_UNSUPPORTED;
    if (!workspace ||
        workspace_bytes < pa::tc_prefill_workspace_bytes(num_seqs, num_query_tokens,
                                                          num_q_heads, num_kv_heads) ||
        !aligned16(workspace))
      return PA_ERR_WORKSPACE;
    DeviceInfo dev;
    if ((st = device_info(&dev)) != PA_OK) return st;
    if (static_cast<size_t>(pa::tc_launch_smem(head_dim)) > static_cast<size_t>(dev.smem_optin))
      return PA_ERR_UNSUPPORTED;
    CUtensorMap tk, tv;
    if ((st = encode_cache_map(&tk, k_cache, rows, head_dim)) != PA_OK ||
        (st = encode_cache_map(&tv, v_cache, rows, head_dim)) != PA_OK)
      return st;
    pa::TcPrefillLaunch l{};
    l.q = q;
    l.out = out;
    l.block_tables = block_tables;
    l.context_lens = context_lens;
    l.query_start = query_start;
    l.num_seqs = num_seqs;
    l.num_query_rows = num_query_tokens;
    l.num_q_heads = num_q_heads;
    l.num_kv_heads = num_kv_heads;
    l.head_dim = head_dim;
    l.max_blocks_per_seq = max_blocks_per_seq;
    l.num_blocks = num_blocks;
    const long long cap = static_cast<long long>(max_blocks_per_seq) * pa::kBlockSize;
    l.len_cap = static_cast<int>(max_context_len < cap ? max_context_len : cap);
    l.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    l.workspace = workspace;
    l.err_flag = err_flag;
    l.tm_k = &tk;
    l.tm_v = &tv;
    CUtensorMap to;
    l.tm_out = pa::encode_prefill_out_map(&to, out, num_query_tokens, num_q_heads, head_dim,
                                          num_q_heads / num_kv_heads)
                   ? &to
                   : nullptr;
    if (pa::launch_tc_prefill(l, dev.sms, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
      cudaGetLastError();
      return PA_ERR_CUDA;
    }
    return PA_OK;
  }
  const int items = prefill_items(num_seqs, num_query_tokens, num_q_heads, num_kv_heads,
                                  head_dim, dtype);
  return decode_impl(out, q, nullptr, nullptr, k_cache, v_cache, block_tables, context_lens,
                     items, num_q_heads, num_kv_heads, head_dim, block_size,
                     max_blocks_per_seq, num_blocks, max_context_len, scale, partition_size,
                     dtype, workspace, workspace_bytes, err_flag, stream, query_start, num_seqs,
                     num_query_tokens);
}

pa_status pa_shared_prefix_workspace_size(int num_seqs, int num_listed, int num_q_heads,
                                          int num_kv_heads, int head_dim,
                                          int max_blocks_per_seq, int max_context_len,
                                          int partition_size, pa_dtype dtype, size_t* bytes) {
  if (!bytes || num_listed < 0 || max_blocks_per_seq <= 0) return PA_ERR_INVALID_ARG;
  if (dtype != PA_BF16) return dtype == PA_F32 ? PA_ERR_UNSUPPORTED : PA_ERR_INVALID_ARG;
  DecodePlan p;
  const pa_status st = make_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                                 partition_size, dtype, &p);
  if (st != PA_OK) return st;
  const size_t extra = pa::shared_prefix_workspace_bytes(num_seqs, num_listed, num_q_heads,
                                                         head_dim, max_blocks_per_seq);
  if (extra == 0) return PA_ERR_UNSUPPORTED;
  *bytes = round_up(p.ws_bytes, 256) + extra;
  return PA_OK;
}

pa_status pa_decode_shared_prefix(void* out, const void* q, const void* key, const void* value,
                                  void* k_cache, void* v_cache, const int32_t* block_tables,
                                  const int32_t* context_lens, const int32_t* group_seqs,
                                  const int32_t* group_start, const int32_t* group_blocks,
                                  int num_groups, int num_listed, int num_seqs, int num_q_heads,
                                  int num_kv_heads, int head_dim, int block_size,
                                  int max_blocks_per_seq, int num_blocks, int max_context_len,
                                  float scale, int partition_size, pa_dtype dtype,
                                  void* workspace, size_t workspace_bytes, int32_t* err_flag,
                                  void* stream) {
  pa_status st = check_decode_shape(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                    max_context_len, partition_size, dtype);
  if (st != PA_OK) return st;
  if (dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
  if (num_groups < 0 || num_listed < 0 || (key == nullptr) != (value == nullptr))
    return PA_ERR_INVALID_ARG;
  if (max_blocks_per_seq <= 0 || num_blocks <= 0 || block_size <= 0 || !std::isfinite(scale))
    return PA_ERR_INVALID_ARG;
  if (block_size != pa::kBlockSize) return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0) return PA_OK;
  if (num_groups > 0 && (!group_seqs || !group_start || !group_blocks || num_listed == 0))
    return PA_ERR_INVALID_ARG;
  if (num_groups > 16384) return PA_ERR_UNSUPPORTED;  // (the pass keeps one int per group on chip)
  if (num_groups > num_listed) return PA_ERR_INVALID_ARG;  // (a group lists one member at least)
  if (key && (!aligned16(key) || !aligned16(value))) return PA_ERR_INVALID_ARG;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID_ARG;
  size_t need = 0;
  if ((st = pa_shared_prefix_workspace_size(num_seqs, num_listed, num_q_heads, num_kv_heads,
                                            head_dim, max_blocks_per_seq, max_context_len,
                                            partition_size, dtype, &need)) != PA_OK)
    return st;
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return PA_ERR_WORKSPACE;
  DecodePlan p;
  if ((st = make_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                      partition_size, dtype, &p)) != PA_OK)
    return st;
  const size_t dec_bytes = round_up(p.ws_bytes, 256);
  pa::SharedPrefixLaunch l{};
  l.q = q;
  l.k_cache = k_cache;
  l.v_cache = v_cache;
  l.block_tables = block_tables;
  l.context_lens = context_lens;
  l.group_seqs = group_seqs;
  l.group_start = group_start;
  l.group_blocks = group_blocks;
  l.num_groups = num_groups;
  l.num_listed = num_listed;
  l.num_seqs = num_seqs;
  l.num_q_heads = num_q_heads;
  l.num_kv_heads = num_kv_heads;
  l.head_dim = head_dim;
  l.max_blocks_per_seq = max_blocks_per_seq;
  l.num_blocks = num_blocks;
  const long long cap = static_cast<long long>(max_blocks_per_seq) * pa::kBlockSize;
  l.len_cap = static_cast<int>(max_context_len < cap ? max_context_len : cap);
  l.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  l.workspace = static_cast<char*>(workspace) + dec_bytes;
  l.err_flag = err_flag;
  CUtensorMap tk, tv;
  const long long rows = static_cast<long long>(num_blocks) * num_kv_heads * pa::kBlockSize;
  if (rows + pa::kBlockSize < (1LL << 31) && num_groups > 0 &&
      encode_cache_map(&tk, k_cache, rows, head_dim) == PA_OK &&
      encode_cache_map(&tv, v_cache, rows, head_dim) == PA_OK) {
    l.tm_k = &tk;
    l.tm_v = &tv;
  }
  if (pa::launch_shared_prefix(l, p.sms, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return PA_ERR_CUDA;
  }
  return decode_impl(out, q, key, value, k_cache, v_cache, block_tables, context_lens, num_seqs,
                     num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                     num_blocks, max_context_len, scale, partition_size, dtype, workspace,
                     dec_bytes, err_flag, stream, nullptr, -1, 0, &l);
}

pa_status pa_reshape_and_cache(const void* key, const void* value, void* k_cache, void* v_cache,
                               const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                               int head_dim, int block_size, int num_blocks, pa_dtype dtype,
                               int32_t* err_flag, void* stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      num_blocks <= 0 || !valid_dtype(dtype))
    return PA_ERR_INVALID_ARG;
  const long long row = static_cast<long long>(head_dim) * elem_bytes(dtype);
  if (row % 16 != 0) return PA_ERR_INVALID_ARG;
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !k_cache || !v_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
  if (!aligned16(key) || !aligned16(value) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID_ARG;
  DeviceInfo dev;
  const pa_status st = device_info(&dev);
  if (st != PA_OK) return st;
  const cudaError_t e = pa::launch_reshape_and_cache(
      key, value, k_cache, v_cache, slot_mapping, num_tokens, num_kv_heads,
      static_cast<int>(row), block_size, static_cast<long long>(num_blocks) * block_size,
      err_flag, dev.sms, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_copy_blocks(void* k_cache, void* v_cache, const int32_t* block_mapping,
                         int num_pairs, int num_kv_heads, int head_dim, int block_size,
                         int num_blocks, pa_dtype dtype, int32_t* err_flag, void* stream) {
  if (num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      num_blocks <= 0 || !valid_dtype(dtype))
    return PA_ERR_INVALID_ARG;
  const long long blk =
      static_cast<long long>(num_kv_heads) * block_size * head_dim * elem_bytes(dtype);
  if (blk % 16 != 0) return PA_ERR_INVALID_ARG;
  if (num_pairs == 0) return PA_OK;
  if (!k_cache || !v_cache || !block_mapping) return PA_ERR_INVALID_ARG;
  if (!aligned16(k_cache) || !aligned16(v_cache)) return PA_ERR_INVALID_ARG;
  DeviceInfo dev;
  const pa_status st = device_info(&dev);
  if (st != PA_OK) return st;
  const cudaError_t e = pa::launch_copy_blocks(k_cache, v_cache, block_mapping, num_pairs, blk,
                                               num_blocks, err_flag, dev.sms,
                                               static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // extern "C"
