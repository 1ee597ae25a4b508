// tc_attention.cu -- attention of many query columns at once on the tcgen05
// tensor cores: several query tokens per sequence (chunked prefill) and the
// shared-prefix pass of prefix-deduplicated decode.
//
// Both stream a sequence's K/V blocks past many query columns.  A prompt
// chunk's rows attend causally to the cache that grows by each of their
// tokens before they attend ("vLLM Solved the Wrong Bottleneck...", section
// "Paged Attention"); the members of a group of requests forked from one
// prompt all attend to the blocks they share (skandtandon day-9 post,
// section "Idea 1: PagedAttention").  Here a column is one (query row, query
// head) pair of one KV head, and 128 of them form the M side of the MMAs:
//
//   S[128 columns x 64 keys]  = Q[128 x D] . K[64 keys x D]^T    (TMEM, fp32)
//   P = exp2(S * scale * log2 e - m)  (one thread per column, bf16, into TMEM
//                                      over the S columns it was made from)
//   O[128 columns x D]       += P[128 x 64 keys] . V[64 keys x D]  (TMEM)
//
// with the online softmax of the decode kernels (running max m in log2 units,
// rescaled only when it grows by more than 2^8; the sum l takes the weights
// as rounded for the product).  The keys of a tile are 4 blocks of 16 tokens,
// each fetched by 2-D tensor loads (16 rows x 64 elements, 128-byte swizzle)
// through the block table; a block past the range is loaded from outside the
// tensor, which fills it with zeros.
//
// A CTA works on two column tiles (A and B) of the same work at once, which
// share every K/V tile, so that one tile's softmax overlaps the other's
// MMAs and waits.  CTA roles (320 threads, one CTA per SM, persistent over
// the work units):
//   warps 0-3  softmax of tile A, warps 4-7 of tile B: thread t of a
//              warpgroup owns column t (TMEM lane t): loads its q row,
//              reads its row of S, writes its row of P, rescales and finally
//              reads its row of O -- no cross-thread reduction anywhere;
//   warp 8     producer: K and V tiles into two 3-slot rings (K runs one tile
//              ahead of V, so each wait is in the order the slots free up);
//   warp 9     MMA issuer (one elected lane per group of MMAs; P.V takes P
//              straight from TMEM) and TMEM owner (512 columns: two S
//              buffers per tile, so that S of tile j+2 is computed while the
//              softmax works on tile j, and O of each tile).
// Every mbarrier wait is bounded; a wait that runs out sets PA_ERRBIT_TIMEOUT,
// and every role then leaves its loop; the TMEM is freed on every exit path
// once the MMAs issued so far have completed.
//
// Work units:
//   prefill  (sequence, KV head, pair of column tiles): a tile is 128/G
//            consecutive query rows x G heads; keys 0 .. the position of the
//            pair's last row; the normalised output is stored.
//   shared   (group, range of shared blocks, KV head, pair of column tiles):
//            a tile is 128/G members x G heads; the range's partial state is
//            stored, and a fold kernel launched behind the pass combines the
//            ranges by log-sum-exp into the state the decode kernel
//            continues from (after checking each member's table).
// A one-CTA plan kernel writes the units' records into the workspace first;
// the attention kernel (and the fold kernel behind it) are launched with
// programmatic dependent launch.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <utility>

#include "paged_attention.h"
#include "pa_internal.h"
#include "ptx.cuh"
#include "tc.cuh"

namespace pa {
namespace {

constexpr int kCols = 128;                      // M: query columns of a tile
constexpr int kPair = 2;                        // column tiles a CTA works on together
constexpr int kKeys = 64;                       // N: keys of a K/V tile
constexpr int kTileBlocks = kKeys / kBlockSize; // 4 blocks per K/V tile
constexpr int kStages = 3;                      // slots of the K ring and of the V ring
constexpr int kWgThreads = 128;                 // softmax warpgroup: one thread per column
constexpr int kSoftmaxThreads = kPair * kWgThreads;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kThreads = 320;
constexpr int kTmemCols = 512;                  // S of tile t at 128 t (+64), O of tile t at 256 + 128 t
constexpr int kPlanThreads = 1024;
constexpr int kSortBuckets = 256;               // unit lengths the plan kernel tells apart
constexpr int kPlanRowsOnChip = 2048;           // rows whose metadata and unit starts the plan
                                                // kernel keeps on chip
constexpr int kPlanAhead = 4;                   // block ids per lane the plan loads beside a row's
                                                // lengths
constexpr int kMaxFoldRanges = 16;              // shared: ranges of a group's shared blocks, at most
constexpr int kModePrefill = 0;
constexpr int kModeShared = 1;

struct TcArgs {
  const __nv_bfloat16* q;
  __nv_bfloat16* out;               // prefill: [query rows][Hq][D]
  const int32_t* block_tables;
  const int32_t* context_lens;
  const int32_t* query_start;       // prefill: [rows + 1]
  const int32_t* group_seqs;        // shared: members, group by group
  const int32_t* group_start;       // shared: [groups + 1]
  const int32_t* group_blocks;      // shared: [groups]
  int rows;                         // prefill: sequences (table rows); shared: groups
  int num_query_rows;               // prefill: rows of q and out
  int num_seqs;                     // shared: sequences
  int num_listed;                   // shared: group_seqs entries
  int num_q_heads, num_kv_heads, max_blocks_per_seq, num_blocks, len_cap;
  int num_sms;                      // shared: the plan sizes ranges to fill this many CTAs
  int max_ranges;                   // shared: ranges the partial arrays hold per column
  int oob_row;                      // a row of the cache tensors' 2-D view past their end
  int v8_out;                       // prefill: out is 32-byte aligned (32-byte stores)
  int tma_out;                      // prefill: tm_out is set (full column tiles by tensor stores)
  int v8_part;                      // shared: part_o is 32-byte aligned
  float scale_log2;
  int* unit_start;                  // [rows + 1] work units before each sequence / group
  int4* units;                      // [max_units][2] one record per work unit, longest first
  int max_units;
  int* group_ranges;                // shared: [groups] ranges of each group (0: none folded)
  int* claim;                       // shared: [num_seqs] blocks attended per sequence
  float2* part_ml;                  // shared: [num_listed * Hq][max_ranges]
  float* part_o;                    // shared: [num_listed * Hq][max_ranges][D]
  float2* pre_ml;                   // shared: [num_seqs * Hq]
  float* pre_o;                     // shared: [num_seqs * Hq][D]
  int32_t* err_flag;
  CUtensorMap tm_k;                 // caches as [num_blocks * Hkv * 16][D], boxes 16 x 64, SW128
  CUtensorMap tm_v;
  CUtensorMap tm_out;               // prefill: out as (head_dim, Hq, rows), boxes 64 x G x 128/G
};

// A bounded mbarrier wait whose polls carry no suspend-time hint.  The roles
// of the attention kernel hand off to one another every few hundred cycles;
// a poll with a hint of tens of microseconds let the waiting warps wake
// later after the phase completed (the prefill call took 1.4 us longer),
// while the plain form suspends a thread only for a short time of the
// hardware's choosing.
__device__ __forceinline__ bool mbar_test_plain(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_handoff(uint32_t bar, uint32_t parity) {
  if (mbar_test_plain(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (!mbar_test_plain(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}

__device__ __forceinline__ void seterr(const TcArgs& a, int bit) {
  if (a.err_flag) atomicOr(a.err_flag, bit);
}

// Prefill: sequence s's query rows [a0, a1) and context length len checked;
// its first query row, rows and length, or false (with the error bit to set
// in *bit, 0 if none) when it has none to compute.
__device__ __forceinline__ bool prefill_row(const TcArgs& a, int a0, int a1, int len, int* q0,
                                            int* Q, int* n, int* bit) {
  *bit = 0;
  if (!(0 <= a0 && a0 <= a1 && a1 <= a.num_query_rows)) {
    *bit = kErrQuery;
    return false;
  }
  *q0 = a0;
  *Q = a1 - a0;
  *n = len;
  if (*Q == 0) return false;
  if (len < 0 || len > a.len_cap) {
    *bit = kErrContextLen;
    return false;
  }
  if (*Q > len) {
    *bit = kErrQuery;
    return false;
  }
  return true;
}

// The same from the arrays (all three loads issued together: s is a row of
// the table, so each is in bounds whatever the values).
__device__ __forceinline__ bool prefill_seq(const TcArgs& a, int s, int* q0, int* Q, int* n,
                                            int* bit) {
  const int a0 = a.query_start[s], a1 = a.query_start[s + 1], len = a.context_lens[s];
  return prefill_row(a, a0, a1, len, q0, Q, n, bit);
}

// Shared: group g's members and shared blocks, if well formed.
__device__ __forceinline__ bool shared_group(const TcArgs& a, int g, int* gs, int* m, int* P,
                                             int* leader) {
  const int s0 = a.group_start[g], s1 = a.group_start[g + 1], p = a.group_blocks[g];
  if (!(0 <= s0 && s0 < s1 && s1 <= a.num_listed)) return false;
  if (p < 1 || p > a.max_blocks_per_seq) return false;
  const int l = a.group_seqs[s0];
  if (l < 0 || l >= a.num_seqs) return false;
  *gs = s0;
  *m = s1 - s0;
  *P = p;
  *leader = l;
  return true;
}

// ---------------------------------------------------------------------------
// plan: work units per sequence / group and their prefix sums
// ---------------------------------------------------------------------------
template <int D, int G, int MODE>
__global__ void __launch_bounds__(kPlanThreads, 1) tc_plan_kernel(const __grid_constant__ TcArgs a) {
  // the attention kernel may start its prologue now
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ int s_wsum[kPlanThreads / 32];
  __shared__ int s_target, s_total;
  __shared__ int s_hist[kSortBuckets];
  __shared__ int s_pos[kSortBuckets];
  // per-row scratch on chip when the rows fit (else unit_start holds the
  // counts and starts and the metadata is read again where it is needed):
  // unit counts, then unit starts (the attention kernel reads only
  // unit_start[R]); each row's metadata, prefill {first query row, rows,
  // context length, 0}, shared {first member, members, shared blocks, leader}
  __shared__ int s_us[kPlanRowsOnChip + 1];
  __shared__ int4 s_meta[kPlanRowsOnChip];
  constexpr int RPT = kCols / G;  // query rows (members) per column tile
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int R = a.rows, Hkv = a.num_kv_heads, Hq = a.num_q_heads;
  const int per = (R + kPlanThreads - 1) / kPlanThreads;
  const int r0 = min(R, tid * per), r1 = min(R, r0 + per);
  const bool on_chip = R <= kPlanRowsOnChip;
  auto row_set = [&](int r, int v) {
    if (on_chip) s_us[r] = v; else a.unit_start[r] = v;
  };
  auto row_get = [&](int r) -> int { return on_chip ? s_us[r] : __ldcg(a.unit_start + r); };
  // (only rows with units are asked for: their metadata is well formed)
  auto meta_of = [&](int r) -> int4 {
    if (on_chip) return s_meta[r];
    int4 m = make_int4(0, 0, 0, 0);
    if constexpr (MODE == kModePrefill) {
      int bit;
      prefill_seq(a, r, &m.x, &m.y, &m.z, &bit);
    } else {
      shared_group(a, r, &m.x, &m.y, &m.z, &m.w);
    }
    return m;
  };
  for (int b = tid; b < kSortBuckets; b += kPlanThreads) s_hist[b] = 0;
  int local = 0;  // units of this thread's rows
  if constexpr (MODE == kModePrefill) {
    // One warp per sequence: its lengths and its first block ids are loaded
    // together (each load in bounds of its array whatever the values), then
    // every block a computable sequence attends to must be a block of the
    // cache.  A sequence that cannot be computed gets no units, its
    // (well-placed) query rows are zeroed here and the error bit is set.
    for (int r = warp; r < R; r += kPlanThreads / 32) {
      const int32_t* trow = a.block_tables + static_cast<size_t>(r) * a.max_blocks_per_seq;
      const int a0 = a.query_start[r], a1 = a.query_start[r + 1], len = a.context_lens[r];
      int ids[kPlanAhead];
#pragma unroll
      for (int k = 0; k < kPlanAhead; ++k) {
        const int b = lane + 32 * k;
        ids[k] = b < a.max_blocks_per_seq ? __ldg(trow + b) : 0;
      }
      int q0 = 0, Q = 0, n = 0, bit = 0;
      const bool ok = prefill_row(a, a0, a1, len, &q0, &Q, &n, &bit);
      bool bad = false;
      if (ok) {
        const int nb = (n + kBlockSize - 1) / kBlockSize;  // (at most max_blocks_per_seq)
#pragma unroll
        for (int k = 0; k < kPlanAhead; ++k)
          bad |= lane + 32 * k < nb && !(ids[k] >= 0 && ids[k] < a.num_blocks);
        for (int b = lane + 32 * kPlanAhead; b < nb; b += 32) {
          const int phys = __ldg(trow + b);
          bad |= !(phys >= 0 && phys < a.num_blocks);
        }
        bad = __any_sync(0xffffffffu, bad);
        if (bad) bit = kErrBlockId;
      }
      if (bit) {
        if (lane == 0) seterr(a, bit);
        if (0 <= a0 && a0 <= a1 && a1 <= a.num_query_rows) {
          uint4* dst = reinterpret_cast<uint4*>(a.out + static_cast<size_t>(a0) * Hq * D);
          const size_t cnt = static_cast<size_t>(a1 - a0) * Hq * D * 2 / 16;
          for (size_t i = lane; i < cnt; i += 32) dst[i] = make_uint4(0, 0, 0, 0);
        }
      }
      if (lane == 0) {
        row_set(r, ok && !bad ? Hkv * (((Q + RPT - 1) / RPT + kPair - 1) / kPair) : 0);
        if (on_chip) s_meta[r] = make_int4(q0, Q, n, 0);
      }
    }
    __syncthreads();
    for (int r = r0; r < r1; ++r) local += row_get(r);
  } else {
    // Ranges per group, so that all units together about fill the SMs: the
    // pairs of column tiles x KV heads of every group are counted first, and
    // each group's shared blocks are then cut into as many ranges (of whole
    // K/V tiles, at least two) as one wave needs.
    int base = 0;
    for (int r = r0; r < r1; ++r) {
      int4 m = make_int4(0, 0, 0, -1);
      if (shared_group(a, r, &m.x, &m.y, &m.z, &m.w))
        base += Hkv * (((m.y * G + kCols - 1) / kCols + kPair - 1) / kPair);
      else
        m = make_int4(0, 0, 0, -1);
      if (on_chip) s_meta[r] = m;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) base += __shfl_xor_sync(0xffffffffu, base, o);
    if (lane == 0) s_wsum[warp] = base;
    __syncthreads();
    if (tid == 0) {
      int tot = 0;
      for (int w = 0; w < kPlanThreads / 32; ++w) tot += s_wsum[w];
      s_target = tot > 0 ? max(1, (a.num_sms + tot - 1) / tot) : 1;
    }
    __syncthreads();
  }
  // a group's ranges: count and length in blocks (a multiple of a K/V tile)
  auto ranges_of = [&](int P, int* rb) -> int {
    int Rg = min(min(min(a.max_ranges, kMaxFoldRanges), max(1, P / (2 * kTileBlocks))), s_target);
    int b = (P + Rg - 1) / Rg;
    b = (b + kTileBlocks - 1) / kTileBlocks * kTileBlocks;
    *rb = b;
    return (P + b - 1) / b;
  };
  if constexpr (MODE == kModeShared) {
    for (int r = r0; r < r1; ++r) {
      int units = 0, Rg = 0;
      int4 m = on_chip ? s_meta[r] : make_int4(0, 0, 0, -1);
      if (!on_chip && !shared_group(a, r, &m.x, &m.y, &m.z, &m.w)) m.w = -1;
      if (m.w >= 0) {
        const int npair = ((m.y * G + kCols - 1) / kCols + kPair - 1) / kPair;
        int rb;
        Rg = ranges_of(m.z, &rb);
        units = npair * Hkv * Rg;
      } else {
        seterr(a, kErrGroup);
      }
      a.group_ranges[r] = Rg;
      row_set(r, units);  // (turned into starts below)
      local += units;
    }
  }
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  auto publish_total = [&](int total) {
    // (the workspace is sized for the most units a call can have)
    row_set(R, total);
    s_total = total;
    a.unit_start[R] = min(total, a.max_units);
    if (total > a.max_units) seterr(a, kErrTimeout);
  };
  if (R <= 32) {
    // every row is a lane of warp 0, whose scan is then the whole one
    if (warp == 0) {
      if (r0 < r1) {
        row_set(r0, incl - local);
        // (a group whose units do not all fit the workspace is not folded)
        if (MODE == kModeShared && incl > a.max_units) a.group_ranges[r0] = 0;
      }
      const int total = __shfl_sync(0xffffffffu, incl, 31);
      if (lane == 0) publish_total(total);
    }
  } else {
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    // (only the threads with rows, and thread 0 for the total, need the warps'
    // sums: with few rows most warps skip them)
    if (r0 < r1 || tid == 0) {
      int run = incl - local, total = 0;
#pragma unroll
      for (int w = 0; w < kPlanThreads / 32; ++w) {
        if (w < warp) run += s_wsum[w];
        total += s_wsum[w];
      }
      for (int r = r0; r < r1; ++r) {
        const int units = row_get(r);
        row_set(r, run);
        // (a group whose units do not all fit the workspace is not folded)
        if (MODE == kModeShared && run + units > a.max_units) a.group_ranges[r] = 0;
        run += units;
      }
      if (tid == 0) publish_total(total);
    }
  }
  __syncthreads();
  const int T = min(s_total, a.max_units);
  // Each unit as a record {row, kv head | pair of column tiles << 16, first
  // key, last key + 1} {prefill: first query row, rows, context length, 0 |
  // shared: first member, members, shared blocks, range | ranges << 16}, so
  // that the attention kernel finds a unit with one load instead of a search.
  // A thread finds unit u's row by a search over the unit starts.
  auto record = [&](int u, int4* x0, int4* x1) {
    int lo = 0, up = R - 1;  // largest row with row_get(row) <= u
    while (lo < up) {
      const int mid = (lo + up + 1) >> 1;
      if (row_get(mid) <= u) lo = mid; else up = mid - 1;
    }
    const int r = lo, k = u - row_get(lo);
    const int4 m = meta_of(r);
    if constexpr (MODE == kModePrefill) {
      const int q0 = m.x, Q = m.y, n = m.z;
      const int npair = ((Q + RPT - 1) / RPT + kPair - 1) / kPair;
      const int pr = k % npair, kvh = k / npair;
      const int jl = min(Q, (pr + 1) * kPair * RPT) - 1;  // the pair's last query row
      *x0 = make_int4(r, kvh | (pr << 16), 0, n - Q + jl + 1);
      *x1 = make_int4(q0, Q, n, 0);
    } else {
      const int gs = m.x, P = m.z, leader = m.w;
      const int npair = ((m.y * G + kCols - 1) / kCols + kPair - 1) / kPair;
      int rb;
      const int Rr = ranges_of(P, &rb);
      const int pr = k % npair, kvh = (k / npair) % Hkv, rr = k / (npair * Hkv);
      const int k1 = min(P, (rr + 1) * rb) * kBlockSize;
      *x0 = make_int4(leader, kvh | (pr << 16), rr * rb * kBlockSize, k1);
      *x1 = make_int4(gs, m.y, P, rr | (Rr << 16));
    }
  };
  // Units differ in length (a causal tile's keys end at its last row; ranges
  // and sequences differ), and the attention kernel deals them to its CTAs in
  // rounds, so they are ordered longest first (a counting sort by K/V tiles)
  // and the CTAs take them in snake order: that spreads the long ones.  The
  // records are made twice -- for the histogram, then to be written straight
  // to their place -- rather than stored and read back.  (s_hist was zeroed
  // at the start.)
  auto bucket_of = [](const int4& x0) -> int {
    const int nt = (x0.w - x0.z + kKeys - 1) / kKeys;
    return nt < kSortBuckets - 1 ? nt : kSortBuckets - 1;
  };
  // (lanes with the same bucket add together: one shared-memory atomic per
  // distinct bucket and warp, not one per unit -- equal lengths are common)
  const int Tw = (T + 31) / 32 * 32;
  for (int u = tid; u < Tw; u += kPlanThreads) {
    int b = -1;
    if (u < T) {
      int4 x0, x1;
      record(u, &x0, &x1);
      b = bucket_of(x0);
    }
    const unsigned same = __match_any_sync(0xffffffffu, b);
    if (b >= 0 && lane == __ffs(same) - 1) atomicAdd(&s_hist[b], __popc(same));
  }
  __syncthreads();
  if (warp == 0) {
    // bucket starts, longest first: an exclusive scan from the top bucket down
    constexpr int PER = kSortBuckets / 32;
    int v[PER], sum = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      v[i] = s_hist[kSortBuckets - 1 - (lane * PER + i)];
      sum += v[i];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int tt = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += tt;
    }
    int run2 = incl - sum;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      s_pos[kSortBuckets - 1 - (lane * PER + i)] = run2;
      run2 += v[i];
    }
  }
  __syncthreads();
  for (int u = tid; u < Tw; u += kPlanThreads) {
    int b = -1;
    int4 x0, x1;
    if (u < T) {
      record(u, &x0, &x1);
      b = bucket_of(x0);
    }
    const unsigned same = __match_any_sync(0xffffffffu, b);
    const int leader = __ffs(same) - 1;
    int base = 0;
    if (b >= 0 && lane == leader) base = atomicAdd(&s_pos[b], __popc(same));
    base = __shfl_sync(0xffffffffu, base, leader);
    if (b >= 0) {
      const int pos = base + __popc(same & ((1u << lane) - 1));
      a.units[2 * pos] = x0;
      a.units[2 * pos + 1] = x1;
    }
  }
}

// ---------------------------------------------------------------------------
// the attention kernel
// ---------------------------------------------------------------------------
struct Unit {
  int row;    // block-table row
  int kvh;
  int pr;     // pair of column tiles: tiles 2 pr and 2 pr + 1
  int k0;     // first key of the unit
  int k1;     // one past its last key
  int nt;     // K/V tiles
  // prefill
  int q0, Q, n;
  // shared
  int gs, m, P, r, R;
};

// Work unit u's record from the plan kernel.  The plan kernel writes the
// records while this grid may already be running (programmatic dependent
// launch), so they are read through L2 (ld.global.cg), never through the
// non-coherent read-only path: on B200 that path returned a previous call's
// records when a workspace was reused, and whole units went missing.  Each
// role loads the next unit's record a unit ahead and decodes it only when
// it moves on, so that it does not wait for the load where it issues it.
struct UnitRecord {
  int4 r0, r1;
};
__device__ __forceinline__ UnitRecord load_record(const TcArgs& a, int u) {
  return UnitRecord{__ldcg(a.units + 2 * u), __ldcg(a.units + 2 * u + 1)};
}
template <int MODE>
__device__ __forceinline__ Unit decode_unit(const UnitRecord& rec) {
  const int4 r0 = rec.r0, r1 = rec.r1;
  Unit x;
  x.row = r0.x;
  x.kvh = r0.y & 0xffff;
  x.pr = r0.y >> 16;
  x.k0 = r0.z;
  x.k1 = r0.w;
  if constexpr (MODE == kModePrefill) {
    x.q0 = r1.x;
    x.Q = r1.y;
    x.n = r1.z;
  } else {
    x.gs = r1.x;
    x.m = r1.y;
    x.P = r1.z;
    x.r = r1.w & 0xffff;
    x.R = r1.w >> 16;
  }
  x.nt = (x.k1 - x.k0 + kKeys - 1) / kKeys;
  return x;
}

// 2^x by the ex2.approx.ftz.f32 instruction.  Results below the smallest
// normal float flush to zero; the weights it makes are rounded to bf16 and
// are at most 2^8, so nothing of them is lost that the sum could see.
__device__ __forceinline__ float ex2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two fp32 lanes per instruction (sm_100a packed f32x2): each lane is
// rounded as the scalar fma / add would be.
__device__ __forceinline__ uint64_t f2_bits(float lo, float hi) {
  return static_cast<uint64_t>(__float_as_uint(lo)) |
         (static_cast<uint64_t>(__float_as_uint(hi)) << 32);
}
__device__ __forceinline__ void fma2(float a0, float a1, uint64_t b, uint64_t c, float* d0, float* d1) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(f2_bits(a0, a1)), "l"(b), "l"(c));
  *d0 = __uint_as_float(static_cast<uint32_t>(d));
  *d1 = __uint_as_float(static_cast<uint32_t>(d >> 32));
}
// max(a, b, c) in one instruction (a NaN operand is passed over, as by fmaxf)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// 32 bytes to global memory in one instruction (address 32-byte aligned):
// a lane then fills a whole 32-byte sector, where two 16-byte stores from
// lanes whose rows lie 256 bytes apart leave each of their sectors half used.
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t (&w)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w[0]),
               "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void* src, bool fill) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(fill ? 16 : 0)
               : "memory");
}

template <int D, int G, int MODE>
__global__ void __launch_bounds__(kThreads, 1) tc_attention_kernel(const __grid_constant__ TcArgs a) {
  constexpr int KB = D / 64;                 // 64-element (128-byte) blocks of head_dim
  constexpr int QT = kCols * D * 2;          // bytes of a Q tile
  constexpr int KT = kKeys * D * 2;          // bytes of a K (or V) tile
  constexpr int OT = kCols * D * 2;          // bytes of a bf16 O tile (prefill's staging)
  constexpr int HALF = kKeys * 128;          // bytes of a 64-element half of a K/V tile
  constexpr int RPT = kCols / G;
  constexpr uint32_t IDESC_S = tc::idesc_bf16_f32(kCols, kKeys, false);
  constexpr uint32_t IDESC_O = tc::idesc_bf16_f32(kCols, D, true);
  static_assert(D == 64 || D == 128, "head_dim");
  static_assert(kKeys == 64, "a P row is one 128-byte swizzle row");

  extern __shared__ unsigned char smem_raw[];
  // 1024-byte alignment for the swizzled tiles
  unsigned char* sm = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  unsigned char* sQ = sm;                    // [kPair][QT]
  unsigned char* sK = sQ + kPair * QT;       // [kStages][KT]
  unsigned char* sV = sK + kStages * KT;     // [kStages][KT]
  unsigned char* sO = sV + kStages * KT;     // prefill: [kPair][OT] staging
  uint64_t* bars = reinterpret_cast<uint64_t*>(sO + (MODE == kModePrefill ? kPair * OT : 0));
  // barriers: kfull[3] kempty[3] vfull[3] vempty[3] | per tile t: sfull[t][2],
  // pfull[t], odone[t] | qfull drain | osync[t]
  const uint32_t b0 = smem_addr(bars);
  const uint32_t KFULL = b0, KEMPTY = b0 + 24, VFULL = b0 + 48, VEMPTY = b0 + 72;
  const uint32_t TB = b0 + 96;  // tile t's barriers at TB + 32 t: sfull[2], pfull, odone
  const uint32_t QFULL = b0 + 96 + 32 * kPair, DRAIN = QFULL + 8;
  const uint32_t OSYNC = DRAIN + 8;  // osync[t] at OSYNC + 8 t: tile t's warpgroup among itself
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Hq = a.num_q_heads, Hkv = a.num_kv_heads;

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(KFULL + 8 * i, 1);
      mbar_init(KEMPTY + 8 * i, 1);
      mbar_init(VFULL + 8 * i, 1);
      mbar_init(VEMPTY + 8 * i, 1);
    }
    for (int t = 0; t < kPair; ++t) {
      mbar_init(TB + 32 * t, 1);        // sfull[0]
      mbar_init(TB + 32 * t + 8, 1);    // sfull[1]
      mbar_init(TB + 32 * t + 16, kWgThreads);  // pfull
      mbar_init(TB + 32 * t + 24, 1);   // odone
    }
    mbar_init(QFULL, kSoftmaxThreads);
    mbar_init(DRAIN, 1);
    for (int t = 0; t < kPair; ++t) mbar_init(OSYNC + 8 * t, kWgThreads);
    s_abort = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tc::tmem_alloc(smem_addr(&s_tmem), kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = s_tmem;

  // the unit layout comes from the plan kernel
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // shared: the fold kernel behind this one may start its member checks
  if constexpr (MODE == kModeShared) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int total = __ldcg(a.unit_start + a.rows);  // (written by the plan kernel: see load_record)

  auto timeout = [&]() {
    if (atomicExch(&s_abort, 1) == 0) seterr(a, kErrTimeout);
  };
  // this CTA's k-th unit: rounds of gridDim.x units (longest first), taken
  // in snake order so that the long ones spread over the CTAs
  auto unit_of = [&](int k) -> int {
    const int g = static_cast<int>(gridDim.x), b = static_cast<int>(blockIdx.x);
    return k * g + ((k & 1) ? g - 1 - b : b);
  };
  auto aborted_one = [&]() { return *reinterpret_cast<volatile int*>(&s_abort) != 0; };
  // (the producer and softmax warps test it with all lanes and act on one answer)
  auto aborted = [&]() { return __any_sync(0xffffffffu, aborted_one()); };

  if (warp == kProducerWarp) {
    // ---------------- producer: K runs one tile ahead of V ----------------------
    int kidx = 0, vidx = 0;
    int yprev = a.oob_row;  // (lane b < 4: tile row of block b of the previous tile)
    bool have_prev = false, ok = true;
    auto issue_v = [&](int ysrc) -> bool {
      const int st = vidx % kStages;
      if (vidx >= kStages &&
          !__all_sync(0xffffffffu, mbar_wait_handoff(VEMPTY + 8 * st, ((vidx / kStages) - 1) & 1)))
        return false;
      if (lane == 0) mbar_arrive_expect_tx(VFULL + 8 * st, KT);
      __syncwarp();
      if (lane < kTileBlocks) {
        const uint32_t dst = smem_addr(sV + st * KT) + lane * kBlockSize * 128;
#pragma unroll
        for (int hx = 0; hx < KB; ++hx) tma_load_2d(dst + hx * HALF, &a.tm_v, hx * 64, ysrc, VFULL + 8 * st);
      }
      ++vidx;
      return true;
    };
    Unit x{};
    UnitRecord nr{};  // the next unit's record
    if (unit_of(0) < total) x = decode_unit<MODE>(load_record(a, unit_of(0)));
    for (int k = 0, u = unit_of(0); u < total && ok; u = unit_of(++k), x = decode_unit<MODE>(nr)) {
      if (unit_of(k + 1) < total) nr = load_record(a, unit_of(k + 1));
      const int32_t* trow = a.block_tables + static_cast<size_t>(x.row) * a.max_blocks_per_seq;
      // block rows of the unit's first tile; then always one tile ahead
      auto rows_of = [&](int j) -> int {
        const int lb = x.k0 / kBlockSize + j * kTileBlocks + lane;
        int y = a.oob_row;
        if (lane < kTileBlocks && j < x.nt && lb * kBlockSize < x.k1) {
          const int phys = __ldg(trow + lb);
          if (phys >= 0 && phys < a.num_blocks) y = (phys * Hkv + x.kvh) * kBlockSize;
        }
        return y;
      };
      int ynext = rows_of(0);
      for (int j = 0; j < x.nt; ++j) {
        if (aborted()) { ok = false; break; }
        const int y = ynext;
        ynext = rows_of(j + 1);
        const int st = kidx % kStages;
        if (kidx >= kStages &&
            !__all_sync(0xffffffffu, mbar_wait_handoff(KEMPTY + 8 * st, ((kidx / kStages) - 1) & 1))) {
          timeout();
          ok = false;
          break;
        }
        if (lane == 0) mbar_arrive_expect_tx(KFULL + 8 * st, KT);
        __syncwarp();
        if (lane < kTileBlocks) {
          const uint32_t dst = smem_addr(sK + st * KT) + lane * kBlockSize * 128;
#pragma unroll
          for (int hx = 0; hx < KB; ++hx) tma_load_2d(dst + hx * HALF, &a.tm_k, hx * 64, y, KFULL + 8 * st);
        }
        ++kidx;
        if (have_prev && !issue_v(yprev)) {
          timeout();
          ok = false;
          break;
        }
        yprev = y;
        have_prev = true;
      }
    }
    if (ok && have_prev && !issue_v(yprev)) timeout();
    // let every load issued land before the CTA can exit
    for (int i = max(0, kidx - kStages); i < kidx; ++i)
      mbar_wait_handoff(KFULL + 8 * (i % kStages), (i / kStages) & 1);
    for (int i = max(0, vidx - kStages); i < vidx; ++i)
      mbar_wait_handoff(VFULL + 8 * (i % kStages), (i / kStages) & 1);
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issuer -------------------------------------------------
    // Per K/V tile j: S_A(j), S_B(j) were issued two tiles ahead; as each
    // warpgroup releases P_t(j): O_t += P_t(j) V(j), then S_t(j + 2) into the
    // S buffer P_t(j) has freed.  The whole warp runs the loop, so that the
    // descriptors it computes are warp-uniform, and one elected lane issues
    // each group of MMAs with its commits in one branch (always the same lane:
    // the warp is converged at each election, and a commit tracks the MMAs of
    // the thread that issues it).
    int kidx = 0, vidx = 0, qidx = 0;
    int sidx[kPair] = {0, 0}, pidx[kPair] = {0, 0};
    bool ok = true;
    // the operands' descriptors: each Q tile's and each ring slot's start,
    // advanced by constant offsets per K step (sdesc_advance)
    const uint64_t qdesc = tc::sdesc_sw128(smem_addr(sQ), 16, 1024);
    const uint64_t kdesc = tc::sdesc_sw128(smem_addr(sK), 16, 1024);
    const uint64_t vdesc = tc::sdesc_sw128(smem_addr(sV), HALF, 1024);
    auto wait_all = [&](uint32_t bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait_handoff(bar, parity));
    };
    auto commit = [&](uint32_t bar) {
      if (tc::elect_one()) tc::commit(bar);
    };
    // S_t of the K tile in ring slot kidx (its K has landed); after the last
    // tile's S the slot frees once they complete
    auto issue_s = [&](int t) {
      const uint64_t kd = tc::sdesc_advance(kdesc, (kidx % kStages) * KT);
      const uint64_t qd = tc::sdesc_advance(qdesc, t * QT);
      const uint32_t dS = tmem + t * 2 * kKeys + (sidx[t] & 1) * kKeys;
      if (tc::elect_one()) {
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k / 4) * (kCols * 128) + (k % 4) * 32;
          const uint32_t koff = (k / 4) * HALF + (k % 4) * 32;
          tc::mma_bf16_ss(dS, tc::sdesc_advance(qd, off), tc::sdesc_advance(kd, koff), IDESC_S, k > 0);
        }
        tc::commit(TB + 32 * t + 8 * (sidx[t] & 1));
        if (t == kPair - 1) tc::commit(KEMPTY + 8 * (kidx % kStages));
      }
      __syncwarp();
      ++sidx[t];
      if (t == kPair - 1) ++kidx;
    };
    auto k_landed = [&]() -> bool {
      if (!wait_all(KFULL + 8 * (kidx % kStages), (kidx / kStages) & 1)) return false;
      tc::fence_after_sync();
      return true;
    };
    Unit x{};
    UnitRecord nr{};  // the next unit's record
    if (unit_of(0) < total) x = decode_unit<MODE>(load_record(a, unit_of(0)));
    for (int k = 0, u = unit_of(0); u < total && ok; u = unit_of(++k), x = decode_unit<MODE>(nr)) {
      if (unit_of(k + 1) < total) nr = load_record(a, unit_of(k + 1));
      if (aborted() || !wait_all(QFULL, qidx & 1)) { ok = false; break; }
      ++qidx;
      tc::fence_after_sync();
      for (int j = 0; j < 2 && j < x.nt && ok; ++j) {
        if (!(ok = k_landed())) break;
        issue_s(0);
        issue_s(1);
      }
      for (int j = 0; j < x.nt && ok; ++j) {
        const int st = vidx % kStages;
        const uint64_t vd = tc::sdesc_advance(vdesc, st * KT);
        const bool ahead = j + 2 < x.nt;
#pragma unroll
        for (int t = 0; t < kPair; ++t) {
          if ((t == 0 && aborted()) || !wait_all(TB + 32 * t + 16, pidx[t] & 1)) { ok = false; break; }
          // (P of this tile sits in the S buffer its S used: S and P.V go in the same order)
          const uint32_t pa = tmem + t * 2 * kKeys + (pidx[t] & 1) * kKeys;
          ++pidx[t];
          if (t == 0 && !wait_all(VFULL + 8 * st, (vidx / kStages) & 1)) { ok = false; break; }
          tc::fence_after_sync();
          if (tc::elect_one()) {
#pragma unroll
            for (int k = 0; k < kKeys / 16; ++k)
              tc::mma_bf16_ts(tmem + 2 * kPair * kKeys + t * D, pa + k * 8,
                              tc::sdesc_advance(vd, k * 16 * 128), IDESC_O, (j > 0 || k > 0) ? 1u : 0u);
            tc::commit(TB + 32 * t + 24);  // odone[t]
            if (t == kPair - 1) tc::commit(VEMPTY + 8 * st);
          }
          __syncwarp();
          if (t == kPair - 1) ++vidx;
          if (ahead) {
            if (t == 0 && !(ok = k_landed())) break;
            issue_s(t);
          }
        }
      }
    }
    if (!ok) timeout();
    // every MMA issued has completed before the TMEM can be freed
    commit(DRAIN);
    wait_all(DRAIN, 0);
    __syncwarp();
  } else {
    // ---------------- softmax: warpgroup t = warp / 4 serves column tile 2 pr + t;
    // thread col owns column col (TMEM lane col of that tile's S and O)
    const int t = warp / 4, col = tid % kWgThreads;
    const int h = col % G;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp % 4) * 32) << 16);
    const uint32_t SFULL = TB + 32 * t, PFULL = SFULL + 16, ODONE = SFULL + 24;
    const uint32_t s_col = t * 2 * kKeys, o_col = 2 * kPair * kKeys + t * D;  // TMEM columns
    unsigned char* const myQ = sQ + t * QT;
    int sidx = 0, oidx = 0, tile = 0, syncs = 0;
    bool ok = true;
    // a bounded wait whose outcome the whole warp shares, so that no lane
    // leaves ahead of the others (the TMEM moves are warp-wide)
    auto wait_all = [&](uint32_t bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait_handoff(bar, parity));
    };
    auto group_sync = [&]() -> bool {  // the 128 threads of this warpgroup
      mbar_arrive(OSYNC + 8 * t);
      return wait_all(OSYNC + 8 * t, (syncs++) & 1);
    };
    // this column's query row in unit y (-1: none), and the keys it sees
    auto column_of = [&](const Unit& y, int* kend) -> int {
      int qrow = -1;
      const int ct = y.pr * kPair + t;
      if constexpr (MODE == kModePrefill) {
        const int jr = ct * RPT + col / G;
        *kend = 0;
        if (jr < y.Q) {
          qrow = y.q0 + jr;
          *kend = min(y.k1, y.n - y.Q + jr + 1);
        }
      } else {
        const int member = ct * RPT + col / G;
        if (member < y.m) {
          const int seq = a.group_seqs[y.gs + member];
          if (seq >= 0 && seq < a.num_seqs) qrow = seq;
        }
        *kend = y.k1;
      }
      return qrow;
    };
    // this column's q row into its tile's swizzled Q (zeros for no row)
    auto load_q = [&](const Unit& y, int qrow) {
      const __nv_bfloat16* src =
          a.q + (static_cast<size_t>(qrow >= 0 ? qrow : 0) * Hq + y.kvh * G + h) * D;
      const uint32_t qb = smem_addr(myQ) + col * 128;
#pragma unroll
      for (int c = 0; c < D / 8; ++c)
        cp_async16_zfill(qb + (c / 8) * (kCols * 128) + (((c % 8) ^ (col % 8)) << 4), src + c * 8,
                         qrow >= 0);
    };
    Unit x{};
    UnitRecord nr{};  // the next unit's record
    if (unit_of(0) < total) x = decode_unit<MODE>(load_record(a, unit_of(0)));
    bool q_issued = false;  // this unit's Q already requested (during the last unit)
    bool q_ready = false;   // ... and already handed to the MMA warp (QFULL)
    for (int k = 0, u = unit_of(0); u < total && ok; u = unit_of(++k), x = decode_unit<MODE>(nr)) {
      const bool has_next = unit_of(k + 1) < total;
      if (has_next) nr = load_record(a, unit_of(k + 1));
      int kend;
      const int qrow = column_of(x, &kend);
      // (a prefill sequence with a block id out of range has no units: the
      // plan kernel zeroed its rows; a shared group's blocks are checked by
      // the fold, and a bad id here only reads the tensor loads' zero fill)
      // ---- Q: requested now, or already during the previous unit's last
      // tile (and then handed over before that unit's epilogue)
      if (!q_ready) {
        if (!q_issued) load_q(x, qrow);
        asm volatile("cp.async.wait_all;" ::: "memory");
        fence_proxy_async_smem();
        tc::fence_before_sync();
        mbar_arrive(QFULL);
      }
      q_issued = q_ready = false;

      float m_run = -INFINITY, l_run = 0.f;
      for (int j = 0; j < x.nt; ++j, ++tile) {
        bool zeroed = false;  // (this thread wrote zeros into the V tile)
        if (aborted() || !wait_all(SFULL + 8 * (sidx & 1), (sidx >> 1) & 1)) { ok = false; break; }
        tc::fence_after_sync();
        uint32_t sv[kKeys];
        const uint32_t s_addr = lane_base + s_col + (sidx & 1) * kKeys;
        tc::tmem_ld64(s_addr, sv);
        tc::tmem_wait_ld(sv);
        ++sidx;
        if (j == x.nt - 1 && has_next) {
          // every S of this tile in this unit is complete: its Q is free
          int kn;
          const Unit nx = decode_unit<MODE>(nr);
          load_q(nx, column_of(nx, &kn));
          q_issued = true;
        }
        // the maximum over 8 independent chains of the scores in log2 units.
        // A tile the column sees whole, with a positive scale: the maximum of
        // the raw scores times the scale (the rounded product is monotonic, so
        // it is the maximum of the rounded scaled scores), and the scale goes
        // into the exponent's fma below.  Otherwise the scores are scaled here
        // and the keys the column does not see are set to -inf.
        const int kb = x.k0 + j * kKeys;
        float m8[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) m8[c] = -INFINITY;
        float mul = 1.f;  // score in log2 units = sv * mul
        if (kb + kKeys <= kend && a.scale_log2 > 0.f) {
          mul = a.scale_log2;
        } else {
#pragma unroll
          for (int k = 0; k < kKeys; ++k) {
            const float v = kb + k < kend ? __uint_as_float(sv[k]) * a.scale_log2 : -INFINITY;
            sv[k] = __float_as_uint(v);
          }
        }
        // (two keys per three-input max; chain c takes keys c, c + 8, ...)
#pragma unroll
        for (int k = 0; k < kKeys; k += 16) {
#pragma unroll
          for (int c = 0; c < 8; ++c)
            m8[c] = fmax3(m8[c], __uint_as_float(sv[k + c]), __uint_as_float(sv[k + c + 8]));
        }
        const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                               fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7]))) * mul;
        const bool grow = mx > m_run + kRescaleThreshold;
        float al = 1.f;
        if (grow) {
          al = ex2_fast(m_run - mx);  // (0 while nothing was seen)
          l_run *= al;
          m_run = mx;
        }
        // weights, rounded to bf16 for the product; the sum (8 chains) takes
        // them as rounded.  They go to tensor memory over the S columns just
        // read (two per 32-bit column), the A operand of this tile's P.V.
        // (a column that has seen no key yet: every score of this tile is -inf,
        // and an offset of 0 keeps its weights at 0.)  Two keys per fma and
        // per add (f32x2); the sum runs in 8 chains, key k in chain k mod 8.
        const float nm = m_run == -INFINITY ? 0.f : -m_run;
        const uint64_t mul2 = f2_bits(mul, mul), nm2 = f2_bits(nm, nm);
        uint64_t l4[4] = {0, 0, 0, 0};
        uint32_t w[kKeys / 2];
#pragma unroll
        for (int e = 0; e < kKeys / 2; ++e) {
          float x0, x1;
          fma2(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1]), mul2, nm2, &x0, &x1);
          const __nv_bfloat162 pp = __floats2bfloat162_rn(ex2_fast(x0), ex2_fast(x1));
          w[e] = *reinterpret_cast<const uint32_t*>(&pp);
          // (bf16 -> fp32 is the 16 bits moved up)
          l4[e & 3] = add2(l4[e & 3], static_cast<uint64_t>(w[e] << 16) |
                                           (static_cast<uint64_t>(w[e] & 0xffff0000u) << 32));
        }
        float l8[8];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          l8[2 * c] = __uint_as_float(static_cast<uint32_t>(l4[c]));
          l8[2 * c + 1] = __uint_as_float(static_cast<uint32_t>(l4[c] >> 32));
        }
        l_run += ((l8[0] + l8[1]) + (l8[2] + l8[3])) + ((l8[4] + l8[5]) + (l8[6] + l8[7]));
        {
          uint32_t w32[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) w32[e] = w[e];
          tc::tmem_st32(s_addr, w32);
          tc::tmem_wait_st();
        }
        if (j > 0) {
          // O of the previous tile is complete (so that it may be rescaled)
          if (!wait_all(ODONE, oidx & 1)) { ok = false; break; }
          ++oidx;
          tc::fence_after_sync();
        }
        if constexpr (MODE == kModePrefill) {
          // rows past the sequence's end in its last block hold stale data: a
          // zero weight times a NaN would still poison O, so tile A's
          // warpgroup zeroes them before the first of the tile's two P.V
          const int tail = x.n % kBlockSize;
          const int lastb = x.n / kBlockSize;  // logical block holding them
          if (t == 0 && tail && lastb * kBlockSize >= kb && lastb * kBlockSize < kb + kKeys) {
            zeroed = true;
            const int st = tile % kStages;
            if (!wait_all(VFULL + 8 * st, (tile / kStages) & 1)) { ok = false; break; }
            const int b = (lastb * kBlockSize - kb) / kBlockSize;
            unsigned char* vt = sV + st * KT;
            const int nz = (kBlockSize - tail) * 8 * KB;  // 16-byte chunks to clear
            for (int i = col; i < nz; i += kWgThreads) {
              const int hx = i / ((kBlockSize - tail) * 8);
              const int rem = i % ((kBlockSize - tail) * 8);
              const int row = b * kBlockSize + tail + rem / 8;
              *reinterpret_cast<uint4*>(vt + hx * HALF + row * 128 + (((rem % 8) ^ (row % 8)) << 4)) =
                  make_uint4(0, 0, 0, 0);
            }
          }
        }
        // O rows are rescaled by the whole warp together (the TMEM moves are
        // warp-wide; rows that do not grow are multiplied by 1), after the S
        // row is spent and before P is released to the MMA
        if (j > 0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tc::tmem_ld32(lane_base + o_col + c * 32, r);
            tc::tmem_wait_ld(r);
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * al);
            tc::tmem_st32(lane_base + o_col + c * 32, r);
          }
          tc::tmem_wait_st();
        }
        // (the V rows zeroed above are generic writes the MMA reads through
        // the async proxy; P went to tensor memory and needs no such fence)
        if (zeroed) fence_proxy_async_smem();
        tc::fence_before_sync();
        mbar_arrive(PFULL);
      }
      if (!ok) break;
      if (q_issued) {
        // The next unit's Q (requested during the last tile) goes to the MMA
        // warp now, so that the next unit's first S tiles are computed while
        // this unit's O goes out: they fill the S buffers, which the last
        // P.V has read before them (the MMAs run in order), and the next
        // P.V that writes O waits for this warpgroup's next P.
        asm volatile("cp.async.wait_all;" ::: "memory");
        fence_proxy_async_smem();
        tc::fence_before_sync();
        mbar_arrive(QFULL);
        q_ready = true;
      }
      // ---- the unit's O row (in halves of 64 columns)
      if (!wait_all(ODONE, oidx & 1)) { ok = false; break; }
      ++oidx;
      tc::fence_after_sync();
      if constexpr (MODE == kModePrefill) {
        const float inv = 1.f / l_run;
        const int ct = x.pr * kPair + t;
        // A column tile whose rows all belong to this sequence goes out by
        // tensor stores (one box per 64 dims: the TMA engine does the strided
        // writes) from a staging tile in the 128-byte-swizzled layout; the
        // last tile of a sequence goes out row by row.
        const bool staged = a.tma_out && (ct + 1) * RPT <= x.Q;
        if (staged) {
          unsigned char* const stg = sO + t * OT;
          if (col == 0) bulk_wait_group_read0();  // (the previous unit's stores have read it)
          if (!group_sync()) { ok = false; break; }
#pragma unroll
          for (int hf = 0; hf < D / 64; ++hf) {
            uint32_t ov[64];
            tc::tmem_ld64(lane_base + o_col + hf * 64, ov);
            tc::tmem_wait_ld(ov);
            const uint32_t rowb = smem_addr(stg) + hf * (kCols * 128) + col * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {  // 8 dims (16 bytes) per chunk
              uint32_t w[4];
#pragma unroll
              for (int f = 0; f < 4; ++f) {
                const __nv_bfloat162 pp = __floats2bfloat162_rn(
                    __uint_as_float(ov[c * 8 + 2 * f]) * inv, __uint_as_float(ov[c * 8 + 2 * f + 1]) * inv);
                w[f] = *reinterpret_cast<const uint32_t*>(&pp);
              }
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(rowb + ((c ^ (col & 7)) << 4)),
                           "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3])
                           : "memory");
            }
          }
          fence_proxy_async_smem();
          if (!group_sync()) { ok = false; break; }
          if (col == 0) {
#pragma unroll
            for (int hf = 0; hf < D / 64; ++hf)
              tma_store_3d(&a.tm_out, smem_addr(stg) + hf * (kCols * 128), hf * 64, x.kvh * G,
                           x.q0 + ct * RPT);
            bulk_commit_group();
          }
        } else {
        // (every lane runs the warp-wide TMEM loads; only live columns store)
        uint4* dst = reinterpret_cast<uint4*>(
            a.out + (static_cast<size_t>(qrow >= 0 ? qrow : 0) * Hq + x.kvh * G + h) * D);
#pragma unroll
        for (int hf = 0; hf < D / 64; ++hf) {
          uint32_t ov[64];
          tc::tmem_ld64(lane_base + o_col + hf * 64, ov);
          tc::tmem_wait_ld(ov);
          if (qrow >= 0) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {  // 16 dims (32 bytes) at a time
              uint32_t w[8];
#pragma unroll
              for (int f = 0; f < 8; ++f) {
                const __nv_bfloat162 pp = __floats2bfloat162_rn(
                    __uint_as_float(ov[c * 16 + 2 * f]) * inv, __uint_as_float(ov[c * 16 + 2 * f + 1]) * inv);
                w[f] = *reinterpret_cast<const uint32_t*>(&pp);
              }
              if (a.v8_out) {
                st_global_v8(dst + hf * 8 + 2 * c, w);
              } else {
                dst[hf * 8 + 2 * c] = make_uint4(w[0], w[1], w[2], w[3]);
                dst[hf * 8 + 2 * c + 1] = make_uint4(w[4], w[5], w[6], w[7]);
              }
            }
          }
        }
        }
      } else {
        // ---- shared: this range's partial state (the fold kernel combines the ranges)
        const int ct = x.pr * kPair + t;
        const int member = ct * RPT + col / G;
        const bool live = member < x.m;
        const size_t pi = live ? (static_cast<size_t>(x.gs + member) * Hq + x.kvh * G + h) *
                                         a.max_ranges + x.r
                               : 0;
#pragma unroll
        for (int hf = 0; hf < D / 64; ++hf) {
          uint32_t ov[64];
          tc::tmem_ld64(lane_base + o_col + hf * 64, ov);
          tc::tmem_wait_ld(ov);
          if (live) {
            float4* po = reinterpret_cast<float4*>(a.part_o + pi * D + hf * 64);
#pragma unroll
            for (int e = 0; e < 8; ++e) {  // 8 floats (32 bytes) at a time
              if (a.v8_part) {
                uint32_t w[8];
#pragma unroll
                for (int f = 0; f < 8; ++f) w[f] = ov[8 * e + f];
                st_global_v8(po + 2 * e, w);
              } else {
                po[2 * e] = make_float4(__uint_as_float(ov[8 * e]), __uint_as_float(ov[8 * e + 1]),
                                        __uint_as_float(ov[8 * e + 2]), __uint_as_float(ov[8 * e + 3]));
                po[2 * e + 1] = make_float4(__uint_as_float(ov[8 * e + 4]), __uint_as_float(ov[8 * e + 5]),
                                            __uint_as_float(ov[8 * e + 6]), __uint_as_float(ov[8 * e + 7]));
              }
            }
          }
        }
        if (live) a.part_ml[pi] = make_float2(m_run, l_run);
      }
    }
    if (!ok) timeout();
    asm volatile("cp.async.wait_all;" ::: "memory");  // (a prefetch left in flight by an abort)
    if (MODE == kModePrefill && col == 0) bulk_wait_group0();  // (the tensor stores have completed)
  }

  // ---- teardown: every role is out of its loop; the MMAs have drained -------
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == kMmaWarp) tc::tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------------------
// shared: the fold of a group's ranges, per listed member
// ---------------------------------------------------------------------------
// CTA (member i, slice y of the query heads); thread = 4 dims of one head.
// Each range left a partial state (m_r, l_r, o_r) per column; the state over
// all the shared blocks is their log-sum-exp combination
//   M = max_r m_r,  w_r = 2^(m_r - M),  l = sum_r w_r l_r,  o = sum_r w_r o_r,
// stored per (sequence, head) for the decode kernel to go on from.  The
// member is first checked against the block tables -- its row must hold the
// leader's blocks, and its length must leave a token after them -- and is
// claimed once (a sequence that two listings claim is given up, and the
// decode kernel attends to all of it).  The check reads only the call's
// inputs, so it runs while the pass is still going; the partial states are
// read once the pass has finished (griddepcontrol.wait).  CTAs are small
// (128 threads, at most 64 registers each) so that one fits beside an
// attention CTA and starts while the pass runs.
constexpr int kFoldThreads = 128;
constexpr int kFoldBatch = 8;  // ranges whose loads are in flight together

template <int D>
__global__ void __launch_bounds__(kFoldThreads, 8) tc_fold_kernel(const __grid_constant__ TcArgs a) {
  constexpr int V = D / 4;                  // threads of a head (float4 each)
  constexpr int HPC = kFoldThreads / V;     // heads of a CTA
  const int i = blockIdx.x, tid = threadIdx.x;
  const int Hq = a.num_q_heads;
  const int h = blockIdx.y * HPC + tid / V, d4 = tid % V;
  // the group listing member i: the last g with group_start[g] <= i
  int lo = 0, up = a.rows - 1;
  while (lo < up) {
    const int mid = (lo + up + 1) >> 1;
    if (a.group_start[mid] <= i) lo = mid; else up = mid - 1;
  }
  const int g = lo;
  int gs = 0, m = 0, P = 0, leader = 0, seq = -1;
  bool ok = shared_group(a, g, &gs, &m, &P, &leader) && gs <= i && i < gs + m;
  if (ok) {
    seq = a.group_seqs[i];
    ok = seq >= 0 && seq < a.num_seqs;
    if (ok) {
      const int n = a.context_lens[seq];
      ok = n > 0 && n <= a.len_cap && kBlockSize * P <= n - 1;
    }
  }
  bool bad = false;
  if (ok) {
    const int32_t* lrow = a.block_tables + static_cast<size_t>(leader) * a.max_blocks_per_seq;
    const int32_t* mrow = a.block_tables + static_cast<size_t>(seq) * a.max_blocks_per_seq;
    for (int jb = tid; jb < P; jb += kFoldThreads) {
      const int lb = __ldg(lrow + jb), mb = __ldg(mrow + jb);
      bad |= !(lb >= 0 && lb < a.num_blocks && mb == lb);
    }
  }
  ok = ok && !__syncthreads_or(bad);  // (ok was the same in every thread)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (!ok) {
    if (blockIdx.y == 0 && tid == 0) seterr(a, kErrGroup);
    return;
  }
  // (written by the plan kernel ahead of the pass: read through L2)
  const int R = min(__ldcg(a.group_ranges + g), kMaxFoldRanges);
  if (R <= 0) return;  // (a malformed group: nothing was computed for it)
  if (h < Hq) {
    const size_t pb = (static_cast<size_t>(i) * Hq + h) * a.max_ranges;
    float M = -INFINITY;
#pragma unroll
    for (int r = 0; r < kMaxFoldRanges; ++r)
      if (r < R) M = fmaxf(M, __ldcg(&a.part_ml[pb + r].x));
    float L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r0 = 0; r0 < kMaxFoldRanges; r0 += kFoldBatch) {
      if (r0 >= R) break;
      float2 ml[kFoldBatch];
      float4 o4[kFoldBatch];
#pragma unroll
      for (int r = 0; r < kFoldBatch; ++r) {
        if (r0 + r < R) {
          ml[r] = __ldcg(a.part_ml + pb + r0 + r);
          o4[r] = __ldcg(reinterpret_cast<const float4*>(a.part_o + (pb + r0 + r) * D) + d4);
        }
      }
#pragma unroll
      for (int r = 0; r < kFoldBatch; ++r) {
        if (r0 + r < R) {
          const float w = ml[r].x == -INFINITY ? 0.f : exp2f(ml[r].x - M);
          L = fmaf(w, ml[r].y, L);
          acc.x = fmaf(w, o4[r].x, acc.x);
          acc.y = fmaf(w, o4[r].y, acc.y);
          acc.z = fmaf(w, o4[r].z, acc.z);
          acc.w = fmaf(w, o4[r].w, acc.w);
        }
      }
    }
    const size_t orow = static_cast<size_t>(seq) * Hq + h;
    reinterpret_cast<float4*>(a.pre_o + orow * D)[d4] = acc;
    if (d4 == 0) a.pre_ml[orow] = make_float2(M, L);
  }
  if (blockIdx.y == 0 && tid == 0 && atomicCAS(a.claim + seq, 0, P) != 0) {
    atomicExch(a.claim + seq, -1);
    seterr(a, kErrGroup);
  }
}

template <int D, int G, int MODE>
struct TcKernels {
  static const void* plan() { return reinterpret_cast<const void*>(&tc_plan_kernel<D, G, MODE>); }
  static const void* main() { return reinterpret_cast<const void*>(&tc_attention_kernel<D, G, MODE>); }
};

template <int MODE>
bool pick(int head_dim, int group, const void** plan, const void** main) {
  switch (head_dim * 100 + group) {
#define PA_TC_CASE(D_, G_)                      \
  case D_ * 100 + G_:                           \
    *plan = TcKernels<D_, G_, MODE>::plan();    \
    *main = TcKernels<D_, G_, MODE>::main();    \
    return true;
    PA_TC_CASE(64, 1)
    PA_TC_CASE(64, 2)
    PA_TC_CASE(64, 4)
    PA_TC_CASE(64, 8)
    PA_TC_CASE(128, 1)
    PA_TC_CASE(128, 2)
    PA_TC_CASE(128, 4)
    PA_TC_CASE(128, 8)
#undef PA_TC_CASE
    default: return false;
  }
}

size_t tc_smem_bytes(int head_dim, bool prefill) {
  const size_t q = static_cast<size_t>(kCols) * head_dim * 2;
  const size_t kv = static_cast<size_t>(kKeys) * head_dim * 2;
  // (alignment slack; barriers: 12 ring + 4 per tile + 4)
  // (prefill: a bf16 O staging tile per column tile, as large as its Q tile)
  return 1024 + kPair * q + 2 * kStages * kv + (prefill ? kPair * q : 0) + 256;
}

std::mutex g_tc_mu;
std::map<std::pair<int, const void*>, bool> g_tc_ready;

cudaError_t prepare(const void* fn, size_t smem) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_tc_mu);
  bool& ready = g_tc_ready[std::make_pair(dev, fn)];
  if (!ready) {
    if ((e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(smem))) != cudaSuccess)
      return e;
    ready = true;
  }
  return cudaSuccess;
}

// a launch behind the previous kernel of the stream with programmatic
// dependent launch (the kernel waits for it with griddepcontrol.wait)
cudaError_t launch_dependent(const void* fn, dim3 grid, int threads, size_t smem, TcArgs& a,
                             cudaStream_t stream) {
  void* params[] = {&a};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, fn, params);
}

// plan kernel, then the attention kernel behind it
cudaError_t launch_pair(const void* plan, const void* main, TcArgs& a, int grid, size_t smem,
                        cudaStream_t stream) {
  cudaError_t e = prepare(main, smem);
  if (e != cudaSuccess) return e;
  void* params[] = {&a};
  if ((e = cudaLaunchKernel(plan, dim3(1), dim3(kPlanThreads), params, 0, stream)) != cudaSuccess)
    return e;
  return launch_dependent(main, dim3(grid), kThreads, smem, a, stream);
}

}  // namespace

bool tc_prefill_supported(int head_dim, int group) {
  const void *p, *m;
  return pick<kModePrefill>(head_dim, group, &p, &m);
}

// Most work units a prefill call can have: each sequence's pairs of column
// tiles, ceil(Q_s * G / 256) <= Q_s * G / 256 + 1, for every KV head.
static long long prefill_max_units(int num_seqs, int num_query_tokens, int num_q_heads,
                                   int num_kv_heads) {
  const long long G = num_q_heads / num_kv_heads;
  return static_cast<long long>(num_kv_heads) *
         ((static_cast<long long>(num_query_tokens) * G + kPair * kCols - 1) / (kPair * kCols) +
          num_seqs);
}
static size_t prefill_records_offset(int num_seqs) {
  return ((static_cast<size_t>(num_seqs) + 1) * sizeof(int) + 255) / 256 * 256;
}

size_t tc_prefill_workspace_bytes(int num_seqs, int num_query_tokens, int num_q_heads,
                                  int num_kv_heads) {
  // unit starts, then a record per unit
  return prefill_records_offset(num_seqs) +
         static_cast<size_t>(prefill_max_units(num_seqs, num_query_tokens, num_q_heads,
                                               num_kv_heads)) * 2 * sizeof(int4);
}

int tc_launch_smem(int head_dim) { return static_cast<int>(tc_smem_bytes(head_dim, true)); }

cudaError_t launch_tc_prefill(const TcPrefillLaunch& l, int num_sms, cudaStream_t stream) {
  const void *plan, *main;
  if (!pick<kModePrefill>(l.head_dim, l.num_q_heads / l.num_kv_heads, &plan, &main))
    return cudaErrorInvalidValue;
  TcArgs a{};
  a.q = static_cast<const __nv_bfloat16*>(l.q);
  a.out = static_cast<__nv_bfloat16*>(l.out);
  a.block_tables = l.block_tables;
  a.context_lens = l.context_lens;
  a.query_start = l.query_start;
  a.rows = l.num_seqs;
  a.num_query_rows = l.num_query_rows;
  a.num_q_heads = l.num_q_heads;
  a.num_kv_heads = l.num_kv_heads;
  a.max_blocks_per_seq = l.max_blocks_per_seq;
  a.num_blocks = l.num_blocks;
  a.len_cap = l.len_cap;
  a.oob_row = l.num_blocks * l.num_kv_heads * kBlockSize;
  a.v8_out = reinterpret_cast<uintptr_t>(l.out) % 32 == 0;
  if (l.tm_out) {
    a.tm_out = *l.tm_out;
    a.tma_out = 1;
  }
  a.scale_log2 = l.scale_log2;
  a.unit_start = static_cast<int*>(l.workspace);
  a.units = reinterpret_cast<int4*>(static_cast<char*>(l.workspace) +
                                    prefill_records_offset(l.num_seqs));
  a.max_units = static_cast<int>(std::min<long long>(
      prefill_max_units(l.num_seqs, l.num_query_rows, l.num_q_heads, l.num_kv_heads), 1 << 28));
  a.err_flag = l.err_flag;
  a.tm_k = *l.tm_k;
  a.tm_v = *l.tm_v;
  return launch_pair(plan, main, a, num_sms, tc_smem_bytes(l.head_dim, true), stream);
}

bool tc_shared_prefix_supported(int head_dim, int group) {
  const void *p, *m;
  return pick<kModeShared>(head_dim, group, &p, &m);
}

cudaError_t launch_tc_shared_prefix(const TcSharedLaunch& l, int num_sms, cudaStream_t stream) {
  const int group = l.num_q_heads / l.num_kv_heads;
  const void *plan, *main;
  if (!pick<kModeShared>(l.head_dim, group, &plan, &main)) return cudaErrorInvalidValue;
  TcArgs a{};
  a.q = static_cast<const __nv_bfloat16*>(l.q);
  a.block_tables = l.block_tables;
  a.context_lens = l.context_lens;
  a.group_seqs = l.group_seqs;
  a.group_start = l.group_start;
  a.group_blocks = l.group_blocks;
  a.rows = l.num_groups;
  a.num_seqs = l.num_seqs;
  a.num_listed = l.num_listed;
  a.num_q_heads = l.num_q_heads;
  a.num_kv_heads = l.num_kv_heads;
  a.max_blocks_per_seq = l.max_blocks_per_seq;
  a.num_blocks = l.num_blocks;
  a.len_cap = l.len_cap;
  a.oob_row = l.num_blocks * l.num_kv_heads * kBlockSize;
  a.scale_log2 = l.scale_log2;
  a.max_ranges = l.max_ranges;
  a.num_sms = num_sms;
  a.unit_start = l.unit_start;
  a.units = l.units;
  a.max_units = l.max_units;
  a.group_ranges = l.group_ranges;
  a.claim = l.claim;
  a.part_ml = l.part_ml;
  a.part_o = l.part_o;
  a.v8_part = reinterpret_cast<uintptr_t>(l.part_o) % 32 == 0;
  a.pre_ml = l.pre_ml;
  a.pre_o = l.pre_o;
  a.err_flag = l.err_flag;
  a.tm_k = *l.tm_k;
  a.tm_v = *l.tm_v;
  cudaError_t e = launch_pair(plan, main, a, num_sms, tc_smem_bytes(l.head_dim, false), stream);
  if (e != cudaSuccess || l.num_listed == 0) return e;
  // the fold: one CTA per (listed member, slice of kFoldThreads / (D / 4) heads)
  const int hpc = kFoldThreads / (l.head_dim / 4);
  const void* fold = l.head_dim == 64 ? reinterpret_cast<const void*>(&tc_fold_kernel<64>)
                                      : reinterpret_cast<const void*>(&tc_fold_kernel<128>);
  return launch_dependent(fold, dim3(l.num_listed, (l.num_q_heads + hpc - 1) / hpc), kFoldThreads,
                          0, a, stream);
}

}  // namespace pa
