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
//   S[128 columns x 128 keys]  = Q[128 x D] . K[128 keys x D]^T   (TMEM, fp32)
//   P = exp2(S * scale * log2 e - m)  (one thread per column, bf16, to smem)
//   O[128 columns x D]        += P[128 x 128 keys] . V[128 keys x D]  (TMEM)
//
// with the online softmax of the decode kernels (running max m in log2 units,
// rescaled only when it grows by more than 2^8; the sum l takes the weights
// as rounded for the product).  The keys of a tile are 8 blocks of 16 tokens,
// each fetched by 2-D tensor loads (16 rows x 64 elements, 128-byte swizzle)
// through the block table; a block past the range is loaded from outside the
// tensor, which fills it with zeros.
//
// CTA roles (192 threads, one CTA per SM, persistent over the work units):
//   warps 0-3  softmax: thread t owns column t (TMEM lane t): loads its q row,
//              reads its row of S, writes its row of P, rescales and finally
//              reads its row of O -- no cross-thread reduction anywhere;
//   warp 4     producer: K and V tiles into two 2-slot rings (K runs one tile
//              ahead of V, so each wait is in the order the slots free up);
//   warp 5     MMA issuer (one thread) and TMEM owner (512 columns: two S
//              buffers so that S of tile j+1 is computed while the softmax
//              works on tile j, and O).
// Every mbarrier wait is bounded; a wait that runs out sets PA_ERRBIT_TIMEOUT,
// and every role then leaves its loop; the TMEM is freed on every exit path
// once the MMAs issued so far have completed.
//
// Work units:
//   prefill  (sequence, KV head, column tile): a tile is 128/G consecutive
//            query rows x G heads; keys 0 .. the tile's last row's position;
//            the normalised output is stored.
//   shared   (group, range of shared blocks, KV head, column tile): a tile
//            is 128/G members x G heads; the range's partial state is stored
//            and the last range of a (group, tile, KV head) to finish folds
//            them by log-sum-exp into the state the decode kernel continues
//            from (after checking each member's table, as the other pass did).
// A one-CTA plan kernel lays the units out (prefix sums over sequences or
// groups) in the workspace first; the attention kernel is launched behind it
// with programmatic dependent launch.
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
constexpr int kKeys = 128;                      // N: keys of a K/V tile
constexpr int kTileBlocks = kKeys / kBlockSize; // 8 blocks per K/V tile
constexpr int kStages = 2;                      // slots of the K ring and of the V ring
constexpr int kSoftmaxThreads = 256;            // two per column: keys 0-63 / 64-127
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kThreads = 320;
constexpr int kTmemCols = 512;                  // S[2] at columns 0 / 128, O at 256
constexpr int kPlanThreads = 1024;
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
  int range_blocks;                 // shared: shared blocks per range (a multiple of 8)
  int max_ranges;                   // shared: ranges the partial arrays hold per column
  int oob_row;                      // a row of the cache tensors' 2-D view past their end
  float scale_log2;
  int* unit_start;                  // [rows + 1] work units before each sequence / group
  int4* units;                      // [max_units][2] one record per work unit (plan kernel)
  int max_units;
  int* counters;                    // shared: [num_listed * Hq] ranges finished, zero between calls
  int* claim;                       // shared: [num_seqs] blocks attended per sequence
  float2* part_ml;                  // shared: [num_listed * Hq][max_ranges]
  float* part_o;                    // shared: [num_listed * Hq][max_ranges][D]
  float2* pre_ml;                   // shared: [num_seqs * Hq]
  float* pre_o;                     // shared: [num_seqs * Hq][D]
  int32_t* err_flag;
  CUtensorMap tm_k;                 // caches as [num_blocks * Hkv * 16][D], boxes 16 x 64, SW128
  CUtensorMap tm_v;
};

__device__ __forceinline__ void seterr(const TcArgs& a, int bit) {
  if (a.err_flag) atomicOr(a.err_flag, bit);
}

// Prefill: the query rows of sequence s, or false (with the error bit to set
// in *bit, 0 if none) when it has none to compute.
__device__ __forceinline__ bool prefill_seq(const TcArgs& a, int s, int* q0, int* Q, int* n,
                                            int* bit) {
  *bit = 0;
  const int a0 = a.query_start[s], a1 = a.query_start[s + 1];
  if (!(0 <= a0 && a0 <= a1 && a1 <= a.num_query_rows)) {
    *bit = kErrQuery;
    return false;
  }
  *q0 = a0;
  *Q = a1 - a0;
  *n = a.context_lens[s];
  if (*Q == 0) return false;
  if (*n < 0 || *n > a.len_cap) {
    *bit = kErrContextLen;
    return false;
  }
  if (*Q > *n) {
    *bit = kErrQuery;
    return false;
  }
  return true;
}

// Shared: group g's members and shared blocks, if well formed.
__device__ __forceinline__ bool shared_group(const TcArgs& a, int g, int* gs, int* m, int* P,
                                             int* leader) {
  const int s0 = a.group_start[g], s1 = a.group_start[g + 1];
  if (!(0 <= s0 && s0 < s1 && s1 <= a.num_listed)) return false;
  const int p = a.group_blocks[g];
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
__global__ void __launch_bounds__(kPlanThreads) tc_plan_kernel(const __grid_constant__ TcArgs a) {
  // the attention kernel may start its prologue now
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ int s_wsum[kPlanThreads / 32];
  constexpr int RPT = kCols / G;  // query rows (members) per column tile
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int R = a.rows, Hkv = a.num_kv_heads, Hq = a.num_q_heads;
  const int per = (R + kPlanThreads - 1) / kPlanThreads;
  const int r0 = min(R, tid * per), r1 = min(R, r0 + per);
  int local = 0;
  for (int r = r0; r < r1; ++r) {
    int units = 0;
    if constexpr (MODE == kModePrefill) {
      int q0 = 0, Q = 0, n = 0, bit = 0;
      if (prefill_seq(a, r, &q0, &Q, &n, &bit)) {
        units = Hkv * ((Q + RPT - 1) / RPT);
      } else if (bit) {
        seterr(a, bit);
        if (bit != kErrQuery || (a.query_start[r] >= 0 && a.query_start[r] <= a.query_start[r + 1] &&
                                 a.query_start[r + 1] <= a.num_query_rows)) {
          // a sequence that cannot be computed: its (well-placed) rows are zero
          const int b0 = a.query_start[r], b1 = a.query_start[r + 1];
          uint4* dst = reinterpret_cast<uint4*>(a.out + static_cast<size_t>(b0) * Hq * D);
          const size_t cnt = static_cast<size_t>(b1 - b0) * Hq * D * 2 / 16;
          for (size_t i = 0; i < cnt; ++i) dst[i] = make_uint4(0, 0, 0, 0);
        }
      }
    } else {
      int gs, m, P, leader;
      if (shared_group(a, r, &gs, &m, &P, &leader)) {
        const int nct = (m * G + kCols - 1) / kCols;
        units = nct * Hkv * ((P + a.range_blocks - 1) / a.range_blocks);
      } else {
        seterr(a, kErrGroup);
      }
    }
    a.unit_start[r] = units;  // (turned into starts below)
    local += units;
  }
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) s_wsum[warp] = incl;
  __syncthreads();
  int run = incl - local, total = 0;
#pragma unroll
  for (int w = 0; w < kPlanThreads / 32; ++w) {
    if (w < warp) run += s_wsum[w];
    total += s_wsum[w];
  }
  // each row's units as records {row, kv head, column tile, last key + 1}
  // {prefill: first query row, rows, context length, 0 | shared: first
  // member, members, shared blocks, range | ranges << 16}, so that the
  // attention kernel finds a unit with one load instead of a search
  for (int r = r0; r < r1; ++r) {
    const int units = a.unit_start[r];
    a.unit_start[r] = run;
    if constexpr (MODE == kModePrefill) {
      int q0 = 0, Q = 0, n = 0, bit = 0;
      if (units > 0 && prefill_seq(a, r, &q0, &Q, &n, &bit)) {
        const int nct = (Q + RPT - 1) / RPT;
        for (int k = 0; k < units && run + k < a.max_units; ++k) {
          const int ct = k % nct, kvh = k / nct;
          const int jl = min(Q, (ct + 1) * RPT) - 1;  // the tile's last query row
          a.units[2 * (run + k)] = make_int4(r, kvh, ct, n - Q + jl + 1);
          a.units[2 * (run + k) + 1] = make_int4(q0, Q, n, 0);
        }
      }
    } else {
      int gs, m, P, leader;
      if (units > 0 && shared_group(a, r, &gs, &m, &P, &leader)) {
        const int nct = (m * G + kCols - 1) / kCols;
        const int Rr = (P + a.range_blocks - 1) / a.range_blocks;
        for (int k = 0; k < units && run + k < a.max_units; ++k) {
          const int ct = k % nct, kvh = (k / nct) % Hkv, rr = k / (nct * Hkv);
          const int k1 = min(P, (rr + 1) * a.range_blocks) * kBlockSize;
          a.units[2 * (run + k)] = make_int4(leader, kvh, ct, k1);
          a.units[2 * (run + k) + 1] = make_int4(gs, m, P, rr | (Rr << 16));
        }
      }
    }
    run += units;
  }
  if (tid == 0) {
    // (the workspace is sized for the most units a call can have)
    if (total > a.max_units) seterr(a, kErrTimeout);
    a.unit_start[R] = min(total, a.max_units);
  }
}

// ---------------------------------------------------------------------------
// the attention kernel
// ---------------------------------------------------------------------------
struct Unit {
  int row;    // block-table row
  int kvh;
  int ct;     // column tile
  int k0;     // first key of the unit
  int k1;     // one past its last key
  int nt;     // K/V tiles
  // prefill
  int q0, Q, n;
  // shared
  int gs, m, P, r, R;
};

// Work unit u from the plan kernel's records.  The plan kernel writes them
// while this grid may already be running (programmatic dependent launch), so
// they are read through L2 (ld.global.cg), never through the non-coherent
// read-only path: on B200 that path returned a previous call's records when a
// workspace was reused, and whole units went missing.
template <int MODE>
__device__ __forceinline__ void load_unit(const TcArgs& a, int u, Unit* x) {
  const int4 r0 = __ldcg(a.units + 2 * u), r1 = __ldcg(a.units + 2 * u + 1);
  x->row = r0.x;
  x->kvh = r0.y;
  x->ct = r0.z;
  x->k1 = r0.w;
  if constexpr (MODE == kModePrefill) {
    x->q0 = r1.x;
    x->Q = r1.y;
    x->n = r1.z;
    x->k0 = 0;
  } else {
    x->gs = r1.x;
    x->m = r1.y;
    x->P = r1.z;
    x->r = r1.w & 0xffff;
    x->R = r1.w >> 16;
    x->k0 = x->r * a.range_blocks * kBlockSize;
  }
  x->nt = (x->k1 - x->k0 + kKeys - 1) / kKeys;
}

// 2^x by the ex2.approx.ftz.f32 instruction.  Results below the smallest
// normal float flush to zero; the weights it makes are rounded to bf16 and
// are at most 2^8, so nothing of them is lost that the sum could see.
__device__ __forceinline__ float ex2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void* src, bool fill) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(fill ? 16 : 0)
               : "memory");
}

template <int D, int G, int MODE>
__global__ void __launch_bounds__(kThreads, 1) tc_attention_kernel(const __grid_constant__ TcArgs a) {
  constexpr int KB = D / 64;                 // 64-element (128-byte) blocks of head_dim
  constexpr int QT = kCols * D * 2;          // bytes of the Q tile
  constexpr int KT = kKeys * D * 2;          // bytes of a K (or V) tile
  constexpr int PT = kCols * kKeys * 2;      // bytes of the P tile
  constexpr int HALF = kKeys * 128;          // bytes of a 64-element half of a K/V tile
  constexpr int RPT = kCols / G;
  constexpr uint32_t IDESC_S = tc::idesc_bf16_f32(kCols, kKeys, false);
  constexpr uint32_t IDESC_O = tc::idesc_bf16_f32(kCols, D, true);
  static_assert(D == 64 || D == 128, "head_dim");

  extern __shared__ unsigned char smem_raw[];
  // 1024-byte alignment for the swizzled tiles
  unsigned char* sm = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  unsigned char* sQ = sm;
  unsigned char* sK = sQ + QT;               // [kStages][KT]
  unsigned char* sV = sK + kStages * KT;     // [kStages][KT]
  unsigned char* sP = sV + kStages * KT;     // [PT]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + PT);
  // barriers: kfull[2] kempty[2] vfull[2] vempty[2] sfull[2] pfull odone qfull drain sync
  const uint32_t b0 = smem_addr(bars);
  const uint32_t KFULL = b0, KEMPTY = b0 + 16, VFULL = b0 + 32, VEMPTY = b0 + 48, SFULL = b0 + 64;
  const uint32_t PFULL = b0 + 80, ODONE = b0 + 88, QFULL = b0 + 96, DRAIN = b0 + 104;
  const uint32_t SYNC = b0 + 112;  // the softmax threads among themselves (bounded, unlike bar.sync)
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ int s_red[3];
  __shared__ float s_xch[2][2][kCols];  // per half: row maxima of a tile / row sums of a unit
  // shared mode: the fold's member checks
  __shared__ int s_seq[kCols];
  __shared__ unsigned char s_ok[kCols];
  __shared__ int s_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Hq = a.num_q_heads, Hkv = a.num_kv_heads;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(KFULL + 8 * i, 1);
      mbar_init(KEMPTY + 8 * i, 1);
      mbar_init(VFULL + 8 * i, 1);
      mbar_init(VEMPTY + 8 * i, 1);
      mbar_init(SFULL + 8 * i, 1);
    }
    mbar_init(PFULL, kSoftmaxThreads);
    mbar_init(ODONE, 1);
    mbar_init(QFULL, kSoftmaxThreads);
    mbar_init(DRAIN, 1);
    mbar_init(SYNC, kSoftmaxThreads);
    s_abort = 0;
    s_red[0] = s_red[1] = s_red[2] = 0;
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
  const int total = __ldcg(a.unit_start + a.rows);  // (written by the plan kernel: see load_unit)

  auto timeout = [&]() {
    if (atomicExch(&s_abort, 1) == 0) seterr(a, kErrTimeout);
  };
  auto aborted_one = [&]() { return *reinterpret_cast<volatile int*>(&s_abort) != 0; };
  // (the producer and softmax warps test it with all lanes and act on one answer)
  auto aborted = [&]() { return __any_sync(0xffffffffu, aborted_one()); };

  if (warp == kProducerWarp) {
    // ---------------- producer: K runs one tile ahead of V ----------------------
    int kidx = 0, vidx = 0;
    int yprev = a.oob_row;  // (lane b < 8: tile row of block b of the previous tile)
    bool have_prev = false, ok = true;
    auto issue_v = [&](int ysrc) -> bool {
      const int st = vidx % kStages;
      if (vidx >= kStages &&
          !__all_sync(0xffffffffu, mbar_wait_bounded(VEMPTY + 8 * st, ((vidx / kStages) - 1) & 1)))
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
    Unit x, nx;
    if (blockIdx.x < total) load_unit<MODE>(a, blockIdx.x, &x);
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x, x = nx) {
      if (u + static_cast<int>(gridDim.x) < total) load_unit<MODE>(a, u + gridDim.x, &nx);
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
            !__all_sync(0xffffffffu, mbar_wait_bounded(KEMPTY + 8 * st, ((kidx / kStages) - 1) & 1))) {
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
      mbar_wait_bounded(KFULL + 8 * (i % kStages), (i / kStages) & 1);
    for (int i = max(0, vidx - kStages); i < vidx; ++i)
      mbar_wait_bounded(VFULL + 8 * (i % kStages), (i / kStages) & 1);
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issuer -------------------------------------------------
    if (lane == 0) {
      int kidx = 0, vidx = 0, sidx = 0, pidx = 0, qidx = 0;
      bool ok = true;
      const uint32_t qbase = smem_addr(sQ), pbase = smem_addr(sP);
      auto issue_s = [&]() -> bool {
        const int st = kidx % kStages;
        if (!mbar_wait_bounded(KFULL + 8 * st, (kidx / kStages) & 1)) return false;
        tc::fence_after_sync();
        const uint32_t kbase = smem_addr(sK + st * KT);
        const uint32_t dS = tmem + (sidx & 1) * kKeys;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k / 4) * (kCols * 128) + (k % 4) * 32;
          const uint32_t koff = (k / 4) * HALF + (k % 4) * 32;
          tc::mma_bf16_ss(dS, tc::sdesc_sw128(qbase + off, 16, 1024),
                          tc::sdesc_sw128(kbase + koff, 16, 1024), IDESC_S, k > 0);
        }
        tc::commit(KEMPTY + 8 * st);
        tc::commit(SFULL + 8 * (sidx & 1));
        ++kidx;
        ++sidx;
        return true;
      };
      Unit x, nx;
      if (blockIdx.x < total) load_unit<MODE>(a, blockIdx.x, &x);
      for (int u = blockIdx.x; u < total && ok; u += gridDim.x, x = nx) {
        if (u + static_cast<int>(gridDim.x) < total) load_unit<MODE>(a, u + gridDim.x, &nx);
        if (aborted_one() || !mbar_wait_bounded(QFULL, qidx & 1)) { ok = false; break; }
        ++qidx;
        tc::fence_after_sync();
        for (int j = 0; j < 2 && j < x.nt && ok; ++j) ok = issue_s();
        for (int j = 0; j < x.nt && ok; ++j) {
          if (aborted_one() || !mbar_wait_bounded(PFULL, pidx & 1)) { ok = false; break; }
          ++pidx;
          const int st = vidx % kStages;
          if (!mbar_wait_bounded(VFULL + 8 * st, (vidx / kStages) & 1)) { ok = false; break; }
          tc::fence_after_sync();
          const uint32_t vbase = smem_addr(sV + st * KT);
#pragma unroll
          for (int k = 0; k < kKeys / 16; ++k) {
            const uint32_t poff = (k / 4) * (kCols * 128) + (k % 4) * 32;
            tc::mma_bf16_ss(tmem + 2 * kKeys, tc::sdesc_sw128(pbase + poff, 16, 1024),
                            tc::sdesc_sw128(vbase + k * 16 * 128, HALF, 1024), IDESC_O,
                            (j > 0 || k > 0) ? 1u : 0u);
          }
          tc::commit(VEMPTY + 8 * st);
          tc::commit(ODONE);
          ++vidx;
          if (j + 2 < x.nt) ok = issue_s();
        }
      }
      if (!ok) timeout();
      // every MMA issued has completed before the TMEM can be freed
      tc::commit(DRAIN);
      mbar_wait_bounded(DRAIN, 0);
    }
    __syncwarp();
  } else {
    // ---------------- softmax: two threads per column -----------------------------
    // Thread t (0..255) serves column col = t % 128, which is TMEM lane col
    // (warps w and w + 4 share a lane quarter), and half hf = t / 128 of it:
    // keys 64 hf .. 64 hf + 63 of every tile, head_dim D/2 hf .. D/2 hf + D/2 - 1
    // of O, and its own share of the row sum.  The two threads of a column
    // swap their partial row maxima once per tile and their sums once per unit.
    const int col = tid % kCols, hf = tid / kCols;
    const int h = col % G;
    constexpr int HK = kKeys / 2;   // keys per thread and tile
    constexpr int HD = D / 2;       // O columns per thread
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp % 4) * 32) << 16);
    int sidx = 0, oidx = 0, tile = 0, syncs = 0, reds = 0, xs = 0;
    bool ok = true;
    // a bounded wait whose outcome the whole warp shares, so that no lane
    // leaves ahead of the others (the TMEM moves are warp-wide)
    auto wait_all = [&](uint32_t bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait_bounded(bar, parity));
    };
    auto group_sync = [&]() -> bool {
      mbar_arrive(SYNC);
      return wait_all(SYNC, (syncs++) & 1);
    };
    // OR of a flag over the softmax threads; slot reds % 3 is cleared two uses ahead
    auto group_or = [&](bool v, bool* res) -> bool {
      const int slot = reds % 3;
      if (v) atomicOr(&s_red[slot], 1);
      if (!group_sync()) return false;
      *res = *reinterpret_cast<volatile int*>(&s_red[slot]) != 0;
      if (tid == 0) s_red[(reds + 2) % 3] = 0;
      ++reds;
      return true;
    };
    // the other half's value of this column (the exchange slot alternates, so
    // that one sync per exchange suffices)
    auto swap_half = [&](float v, float* other) -> bool {
      const int sl = (xs++) & 1;
      s_xch[sl][hf][col] = v;
      if (!group_sync()) return false;
      *other = s_xch[sl][hf ^ 1][col];
      return true;
    };
    // this column's query row in unit y (-1: none), and the keys it sees
    auto column_of = [&](const Unit& y, int* kend) -> int {
      int qrow = -1;
      if constexpr (MODE == kModePrefill) {
        const int jr = y.ct * RPT + col / G;
        *kend = 0;
        if (jr < y.Q) {
          qrow = y.q0 + jr;
          *kend = min(y.k1, y.n - y.Q + jr + 1);
        }
      } else {
        const int member = y.ct * RPT + col / G;
        if (member < y.m) {
          const int seq = a.group_seqs[y.gs + member];
          if (seq >= 0 && seq < a.num_seqs) qrow = seq;
        }
        *kend = y.k1;
      }
      return qrow;
    };
    // this thread's half of its column's q row into the swizzled Q tile
    // (zeros for no row)
    auto load_q = [&](const Unit& y, int qrow) {
      const __nv_bfloat16* src =
          a.q + (static_cast<size_t>(qrow >= 0 ? qrow : 0) * Hq + y.kvh * G + h) * D;
      const uint32_t qb = smem_addr(sQ) + col * 128;
#pragma unroll
      for (int cc = 0; cc < D / 16; ++cc) {
        const int c = hf * (D / 16) + cc;  // 16-byte chunk of the row
        cp_async16_zfill(qb + (c / 8) * (kCols * 128) + (((c % 8) ^ (col % 8)) << 4), src + c * 8,
                         qrow >= 0);
      }
    };
    Unit x, nx;
    if (blockIdx.x < total) load_unit<MODE>(a, blockIdx.x, &x);
    bool q_issued = false;  // this unit's Q already requested (during the last unit)
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x, x = nx) {
      const bool has_next = u + static_cast<int>(gridDim.x) < total;
      if (has_next) load_unit<MODE>(a, u + gridDim.x, &nx);
      int kend;
      const int qrow = column_of(x, &kend);
      // ---- the unit's blocks must be in range (prefill: a bad one empties the sequence)
      bool bad = false;
      if constexpr (MODE == kModePrefill) {
        const int nb = (x.n + kBlockSize - 1) / kBlockSize;
        const int32_t* trow = a.block_tables + static_cast<size_t>(x.row) * a.max_blocks_per_seq;
        for (int b = tid; b < nb; b += kSoftmaxThreads) {
          const int phys = __ldg(trow + b);
          bad |= !(phys >= 0 && phys < a.num_blocks);
        }
        if (!group_or(bad, &bad)) { ok = false; break; }
        if (bad && tid == 0) seterr(a, kErrBlockId);
      }
      // ---- Q: requested now, or already during the previous unit's last tile
      if (!q_issued) load_q(x, qrow);
      q_issued = false;
      asm volatile("cp.async.wait_all;" ::: "memory");
      fence_proxy_async_smem();
      tc::fence_before_sync();
      mbar_arrive(QFULL);

      float m_run = -INFINITY, l_run = 0.f;
      for (int j = 0; j < x.nt; ++j, ++tile) {
        if (aborted() || !wait_all(SFULL + 8 * (sidx & 1), (sidx >> 1) & 1)) { ok = false; break; }
        tc::fence_after_sync();
        uint32_t sv[HK];
        tc::tmem_ld64(lane_base + (sidx & 1) * kKeys + hf * HK, sv);
        tc::tmem_wait_ld(sv);
        ++sidx;
        if (j == x.nt - 1 && has_next) {
          // every S of this unit is complete: the Q tile is free for the next unit
          int kn;
          load_q(nx, column_of(nx, &kn));
          q_issued = true;
        }
        // scale to log2 units, mask the keys this column does not see, and take
        // the maximum over 8 independent chains, then with the other half's
        const int kb = x.k0 + j * kKeys + hf * HK;
        float m8[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) m8[c] = -INFINITY;
        if (kb + HK <= kend) {
#pragma unroll
          for (int t = 0; t < HK; ++t) {
            const float v = __uint_as_float(sv[t]) * a.scale_log2;
            sv[t] = __float_as_uint(v);
            m8[t & 7] = fmaxf(m8[t & 7], v);
          }
        } else {
#pragma unroll
          for (int t = 0; t < HK; ++t) {
            const float v = kb + t < kend ? __uint_as_float(sv[t]) * a.scale_log2 : -INFINITY;
            sv[t] = __float_as_uint(v);
            m8[t & 7] = fmaxf(m8[t & 7], v);
          }
        }
        float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                         fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
        {
          float mo;
          if (!swap_half(mx, &mo)) { ok = false; break; }
          mx = fmaxf(mx, mo);  // (both halves now hold the same tile maximum)
        }
        if (j > 0) {
          // O of the previous tile is complete: its P slot is free and O is stable
          if (!wait_all(ODONE, oidx & 1)) { ok = false; break; }
          ++oidx;
          tc::fence_after_sync();
        }
        const bool grow = mx > m_run + kRescaleThreshold;
        float al = 1.f;
        if (grow) {
          al = ex2_fast(m_run - mx);  // (0 while nothing was seen)
          l_run *= al;
          m_run = mx;
        }
        // weights, rounded to bf16 for the product; the sum (8 chains) takes
        // them as rounded; this half's 64 keys are P's K-block hf
        const bool none = m_run == -INFINITY;
        const uint32_t pb = smem_addr(sP) + hf * (kCols * 128) + col * 128;
        float l8[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) l8[c] = 0.f;
#pragma unroll
        for (int c = 0; c < HK / 8; ++c) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float p0 = none ? 0.f : ex2_fast(__uint_as_float(sv[c * 8 + 2 * e]) - m_run);
            const float p1 = none ? 0.f : ex2_fast(__uint_as_float(sv[c * 8 + 2 * e + 1]) - m_run);
            const __nv_bfloat162 pp = __floats2bfloat162_rn(p0, p1);
            l8[2 * e] += __low2float(pp);
            l8[2 * e + 1] += __high2float(pp);
            w[e] = *reinterpret_cast<const uint32_t*>(&pp);
          }
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                           pb + (((c % 8) ^ (col % 8)) << 4)),
                       "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3])
                       : "memory");
        }
        l_run += ((l8[0] + l8[1]) + (l8[2] + l8[3])) + ((l8[4] + l8[5]) + (l8[6] + l8[7]));
        if constexpr (MODE == kModePrefill) {
          // rows past the sequence's end in its last block hold stale data: a
          // zero weight times a NaN would still poison O, so they are zeroed
          const int tail = x.n % kBlockSize;
          const int lastb = x.n / kBlockSize;        // logical block holding them
          const int kt = x.k0 + j * kKeys;           // the tile's first key
          if (tail && lastb * kBlockSize >= kt && lastb * kBlockSize < kt + kKeys) {
            const int st = tile % kStages;
            if (!wait_all(VFULL + 8 * st, (tile / kStages) & 1)) { ok = false; break; }
            const int b = (lastb * kBlockSize - kt) / kBlockSize;
            unsigned char* vt = sV + st * KT;
            const int nz = (kBlockSize - tail) * 8 * KB;  // 16-byte chunks to clear
            for (int i = tid; i < nz; i += kSoftmaxThreads) {
              const int hx = i / ((kBlockSize - tail) * 8);
              const int rem = i % ((kBlockSize - tail) * 8);
              const int row = b * kBlockSize + tail + rem / 8;
              *reinterpret_cast<uint4*>(vt + hx * HALF + row * 128 + (((rem % 8) ^ (row % 8)) << 4)) =
                  make_uint4(0, 0, 0, 0);
            }
          }
        }
        // this half of the O row is rescaled by the whole warp together (the
        // TMEM moves are warp-wide; rows that do not grow are multiplied by 1),
        // after the S row is spent and before P is released to the MMA
        if (j > 0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll 1
          for (int c = 0; c < HD / 32; ++c) {
            uint32_t r[32];
            tc::tmem_ld32(lane_base + 2 * kKeys + hf * HD + c * 32, r);
            tc::tmem_wait_ld(r);
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * al);
            tc::tmem_st32(lane_base + 2 * kKeys + hf * HD + c * 32, r);
          }
          tc::tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc::fence_before_sync();
        mbar_arrive(PFULL);
      }
      if (!ok) break;
      // ---- the unit's O row: this thread's half, over the column's whole sum
      if (!wait_all(ODONE, oidx & 1)) { ok = false; break; }
      ++oidx;
      tc::fence_after_sync();
      float lo;
      if (!swap_half(l_run, &lo)) { ok = false; break; }
      const float l_all = l_run + lo;
      uint32_t ov[HD];
      if constexpr (HD == 64) tc::tmem_ld64(lane_base + 2 * kKeys + hf * HD, ov);
      else tc::tmem_ld32(lane_base + 2 * kKeys + hf * HD, ov);
      tc::tmem_wait_ld(ov);
      if constexpr (MODE == kModePrefill) {
        // (every lane ran the warp-wide TMEM load; only live columns store)
        if (qrow >= 0) {
          const float inv = bad ? 0.f : 1.f / l_all;
          uint4* dst = reinterpret_cast<uint4*>(
              a.out + (static_cast<size_t>(qrow) * Hq + x.kvh * G + h) * D + hf * HD);
#pragma unroll
          for (int c = 0; c < HD / 8; ++c) {
            uint32_t w[4];
#pragma unroll
            for (int f = 0; f < 4; ++f) {
              const __nv_bfloat162 pp = __floats2bfloat162_rn(
                  __uint_as_float(ov[c * 8 + 2 * f]) * inv, __uint_as_float(ov[c * 8 + 2 * f + 1]) * inv);
              w[f] = *reinterpret_cast<const uint32_t*>(&pp);
            }
            dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      } else {
        // ---- shared: this range's partial state, then the fold by the last range
        const int member = x.ct * RPT + col / G;
        const bool live = member < x.m;
        const size_t pi = live ? (static_cast<size_t>(x.gs + member) * Hq + x.kvh * G + h) *
                                         a.max_ranges + x.r
                               : 0;
        if (live) {
          float4* po = reinterpret_cast<float4*>(a.part_o + pi * D + hf * HD);
#pragma unroll
          for (int e = 0; e < HD / 4; ++e)
            po[e] = make_float4(__uint_as_float(ov[4 * e]), __uint_as_float(ov[4 * e + 1]),
                                __uint_as_float(ov[4 * e + 2]), __uint_as_float(ov[4 * e + 3]));
          if (hf == 0) a.part_ml[pi] = make_float2(m_run, l_all);
        }
        __threadfence();
        if (!group_sync()) { ok = false; break; }
        if (tid == 0) {
          int* cnt = a.counters + (static_cast<size_t>(x.gs) * G + x.ct * kCols) * Hkv + x.kvh;
          const int prev = atomicAdd(cnt, 1);
          s_last = prev == x.R - 1;
          if (s_last) *cnt = 0;  // every range has arrived: zero again for the next call
        }
        if (!group_sync()) { ok = false; break; }
        if (*reinterpret_cast<volatile int*>(&s_last)) {
          __threadfence();
          const int mlo = x.ct * RPT;
          const int nm = min(x.m - mlo, RPT);  // members of this tile
          const int32_t* lrow = a.block_tables + static_cast<size_t>(x.row) * a.max_blocks_per_seq;
          if (tid < nm) {
            const int seq = a.group_seqs[x.gs + mlo + tid];
            bool okm = seq >= 0 && seq < a.num_seqs;
            if (okm) {
              const int n = a.context_lens[seq];
              okm = n > 0 && n <= a.len_cap && kBlockSize * x.P <= n - 1;
            }
            s_seq[tid] = okm ? seq : -1;
            s_ok[tid] = okm;
          }
          if (!group_sync()) { ok = false; break; }
          // every (member, shared block): the member's table holds the leader's block
          for (int idx = tid; idx < nm * x.P; idx += kSoftmaxThreads) {
            const int i = idx / x.P, jb = idx - i * x.P;
            const int seq = s_seq[i];
            if (seq < 0) continue;
            const int b = __ldg(lrow + jb);
            if (!(b >= 0 && b < a.num_blocks &&
                  __ldg(a.block_tables + static_cast<size_t>(seq) * a.max_blocks_per_seq + jb) == b))
              s_ok[i] = 0;  // (every writer stores the same value)
          }
          if (!group_sync()) { ok = false; break; }
          if (x.kvh == 0 && tid < nm && !s_ok[tid]) seterr(a, kErrGroup);
          if (live && s_ok[col / G]) {
            // this thread folds its half of the column's head_dim
            const size_t pb0 = (static_cast<size_t>(x.gs + member) * Hq + x.kvh * G + h) * a.max_ranges;
            float M = -INFINITY;
            for (int rr = 0; rr < x.R; ++rr) M = fmaxf(M, __ldcg(a.part_ml + pb0 + rr).x);
            const size_t orow = static_cast<size_t>(s_seq[col / G]) * Hq + x.kvh * G + h;
            // (in passes of 32 dims, to keep the accumulators in registers)
            constexpr int QD = HD < 32 ? HD : 32;
            float L = 0.f;
#pragma unroll 1
            for (int q0 = 0; q0 < HD; q0 += QD) {
              float4 acc[QD / 4];
#pragma unroll
              for (int e = 0; e < QD / 4; ++e) acc[e] = make_float4(0.f, 0.f, 0.f, 0.f);
              L = 0.f;
              for (int rr = 0; rr < x.R; ++rr) {
                const float2 ml = __ldcg(a.part_ml + pb0 + rr);
                const float w = ml.x == -INFINITY ? 0.f : exp2f(ml.x - M);
                L += w * ml.y;
                const float4* po =
                    reinterpret_cast<const float4*>(a.part_o + (pb0 + rr) * D + hf * HD + q0);
#pragma unroll
                for (int e = 0; e < QD / 4; ++e) {
                  const float4 o4 = __ldcg(po + e);
                  acc[e].x = fmaf(w, o4.x, acc[e].x);
                  acc[e].y = fmaf(w, o4.y, acc[e].y);
                  acc[e].z = fmaf(w, o4.z, acc[e].z);
                  acc[e].w = fmaf(w, o4.w, acc[e].w);
                }
              }
              float4* dst = reinterpret_cast<float4*>(a.pre_o + orow * D + hf * HD + q0);
#pragma unroll
              for (int e = 0; e < QD / 4; ++e) dst[e] = acc[e];
            }
            if (hf == 0) a.pre_ml[orow] = make_float2(M, L);
          }
          // claim each checked member once (KV head 0; a member's columns all
          // lie in one tile, since 128 is a multiple of G); a sequence claimed
          // twice is given up
          if (x.kvh == 0 && tid < nm && s_ok[tid]) {
            const int seq = s_seq[tid];
            if (atomicCAS(a.claim + seq, 0, x.P) != 0) {
              atomicExch(a.claim + seq, -1);
              seterr(a, kErrGroup);
            }
          }
          if (!group_sync()) { ok = false; break; }  // (s_ok, s_seq rewritten next unit)
        }
      }
    }
    if (!ok) timeout();
    asm volatile("cp.async.wait_all;" ::: "memory");  // (a prefetch left in flight by an abort)
  }

  // ---- teardown: every role is out of its loop; the MMAs have drained -------
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == kMmaWarp) tc::tmem_dealloc(tmem, kTmemCols);
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

size_t tc_smem_bytes(int head_dim) {
  const size_t q = static_cast<size_t>(kCols) * head_dim * 2;
  const size_t kv = static_cast<size_t>(kKeys) * head_dim * 2;
  const size_t p = static_cast<size_t>(kCols) * kKeys * 2;
  return 1024 + q + 2 * kStages * kv + p + 128;  // (alignment slack, barriers)
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

// plan kernel, then the attention kernel behind it (programmatic dependent launch)
cudaError_t launch_pair(const void* plan, const void* main, TcArgs& a, int grid, size_t smem,
                        cudaStream_t stream) {
  cudaError_t e = prepare(main, smem);
  if (e != cudaSuccess) return e;
  void* params[] = {&a};
  if ((e = cudaLaunchKernel(plan, dim3(1), dim3(kPlanThreads), params, 0, stream)) != cudaSuccess)
    return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, main, params);
}

}  // namespace

bool tc_prefill_supported(int head_dim, int group) {
  const void *p, *m;
  return pick<kModePrefill>(head_dim, group, &p, &m);
}

// Most work units a prefill call can have: each sequence's column tiles,
// ceil(Q_s * G / 128) <= Q_s * G / 128 + 1, for every KV head.
static long long prefill_max_units(int num_seqs, int num_query_tokens, int num_q_heads,
                                   int num_kv_heads) {
  const long long G = num_q_heads / num_kv_heads;
  return static_cast<long long>(num_kv_heads) *
         ((static_cast<long long>(num_query_tokens) * G + kCols - 1) / kCols + num_seqs);
}
static size_t prefill_records_offset(int num_seqs) {
  return ((static_cast<size_t>(num_seqs) + 1) * sizeof(int) + 255) / 256 * 256;
}

size_t tc_prefill_workspace_bytes(int num_seqs, int num_query_tokens, int num_q_heads,
                                  int num_kv_heads) {
  return prefill_records_offset(num_seqs) +
         static_cast<size_t>(prefill_max_units(num_seqs, num_query_tokens, num_q_heads,
                                               num_kv_heads)) * 2 * sizeof(int4);
}

int tc_launch_smem(int head_dim) { return static_cast<int>(tc_smem_bytes(head_dim)); }

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
  a.scale_log2 = l.scale_log2;
  a.unit_start = static_cast<int*>(l.workspace);
  a.units = reinterpret_cast<int4*>(static_cast<char*>(l.workspace) +
                                    prefill_records_offset(l.num_seqs));
  a.max_units = static_cast<int>(std::min<long long>(
      prefill_max_units(l.num_seqs, l.num_query_rows, l.num_q_heads, l.num_kv_heads), 1 << 30));
  a.err_flag = l.err_flag;
  a.tm_k = *l.tm_k;
  a.tm_v = *l.tm_v;
  return launch_pair(plan, main, a, num_sms, tc_smem_bytes(l.head_dim), stream);
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
  // ranges of shared blocks: whole K/V tiles, at least 4 of them, and about
  // enough units to fill the SMs from the fewest column tiles the groups form
  const long long tiles =
      std::max(1LL, (static_cast<long long>(l.num_listed) * group + kCols - 1) / kCols);
  const long long per = std::max(1LL, num_sms / (tiles * l.num_kv_heads));
  long long rb = (l.max_blocks_per_seq + per - 1) / per;
  rb = std::max<long long>(rb, 4 * kTileBlocks);
  rb = (rb + kTileBlocks - 1) / kTileBlocks * kTileBlocks;
  // ... and no more ranges than the partial arrays hold
  while ((l.max_blocks_per_seq + rb - 1) / rb > l.max_ranges) rb += kTileBlocks;
  a.range_blocks = static_cast<int>(rb);
  a.unit_start = l.unit_start;
  a.units = l.units;
  a.max_units = l.max_units;
  a.counters = l.counters;
  a.claim = l.claim;
  a.part_ml = l.part_ml;
  a.part_o = l.part_o;
  a.pre_ml = l.pre_ml;
  a.pre_o = l.pre_o;
  a.err_flag = l.err_flag;
  a.tm_k = *l.tm_k;
  a.tm_v = *l.tm_v;
  return launch_pair(plan, main, a, num_sms, tc_smem_bytes(l.head_dim), stream);
}

}  // namespace pa
