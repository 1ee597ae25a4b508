// decode_kernel.cuh -- PagedAttention decode for sm_100a.
//
// What it computes: for every sequence s and query head h, softmax attention
// of q[s][h] over the context_lens[s] cached tokens, each token found through
// the sequence's block table, wherever in the pool its block lies ("What vLLM
// Is and Why It Exists", section "The idea vLLM started from: pages").
//
// How (B200 design):
//  * Work unit = one (sequence, KV head, block) tile: 16 tokens x head_dim,
//    contiguous in the cache, read once for all G = Hq/Hkv query heads that
//    share the KV head.  All units are laid end to end in (seq, kv head,
//    block) order and cut into equal contiguous ranges, one or more per
//    worker of a persistent grid (as many CTAs as fit on the 148 SMs): every
//    worker gets the same number of tiles however skewed the lengths are.
//    A worker is one warp, or on the CUDA-core path with G = 8, HS = 2 warps
//    that split the query heads of a tile between them.
//  * Each worker streams its tiles through a ring of DEPTH shared-memory
//    slots filled by its leader warp: 1-D bulk copies (cp.async.bulk) of the
//    live rows on the CUDA-core path, 2-D tensor loads of whole 16-row tiles
//    with the 128-byte swizzle on the tensor-core path; a "full" mbarrier per
//    slot completes by byte count, an "empty" one per slot when two warps
//    share it.  Block-table entries for the next 32-64 tiles are loaded one
//    per lane well ahead of use, and each slot's descriptor travels with it
//    through shared memory.
//  * Fused slot write (when key/value are given): the newest row of each
//    (sequence, KV head) is fetched from key/value instead of the cache, and
//    the leader writes it from shared memory to its cache slot.
//  * Arithmetic: fp32 on the CUDA cores for G <= 4 and for fp32 caches (a
//    one-token query is a bandwidth-bound gather): lanes split head_dim 16
//    bytes at a time, partial dot products are combined by a butterfly
//    reduce-scatter of warp shuffles, the softmax is online (base 2, rescaled
//    only when the running max grows by more than 2^8), and P.V accumulates
//    in registers.  bf16 with G = 8 runs on the tensor cores (mma.sync,
//    fp32 accumulation): 16 tokens x 8 heads per tile is exactly one MMA
//    shape, and the CUDA cores alone would be bound by issue there.
//  * A (seq, kv head) cut by a range boundary leaves partial results (m, l,
//    o) in the workspace; its first piece lists the item, and a second,
//    programmatically dependent kernel merges the pieces by log-sum-exp.
//    (The CUDA-core path can instead merge few-piece items in the warp that
//    finishes the last piece, behind PA_FUSE_MAX_VALUES; off by default.)
//  * Several query tokens per sequence (prefill): items are query rows, or
//    on the tensor-core path pairs of rows (NR = 2), each over its own
//    causal prefix, found on chip from query_start.
//  * Shared-prefix continuation (pre_blocks): a sequence's first blocks were
//    attended by the shared-prefix pass; the kernel walks the rest and
//    starts the item from that pass's state.
//  * Device-side index checks skip bad items and set err_flag bits; every
//    wait is bounded.
#pragma once

#include <cstdint>
#include <type_traits>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "pa_internal.h"
#include "ptx.cuh"

namespace pa {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kMaxOwnRanges = 4;  // range starts a warp keeps in shared memory

// Order the warps' generic reads of a ring slot before the bulk copy that
// refills it.  Only reads (never generic writes) touch the slots, and every
// refill follows the release of the slot, so the barrier hand-off alone
// orders them as in the usual producer/consumer pipelines; the fence is kept
// as a build option.
#ifndef PA_PROXY_FENCE
#define PA_PROXY_FENCE 1
#endif
constexpr bool kProxyFence = PA_PROXY_FENCE != 0;

// K/V tiles are read once per call: loaded under the L2 evict-first policy
// (1), the partial results the merge pass reads back stay in L2 instead of
// being pushed out by the stream; 0 loads them under the default policy.
// Measured on B200 (fraction of the copy peak, decode + merge): 7b 0.784 ->
// 0.802, gqa70b 0.736 -> 0.759, long 0.869 -> 0.882; a shared prefix re-read
// by many sequences loses a little (prefix_cow 0.928 -> 0.916).
#ifndef PA_KV_EVICT_FIRST
#define PA_KV_EVICT_FIRST 1
#endif
constexpr bool kKvEvictFirst = PA_KV_EVICT_FIRST != 0;

// -- element conversion ---------------------------------------------------------
template <typename T>
struct Elem;

template <>
struct Elem<float> {
  __device__ __forceinline__ static void unpack(const uint4& r, float* f) {
    f[0] = __uint_as_float(r.x);
    f[1] = __uint_as_float(r.y);
    f[2] = __uint_as_float(r.z);
    f[3] = __uint_as_float(r.w);
  }
  __device__ __forceinline__ static uint4 pack(const float* f) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
  }
};

template <>
struct Elem<__nv_bfloat16> {
  // bf16 -> fp32 is exact: the bf16 pattern is the high half of the fp32 one.
  __device__ __forceinline__ static void unpack(const uint4& r, float* f) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  __device__ __forceinline__ static uint4 pack(const float* f) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 b = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&b);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
  }
};

// -- the two inner loops, on packed fp32 pairs (sm_100 FFMA2) or scalar FMAs ---
#ifndef PA_PACKED_FMA
#define PA_PACKED_FMA 1
#endif

// sum_e q[e] * k[e] over one lane's VEC elements
template <int VEC>
__device__ __forceinline__ float dot_vec(const float* q, const float* k) {
#if PA_PACKED_FMA
  float2 acc = __fmul2_rn(make_float2(q[0], q[1]), make_float2(k[0], k[1]));
#pragma unroll
  for (int j = 1; j < VEC / 2; ++j)
    acc = __ffma2_rn(make_float2(q[2 * j], q[2 * j + 1]), make_float2(k[2 * j], k[2 * j + 1]), acc);
  return acc.x + acc.y;
#else
  float acc = 0.f;
#pragma unroll
  for (int e = 0; e < VEC; ++e) acc = fmaf(q[e], k[e], acc);
  return acc;
#endif
}

// o[e] += p * v[e]
template <int VEC>
__device__ __forceinline__ void axpy_vec(float p, const float* v, float* o) {
#if PA_PACKED_FMA
  const float2 pp = make_float2(p, p);
#pragma unroll
  for (int j = 0; j < VEC / 2; ++j) {
    const float2 r =
        __ffma2_rn(pp, make_float2(v[2 * j], v[2 * j + 1]), make_float2(o[2 * j], o[2 * j + 1]));
    o[2 * j] = r.x;
    o[2 * j + 1] = r.y;
  }
#else
#pragma unroll
  for (int e = 0; e < VEC; ++e) o[e] = fmaf(p, v[e], o[e]);
#endif
}

// o[e] *= s
template <int VEC>
__device__ __forceinline__ void scale_vec(float s, float* o) {
#if PA_PACKED_FMA
  const float2 ss = make_float2(s, s);
#pragma unroll
  for (int j = 0; j < VEC / 2; ++j) {
    const float2 r = __fmul2_rn(ss, make_float2(o[2 * j], o[2 * j + 1]));
    o[2 * j] = r.x;
    o[2 * j + 1] = r.y;
  }
#else
#pragma unroll
  for (int e = 0; e < VEC; ++e) o[e] *= s;
#endif
}

constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }
constexpr int cmin(int a, int b) { return a < b ? a : b; }

// -- compile-time geometry --------------------------------------------------------
// MMA: the tensor-core layout of a slot -- K and V tiles as 128-byte-swizzled
// boxes (1024-byte aligned), then q, then a staging row pair for the fused
// slot write -- padded to a multiple of 1024 bytes.
template <typename T, int D, int G, int GT, int HS, int DEPTH, int WARPS, bool MMA = false,
          int NR = 1>
struct DecodeCfg {
  static constexpr int EB = sizeof(T);
  static constexpr int ROW = D * EB;          // bytes of one token's row of one KV head
  static constexpr int VEC = 16 / EB;         // elements a lane holds per row
  static constexpr int LPR = D / VEC;         // lanes per row
  static constexpr int RPI = 32 / LPR;        // rows one warp instruction covers (row groups)
  static constexpr int RL = kBlockSize / RPI; // rows per lane per block
  static constexpr int TILE = kBlockSize * ROW;
  static constexpr int QB = NR * GT * ROW;    // q rows of the whole group (of NR query rows)
  static constexpr int APP = 2 * TILE + QB;   // MMA: staging for the new K and V rows
  static constexpr int SLOT =
      MMA ? ((2 * TILE + QB + 2 * ROW + 1023) / 1024) * 1024 : 2 * TILE + QB;  // K, V, q (, rows)
  static constexpr int XS = kBlockSize * G * 4;
  static constexpr int ALPHA = ((G * 4 + 15) / 16) * 16;
  static constexpr int BND = (kMaxOwnRanges + 1) * 8;
  static constexpr int AUX = XS + ALPHA + BND;        // per warp
  static constexpr int BAR_OFF = DEPTH * SLOT;         // full[DEPTH], empty[DEPTH]
  static constexpr int DESC_OFF = BAR_OFF + 2 * DEPTH * 8;  // one descriptor per slot
  static constexpr int AUX_OFF = DESC_OFF + DEPTH * 16;
  static constexpr int WALIGN = MMA ? 1024 : 128;
  static constexpr int WORKER_BYTES = ((AUX_OFF + HS * AUX + WALIGN - 1) / WALIGN) * WALIGN;
  // (MMA: plus slack to align the dynamic shared memory base to 1024 bytes)
  static constexpr int CTA_BYTES = (WARPS / HS) * WORKER_BYTES + (MMA ? 1024 : 0);
  static constexpr int MT = D / 16;  // MMA: 16-wide slices of head_dim
  // QK is done CH rows at a time; V = CH*G partial dots are reduce-scattered
  // over the LPR lanes of a row, leaving NV finished logits per lane.
  static constexpr int CH = cmin(RL, LPR / G >= 1 ? LPR / G : 1);
  static constexpr int NCH = RL / CH;
  static constexpr int V = CH * G;
  static constexpr int LS = ilog2(LPR);
  static constexpr int LV = ilog2(V);
  static constexpr int LG = ilog2(G);
  static constexpr int LSC = cmin(LS, LV);
  static constexpr int NV = V >> LSC;
  static constexpr int TPL = G >= 2 ? G / 2 : 1;  // softmax tokens per lane
  static_assert(VEC * LPR == D, "head_dim must be a multiple of 16 bytes");
  static_assert(RPI * LPR == 32 && RL * RPI == kBlockSize, "bad lane geometry");
  static_assert(NCH * CH == RL, "bad chunking");
  static_assert(32 % G == 0 && G <= 16 && GT == G * HS, "group size");
  static_assert(!MMA || (EB == 2 && GT == 8 && HS == 1 && D % 64 == 0),
                "the tensor-core path takes bf16, 8 heads per KV head, one warp per worker");
  static_assert(NR == 1 || (MMA && NR <= 2), "several query rows per item: tensor-core path");
};

// -- per-warp ranges of the global tile order ------------------------------------
struct Ranges {
  long long W;   // tiles in total
  long long Ws;  // the static part [0, Ws) is cut into Rs ranges, one or more per worker
  long long Rs;
  long long CS;  // the rest [Ws, W) is cut into chunks of CS tiles, claimed at run time
  long long R;   // all ranges: Rs static + ceil((W - Ws) / CS) chunks
  __device__ __forceinline__ long long start(long long r) const {
    if (r <= Rs) return Rs ? r * Ws / Rs : 0;
    const long long x = Ws + (r - Rs) * CS;
    return x < W ? x : W;
  }
  __device__ __forceinline__ long long of(long long x) const {
    return x < Ws ? ((x + 1) * Rs - 1) / Ws : Rs + (x - Ws) / CS;
  }
  __device__ __forceinline__ bool is_start(long long x) const {
    if (x <= 0 || x >= W) return true;
    return x < Ws ? start(of(x)) == x : (x - Ws) % CS == 0;
  }
};

// Starts of the ranges one warp owns, kept in shared memory so that the
// per-tile "does a range start here" test needs no 64-bit division.
struct OwnRanges {
  const long long* b;  // b[0] = first tile of the warp ... b[n] = one past its last
  int n;               // ranges owned; 0 = more than kMaxOwnRanges (fall back to division)
  __device__ __forceinline__ bool is_start(long long x, const Ranges& rg) const {
    if (n == 0 || x < b[0] || x > b[n]) return rg.is_start(x);
    int l = 0, u = n;
    while (l < u) {
      const int m = (l + u) >> 1;
      if (b[m] < x) l = m + 1; else u = m;
    }
    return b[l] == x;
  }
};

// The cut of W tiles: the first part into static ranges (one per worker, or
// more so that none exceeds part_blocks tiles), the last part (tail_tiles)
// into chunks of chunk_tiles that workers claim as they run out of static
// work, so that slower SMs end up with less of it.
constexpr int kClaimAhead = 4;  // positions the leader keeps assigned beyond its refill point

__device__ __forceinline__ Ranges make_ranges(long long W, long long workers, int part_blocks) {
  Ranges rg;
  rg.W = W;
  rg.CS = chunk_tiles(part_blocks);
  rg.Ws = W - tail_tiles(W, workers);
  long long Rs = workers;
  if (part_blocks > 0) {
    const long long per = workers * part_blocks;
    Rs = workers * max(1LL, (rg.Ws + per - 1) / per);
  }
  rg.Rs = Rs < rg.Ws ? Rs : rg.Ws;
  rg.R = rg.Rs + (W - rg.Ws + rg.CS - 1) / rg.CS;
  return rg;
}

// Partial-result slot of the piece of item [item_a, ...) that lies in range r.
__device__ __forceinline__ long long piece_slot(const Ranges& rg, long long r, long long item_a) {
  return 2 * r + (item_a <= rg.start(r) ? 0 : 1);
}

// One tile of a warp's stream, as 3 words (kept one per lane, 32 tiles per batch).
struct __align__(16) StageDesc {
  int phys;  // physical block id (0 if bad)
  int seq;
  int meta;  // kv head (bits 0-15) | live rows (16-20) | flags
  int g;     // tile index in the global order
};
constexpr int kFirst = 1 << 24;  // first tile of a piece: reset state, fetch q
constexpr int kLast = 1 << 25;   // last tile of a piece: finish it
constexpr int kBad = 1 << 26;    // block-table entry out of range
constexpr int kEnd = 1 << 27;    // no more tiles: the partner warp stops
constexpr int kAppend = 1 << 28; // fused append: the tile's last live row is the new token
constexpr int kPrefix = 1 << 29; // first tile of an item that continues a shared-prefix state

__device__ __forceinline__ StageDesc make_desc(long long g, long long hi, const int* s_start,
                                               const int* s_len, const int* s_row,
                                               const Ranges& rg,
                                               const OwnRanges& own, const DecodeArgs& a) {
  StageDesc d{0, 0, 0, 0};
  if (g >= hi) return d;
  // largest s with s_start[s] <= g (sequences without blocks share their start)
  int lo = 0, up = a.num_seqs - 1;
  while (lo < up) {
    const int mid = (lo + up + 1) >> 1;
    if (s_start[mid] <= g) lo = mid; else up = mid - 1;
  }
  const int s = lo;
  const int n = s_len[s];
  const int nb = (n + kBlockSize - 1) / kBlockSize;
  const int off = static_cast<int>(g - s_start[s]);
  const int kvh = off / nb;
  const int blk = off - kvh * nb;
  const long long item_a = s_start[s] + static_cast<long long>(kvh) * nb;
  int flags = 0;
  if (g == item_a || own.is_start(g, rg)) flags |= kFirst;
  if (g + 1 == item_a + nb || own.is_start(g + 1, rg)) flags |= kLast;
  const int trow = s_row ? s_row[s] : s;  // (query rows share their sequence's table)
  // (shared-prefix decode: the sequence's first boff blocks were attended
  // already; read beside the table entry rather than kept on chip, which
  // would cost the CTA shared memory per sequence)
  const int boff = a.pre_blocks ? max(__ldg(a.pre_blocks + s), 0) : 0;
  if (boff > 0 && g == item_a) flags |= kPrefix;
  int phys = __ldg(a.block_tables + static_cast<size_t>(trow) * a.max_blocks_per_seq + boff + blk);
  if (phys < 0 || phys >= a.num_blocks) {
    flags |= kBad;
    phys = 0;
    if (a.err_flag) atomicOr(a.err_flag, kErrBlockId);
  }
  const int rows = min(kBlockSize, n - blk * kBlockSize);
  if (a.key && blk == nb - 1 && !(flags & kBad)) flags |= kAppend;
  d.phys = phys;
  d.seq = s;
  d.meta = kvh | (rows << 16) | flags;
  d.g = static_cast<int>(g);
  return d;
}

__device__ __forceinline__ StageDesc pick_desc(const StageDesc& A, const StageDesc& B, int rel) {
  const bool in_a = rel < 32;
  const int src = rel & 31;
  StageDesc d;
  d.phys = __shfl_sync(kFull, in_a ? A.phys : B.phys, src);
  d.seq = __shfl_sync(kFull, in_a ? A.seq : B.seq, src);
  d.meta = __shfl_sync(kFull, in_a ? A.meta : B.meta, src);
  d.g = __shfl_sync(kFull, in_a ? A.g : B.g, src);
  return d;
}

// Butterfly reduce-scatter of V values over the LPR lanes of a row group.
// Each lane computes its partials in a lane-dependent order (array index f
// holds logical index f ^ mask, mask = the lane's bits above the kept part),
// so at every stage all lanes keep the lower half and send the upper half:
// no per-element selects.  Afterwards v[0..NV) of lane dl hold complete sums
// of logical indices (dl >> (LS - LSC)) * NV + r.
template <int LPR, int V>
__device__ __forceinline__ void reduce_scatter(float (&v)[V]) {
#pragma unroll
  for (int st = 0; (1 << st) < LPR; ++st) {
    const int o = LPR >> (st + 1);
    const int len = V >> st;
    if (len >= 2) {
#pragma unroll
      for (int i = 0; i < len / 2; ++i) v[i] += __shfl_xor_sync(kFull, v[len / 2 + i], o);
    } else {
      v[0] += __shfl_xor_sync(kFull, v[0], o);
    }
  }
}

// One "worker" = HS warps that stream the same tiles through one ring and
// split the query heads of the group between them (HS = 2 halves the
// registers each warp needs when the group is large).  The first warp of a
// worker (the leader) issues the copies; every warp waits on the slot's
// "full" barrier and releases the slot on its "empty" barrier, which the
// leader waits on (bounded) before refilling the slot.
// NR > 1 (tensor-core path, several query tokens per sequence only): an item
// is a group of NR consecutive query rows of one sequence, whose 8 x NR
// (row, head) columns share every K/V tile of the group's longest prefix.
template <typename T, int D, int GT, int HS, int DEPTH, int WARPS, int MIN_CTAS, bool MMA = false,
          int NR = 1>
__global__ void __launch_bounds__(WARPS * 32, MIN_CTAS)
paged_decode_kernel(const __grid_constant__ DecodeArgs a) {
  constexpr int G = GT / HS;  // query heads handled by one warp
  using C = DecodeCfg<T, D, G, GT, HS, DEPTH, WARPS, MMA, NR>;
  using E = Elem<T>;
  static_assert(WARPS % HS == 0, "warps per CTA must be a multiple of the head split");
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_wsum[WARPS];

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int half = warp % HS;      // which share of the heads this warp computes
  const int hoff = half * G;       // first head (within the group) of that share
  const bool leader = half == 0;
  const int S = a.num_seqs;
  const int Hkv = a.num_kv_heads;
  const int Hq = a.num_q_heads;
  constexpr int WORKERS = WARPS / HS;
  // the swizzled tiles of the tensor-core path need 1024-byte alignment
  unsigned char* sbase = MMA ? smem + ((1024u - (smem_addr(smem) & 1023u)) & 1023u) : smem;
  unsigned char* wkbase = sbase + (warp / HS) * C::WORKER_BYTES;
  unsigned char* aux = wkbase + C::AUX_OFF + half * C::AUX;
  const uint32_t slot0 = smem_addr(wkbase);
  const uint32_t full0 = smem_addr(wkbase + C::BAR_OFF);
  const uint32_t empty0 = full0 + 8 * DEPTH;
  int* s_start = reinterpret_cast<int*>(sbase + WORKERS * C::WORKER_BYTES);  // [S + 1]
  int* s_len = s_start + S + 1;                                              // [S]
  // several query tokens per sequence: table row of each query row, query_start
  const bool prefill = a.query_start != nullptr;
  int* s_row = prefill ? s_len + S : nullptr;                                // [S]
  int* s_qs = s_len + 2 * S;                                                 // [rows + 1]
  // NR > 1: first query row | (rows << 24) of each group; first group of each sequence
  int* s_r0 = s_qs + a.num_table_rows + 1;                                   // [S]
  int* s_gs = s_r0 + S;                                                      // [rows + 1]

  if (leader && lane == 0) {
#pragma unroll
    for (int j = 0; j < DEPTH; ++j) {
      mbar_init(full0 + 8 * j, 1);
      mbar_init(empty0 + 8 * j, HS);
    }
    fence_barrier_init();
  }

  // Tokens sequence s attends to, or minus the error bit that empties it.
  // Decode: context_lens[s].  Several query tokens per sequence: s is a query
  // row; its sequence (row of the block table) is found in query_start, and
  // query j of a sequence of n tokens and Q queries sees n - Q + j + 1 tokens.
  auto attended = [&](int s, int& row, int& r0nr) -> int {
    if (!prefill) {
      row = s;
      r0nr = s | (1 << 24);
      const int n = a.context_lens[s];
      if (n < 0 || n > a.len_cap) return -kErrContextLen;
      // (a claimed shared prefix always leaves at least one token)
      return a.pre_blocks ? n - kBlockSize * max(a.pre_blocks[s], 0) : n;
    }
    if constexpr (NR > 1) {
      // s is a group of up to NR consecutive query rows; it attends to the
      // prefix of its last row
      const int R = a.num_table_rows;
      row = 0;
      r0nr = 0;
      if (s >= s_gs[R]) return 0;  // no such group (the launch sizes for the most)
      int lo = 0, up = R - 1;      // largest sequence with s_gs[sequence] <= s
      while (lo < up) {
        const int mid = (lo + up + 1) >> 1;
        if (s_gs[mid] <= s) lo = mid; else up = mid - 1;
      }
      row = lo;
      const int q0 = s_qs[lo], Q = s_qs[lo + 1] - q0;
      const int j0 = NR * (s - s_gs[lo]);
      const int nr = min(NR, Q - j0);
      r0nr = (q0 + j0) | (nr << 24);
      const int n = a.context_lens[lo];
      if (n < 0 || n > a.len_cap) return -kErrContextLen;
      if (Q > n) return -kErrQuery;
      return n - Q + j0 + nr;
    }
    int lo = 0, up = a.num_table_rows - 1;  // largest row with query_start[row] <= s
    while (lo < up) {
      const int mid = (lo + up + 1) >> 1;
      if (s_qs[mid] <= s) lo = mid; else up = mid - 1;
    }
    row = lo;
    r0nr = s | (1 << 24);
    const int q0 = s_qs[lo], q1 = s_qs[lo + 1];
    if (!(q0 <= s && s < q1)) return -kErrQuery;
    const int n = a.context_lens[lo];
    if (n < 0 || n > a.len_cap) return -kErrContextLen;
    if (q1 - q0 > n) return -kErrQuery;
    return n - (q1 - q0) + (s - q0) + 1;
  };
  if (prefill) {
    for (int i = tid; i <= a.num_table_rows; i += WARPS * 32) s_qs[i] = a.query_start[i];
    __syncthreads();
    if (NR > 1 && warp == 0) {
      // groups of each sequence, ceil(Q / NR), and their prefix sums
      const int R = a.num_table_rows;
      int carry = 0;
      for (int base = 0; base < R; base += 32) {
        const int i = base + lane;
        // a sequence's rows must lie in [0, rows of q); one that breaks this
        // gets no group (its rows are not touched) and the error bit
        const bool ok = i >= R || (s_qs[i] >= 0 && s_qs[i] <= s_qs[i + 1] &&
                                   s_qs[i + 1] <= a.num_query_rows);
        if (!ok && blockIdx.x == 0 && a.err_flag) atomicOr(a.err_flag, kErrQuery);
        const int q = i < R && ok ? s_qs[i + 1] - s_qs[i] : 0;
        const int ng = q > 0 ? (q + NR - 1) / NR : 0;
        int incl = ng;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int t = __shfl_up_sync(kFull, incl, o);
          if (lane >= o) incl += t;
        }
        if (i < R) s_gs[i] = carry + incl - ng;
        carry += __shfl_sync(kFull, incl, 31);
      }
      if (lane == 0) s_gs[R] = carry;
    }
    __syncthreads();
  }

  // ---- prologue: block counts and their prefix sums, in tiles ----------------
  {
    const int per = (S + WARPS * 32 - 1) / (WARPS * 32);
    const int s0 = min(S, tid * per);
    const int s1 = min(S, s0 + per);
    int local = 0;
    for (int s = s0; s < s1; ++s) {
      int row, r0nr;
      int n = attended(s, row, r0nr);
      if (n < 0) n = 0;
      s_len[s] = n;
      if (prefill) s_row[s] = row;
      if (NR > 1) s_r0[s] = r0nr;
      local += (n + kBlockSize - 1) / kBlockSize;
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    int before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) {
      const int v = s_wsum[w];
      if (w < warp) before += v;
      total += v;
    }
    int run = before + incl - local;
    for (int s = s0; s < s1; ++s) {
      s_start[s] = run * Hkv;
      run += (s_len[s] + kBlockSize - 1) / kBlockSize;
    }
    if (tid == 0) s_start[S] = total * Hkv;
    __syncthreads();  // also publishes the barrier initialisation to the whole CTA
  }

  // ---- rows of empty or invalid sequences are zero --------------------------------
  for (int s = blockIdx.x; s < S; s += gridDim.x) {
    if (s_len[s] != 0) continue;
    int row, r0nr;
    const int n = attended(s, row, r0nr);
    if (tid == 0 && a.err_flag && n < 0) atomicOr(a.err_flag, -n);
    // (its query rows: one, or a group's; a group that does not exist has none)
    const int nrows = NR > 1 ? (r0nr >> 24) : 1;
    const int r0 = NR > 1 ? (r0nr & 0xffffff) : s;
    uint4* dst = reinterpret_cast<uint4*>(static_cast<char*>(a.out) +
                                          static_cast<size_t>(r0) * Hq * C::ROW);
    for (int i = tid; i < nrows * Hq * C::ROW / 16; i += WARPS * 32) dst[i] = make_uint4(0, 0, 0, 0);
  }

  // ---- this worker's share of the tiles -------------------------------------------
  // the merge pass (launched after this kernel) may start its prologue now
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const long long W = s_start[S];
  if (W == 0) return;
  const long long NWK = static_cast<long long>(gridDim.x) * WORKERS;
  const Ranges rg = make_ranges(W, NWK, a.part_blocks);
  const long long gw = static_cast<long long>(blockIdx.x) * WORKERS + warp / HS;
  const long long r0 = gw * rg.Rs / NWK;  // this worker's static ranges [r0, r1)
  const long long r1 = (gw + 1) * rg.Rs / NWK;

  long long* bnd = reinterpret_cast<long long*>(aux + C::XS + C::ALPHA);
  OwnRanges own{bnd, r1 - r0 <= kMaxOwnRanges ? static_cast<int>(r1 - r0) : 0};
  long long lo, hi;
  if (own.n > 0) {
    if (lane <= own.n) bnd[lane] = rg.start(r0 + lane);  // one division per lane, in parallel
    __syncwarp();
    lo = bnd[0];
    hi = bnd[own.n];
  } else {
    lo = rg.start(r0);
    hi = rg.start(r1);
  }
  float* xs = reinterpret_cast<float*>(aux);
  float* alpha_s = reinterpret_cast<float*>(aux + C::XS);
  StageDesc* ring_desc = reinterpret_cast<StageDesc*>(wkbase + C::DESC_OFF);
  // An item for the merge pass, listed by its first piece as a record
  // {first out row * Hkv + kv head, first range, pieces | (out rows << 24),
  // partial slot of the first piece}: each later piece starts its range r, so
  // its partial is in slot 2r.  Few pieces go to the one-warp list, more to the
  // one-CTA-per-head list.
  auto list_for_merge = [&](long long ra, long long rb, long long item_a, int item, int nr = 1) {
    const int4 rec = make_int4(item, static_cast<int>(ra), static_cast<int>(rb - ra + 1) | (nr << 24),
                               static_cast<int>(piece_slot(rg, ra, item_a)));
    if (rb - ra + 1 <= kWarpMergeMaxPieces)
      reinterpret_cast<int4*>(a.light_list)[atomicAdd(a.heavy + 4, 1)] = rec;
    else
      reinterpret_cast<int4*>(a.heavy_list)[atomicAdd(a.heavy, 1)] = rec;
  };

  const int dl = lane % C::LPR;  // which 16 bytes of a row
  const int rgp = lane / C::LPR; // which row group
  const int hs = lane % G;       // softmax: head of this lane
  // reduce-scatter order of this lane: its partial at array index i*G + h is
  // the logical (row i ^ imask, head h ^ hmask) of the chunk
  const int perm = (dl >> (C::LS - C::LSC)) << (C::LV - C::LSC);
  const int imask = perm >> C::LG;
  const int hmask = perm & (G - 1);

  // ---- the leader's stream: positions 0, 1, ... are its static tiles [lo, hi)
  // followed by the chunks it claims; descriptors of positions [base, base+64)
  // are held one per lane in A and B.
  const int n0 = static_cast<int>(hi - lo);
  int known = n0;                      // positions with a tile assigned
  bool no_more = rg.R == rg.Rs;        // no chunks left to claim
  auto static_desc = [&](int p) -> StageDesc {
    return p < n0 ? make_desc(lo + p, hi, s_start, s_len, s_row, rg, own, a) : StageDesc{0, 0, 0, 0};
  };
  StageDesc A{0, 0, 0, 0}, B{0, 0, 0, 0};
  int base = 0;
  if (leader) {
    A = static_desc(lane);
    B = static_desc(32 + lane);
  }
  // claim the next chunk of the tail and give its tiles the next positions
  auto claim = [&]() {
    int c = 0;
    if (lane == 0) c = atomicAdd(a.heavy + 2, 1);
    c = __shfl_sync(kFull, c, 0);
    if (c >= rg.R - rg.Rs) {
      no_more = true;
      return;
    }
    const long long g0 = rg.Ws + static_cast<long long>(c) * rg.CS;
    const int len = static_cast<int>(rg.CS < W - g0 ? rg.CS : W - g0);
    const int pa = base + lane, pb = base + 32 + lane;
    if (pa >= known && pa < known + len) A = make_desc(g0 + (pa - known), W, s_start, s_len, s_row, rg, own, a);
    if (pb >= known && pb < known + len) B = make_desc(g0 + (pb - known), W, s_start, s_len, s_row, rg, own, a);
    known += len;
  };
  auto top_up = [&](int frontier) {
    while (!no_more && known - frontier < kClaimAhead) claim();
  };

  const uint64_t kv_policy = kKvEvictFirst ? l2_policy_evict_first() : 0;
  // Leader: fill ring slot j % DEPTH with tile j (K and V rows, plus the q rows
  // of all GT heads on a piece start) -- or with the end marker -- once every
  // warp has released the slot.  The slot's descriptor goes with it.
  auto issue = [&](int j, bool end_marker) -> bool {
    const StageDesc e = end_marker ? StageDesc{0, 0, kEnd, 0} : pick_desc(A, B, j - base);
    const int slot = j % DEPTH;
    if (HS > 1 && j >= DEPTH) {
      if (!__all_sync(kFull, mbar_wait_bounded(empty0 + 8 * slot, ((j / DEPTH) - 1) & 1)))
        return false;
    }
    if (lane == 0) {
      ring_desc[slot] = e;
      const uint32_t bar = full0 + 8 * slot;
      if (e.meta & (kBad | kEnd)) {
        mbar_arrive(bar);  // nothing to fetch; complete the phase
      } else {
        const int kvh = e.meta & 0xffff;
        const int rows = (e.meta >> 16) & 31;
        const bool with_q = (e.meta & kFirst) != 0;
        const uint32_t kv_bytes = static_cast<uint32_t>(rows) * C::ROW;
        const uint32_t dst = slot0 + slot * C::SLOT;
        const size_t off = (static_cast<size_t>(e.phys) * Hkv + kvh) * C::TILE;
        if constexpr (MMA) {
          // whole 16-row tiles through the tensor maps (rows past the end are
          // masked or zeroed after arrival); the new rows go to the staging pair
          const bool app = (e.meta & kAppend) != 0;
          fence_proxy_async_smem();  // the slot may have been written (staged rows, zeroed rows)
          const int q_rows = !with_q ? 0 : NR > 1 ? (s_r0[e.seq] >> 24) : 1;
          mbar_arrive_expect_tx(bar, 2 * C::TILE + q_rows * GT * C::ROW + (app ? 2 * C::ROW : 0));
          const int y = (e.phys * Hkv + kvh) * kBlockSize;
#pragma unroll
          for (int hx = 0; hx < D / 64; ++hx) {
            if (kKvEvictFirst) {
              tma_load_2d_hint(dst + hx * 2048, &a.tm_k, hx * 64, y, bar, kv_policy);
              tma_load_2d_hint(dst + C::TILE + hx * 2048, &a.tm_v, hx * 64, y, bar, kv_policy);
            } else {
              tma_load_2d(dst + hx * 2048, &a.tm_k, hx * 64, y, bar);
              tma_load_2d(dst + C::TILE + hx * 2048, &a.tm_v, hx * 64, y, bar);
            }
          }
          if (app) {
            const size_t src = (static_cast<size_t>(e.seq) * Hkv + kvh) * C::ROW;
            bulk_copy_g2s(dst + C::APP, static_cast<const char*>(a.key) + src, C::ROW, bar);
            bulk_copy_g2s(dst + C::APP + C::ROW, static_cast<const char*>(a.value) + src, C::ROW,
                          bar);
          }
          if (with_q) {
            // the q rows of the item's query rows (one, or a group's)
            const int r0nr = NR > 1 ? s_r0[e.seq] : (e.seq | (1 << 24));
            const int r0 = r0nr & 0xffffff, nr = r0nr >> 24;
            for (int j = 0; j < nr; ++j)
              bulk_copy_g2s(dst + 2 * C::TILE + j * GT * C::ROW,
                            static_cast<const char*>(a.q) +
                                (static_cast<size_t>(r0 + j) * Hq + static_cast<size_t>(kvh) * GT) *
                                    C::ROW,
                            GT * C::ROW, bar);
          }
          return true;
        }
        if (kProxyFence) fence_proxy_async_smem();
        mbar_arrive_expect_tx(bar, 2 * kv_bytes + (with_q ? C::QB : 0));
        // with a fused append the last live row comes from key/value, not the cache
        const uint32_t cached = (e.meta & kAppend) ? kv_bytes - C::ROW : kv_bytes;
        if (cached) {
          if (kKvEvictFirst) {
            bulk_copy_g2s_hint(dst, static_cast<const char*>(a.k_cache) + off, cached, bar, kv_policy);
            bulk_copy_g2s_hint(dst + C::TILE, static_cast<const char*>(a.v_cache) + off, cached, bar,
                               kv_policy);
          } else {
            bulk_copy_g2s(dst, static_cast<const char*>(a.k_cache) + off, cached, bar);
            bulk_copy_g2s(dst + C::TILE, static_cast<const char*>(a.v_cache) + off, cached, bar);
          }
        }
        if (e.meta & kAppend) {
          const size_t src = (static_cast<size_t>(e.seq) * Hkv + kvh) * C::ROW;
          bulk_copy_g2s(dst + cached, static_cast<const char*>(a.key) + src, C::ROW, bar);
          bulk_copy_g2s(dst + C::TILE + cached, static_cast<const char*>(a.value) + src, C::ROW,
                        bar);
        }
        if (with_q)
          bulk_copy_g2s(dst + 2 * C::TILE,
                        static_cast<const char*>(a.q) +
                            (static_cast<size_t>(e.seq) * Hq + static_cast<size_t>(kvh) * GT) *
                                C::ROW,
                        C::QB, bar);
      }
    }
    return true;
  };
  // Leader, after consuming position k: keep positions assigned ahead and
  // refill the ring with position k + DEPTH (or the end marker, once).
  auto advance = [&](int k) -> bool {
    top_up(k + DEPTH + 1);
    const int j = k + DEPTH;
    if (j < known) return issue(j, false);
    if (HS > 1 && j == known && no_more) return issue(j, true);
    return true;
  };

  // A bounded wait ran out: flag it, let this warp's copies in flight land, leave.
  auto bail_out = [&](int k) {
    if (lane == 0 && a.err_flag) atomicOr(a.err_flag, kErrTimeout);
    if (leader)
      for (int j = k; j < known && j < k + DEPTH; ++j)
        mbar_wait_bounded(full0 + 8 * (j % DEPTH), (j / DEPTH) & 1);
  };

  if (leader) {
    top_up(DEPTH);
    for (int j = 0; j < DEPTH; ++j) {
      if (j < known) issue(j, false);
      else if (HS > 1 && j == known && no_more) issue(j, true);
    }
  }

  float qv[G][C::VEC];
  float o[G][C::VEC];
  float m_run = -INFINITY, l_run = 0.f;
  bool poisoned = false;
  // tensor-core path: lane (g = lane / 4, t = lane % 4) holds q as the B
  // operand of S^T = K q^T (heads g; head_dim pairs 2t, 2t+1 and 2t+8, 2t+9
  // of each 16-wide slice), o^T[head_dim x heads] as C fragments (head_dim
  // g and g + 8 of each slice; heads 2t and 2t+1), and the running max / sum
  // of heads 2t and 2t+1 (the sums over this lane's tokens only) -- one set
  // per query row of the item (NR).
  uint32_t qb[NR][C::MT][2];
  float oa[NR][C::MT][4];
  float mh[NR][2], lh[NR][2];
#pragma unroll
  for (int j = 0; j < NR; ++j) mh[j][0] = mh[j][1] = -INFINITY, lh[j][0] = lh[j][1] = 0.f;
  const int mg = lane >> 2, mtq = lane & 3;

  for (int k = 0;; ++k) {
    if (leader && k >= known) break;  // (the partner warp stops at the end marker)
    const int slot = k % DEPTH;
    if (!__all_sync(kFull, mbar_wait_bounded(full0 + 8 * slot, (k / DEPTH) & 1))) {
      bail_out(k);
      return;
    }
    const StageDesc d = ring_desc[slot];
    if (d.meta & kEnd) break;
    if (MMA && (d.meta & kAppend)) {
      // fused append: the new token's rows arrived in the staging pair; they
      // go to their cache slot and into the swizzled tiles in place of the
      // (stale) cache row the tensor load brought
      const int nrow = ((d.meta >> 16) & 31) - 1;
      const size_t off = (static_cast<size_t>(d.phys) * Hkv + (d.meta & 0xffff)) * C::TILE +
                         static_cast<size_t>(nrow) * C::ROW;
      unsigned char* sl = wkbase + slot * C::SLOT;
      for (int c = lane; c < C::ROW / 16; c += 32) {
        const uint4 kr = *reinterpret_cast<const uint4*>(sl + C::APP + 16 * c);
        const uint4 vr = *reinterpret_cast<const uint4*>(sl + C::APP + C::ROW + 16 * c);
        *reinterpret_cast<uint4*>(static_cast<char*>(const_cast<void*>(a.k_cache)) + off + 16 * c) = kr;
        *reinterpret_cast<uint4*>(static_cast<char*>(const_cast<void*>(a.v_cache)) + off + 16 * c) = vr;
        const int so = (c >> 3) * 2048 + nrow * 128 + (((c & 7) ^ (nrow & 7)) << 4);
        *reinterpret_cast<uint4*>(sl + so) = kr;
        *reinterpret_cast<uint4*>(sl + C::TILE + so) = vr;
      }
      __syncwarp();
    } else if ((d.meta & kAppend) && leader) {
      // fused append: the new token's row, now in shared memory, goes to its cache slot
      const int nrow = ((d.meta >> 16) & 31) - 1;
      const size_t off = (static_cast<size_t>(d.phys) * Hkv + (d.meta & 0xffff)) * C::TILE +
                         static_cast<size_t>(nrow) * C::ROW;
      const unsigned char* sk = wkbase + slot * C::SLOT + nrow * C::ROW;
      for (int c = lane; c < C::ROW / 16; c += 32) {
        *reinterpret_cast<uint4*>(static_cast<char*>(const_cast<void*>(a.k_cache)) + off + 16 * c) =
            *reinterpret_cast<const uint4*>(sk + 16 * c);
        *reinterpret_cast<uint4*>(static_cast<char*>(const_cast<void*>(a.v_cache)) + off + 16 * c) =
            *reinterpret_cast<const uint4*>(sk + C::TILE + 16 * c);
      }
    }
    const int flags = d.meta;
    const int kvh = d.meta & 0xffff;
    const int rows = (d.meta >> 16) & 31;
    const unsigned char* pk = wkbase + slot * C::SLOT;
    const unsigned char* pv = pk + C::TILE;

    if (MMA && (flags & kFirst)) {
#pragma unroll
      for (int j = 0; j < NR; ++j) {
        // (a group's missing second row reads stale q; its columns are masked)
        const unsigned char* pq = pk + 2 * C::TILE + (j * GT + mg) * C::ROW + mtq * 4;
#pragma unroll
        for (int ks = 0; ks < C::MT; ++ks) {
          qb[j][ks][0] = *reinterpret_cast<const uint32_t*>(pq + ks * 32);
          qb[j][ks][1] = *reinterpret_cast<const uint32_t*>(pq + ks * 32 + 16);
#pragma unroll
          for (int e = 0; e < 4; ++e) oa[j][ks][e] = 0.f;
        }
        mh[j][0] = mh[j][1] = -INFINITY;
        lh[j][0] = lh[j][1] = 0.f;
      }
      if (NR == 1 && (flags & kPrefix)) {
        // continue from the shared-prefix state: this lane's heads 2t, 2t+1,
        // head_dim g, g + 8 of each slice; the sums go to one lane per head
        const size_t hb = static_cast<size_t>(d.seq) * Hq + static_cast<size_t>(kvh) * GT + 2 * mtq;
        const float2 m0 = a.pre_ml[hb], m1 = a.pre_ml[hb + 1];
        mh[0][0] = m0.x;
        mh[0][1] = m1.x;
        lh[0][0] = mg == 0 ? m0.y : 0.f;
        lh[0][1] = mg == 0 ? m1.y : 0.f;
        const float* po = a.pre_o + hb * D + mg;
#pragma unroll
        for (int mt = 0; mt < C::MT; ++mt) {
          oa[0][mt][0] = po[mt * 16];
          oa[0][mt][1] = po[D + mt * 16];
          oa[0][mt][2] = po[mt * 16 + 8];
          oa[0][mt][3] = po[D + mt * 16 + 8];
        }
      }
      poisoned = false;
    } else if (flags & kFirst) {
      const unsigned char* pq = pk + 2 * C::TILE;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        // one head keeps the natural order; more heads are permuted (see reduce_scatter)
        const int hq = hoff + (G == 1 ? h : (h ^ hmask));
        const uint4 raw = *reinterpret_cast<const uint4*>(pq + hq * C::ROW + dl * 16);
        E::unpack(raw, qv[h]);
#pragma unroll
        for (int e = 0; e < C::VEC; ++e) {
          qv[h][e] *= a.scale_log2;
          o[h][e] = 0.f;
        }
      }
      m_run = -INFINITY;
      l_run = 0.f;
      if (flags & kPrefix) {
        // continue from the shared-prefix state.  The final reductions add
        // o over row groups and l over the lanes that share a head, so both
        // start in one of them; the running max is per head (per warp at G = 1).
        const size_t hb = static_cast<size_t>(d.seq) * Hq + static_cast<size_t>(kvh) * GT + hoff;
        const float2 ml = a.pre_ml[hb + hs];
        m_run = ml.x;
        l_run = (G == 1 ? rgp == 0 : lane < G) ? ml.y : 0.f;
        if (rgp == 0) {
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float* po = a.pre_o + (hb + h) * D + dl * C::VEC;
#pragma unroll
            for (int e = 0; e < C::VEC; e += 4) {
              const float4 t4 = *reinterpret_cast<const float4*>(po + e);
              o[h][e] = t4.x;
              o[h][e + 1] = t4.y;
              o[h][e + 2] = t4.z;
              o[h][e + 3] = t4.w;
            }
          }
        }
      }
      poisoned = false;
    }

    // Hand the slot back (this warp has read what it needs) and, on the leader,
    // refill it with position k + DEPTH.  Called exactly once per tile, after it.
    bool refill_ok = true;
    auto release = [&]() {
      __syncwarp();
      if (HS > 1 && lane == 0) mbar_arrive(empty0 + 8 * slot);
      if (leader) refill_ok = advance(k);
    };

    auto compute_tile = [&](auto mask_tag) {
      constexpr bool MASK = decltype(mask_tag)::value;
      if constexpr (MMA) {
        // ---- 8 heads on the tensor cores: S^T = K q^T, online softmax on the
        // fragments, o^T += V^T P^T.  Rows past the end of a partial tile:
        // their logits are masked and their V rows zeroed (a stale or NaN row
        // times a zero weight would still poison the sum).
        if (MASK) {
          unsigned char* vt = const_cast<unsigned char*>(pv);
          for (int c = lane; c < (kBlockSize - rows) * (C::ROW / 16); c += 32) {
            const int r = rows + c / (C::ROW / 16), cc = c % (C::ROW / 16);
            *reinterpret_cast<uint4*>(vt + (cc >> 3) * 2048 + r * 128 + ((cc & 7) << 4)) =
                make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();  // before the tensor load that next refills the slot
          __syncwarp();
        }
        const uint32_t kb = smem_addr(pk), vb = kb + C::TILE;
        const int lr = lane & 7, lm = lane >> 3;  // ldmatrix: row within matrix, matrix
        // a group of NR query rows: row j sees token t of this tile iff
        // t <= lim[j] (its causal limit); a missing row sees nothing
        int lim[NR];
        if constexpr (NR > 1) {
          const int v = d.seq;
          const int len = s_len[v];
          const long long item_a =
              s_start[v] + static_cast<long long>(kvh) * ((len + kBlockSize - 1) / kBlockSize);
          const int tb = static_cast<int>(d.g - item_a) * kBlockSize;
          const int nr = s_r0[v] >> 24;
#pragma unroll
          for (int j = 0; j < NR; ++j) lim[j] = j < nr ? len - nr + j - tb : -1;
        }
        float sc[NR][4];
#pragma unroll
        for (int j = 0; j < NR; ++j) sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < C::MT; ++ks) {
          // matrices: tokens 0-7 / 8-15 x head_dim ks*16 + 0-7, then + 8-15
          const int tok = (lm & 1) * 8 + lr;
          const int ch = ks * 2 + (lm >> 1);
          uint32_t af[4];
          ldmatrix_x4(kb + (ch >> 3) * 2048 + tok * 128 + (((ch & 7) ^ (tok & 7)) << 4), af);
#pragma unroll
          for (int j = 0; j < NR; ++j) mma_bf16_16816(sc[j], af, qb[j][ks][0], qb[j][ks][1]);
        }
        // sc[j]: tokens mg, mg, mg+8, mg+8 x heads 2t, 2t+1, 2t, 2t+1 (t = mtq)
        uint32_t b0[NR], b1[NR];
#pragma unroll
        for (int j = 0; j < NR; ++j) {
          float x[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int tok = mg + (e >> 1) * 8;
            const bool seen = NR > 1 ? tok <= lim[j] : (!MASK || tok < rows);
            x[e] = seen ? sc[j][e] * a.scale_log2 : -INFINITY;
          }
          float mx[2] = {fmaxf(x[0], x[2]), fmaxf(x[1], x[3])};
#pragma unroll
          for (int off = 4; off < 32; off <<= 1) {
            mx[0] = fmaxf(mx[0], __shfl_xor_sync(kFull, mx[0], off));
            mx[1] = fmaxf(mx[1], __shfl_xor_sync(kFull, mx[1], off));
          }
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            if (mx[c] > mh[j][c] + kRescaleThreshold) {
              const float al = exp2f(mh[j][c] - mx[c]);
              mh[j][c] = mx[c];
              lh[j][c] *= al;
#pragma unroll
              for (int mt = 0; mt < C::MT; ++mt) {
                oa[j][mt][c] *= al;
                oa[j][mt][c + 2] *= al;
              }
            }
          }
          __syncwarp();
          // (a logit masked out weighs 0, also while its running max is still -inf)
          auto wgt = [](float xv, float m) { return xv == -INFINITY ? 0.f : exp2f(xv - m); };
          const __nv_bfloat162 p01 =
              __floats2bfloat162_rn(wgt(x[0], mh[j][0]), wgt(x[1], mh[j][1]));
          const __nv_bfloat162 p23 =
              __floats2bfloat162_rn(wgt(x[2], mh[j][0]), wgt(x[3], mh[j][1]));
          // the sums take the weights as rounded for the product
          lh[j][0] += __low2float(p01) + __low2float(p23);
          lh[j][1] += __high2float(p01) + __high2float(p23);
          b0[j] = movmatrix_trans(*reinterpret_cast<const uint32_t*>(&p01));
          b1[j] = movmatrix_trans(*reinterpret_cast<const uint32_t*>(&p23));
        }
#pragma unroll
        for (int mt = 0; mt < C::MT; ++mt) {
          // matrices (transposed on load): tokens 0-7 x head_dim mt*16 + 0-7 /
          // + 8-15, then tokens 8-15 x the same
          const int tok = (lm >> 1) * 8 + lr;
          const int ch = mt * 2 + (lm & 1);
          uint32_t af[4];
          ldmatrix_x4_trans(vb + (ch >> 3) * 2048 + tok * 128 + (((ch & 7) ^ (tok & 7)) << 4), af);
#pragma unroll
          for (int j = 0; j < NR; ++j) mma_bf16_16816(oa[j][mt], af, b0[j], b1[j]);
        }
      } else if constexpr (G == 1) {
        // ---- one query head: every lane keeps the logits of its row group
        float x[C::RL];
#pragma unroll
        for (int i = 0; i < C::RL; ++i) {
          const int row = i * C::RPI + rgp;
          x[i] = 0.f;
          if (!MASK || row < rows) {
            float kf[C::VEC];
            E::unpack(*reinterpret_cast<const uint4*>(pk + row * C::ROW + dl * 16), kf);
            x[i] = dot_vec<C::VEC>(qv[0], kf);
          }
        }
#pragma unroll
        for (int off = C::LPR / 2; off >= 1; off >>= 1)
#pragma unroll
          for (int i = 0; i < C::RL; ++i) x[i] += __shfl_xor_sync(kFull, x[i], off);
        float mb = -INFINITY;
#pragma unroll
        for (int i = 0; i < C::RL; ++i) {
          if (MASK && i * C::RPI + rgp >= rows) x[i] = -INFINITY;
          mb = fmaxf(mb, x[i]);
        }
#pragma unroll
        for (int off = C::LPR; off < 32; off <<= 1) mb = fmaxf(mb, __shfl_xor_sync(kFull, mb, off));
        if (mb > m_run + kRescaleThreshold) {  // warp-uniform
          const float alpha = exp2f(m_run - mb);
          m_run = mb;
          l_run *= alpha;
          scale_vec<C::VEC>(alpha, o[0]);
        }
#pragma unroll
        for (int i = 0; i < C::RL; ++i) {
          const int row = i * C::RPI + rgp;
          const float p = exp2f(x[i] - m_run);
          l_run += p;
          if (!MASK || row < rows) {
            float vf[C::VEC];
            E::unpack(*reinterpret_cast<const uint4*>(pv + row * C::ROW + dl * 16), vf);
            axpy_vec<C::VEC>(p, vf, o[0]);
          }
        }
      } else {
        // ---- logits x = q.k (base-2 scaled) for the 16 rows x G heads --------
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) {
          float v[C::V];
#pragma unroll
          for (int i = 0; i < C::CH; ++i) {
            const int row = (c * C::CH + (i ^ imask)) * C::RPI + rgp;
            if (!MASK || row < rows) {
              float kf[C::VEC];
              E::unpack(*reinterpret_cast<const uint4*>(pk + row * C::ROW + dl * 16), kf);
#pragma unroll
              for (int h = 0; h < G; ++h) v[i * G + h] = dot_vec<C::VEC>(qv[h], kf);
            } else {
#pragma unroll
              for (int h = 0; h < G; ++h) v[i * G + h] = 0.f;
            }
          }
          reduce_scatter<C::LPR, C::V>(v);
          if ((dl & ((C::LPR >> C::LSC) - 1)) == 0) {
            const int sel = dl >> (C::LS - C::LSC);
#pragma unroll
            for (int r = 0; r < C::NV; ++r) {
              const int f = sel * C::NV + r;
              const int row = (c * C::CH + f / G) * C::RPI + rgp;
              xs[row * G + f % G] = (!MASK || row < rows) ? v[r] : -INFINITY;
            }
          }
        }
        __syncwarp();

        // ---- online softmax: lane owns head hs, tokens lane/G + k*(32/G) -------
        float xv[C::TPL];
        float mb = -INFINITY;
#pragma unroll
        for (int t = 0; t < C::TPL; ++t) {
          const int tok = lane / G + t * (32 / G);
          xv[t] = tok < kBlockSize ? xs[tok * G + hs] : -INFINITY;
          mb = fmaxf(mb, xv[t]);
        }
#pragma unroll
        for (int off = G; off < 32; off <<= 1) mb = fmaxf(mb, __shfl_xor_sync(kFull, mb, off));
        const bool grow = mb > m_run + kRescaleThreshold;
        float alpha = 1.f;
        if (grow) {
          alpha = exp2f(m_run - mb);
          m_run = mb;
          l_run *= alpha;
        }
        if (__any_sync(kFull, grow)) {
          if (lane < G) alpha_s[lane] = alpha;
          __syncwarp();
#pragma unroll
          for (int h = 0; h < G; ++h) scale_vec<C::VEC>(alpha_s[h], o[h]);
        }
#pragma unroll
        for (int t = 0; t < C::TPL; ++t) {
          const int tok = lane / G + t * (32 / G);
          const float p = exp2f(xv[t] - m_run);
          if (tok < kBlockSize) {
            l_run += p;
            xs[tok * G + hs] = p;
          }
        }
        __syncwarp();

        // ---- o += p . V ------------------------------------------------------
#pragma unroll
        for (int i = 0; i < C::RL; ++i) {
          const int row = i * C::RPI + rgp;
          if (!MASK || row < rows) {
            float vf[C::VEC];
            E::unpack(*reinterpret_cast<const uint4*>(pv + row * C::ROW + dl * 16), vf);
            float p[G];
#pragma unroll
            for (int h = 0; h < G; ++h) p[h] = xs[row * G + h];
#pragma unroll
            for (int h = 0; h < G; ++h) axpy_vec<C::VEC>(p[h], vf, o[h]);
          }
        }
      }
    };

    if (flags & kBad) {
      poisoned = true;
    } else if (rows == kBlockSize) {
      compute_tile(std::false_type{});
    } else {
      compute_tile(std::true_type{});
    }
    release();
    if (!refill_ok) {
      bail_out(k + 1);
      return;
    }

    // ---- end of a piece: write the output or a partial -------------------------
    if (MMA && (flags & kLast)) {
      const bool bad = __any_sync(kFull, poisoned);
      const int s = d.seq;
      const int nb = (s_len[s] + kBlockSize - 1) / kBlockSize;
      const long long item_a = s_start[s] + static_cast<long long>(kvh) * nb;
      const long long ra = rg.of(item_a);
      const long long rb = rg.of(item_a + nb - 1);
      const int h0 = 2 * mtq;  // this lane's heads h0, h0 + 1; head_dim mg, mg + 8 of each slice
      // the item's query rows: out rows r0 .. r0 + nr - 1 (decode: the sequence's)
      const int r0nr = NR > 1 ? s_r0[s] : (s | (1 << 24));
      const int r0 = r0nr & 0xffffff, nr = r0nr >> 24;
      const long long r = rg.of(d.g);
      const long long sl = piece_slot(rg, r, item_a);
#pragma unroll
      for (int j = 0; j < NR; ++j) {
        float lt[2] = {lh[j][0], lh[j][1]};
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          lt[0] += __shfl_xor_sync(kFull, lt[0], off);
          lt[1] += __shfl_xor_sync(kFull, lt[1], off);
        }
        if (j >= nr) continue;
        if (ra == rb) {
          // the whole item was this piece: normalise and store
          T* dst = static_cast<T*>(a.out) +
                   (static_cast<size_t>(r0 + j) * Hq + static_cast<size_t>(kvh) * GT + h0) * D + mg;
          const float i0 = bad ? 0.f : 1.f / lt[0], i1 = bad ? 0.f : 1.f / lt[1];
#pragma unroll
          for (int mt = 0; mt < C::MT; ++mt) {
            dst[mt * 16] = static_cast<T>(oa[j][mt][0] * i0);
            dst[D + mt * 16] = static_cast<T>(oa[j][mt][1] * i1);
            dst[mt * 16 + 8] = static_cast<T>(oa[j][mt][2] * i0);
            dst[D + mt * 16 + 8] = static_cast<T>(oa[j][mt][3] * i1);
          }
        } else {
          // a partial (columns j * 8 + head of the slot): no fence or counter
          // here; the merge pass, which starts once this grid has finished,
          // combines the pieces
          float* wo = a.ws_o + (sl * (NR * GT) + j * GT + h0) * D + mg;
#pragma unroll
          for (int mt = 0; mt < C::MT; ++mt) {
            wo[mt * 16] = oa[j][mt][0];
            wo[D + mt * 16] = oa[j][mt][1];
            wo[mt * 16 + 8] = oa[j][mt][2];
            wo[D + mt * 16 + 8] = oa[j][mt][3];
          }
          if (mg == 0) {
            a.ws_ml[sl * (NR * GT) + j * GT + h0] = make_float2(mh[j][0], bad ? -1.f : lt[0]);
            a.ws_ml[sl * (NR * GT) + j * GT + h0 + 1] = make_float2(mh[j][1], bad ? -1.f : lt[1]);
          }
        }
      }
      // the merge pass combines the pieces; the first piece lists the item
      if (ra != rb && r == ra && lane == 0) list_for_merge(ra, rb, item_a, r0 * Hkv + kvh, nr);
    } else if (flags & kLast) {
#pragma unroll
      for (int off = C::LPR; off < 32; off <<= 1)
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
          for (int e = 0; e < C::VEC; ++e) o[h][e] += __shfl_xor_sync(kFull, o[h][e], off);
      // l: with one head every lane of a row group holds that group's sum;
      // otherwise lanes sharing a head hold disjoint token sums
      float lsum = l_run;
#pragma unroll
      for (int off = (G == 1 ? C::LPR : G); off < 32; off <<= 1)
        lsum += __shfl_xor_sync(kFull, lsum, off);
      const bool bad = __any_sync(kFull, poisoned);
      const int s = d.seq;
      const int nb = (s_len[s] + kBlockSize - 1) / kBlockSize;
      const long long item_a = s_start[s] + static_cast<long long>(kvh) * nb;
      const long long ra = rg.of(item_a);
      const long long rb = rg.of(item_a + nb - 1);
      const size_t orow =
          (static_cast<size_t>(s) * Hq + static_cast<size_t>(kvh) * GT + hoff) * D;
      if (ra == rb) {
        // the whole (seq, kv head) was this piece: normalise and store
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float lh = __shfl_sync(kFull, lsum, h);
          if (h % C::RPI != rgp) continue;
          float r[C::VEC];
          const float inv = bad ? 0.f : 1.f / lh;
#pragma unroll
          for (int e = 0; e < C::VEC; ++e) r[e] = bad ? 0.f : o[h][e] * inv;
          *reinterpret_cast<uint4*>(static_cast<T*>(a.out) + orow + h * D + dl * C::VEC) =
              E::pack(r);
        }
      } else {
        const long long r = rg.of(d.g);
        const long long sl = piece_slot(rg, r, item_a);
        float* wo = a.ws_o + (sl * GT + hoff) * D;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          if (h % C::RPI != rgp) continue;
#pragma unroll
          for (int e = 0; e < C::VEC; e += 4)
            *reinterpret_cast<float4*>(wo + h * D + dl * C::VEC + e) =
                make_float4(o[h][e], o[h][e + 1], o[h][e + 2], o[h][e + 3]);
        }
        if (lane < G) a.ws_ml[sl * GT + hoff + lane] = make_float2(m_run, bad ? -1.f : lsum);
        const bool heavy = (rb - ra + 1) * G > kFuseMaxValues;
        if (heavy) {
          // many pieces: the merge pass combines them; the first piece lists the item
          if (r == ra && lane == 0 && half == 0) {
            list_for_merge(ra, rb, item_a, s * Hkv + kvh);
          }
        } else {
          __threadfence();
          __syncwarp();
          int prev = 0;
          int* cnt = a.counters + (static_cast<size_t>(s) * Hkv + kvh) * 2 + half;
          if (lane == 0) prev = atomicAdd(cnt, 1);
          prev = __shfl_sync(kFull, prev, 0);
          if (prev == static_cast<int>(rb - ra)) {
            // last piece of this (seq, kv head): merge all pieces by log-sum-exp
            __threadfence();
#pragma unroll
            for (int h = 0; h < G; ++h) {
              if (h % C::RPI != rgp) continue;
              float M = -INFINITY;
              bool any_bad = false;
              for (long long rr = ra; rr <= rb; ++rr) {
                const long long ss = piece_slot(rg, rr, item_a);
                const float2 ml = __ldcg(a.ws_ml + ss * GT + hoff + h);
                any_bad |= ml.y < 0.f;
                M = fmaxf(M, ml.x);
              }
              float L = 0.f;
              float acc[C::VEC];
#pragma unroll
              for (int e = 0; e < C::VEC; ++e) acc[e] = 0.f;
              for (long long rr = ra; rr <= rb; ++rr) {
                const long long ss = piece_slot(rg, rr, item_a);
                const float2 ml = __ldcg(a.ws_ml + ss * GT + hoff + h);
                const float w = exp2f(ml.x - M);
                L += w * ml.y;
                const float* po = a.ws_o + (ss * GT + hoff + h) * D + dl * C::VEC;
#pragma unroll
                for (int e = 0; e < C::VEC; e += 4) {
                  const float4 t4 = __ldcg(reinterpret_cast<const float4*>(po + e));
                  acc[e] = fmaf(w, t4.x, acc[e]);
                  acc[e + 1] = fmaf(w, t4.y, acc[e + 1]);
                  acc[e + 2] = fmaf(w, t4.z, acc[e + 2]);
                  acc[e + 3] = fmaf(w, t4.w, acc[e + 3]);
                }
              }
              const float inv = any_bad ? 0.f : 1.f / L;
#pragma unroll
              for (int e = 0; e < C::VEC; ++e) acc[e] = any_bad ? 0.f : acc[e] * inv;
              *reinterpret_cast<uint4*>(static_cast<T*>(a.out) + orow + h * D + dl * C::VEC) =
                  E::pack(acc);
            }
            if (lane == 0) *cnt = 0;  // leave the workspace zeroed for the next call
          }
        }
      }
    }

    if (leader && k - base == 31) {
      A = B;
      base += 32;
      B = static_desc(base + 32 + lane);
    }
  }
  // the last worker out resets the chunk counter for the next call (only a
  // claimed tail uses it)
  if (kTailDiv > 0 && leader && lane == 0) {
    if (atomicAdd(a.heavy + 3, 1) == static_cast<int>(NWK) - 1) {
      a.heavy[2] = 0;
      a.heavy[3] = 0;
    }
  }
}

}  // namespace pa
