// shared_prefix.cu -- prefix-deduplicated decode: the pass over the blocks
// that several sequences share, and the host planner that finds them.
//
// Requests with a common prefix hold the same physical blocks for it, and a
// shared block is copied only when one of them must change it (skandtandon
// day-9 post, section "Idea 1: PagedAttention", the sharing and
// copy-on-write points).  Plain paged decode reads a shared block once per
// sequence.  Here the (member, query head) pairs of a group are the columns
// of one tensor-core product per shared block: each K/V tile of the shared
// prefix is read once for up to 64 columns.  Each column's online-softmax
// state over the shared blocks -- running max m (log2 units), sum of weights
// l, unnormalised output o -- is handed to the decode kernel, which goes on
// from it over the sequence's own blocks.  Attention over a union of token
// sets is the log-sum-exp combination of the parts, so the result is the
// same attention up to rounding.
//
// The pass runs on the tcgen05 tensor cores (tc_attention.cu: units of 128
// columns, a separate fold kernel).  The warp-level MMA pass below is kept
// as a build option.  Its work: a unit is (group, chunk of 64 columns, kv
// head, range of shared blocks); the host picks the range length so that the
// units fill the resident CTAs.  Each unit writes a partial state per column;
// the last unit of a (group, chunk, kv head) to finish folds the ranges and
// stores the state per (sequence, head).  Either way members are checked against the
// block tables before their state is published: a member whose table does
// not hold the group's blocks, whose length leaves no token after them, or
// that two groups list, is not claimed (PA_ERRBIT_GROUP) and the decode
// kernel attends to all of its tokens itself.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <utility>
#include <vector>

#include "paged_attention.h"
#include "pa_internal.h"
#include "ptx.cuh"

namespace pa {
namespace {

// Shape of a CTA: warps, and 8-column blocks per warp (build-time knobs).
// 8 warps of 8 columns measured fastest on prefix_cow (121.6 us for the
// deduplicated call), ahead of 4 x 16 (131.2 us) and 4 x 8 (127.8 us): more
// warps per SM hide the latency of each warp's dependent MMA / softmax chain.
#ifndef PA_SP_WARPS
#define PA_SP_WARPS 8
#endif
#ifndef PA_SP_NTW
#define PA_SP_NTW 1
#endif
#ifndef PA_SP_MINB
#define PA_SP_MINB 2
#endif
#ifndef PA_SP_MINRANGE
#define PA_SP_MINRANGE 16
#endif
constexpr int kPWarps = PA_SP_WARPS;
constexpr int NTW = PA_SP_NTW;                // 8-column blocks of a warp
constexpr int kPCols = 8 * NTW * kPWarps;     // (member, head) columns of a unit
constexpr int kPStages = 6;           // ring of K/V tiles: 5 in flight while one is used
constexpr int kMinRangeTiles = PA_SP_MINRANGE;  // shortest range of shared blocks per unit
constexpr int kMaxChunkMembers = kPCols + 1;
// The pass runs on the tcgen05 tensor cores (tc_attention.cu) unless built
// with PA_SHARED_TC=0, which keeps the warp-level MMA pass below.
#ifndef PA_SHARED_TC
#define PA_SHARED_TC 1
#endif
constexpr bool kSharedOnTensorCores = PA_SHARED_TC != 0;

struct PrefixArgs {
  const __nv_bfloat16* q;
  const unsigned char* k_cache;
  const unsigned char* v_cache;
  const int32_t* block_tables;
  const int32_t* context_lens;
  const int32_t* group_seqs;
  const int32_t* group_start;
  const int32_t* group_blocks;
  int num_groups, num_listed, num_seqs, num_q_heads, num_kv_heads;
  int max_blocks_per_seq, num_blocks, len_cap, max_ranges, range_tiles;
  float scale_log2;
  int* counters;     // [num_listed * Hq] units finished per (chunk, kv head); zero between calls
  int* claim;        // [num_seqs] = pre_blocks; zeroed before the pass
  float2* part_ml;   // [num_listed][Hq][max_ranges]
  float* part_o;     // [num_listed][Hq][max_ranges][D]
  float2* pre_ml;    // [num_seqs][Hq]
  float* pre_o;      // [num_seqs][Hq][D]
  int32_t* err_flag;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool fill) {
  // (src-size 0 writes zeros and reads nothing)
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(fill ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Byte offset of 16-byte chunk ch of row tok in a swizzled tile: rows of 64
// elements (128 bytes) with chunk' = chunk ^ (row & 7), head_dim 64-127 in a
// second 2 KB half.  ldmatrix of 8 rows at one chunk then hits 8 distinct bank groups.
__device__ __forceinline__ uint32_t swz(int tok, int ch) {
  return static_cast<uint32_t>((ch >> 3) * 2048 + tok * 128 + (((ch & 7) ^ (tok & 7)) << 4));
}

// Group g, if well formed: members [*gs, *gs + *m) of group_seqs, *P shared
// blocks, *leader = its first member (whose table row is read).
__device__ __forceinline__ bool group_ok(const PrefixArgs& a, int g, int* gs, int* m, int* P,
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

template <int D, int G>
__global__ void __launch_bounds__(kPWarps * 32, PA_SP_MINB)
shared_prefix_kernel(const __grid_constant__ PrefixArgs a) {
  constexpr int ROW = D * 2;              // bytes of one K or V row (bf16)
  constexpr int TILE = kBlockSize * ROW;  // one block of one kv head
  constexpr int CPR = ROW / 16;           // 16-byte chunks per row
  constexpr int MT = D / 16;              // 16-wide head_dim slices
  constexpr int NT = kBlockSize * CPR;    // chunks per tile
  constexpr int NTHR = kPWarps * 32;
  extern __shared__ unsigned char smem_raw[];
  __shared__ int s_wsum[kPWarps];
  __shared__ int s_last;
  __shared__ unsigned char s_ok[kMaxChunkMembers];
  __shared__ int s_seq[kMaxChunkMembers];
  __shared__ float s_M[kPCols], s_L[kPCols];
  // tiles 128-byte aligned for the swizzle; the unit prefix sums behind them
  unsigned char* ring = smem_raw + ((128u - (smem_addr(smem_raw) & 127u)) & 127u);
  int* s_ubase = reinterpret_cast<int*>(ring + kPStages * 2 * TILE);  // [num_groups + 1]
  int* s_phys = s_ubase + a.num_groups + 1;                            // [range_tiles]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int mg = lane >> 2, mtq = lane & 3;  // mma fragment row group / thread in group
  const int lr = lane & 7, lm = lane >> 3;    // ldmatrix row within matrix / matrix
  const int Hq = a.num_q_heads, Hkv = a.num_kv_heads;

  // ---- units per group and their prefix sums (every CTA computes them) ------
  {
    const int NGr = a.num_groups;
    const int per = (NGr + NTHR - 1) / NTHR;
    const int g0 = min(NGr, tid * per), g1 = min(NGr, g0 + per);
    int local = 0;
    for (int g = g0; g < g1; ++g) {
      int gs, m, P, leader;
      int units = 0;
      if (group_ok(a, g, &gs, &m, &P, &leader)) {
        units = ((m * G + kPCols - 1) / kPCols) * Hkv * ((P + a.range_tiles - 1) / a.range_tiles);
      } else if (blockIdx.x == 0 && a.err_flag) {
        atomicOr(a.err_flag, kErrGroup);
      }
      s_ubase[g] = units;  // (turned into starts below)
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
    for (int w = 0; w < kPWarps; ++w) {
      if (w < warp) run += s_wsum[w];
      total += s_wsum[w];
    }
    for (int g = g0; g < g1; ++g) {
      const int units = s_ubase[g];
      s_ubase[g] = run;
      run += units;
    }
    if (tid == 0) s_ubase[NGr] = total;
    __syncthreads();
  }
  const int total = s_ubase[a.num_groups];

  for (int u = blockIdx.x; u < total; u += gridDim.x) {
    // largest g with s_ubase[g] <= u (groups without units share their start)
    int lo = 0, up = a.num_groups - 1;
    while (lo < up) {
      const int mid = (lo + up + 1) >> 1;
      if (s_ubase[mid] <= u) lo = mid; else up = mid - 1;
    }
    const int g = lo;
    int gs = 0, m = 0, P = 0, leader = 0;
    group_ok(a, g, &gs, &m, &P, &leader);  // (true: only such groups have units)
    const int NC = (m * G + kPCols - 1) / kPCols;
    const int R = (P + a.range_tiles - 1) / a.range_tiles;
    int local = u - s_ubase[g];
    const int c = local % NC;  // (consecutive units share the same K/V tiles)
    local /= NC;
    const int kvh = local % Hkv;
    const int r = local / Hkv;
    const int t0 = r * a.range_tiles, t1 = min(P, t0 + a.range_tiles);
    const int32_t* trow = a.block_tables + static_cast<size_t>(leader) * a.max_blocks_per_seq;

    // ---- q of this warp's 8 * NTW columns as the B operand of S^T = K q^T: lane
    // (g, t) holds column g of each 8-column block, head_dim pairs 2t, 2t+1
    // and 2t+8, 2t+9 of every 16-wide slice.  Columns past the group: zero.
    uint32_t qb[NTW][MT][2];
#pragma unroll
    for (int n = 0; n < NTW; ++n) {
      const int col = c * kPCols + warp * 8 * NTW + n * 8 + mg;
      const int member = col / G;
      int seq = member < m ? a.group_seqs[gs + member] : -1;
      const bool ok = seq >= 0 && seq < a.num_seqs;
      const uint32_t* qp = reinterpret_cast<const uint32_t*>(
          a.q + (static_cast<size_t>(ok ? seq : 0) * Hq + kvh * G + col % G) * D) + mtq;
#pragma unroll
      for (int ks = 0; ks < MT; ++ks) {
        qb[n][ks][0] = ok ? __ldg(qp + ks * 8) : 0u;
        qb[n][ks][1] = ok ? __ldg(qp + ks * 8 + 4) : 0u;
      }
    }
    // o^T[head_dim x columns] as C fragments (head_dim g, g + 8 of each slice;
    // columns 2t, 2t+1); running max and this lane's share of the sums
    float oa[NTW][MT][4];
    float mh[NTW][2], lh[NTW][2];
#pragma unroll
    for (int n = 0; n < NTW; ++n) {
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) oa[n][mt][0] = oa[n][mt][1] = oa[n][mt][2] = oa[n][mt][3] = 0.f;
      mh[n][0] = mh[n][1] = -INFINITY;
      lh[n][0] = lh[n][1] = 0.f;
    }

    // the range's block ids, once (-1: out of range)
    for (int i = tid; i < t1 - t0; i += NTHR) {
      const int b = __ldg(trow + t0 + i);
      s_phys[i] = b >= 0 && b < a.num_blocks ? b : -1;
    }
    __syncthreads();
    // all threads of the CTA stage tile t (K then V, swizzled); a bad id reads nothing
    auto load = [&](int t) {
      const uint32_t dst = smem_addr(ring) + ((t - t0) % kPStages) * 2 * TILE;
      int phys = s_phys[t - t0];
      const bool ok = phys >= 0;
      if (!ok) phys = 0;
      const size_t off = (static_cast<size_t>(phys) * Hkv + kvh) * TILE;
#pragma unroll
      for (int i = tid; i < 2 * NT; i += NTHR) {
        const int which = i / NT, rem = i % NT;
        const int row = rem / CPR, ch = rem % CPR;
        const unsigned char* src = (which ? a.v_cache : a.k_cache) + off + row * ROW + ch * 16;
        cp_async16(dst + which * TILE + swz(row, ch), src, ok);
      }
    };
#pragma unroll
    for (int i = 0; i < kPStages - 1; ++i) {
      if (t0 + i < t1) load(t0 + i);
      cp_async_commit();
    }
    for (int t = t0; t < t1; ++t) {
      cp_async_wait<kPStages - 2>();  // this thread's copies of tile t are done
      __syncthreads();                // ... and everyone's; every warp is past tile t - 1
      // refill the stage of tile t - 1 with tile t + kPStages - 1
      if (t + kPStages - 1 < t1) load(t + kPStages - 1);
      cp_async_commit();
      const uint32_t kb = smem_addr(ring) + ((t - t0) % kPStages) * 2 * TILE, vb = kb + TILE;
      // S^T[16 tokens x 8 * NTW columns] = K q^T (even and odd head_dim slices
      // in separate accumulators: dependent chains of MT / 2)
      float sc[NTW][4], sd[NTW][4];
#pragma unroll
      for (int n = 0; n < NTW; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[n][e] = sd[n][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < MT; ++ks) {
        uint32_t af[4];  // tokens 0-7 / 8-15 x head_dim ks*16 + 0-7, then + 8-15
        ldmatrix_x4(kb + swz((lm & 1) * 8 + lr, ks * 2 + (lm >> 1)), af);
#pragma unroll
        for (int n = 0; n < NTW; ++n)
          mma_bf16_16816(ks & 1 ? sd[n] : sc[n], af, qb[n][ks][0], qb[n][ks][1]);
      }
#pragma unroll
      for (int n = 0; n < NTW; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[n][e] += sd[n][e];
      // online softmax per column on the fragments: sc[n] holds tokens g and
      // g + 8 of columns 2t, 2t+1
      uint32_t b0[NTW], b1[NTW];
#pragma unroll
      for (int n = 0; n < NTW; ++n) {
        float x[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] = sc[n][e] * a.scale_log2;
        float mx[2] = {fmaxf(x[0], x[2]), fmaxf(x[1], x[3])};
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          mx[0] = fmaxf(mx[0], __shfl_xor_sync(0xffffffffu, mx[0], off));
          mx[1] = fmaxf(mx[1], __shfl_xor_sync(0xffffffffu, mx[1], off));
        }
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          if (mx[cc] > mh[n][cc] + kRescaleThreshold) {
            const float al = exp2f(mh[n][cc] - mx[cc]);
            mh[n][cc] = mx[cc];
            lh[n][cc] *= al;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
              oa[n][mt][cc] *= al;
              oa[n][mt][cc + 2] *= al;
            }
          }
        }
        __syncwarp();
        const __nv_bfloat162 p01 =
            __floats2bfloat162_rn(exp2f(x[0] - mh[n][0]), exp2f(x[1] - mh[n][1]));
        const __nv_bfloat162 p23 =
            __floats2bfloat162_rn(exp2f(x[2] - mh[n][0]), exp2f(x[3] - mh[n][1]));
        // the sums take the weights as rounded for the product
        lh[n][0] += __low2float(p01) + __low2float(p23);
        lh[n][1] += __high2float(p01) + __high2float(p23);
        b0[n] = movmatrix_trans(*reinterpret_cast<const uint32_t*>(&p01));
        b1[n] = movmatrix_trans(*reinterpret_cast<const uint32_t*>(&p23));
      }
      // o^T += V^T P^T
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        uint32_t af[4];  // (transposed on load) tokens 0-7 x head_dim mt*16 + 0-7 / + 8-15, then tokens 8-15
        ldmatrix_x4_trans(vb + swz((lm >> 1) * 8 + lr, mt * 2 + (lm & 1)), af);
#pragma unroll
        for (int n = 0; n < NTW; ++n) mma_bf16_16816(oa[n][mt], af, b0[n], b1[n]);
      }
    }

    // ---- the range's partial state per column ------------------------------
#pragma unroll
    for (int n = 0; n < NTW; ++n) {
      float lt[2] = {lh[n][0], lh[n][1]};
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        lt[0] += __shfl_xor_sync(0xffffffffu, lt[0], off);
        lt[1] += __shfl_xor_sync(0xffffffffu, lt[1], off);
      }
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int col = c * kPCols + warp * 8 * NTW + n * 8 + 2 * mtq + cc;
        const int member = col / G;
        if (member >= m) continue;
        const size_t pi =
            (static_cast<size_t>(gs + member) * Hq + kvh * G + col % G) * a.max_ranges + r;
        float* po = a.part_o + pi * D + mg;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          po[mt * 16] = oa[n][mt][cc];
          po[mt * 16 + 8] = oa[n][mt][cc + 2];
        }
        if (mg == 0) a.part_ml[pi] = make_float2(mh[n][cc], lt[cc]);
      }
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) {
      int* cnt = a.counters + (static_cast<size_t>(gs) * G + c * kPCols) * Hkv + kvh;
      const int prev = atomicAdd(cnt, 1);
      s_last = prev == R - 1;
      if (s_last) *cnt = 0;  // every range has arrived: leave it zero for the next call
    }
    __syncthreads();
    if (!s_last) continue;
    __threadfence();

    // ---- last range of (group, chunk, kv head): check the members, fold ----
    // (spread over all threads: each step's loads are independent, so they
    // overlap instead of paying the L2 latency one after the other)
    const int mlo = (c * kPCols) / G;
    const int nm = (min(m * G, (c + 1) * kPCols) - 1) / G - mlo + 1;  // members in the chunk
    for (int i = tid; i < nm; i += NTHR) {
      const int seq = a.group_seqs[gs + mlo + i];
      bool ok = seq >= 0 && seq < a.num_seqs;
      if (ok) {
        const int n = a.context_lens[seq];
        ok = n > 0 && n <= a.len_cap && kBlockSize * P <= n - 1;
      }
      s_seq[i] = ok ? seq : -1;
      s_ok[i] = ok;
    }
    __syncthreads();
    // every (member, shared block): the member's table holds the leader's block
#pragma unroll 4
    for (int idx = tid; idx < nm * P; idx += NTHR) {
      const int i = idx / P, j = idx - i * P;
      const int seq = s_seq[i];
      if (seq < 0) continue;
      const int b = __ldg(trow + j);
      if (!(b >= 0 && b < a.num_blocks &&
            __ldg(a.block_tables + static_cast<size_t>(seq) * a.max_blocks_per_seq + j) == b))
        s_ok[i] = 0;  // (every writer stores the same value)
    }
    __syncthreads();
    if (kvh == 0 && a.err_flag)
      for (int i = tid; i < nm; i += NTHR)
        if (!s_ok[i]) atomicOr(a.err_flag, kErrGroup);
    // column weights of the ranges, w = 2^(m_r - M), into the idle ring
    float* s_w = reinterpret_cast<float*>(ring);  // [kPCols][R]
    for (int cl = tid; cl < kPCols; cl += NTHR) {
      const int col = c * kPCols + cl;
      const int member = col / G;
      if (member >= m || !s_ok[member - mlo]) continue;
      const size_t pb = (static_cast<size_t>(gs + member) * Hq + kvh * G + col % G) * a.max_ranges;
      float M = -INFINITY;
#pragma unroll 4
      for (int rr = 0; rr < R; ++rr) M = fmaxf(M, __ldcg(a.part_ml + pb + rr).x);
      float L = 0.f;
#pragma unroll 4
      for (int rr = 0; rr < R; ++rr) {
        const float2 ml = __ldcg(a.part_ml + pb + rr);
        const float w = exp2f(ml.x - M);
        s_w[cl * R + rr] = w;
        L += w * ml.y;
      }
      s_M[cl] = M;
      s_L[cl] = L;
    }
    __syncthreads();
    // outputs: thread t owns (column, 4 head_dim) items t, t + 128, ...; in
    // batches of KB items, one pass over the ranges with the batch's loads
    // in flight together
    constexpr int Q4 = D / 4;
    constexpr int NI = kPCols * Q4 / NTHR;
    static_assert(kPCols * Q4 % NTHR == 0, "fold items must split evenly over the threads");
    constexpr int KB = NI < 8 ? NI : 8;
    for (int k0 = 0; k0 < NI; k0 += KB) {
      const float4* src[KB];
      float4 acc[KB];
#pragma unroll
      for (int k = 0; k < KB; ++k) {
        const int idx = tid + (k0 + k) * NTHR, cl = idx / Q4, q4 = idx % Q4;
        const int col = c * kPCols + cl;
        const int member = col / G;
        const bool live = member < m && s_ok[member - mlo];
        const size_t pb =
            (static_cast<size_t>(gs + (live ? member : 0)) * Hq + kvh * G + col % G) * a.max_ranges;
        src[k] = live ? reinterpret_cast<const float4*>(a.part_o + pb * D) + q4 : nullptr;
        acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      for (int rr = 0; rr < R; ++rr) {
#pragma unroll
        for (int k = 0; k < KB; ++k) {
          if (!src[k]) continue;
          const int cl = (tid + (k0 + k) * NTHR) / Q4;
          const float4 o = __ldcg(src[k] + static_cast<size_t>(rr) * Q4);
          const float w = s_w[cl * R + rr];
          acc[k].x = fmaf(w, o.x, acc[k].x);
          acc[k].y = fmaf(w, o.y, acc[k].y);
          acc[k].z = fmaf(w, o.z, acc[k].z);
          acc[k].w = fmaf(w, o.w, acc[k].w);
        }
      }
#pragma unroll
      for (int k = 0; k < KB; ++k) {
        if (!src[k]) continue;
        const int idx = tid + (k0 + k) * NTHR, cl = idx / Q4, q4 = idx % Q4;
        const int col = c * kPCols + cl;
        const int member = col / G;
        const size_t row = static_cast<size_t>(s_seq[member - mlo]) * Hq + kvh * G + col % G;
        reinterpret_cast<float4*>(a.pre_o + row * D)[q4] = acc[k];
        if (q4 == 0) a.pre_ml[row] = make_float2(s_M[cl], s_L[cl]);
      }
    }
    // claim each checked member once (the chunk of its first column, kv head
    // 0); a sequence claimed twice is given up
    if (kvh == 0) {
      for (int i = tid; i < nm; i += NTHR) {
        const int member = mlo + i;
        if (member * G < c * kPCols || !s_ok[i]) continue;
        const int seq = s_seq[i];
        if (atomicCAS(a.claim + seq, 0, P) != 0) {
          atomicExch(a.claim + seq, -1);
          if (a.err_flag) atomicOr(a.err_flag, kErrGroup);
        }
      }
    }
    __syncthreads();  // (s_ok, s_seq and the ring are rewritten by the next unit)
  }
}

size_t round_up(size_t x, size_t al) { return (x + al - 1) / al * al; }

// Shortest range a launch may use: kMinRangeTiles, and long enough that the
// fold's weights (kPCols x ranges floats) fit the ring they reuse.
int min_range_tiles(int max_blocks_per_seq, int head_dim) {
  const int cap = kPStages * 2 * kBlockSize * head_dim * 2 / (4 * kPCols);  // ranges that fit
  return std::max(kMinRangeTiles, (max_blocks_per_seq + cap - 1) / cap);
}

struct Layout {
  size_t counters, claim, part_ml, part_o, pre_ml, pre_o, unit_start, group_ranges, units, bytes;
  int max_ranges;
  long long max_units;
};

Layout layout(int num_seqs, int num_listed, int num_q_heads, int head_dim,
              int max_blocks_per_seq) {
  Layout l{};
  const int rt = min_range_tiles(max_blocks_per_seq, head_dim);
  l.max_ranges = (max_blocks_per_seq + rt - 1) / rt;
  const size_t cols = static_cast<size_t>(num_listed) * num_q_heads;
  const size_t rows = static_cast<size_t>(num_seqs) * num_q_heads;
  l.counters = 0;
  l.claim = round_up(cols * sizeof(int), 256);
  l.part_ml = round_up(l.claim + static_cast<size_t>(num_seqs) * sizeof(int), 256);
  l.part_o = round_up(l.part_ml + cols * l.max_ranges * sizeof(float2), 256);
  l.pre_ml = round_up(l.part_o + cols * l.max_ranges * head_dim * sizeof(float), 256);
  l.pre_o = round_up(l.pre_ml + rows * sizeof(float2), 256);
  // (the tensor-core pass: work units before each group and each group's
  // ranges; a group lists at least one member, so groups <= listed)
  l.unit_start = round_up(l.pre_o + rows * head_dim * sizeof(float), 256);
  l.group_ranges = round_up(l.unit_start + (static_cast<size_t>(num_listed) + 1) * sizeof(int), 256);
  // its unit records: per group ceil(members * G / 128) <= members * G / 128 + 1
  // column tiles for each KV head and range, so at most
  // (ceil(listed * Hq / 128) + listed * Hq) x max_ranges in all
  l.units = round_up(l.group_ranges + static_cast<size_t>(num_listed) * sizeof(int), 256);
  l.max_units = ((static_cast<long long>(num_listed) * num_q_heads + 127) / 128 +
                 static_cast<long long>(num_listed) * num_q_heads) * l.max_ranges;
  // (a record is two int4)
  l.bytes = round_up(l.units + static_cast<size_t>(l.max_units) * 32, 256);
  return l;
}

template <int D, int G>
const void* kernel_fn() {
  return reinterpret_cast<const void*>(&shared_prefix_kernel<D, G>);
}

const void* pick_kernel(int head_dim, int group) {
  switch (head_dim * 100 + group) {
    case 6401: return kernel_fn<64, 1>();
    case 6402: return kernel_fn<64, 2>();
    case 6404: return kernel_fn<64, 4>();
    case 6408: return kernel_fn<64, 8>();
    case 12801: return kernel_fn<128, 1>();
    case 12802: return kernel_fn<128, 2>();
    case 12804: return kernel_fn<128, 4>();
    case 12808: return kernel_fn<128, 8>();
    default: return nullptr;
  }
}

std::mutex g_pmu;
// (device, kernel) -> dynamic smem limit set so far (only grows); (device,
// kernel, smem) -> resident CTAs per SM
std::map<std::pair<int, const void*>, size_t> g_plimit;
std::map<std::pair<std::pair<int, const void*>, size_t>, int> g_pocc;

}  // namespace

size_t shared_prefix_workspace_bytes(int num_seqs, int num_listed, int num_q_heads, int head_dim,
                                     int max_blocks_per_seq) {
  if (num_seqs < 0 || num_listed < 0 || num_q_heads <= 0 || max_blocks_per_seq <= 0 ||
      (head_dim != 64 && head_dim != 128))
    return 0;
  return layout(num_seqs, num_listed, num_q_heads, head_dim, max_blocks_per_seq).bytes;
}

cudaError_t launch_shared_prefix(SharedPrefixLaunch& l, int num_sms, cudaStream_t stream) {
  const int group = l.num_q_heads / l.num_kv_heads;
  const void* fn = pick_kernel(l.head_dim, group);
  if (!fn) return cudaErrorInvalidValue;
  const Layout lo = layout(l.num_seqs, l.num_listed, l.num_q_heads, l.head_dim,
                           l.max_blocks_per_seq);
  char* ws = static_cast<char*>(l.workspace);
  l.pre_blocks = reinterpret_cast<int32_t*>(ws + lo.claim);
  l.pre_o = reinterpret_cast<float*>(ws + lo.pre_o);
  l.pre_ml = reinterpret_cast<float2*>(ws + lo.pre_ml);
  cudaError_t e = cudaMemsetAsync(l.pre_blocks, 0, static_cast<size_t>(l.num_seqs) * sizeof(int),
                                  stream);
  if (e != cudaSuccess || l.num_groups == 0) return e;
  if (kSharedOnTensorCores && l.tm_k && tc_shared_prefix_supported(l.head_dim, group)) {
    TcSharedLaunch t{};
    t.q = l.q;
    t.block_tables = l.block_tables;
    t.context_lens = l.context_lens;
    t.group_seqs = l.group_seqs;
    t.group_start = l.group_start;
    t.group_blocks = l.group_blocks;
    t.num_groups = l.num_groups;
    t.num_listed = l.num_listed;
    t.num_seqs = l.num_seqs;
    t.num_q_heads = l.num_q_heads;
    t.num_kv_heads = l.num_kv_heads;
    t.head_dim = l.head_dim;
    t.max_blocks_per_seq = l.max_blocks_per_seq;
    t.num_blocks = l.num_blocks;
    t.len_cap = l.len_cap;
    t.max_ranges = lo.max_ranges;
    t.scale_log2 = l.scale_log2;
    t.unit_start = reinterpret_cast<int*>(ws + lo.unit_start);
    t.units = reinterpret_cast<int4*>(ws + lo.units);
    t.max_units = static_cast<int>(std::min<long long>(lo.max_units, 1 << 28));
    t.group_ranges = reinterpret_cast<int*>(ws + lo.group_ranges);
    t.claim = l.pre_blocks;
    t.part_ml = reinterpret_cast<float2*>(ws + lo.part_ml);
    t.part_o = reinterpret_cast<float*>(ws + lo.part_o);
    t.pre_ml = l.pre_ml;
    t.pre_o = l.pre_o;
    t.err_flag = l.err_flag;
    t.tm_k = l.tm_k;
    t.tm_v = l.tm_v;
    return launch_tc_shared_prefix(t, num_sms, stream);
  }

  PrefixArgs a;
  a.q = static_cast<const __nv_bfloat16*>(l.q);
  a.k_cache = static_cast<const unsigned char*>(l.k_cache);
  a.v_cache = static_cast<const unsigned char*>(l.v_cache);
  a.block_tables = l.block_tables;
  a.context_lens = l.context_lens;
  a.group_seqs = l.group_seqs;
  a.group_start = l.group_start;
  a.group_blocks = l.group_blocks;
  a.num_groups = l.num_groups;
  a.num_listed = l.num_listed;
  a.num_seqs = l.num_seqs;
  a.num_q_heads = l.num_q_heads;
  a.num_kv_heads = l.num_kv_heads;
  a.max_blocks_per_seq = l.max_blocks_per_seq;
  a.num_blocks = l.num_blocks;
  a.len_cap = l.len_cap;
  a.max_ranges = lo.max_ranges;
  a.range_tiles = 0;  // (set below, once the resident CTAs are known)
  a.scale_log2 = l.scale_log2;
  a.counters = reinterpret_cast<int*>(ws + lo.counters);
  a.claim = l.pre_blocks;
  a.part_ml = reinterpret_cast<float2*>(ws + lo.part_ml);
  a.part_o = reinterpret_cast<float*>(ws + lo.part_o);
  a.pre_ml = l.pre_ml;
  a.pre_o = l.pre_o;
  a.err_flag = l.err_flag;

  const size_t tile = static_cast<size_t>(kBlockSize) * l.head_dim * 2;
  // (the range's block ids follow the unit starts; sized for the longest range below)
  const size_t smem = 128 + kPStages * 2 * tile +
                      (static_cast<size_t>(l.num_groups) + 1 + l.max_blocks_per_seq) * sizeof(int);
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  int occ = 0;
  {
    std::lock_guard<std::mutex> lock(g_pmu);
    size_t& limit = g_plimit[std::make_pair(dev, fn)];
    if (smem > limit) {
      if ((e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(smem))) != cudaSuccess)
        return e;
      limit = smem;
    }
    const auto key = std::make_pair(std::make_pair(dev, fn), smem);
    auto it = g_pocc.find(key);
    if (it != g_pocc.end()) {
      occ = it->second;
    } else {
      if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, kPWarps * 32, smem)) !=
          cudaSuccess)
        return e;
      g_pocc[key] = occ;
    }
  }
  if (occ < 1) return cudaErrorInvalidConfiguration;
  // ranges per (chunk, kv head) so that the units about fill the resident
  // CTAs (from the fewest chunks the columns can form), but no shorter than
  // min_range_tiles
  const long long resident = static_cast<long long>(num_sms) * occ;
  const long long min_chunks =
      std::max(1LL, (static_cast<long long>(l.num_listed) * group + kPCols - 1) / kPCols);
  const long long per = std::max(1LL, resident / (min_chunks * l.num_kv_heads));
  a.range_tiles = static_cast<int>(std::max<long long>(
      min_range_tiles(l.max_blocks_per_seq, l.head_dim), (l.max_blocks_per_seq + per - 1) / per));
  // units: at most (chunks of all groups) x kv heads x ranges
  const long long chunks = (static_cast<long long>(l.num_listed) * group + kPCols - 1) / kPCols +
                           l.num_groups;
  const long long bound = chunks * l.num_kv_heads *
                          ((l.max_blocks_per_seq + a.range_tiles - 1) / a.range_tiles);
  const int grid = static_cast<int>(std::max(1LL, std::min(bound, resident)));
  void* params[] = {&a};
  return cudaLaunchKernel(fn, dim3(grid), dim3(kPWarps * 32), params, smem, stream);
}

}  // namespace pa

extern "C" pa_status pa_shared_prefix_plan(const int32_t* block_tables,
                                           const int32_t* context_lens, int num_seqs,
                                           int max_blocks_per_seq, int block_size,
                                           int min_shared_blocks, int32_t* group_seqs,
                                           int32_t* group_start, int32_t* group_blocks,
                                           int* num_groups, int* num_listed) {
  if (num_seqs < 0 || max_blocks_per_seq <= 0 || block_size <= 0 || !num_groups || !num_listed)
    return PA_ERR_INVALID_ARG;
  if (block_size != pa::kBlockSize) return PA_ERR_UNSUPPORTED;
  *num_groups = 0;
  *num_listed = 0;
  if (num_seqs == 0) return PA_OK;
  if (!block_tables || !context_lens || !group_seqs || !group_start || !group_blocks)
    return PA_ERR_INVALID_ARG;
  const int min_blocks = min_shared_blocks > 1 ? min_shared_blocks : 1;
  const long long cap_len = static_cast<long long>(max_blocks_per_seq) * pa::kBlockSize;
  // candidates by first physical block: blocks strictly before the block of
  // the sequence's last token can be shared (the pass needs whole blocks and
  // the decode kernel at least one token of its own)
  std::map<int, std::vector<int>> by_first;
  for (int s = 0; s < num_seqs; ++s) {
    const int n = context_lens[s];
    if (n <= 0 || n > cap_len) continue;
    if ((n - 1) / pa::kBlockSize < min_blocks) continue;
    by_first[block_tables[static_cast<size_t>(s) * max_blocks_per_seq]].push_back(s);
  }
  std::vector<std::pair<int, int>> groups;  // (first member, shared blocks) -> members
  std::map<int, const std::vector<int>*> members_of;
  for (const auto& kv : by_first) {
    const std::vector<int>& mem = kv.second;
    if (mem.size() < 2) continue;
    int P = max_blocks_per_seq;
    for (int s : mem) P = std::min(P, (context_lens[s] - 1) / pa::kBlockSize);
    // the longest run of leading blocks every member holds
    const int32_t* lead = block_tables + static_cast<size_t>(mem[0]) * max_blocks_per_seq;
    for (int j = 1; j < P; ++j) {
      bool same = true;
      for (size_t i = 1; i < mem.size() && same; ++i)
        same = block_tables[static_cast<size_t>(mem[i]) * max_blocks_per_seq + j] == lead[j];
      if (!same) {
        P = j;
        break;
      }
    }
    if (P < min_blocks) continue;
    groups.emplace_back(mem[0], P);
    members_of[mem[0]] = &mem;
  }
  std::sort(groups.begin(), groups.end());
  int listed = 0;
  group_start[0] = 0;
  for (size_t g = 0; g < groups.size(); ++g) {
    for (int s : *members_of[groups[g].first]) group_seqs[listed++] = s;
    group_start[g + 1] = listed;
    group_blocks[g] = groups[g].second;
  }
  *num_groups = static_cast<int>(groups.size());
  *num_listed = listed;
  return PA_OK;
}
