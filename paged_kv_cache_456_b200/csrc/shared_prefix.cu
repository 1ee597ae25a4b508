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
// Work: a unit is (group, chunk of 64 columns, kv head, range of up to
// kRangeTiles shared blocks).  Each unit writes a partial state per column;
// the last unit of a (group, chunk, kv head) to finish folds the ranges and
// stores the state per (sequence, head).  Members are checked against the
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

constexpr int kPWarps = 4;
constexpr int kPCols = 16 * kPWarps;  // (member, head) columns of a unit: 16 per warp
constexpr int kPStages = 3;           // K/V tiles in flight per CTA
constexpr int kRangeTiles = 32;       // shared blocks per unit (512 tokens)
constexpr int kMaxChunkMembers = kPCols + 1;

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
  int max_blocks_per_seq, num_blocks, len_cap, max_ranges;
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
__global__ void __launch_bounds__(kPWarps * 32)
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
  // tiles 128-byte aligned for the swizzle; the unit prefix sums behind them
  unsigned char* ring = smem_raw + ((128u - (smem_addr(smem_raw) & 127u)) & 127u);
  int* s_ubase = reinterpret_cast<int*>(ring + kPStages * 2 * TILE);  // [num_groups + 1]

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
        units = ((m * G + kPCols - 1) / kPCols) * Hkv * ((P + kRangeTiles - 1) / kRangeTiles);
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
    const int R = (P + kRangeTiles - 1) / kRangeTiles;
    int local = u - s_ubase[g];
    const int c = local % NC;  // (consecutive units share the same K/V tiles)
    local /= NC;
    const int kvh = local % Hkv;
    const int r = local / Hkv;
    const int t0 = r * kRangeTiles, t1 = min(P, t0 + kRangeTiles);
    const int32_t* trow = a.block_tables + static_cast<size_t>(leader) * a.max_blocks_per_seq;

    // ---- q of this warp's 16 columns as the B operand of S^T = K q^T: lane
    // (g, t) holds column g of each 8-column half, head_dim pairs 2t, 2t+1
    // and 2t+8, 2t+9 of every 16-wide slice.  Columns past the group: zero.
    uint32_t qb[2][MT][2];
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      const int col = c * kPCols + warp * 16 + n * 8 + mg;
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
    float oa[2][MT][4];
    float mh[2][2], lh[2][2];
#pragma unroll
    for (int n = 0; n < 2; ++n) {
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) oa[n][mt][0] = oa[n][mt][1] = oa[n][mt][2] = oa[n][mt][3] = 0.f;
      mh[n][0] = mh[n][1] = -INFINITY;
      lh[n][0] = lh[n][1] = 0.f;
    }

    // all 128 threads stage tile t (K then V, swizzled); a bad id reads nothing
    auto load = [&](int t) {
      const uint32_t dst = smem_addr(ring) + ((t - t0) % kPStages) * 2 * TILE;
      int phys = __ldg(trow + t);
      const bool ok = phys >= 0 && phys < a.num_blocks;
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
    load(t0);
    cp_async_commit();
    if (t0 + 1 < t1) load(t0 + 1);
    cp_async_commit();
    for (int t = t0; t < t1; ++t) {
      if (t + 2 < t1) load(t + 2);
      cp_async_commit();
      cp_async_wait<2>();  // this thread's copies of tile t are done
      __syncthreads();     // ... and everyone's
      const uint32_t kb = smem_addr(ring) + ((t - t0) % kPStages) * 2 * TILE, vb = kb + TILE;
      // S^T[16 tokens x 16 columns] = K q^T
      float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int ks = 0; ks < MT; ++ks) {
        uint32_t af[4];  // tokens 0-7 / 8-15 x head_dim ks*16 + 0-7, then + 8-15
        ldmatrix_x4(kb + swz((lm & 1) * 8 + lr, ks * 2 + (lm >> 1)), af);
        mma_bf16_16816(sc[0], af, qb[0][ks][0], qb[0][ks][1]);
        mma_bf16_16816(sc[1], af, qb[1][ks][0], qb[1][ks][1]);
      }
      // online softmax per column on the fragments: sc[n] holds tokens g and
      // g + 8 of columns 2t, 2t+1
      uint32_t b0[2], b1[2];
#pragma unroll
      for (int n = 0; n < 2; ++n) {
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
        mma_bf16_16816(oa[0][mt], af, b0[0], b1[0]);
        mma_bf16_16816(oa[1][mt], af, b0[1], b1[1]);
      }
      __syncthreads();  // the stage is refilled two tiles later
    }

    // ---- the range's partial state per column ------------------------------
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      float lt[2] = {lh[n][0], lh[n][1]};
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        lt[0] += __shfl_xor_sync(0xffffffffu, lt[0], off);
        lt[1] += __shfl_xor_sync(0xffffffffu, lt[1], off);
      }
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int col = c * kPCols + warp * 16 + n * 8 + 2 * mtq + cc;
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
    const int mlo = (c * kPCols) / G;
    const int mhi = (min(m * G, (c + 1) * kPCols) - 1) / G;  // inclusive
    for (int i = warp; i <= mhi - mlo; i += kPWarps) {
      const int seq = a.group_seqs[gs + mlo + i];
      bool ok = seq >= 0 && seq < a.num_seqs;
      if (ok) {
        const int n = a.context_lens[seq];
        ok = n > 0 && n <= a.len_cap && kBlockSize * P <= n - 1;
      }
      bool same = true;
      if (ok) {
        const int32_t* srow = a.block_tables + static_cast<size_t>(seq) * a.max_blocks_per_seq;
        for (int j = lane; j < P; j += 32) {
          const int b = __ldg(trow + j);
          same &= b >= 0 && b < a.num_blocks && __ldg(srow + j) == b;
        }
      }
      ok = __all_sync(0xffffffffu, ok && same);
      if (lane == 0) {
        s_ok[i] = ok;
        if (!ok && kvh == 0 && a.err_flag) atomicOr(a.err_flag, kErrGroup);
      }
    }
    __syncthreads();
    for (int cl = warp; cl < kPCols; cl += kPWarps) {
      const int col = c * kPCols + cl;
      const int member = col / G;
      if (member >= m || !s_ok[member - mlo]) continue;
      const int seq = a.group_seqs[gs + member];
      const int head = kvh * G + col % G;
      const size_t pb = (static_cast<size_t>(gs + member) * Hq + head) * a.max_ranges;
      float M = -INFINITY;
      for (int rr = 0; rr < R; ++rr) M = fmaxf(M, __ldcg(a.part_ml + pb + rr).x);
      float L = 0.f;
      float acc[D / 32];
#pragma unroll
      for (int e = 0; e < D / 32; ++e) acc[e] = 0.f;
      for (int rr = 0; rr < R; ++rr) {
        const float2 ml = __ldcg(a.part_ml + pb + rr);
        const float w = exp2f(ml.x - M);
        L += w * ml.y;
        const float* po = a.part_o + (pb + rr) * D + lane;
#pragma unroll
        for (int e = 0; e < D / 32; ++e) acc[e] = fmaf(w, __ldcg(po + 32 * e), acc[e]);
      }
      float* dst = a.pre_o + (static_cast<size_t>(seq) * Hq + head) * D + lane;
#pragma unroll
      for (int e = 0; e < D / 32; ++e) dst[32 * e] = acc[e];
      if (lane == 0) a.pre_ml[static_cast<size_t>(seq) * Hq + head] = make_float2(M, L);
    }
    // claim each checked member once (the chunk of its first column, kv head
    // 0); a sequence claimed twice is given up
    if (kvh == 0) {
      for (int i = tid; i <= mhi - mlo; i += NTHR) {
        const int member = mlo + i;
        if (member * G < c * kPCols || !s_ok[i]) continue;
        const int seq = a.group_seqs[gs + member];
        if (atomicCAS(a.claim + seq, 0, P) != 0) {
          atomicExch(a.claim + seq, -1);
          if (a.err_flag) atomicOr(a.err_flag, kErrGroup);
        }
      }
    }
    __syncthreads();  // (s_ok is rewritten by the next unit)
  }
}

size_t round_up(size_t x, size_t al) { return (x + al - 1) / al * al; }

struct Layout {
  size_t counters, claim, part_ml, part_o, pre_ml, pre_o, bytes;
  int max_ranges;
};

Layout layout(int num_seqs, int num_listed, int num_q_heads, int head_dim,
              int max_blocks_per_seq) {
  Layout l{};
  l.max_ranges = (max_blocks_per_seq + kRangeTiles - 1) / kRangeTiles;
  const size_t cols = static_cast<size_t>(num_listed) * num_q_heads;
  const size_t rows = static_cast<size_t>(num_seqs) * num_q_heads;
  l.counters = 0;
  l.claim = round_up(cols * sizeof(int), 256);
  l.part_ml = round_up(l.claim + static_cast<size_t>(num_seqs) * sizeof(int), 256);
  l.part_o = round_up(l.part_ml + cols * l.max_ranges * sizeof(float2), 256);
  l.pre_ml = round_up(l.part_o + cols * l.max_ranges * head_dim * sizeof(float), 256);
  l.pre_o = round_up(l.pre_ml + rows * sizeof(float2), 256);
  l.bytes = round_up(l.pre_o + rows * head_dim * sizeof(float), 256);
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
  a.scale_log2 = l.scale_log2;
  a.counters = reinterpret_cast<int*>(ws + lo.counters);
  a.claim = l.pre_blocks;
  a.part_ml = reinterpret_cast<float2*>(ws + lo.part_ml);
  a.part_o = reinterpret_cast<float*>(ws + lo.part_o);
  a.pre_ml = l.pre_ml;
  a.pre_o = l.pre_o;
  a.err_flag = l.err_flag;

  const size_t tile = static_cast<size_t>(kBlockSize) * l.head_dim * 2;
  const size_t smem = 128 + kPStages * 2 * tile + (static_cast<size_t>(l.num_groups) + 1) * sizeof(int);
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
  // units: at most (chunks of all groups) x kv heads x ranges
  const long long chunks = (static_cast<long long>(l.num_listed) * group + kPCols - 1) / kPCols +
                           l.num_groups;
  const long long bound = chunks * l.num_kv_heads * lo.max_ranges;
  const long long resident = static_cast<long long>(num_sms) * occ;
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
