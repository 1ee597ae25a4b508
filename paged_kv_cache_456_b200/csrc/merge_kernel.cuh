// merge_kernel.cuh -- the second pass of split-K decode: combines the
// partial results (m, l, o) of (sequence, KV head) items that the decode
// kernel cut into pieces, by log-sum-exp.
#pragma once

#include <cstdint>
#include <type_traits>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "pa_internal.h"

namespace pa {

// Merge pass for the (seq, kv head) items listed by the decode kernel.  An
// item of few pieces is merged by one warp; an item of many pieces (long
// contexts) gets one CTA per (item, query head), kMergeThreads / 32 groups of
// lanes taking every GROUPS-th piece, combined in shared memory:
//     M = max_j m_j,  out = sum_j 2^(m_j - M) o_j / sum_j 2^(m_j - M) l_j.
// Launched right behind the decode kernel with programmatic dependent launch;
// griddepcontrol.wait returns once the decode grid has finished and its
// writes are visible.  The last CTA to finish resets the item list.
// G partial columns per item: GH query heads of a KV head for each of the
// item's G / GH query rows (one row in decode).
template <typename T, int D, int G, int GH = G>
__global__ void __launch_bounds__(kMergeThreads)
paged_decode_merge_kernel(const DecodeArgs a, int workers) {
  constexpr int GROUPS = kMergeThreads / 32;
  constexpr int DPL = D / 32;  // dims per lane
  __shared__ float s_m[GROUPS];
  __shared__ float s_l[GROUPS];
  __shared__ int s_bad[GROUPS];
  __shared__ __align__(16) float s_acc[GROUPS][D];
  asm volatile("griddepcontrol.wait;" ::: "memory");

  const int tid = threadIdx.x, grp = tid >> 5, lane = tid & 31;
  const int S = a.num_seqs, Hkv = a.num_kv_heads, Hq = a.num_q_heads;
  // this warp's first record is read together with the counts (the list has
  // room for S * Hkv records; one past the count is simply not used)
  const int it0 = blockIdx.x * GROUPS + grp;
  const int4 rec0 = it0 < S * Hkv ? __ldcg(reinterpret_cast<const int4*>(a.light_list) + it0)
                                  : make_int4(0, 0, 0, 0);
  const int count = __ldcg(a.heavy);        // items of many pieces
  const int light = __ldcg(a.heavy + 4);    // items of few pieces
  if (count == 0 && light == 0) return;     // nothing listed, nothing to reset
  {
    // items of few pieces: one warp each.  Lane l takes head_dim
    // [DPL*l, DPL*l + DPL) of every head, so each load and store of the warp
    // is contiguous, and all of an item's loads are in flight together.
    constexpr int NP = kWarpMergeMaxPieces;
    using VecF = typename std::conditional<DPL == 4, float4, float2>::type;
    for (int it = it0; it < light; it += gridDim.x * GROUPS) {
      const int4 rec =
          it == it0 ? rec0 : __ldcg(reinterpret_cast<const int4*>(a.light_list) + it);
      const int r0 = rec.x / Hkv, kvh = rec.x - r0 * Hkv;  // first out row, KV head
      const int np = rec.z & 0xffffff;  // (at most NP: listed so)
      const int nr = rec.z >> 24;       // out rows of the item
      auto slot_of = [&](int r) -> long long {  // piece r's partial slot
        return r == 0 ? rec.w : 2 * (static_cast<long long>(rec.y) + r);
      };
      // pieces two at a time, every load of a pair issued before any is used
      // (one memory round trip per pair), merged with a running maximum
      float M[G], L[G], acc[G][DPL];
      int bad = 0;  // bit h: head h poisoned
#pragma unroll
      for (int h = 0; h < G; ++h) {
        M[h] = -INFINITY;
        L[h] = 0.f;
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[h][e] = 0.f;
      }
#pragma unroll
      for (int r0 = 0; r0 < NP; r0 += 2) {
        if (r0 < np) {
          const bool two = r0 + 1 < np;
          float2 ml[2][G];
          VecF ov[2][G];
#pragma unroll
          for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int h = 0; h < G; ++h) {
              const long long sj = slot_of(r0 + (two ? j : 0));  // (a lone last piece: twice)
              ml[j][h] = __ldcg(a.ws_ml + sj * G + h);
              ov[j][h] = __ldcg(reinterpret_cast<const VecF*>(a.ws_o + (sj * G + h) * D) + lane);
            }
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float2 m0 = ml[0][h], m1 = two ? ml[1][h] : make_float2(-INFINITY, 0.f);
            bad |= ((m0.y < 0.f) | (m1.y < 0.f)) << h;
            const float mn = fmaxf(M[h], fmaxf(m0.x, m1.x));
            // (an empty running state, M = -inf, has nothing to scale)
            const float sc = M[h] == -INFINITY ? 0.f : exp2f(M[h] - mn);
            const float w0 = exp2f(m0.x - mn), w1 = two ? exp2f(m1.x - mn) : 0.f;
            L[h] = L[h] * sc + w0 * m0.y + w1 * m1.y;
            const float* t0 = reinterpret_cast<const float*>(&ov[0][h]);
            const float* t1 = reinterpret_cast<const float*>(&ov[1][h]);
#pragma unroll
            for (int e = 0; e < DPL; ++e) acc[h][e] = acc[h][e] * sc + w0 * t0[e] + w1 * t1[e];
            M[h] = mn;
          }
        }
      }
      // column h is head h % GH of out row r0 + h / GH
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const bool hb = (bad >> h) & 1;
        const float inv = hb ? 0.f : 1.f / L[h];
        if (h / GH >= nr) continue;
        T* dst = static_cast<T*>(a.out) +
                 (static_cast<size_t>(r0 + h / GH) * Hq + static_cast<size_t>(kvh) * GH + h % GH) * D +
                 lane * DPL;
#pragma unroll
        for (int e = 0; e < DPL; ++e) dst[e] = static_cast<T>(hb ? 0.f : acc[h][e] * inv);
      }
    }
    // items of many pieces: one CTA per (item, head)
    for (int p = blockIdx.x; p < count * G; p += gridDim.x) {
      const int4 rec = __ldcg(reinterpret_cast<const int4*>(a.heavy_list) + p / G);
      const int hl = p % G;
      const int r0 = rec.x / Hkv, kvh = rec.x - r0 * Hkv;  // first out row, KV head
      const long long ra = rec.y, rb = ra + (rec.z & 0xffffff) - 1;
      const int nr = rec.z >> 24;
      if (hl / GH >= nr) continue;  // (the same for the whole CTA)
      auto slot_of = [&](long long r) -> long long { return r == ra ? rec.w : 2 * r; };

      // each warp takes pieces ra + grp, + GROUPS, ..., four at a time with all
      // their loads in flight, merged with a running maximum; then the warps'
      // (M, L, acc) are combined through shared memory
      constexpr int CHUNK = 4;
      float M = -INFINITY, L = 0.f, acc[DPL];
      int bad = 0;
#pragma unroll
      for (int d = 0; d < DPL; ++d) acc[d] = 0.f;
      for (long long base = ra + grp; base <= rb; base += CHUNK * GROUPS) {
        float2 ml[CHUNK];
        VecF ov[CHUNK];
#pragma unroll
        for (int j = 0; j < CHUNK; ++j) {
          const long long r = base + j * GROUPS;
          const long long sl = slot_of(r <= rb ? r : base);
          ml[j] = __ldcg(a.ws_ml + sl * G + hl);
          ov[j] = __ldcg(reinterpret_cast<const VecF*>(a.ws_o + (sl * G + hl) * D) + lane);
          if (r > rb) ml[j] = make_float2(-INFINITY, 0.f);   // (a repeat, weighed 0)
        }
        float mn = M;
#pragma unroll
        for (int j = 0; j < CHUNK; ++j) {
          mn = fmaxf(mn, ml[j].x);
          bad |= ml[j].y < 0.f;
        }
        const float sc = M == -INFINITY ? 0.f : exp2f(M - mn);
        L *= sc;
#pragma unroll
        for (int d = 0; d < DPL; ++d) acc[d] *= sc;
#pragma unroll
        for (int j = 0; j < CHUNK; ++j) {
          const float w = ml[j].x == -INFINITY ? 0.f : exp2f(ml[j].x - mn);
          L = fmaf(w, ml[j].y, L);
          const float* t = reinterpret_cast<const float*>(&ov[j]);
#pragma unroll
          for (int d = 0; d < DPL; ++d) acc[d] = fmaf(w, t[d], acc[d]);
        }
        M = mn;
      }
      if (lane == 0) {
        s_m[grp] = M;
        s_l[grp] = L;
        s_bad[grp] = bad;
      }
#pragma unroll
      for (int d = 0; d < DPL; ++d) s_acc[grp][lane * DPL + d] = acc[d];
      __syncthreads();
      if (grp == 0) {
        float Mt = -INFINITY;
        int bt = 0;
#pragma unroll
        for (int g = 0; g < GROUPS; ++g) {
          Mt = fmaxf(Mt, s_m[g]);
          bt |= s_bad[g];
        }
        float Lt = 0.f, r[DPL];
#pragma unroll
        for (int d = 0; d < DPL; ++d) r[d] = 0.f;
#pragma unroll
        for (int g = 0; g < GROUPS; ++g) {
          const float f = s_m[g] == -INFINITY ? 0.f : exp2f(s_m[g] - Mt);
          Lt = fmaf(f, s_l[g], Lt);
#pragma unroll
          for (int d = 0; d < DPL; ++d) r[d] = fmaf(f, s_acc[g][lane * DPL + d], r[d]);
        }
        T* dst = static_cast<T*>(a.out) +
                 (static_cast<size_t>(r0 + hl / GH) * Hq + static_cast<size_t>(kvh) * GH + hl % GH) *
                     D +
                 lane * DPL;
#pragma unroll
        for (int d = 0; d < DPL; ++d) dst[d] = static_cast<T>(bt ? 0.f : r[d] / Lt);
      }
      __syncthreads();
    }
  }
  // the last CTA out clears the item list for the next call
  __syncthreads();
  // (every thread of this CTA has used the count it read before this point)
  if (tid == 0 && atomicAdd(a.heavy + 1, 1) == static_cast<int>(gridDim.x) - 1) {
    a.heavy[0] = 0;
    a.heavy[1] = 0;
    a.heavy[4] = 0;
  }
}

}  // namespace pa
