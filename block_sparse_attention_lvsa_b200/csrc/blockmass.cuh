// blockmass.cuh - LoSA block mass from the one-pass dense measuring step.
//
// Source: "LoSA (Near-Lossless Sparse Attention)" article, section
// "Balancing efficiency and quality" (one dense step measures the exact
// inter-block attention mass).  The dense forward in mass mode leaves, per
// local head hl, key tile kt and query row q,
//   lpart[hl][kt][q] = log2(sum_{k in kt} exp2(s_qk * scale * log2e - m)) + m
// (m the stabiliser the row used for that tile).  With the row's final
// log-sum-exp lse[h][q] (natural log), the probability mass of (qb, kt) is
//   mass[h][qb][kt] = sum_{q in qb, q < N} exp2(lpart[hl][kt][q] - lse[h][q] * log2e).
//
// Grid (query-block groups, key-tile groups, local heads): one warp per query
// block qb, looping over kMassKt key tiles.  A lane owns 4 consecutive rows
// (16-byte loads of lpart and lse where aligned), loads their LSE once and
// adds its rows in a fixed order before a butterfly over the lanes, so the
// result does not depend on scheduling.  Lane j keeps the sum of the j-th
// key tile and the warp writes its kMassKt results with one contiguous store.
// The loads of kMassBatch key tiles are issued before any of their sums, so
// that a warp keeps that many 512-byte loads in flight (one at a time left
// the kernel at ~70% of HBM bandwidth: too few bytes in flight per SM).
// Algorithmic bytes: lpart read once (H * nB * N * 4), mass written once; the
// LSE of a row is read once per key-tile group (from L2).
#pragma once
#include "ptx.cuh"

namespace bsa {

constexpr int kMassThreads = 256;                  // 8 warps = 8 query blocks per CTA
constexpr int kMassWarps = kMassThreads / 32;
constexpr int kMassKt = 16;                        // key tiles per warp
constexpr int kMassBatch = 4;                      // key tiles whose loads are in flight together

__device__ __forceinline__ void load4(const float* p, int q0, int N, bool vec, float (&v)[4], float fill) {
  if (vec) {
    const float4 t = __ldg(reinterpret_cast<const float4*>(p + q0));
    v[0] = t.x;
    v[1] = t.y;
    v[2] = t.z;
    v[3] = t.w;
  } else {
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = (q0 + u < N) ? __ldg(p + q0 + u) : fill;
  }
}

__global__ void __launch_bounds__(kMassThreads)
blockmass_reduce_kernel(const float* __restrict__ lpart, const float* __restrict__ lse, float* __restrict__ mass,
                        int N, int nB, int h_off) {
  const int lane = threadIdx.x & 31;
  const int qb = blockIdx.x * kMassWarps + (threadIdx.x >> 5);
  const int kt0 = blockIdx.y * kMassKt;
  const int hl = blockIdx.z;
  if (qb >= nB) return;
  const int h = hl + h_off;
  const int q0 = qb * 128 + 4 * lane;
  const float* ls = lse + static_cast<size_t>(h) * N;
  // 16-byte loads when the lane's 4 rows are in range and both rows start aligned
  const bool vec = (q0 + 3 < N) && ((N & 3) == 0) &&
                   (((reinterpret_cast<uintptr_t>(ls) | reinterpret_cast<uintptr_t>(lpart)) & 15u) == 0);
  float l2[4];
  load4(ls, q0, N, vec, l2, -INFINITY);
#pragma unroll
  for (int u = 0; u < 4; ++u) l2[u] *= 1.4426950408889634f;
  const int nkt = min(kMassKt, nB - kt0);
  float keep = 0.f;
  for (int j0 = 0; j0 < nkt; j0 += kMassBatch) {
    float v[kMassBatch][4];
#pragma unroll
    for (int t = 0; t < kMassBatch; ++t) {
      if (j0 + t < nkt) {
        load4(lpart + (static_cast<size_t>(hl) * nB + kt0 + j0 + t) * N, q0, N, vec, v[t], -INFINITY);
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) v[t][u] = -INFINITY;
      }
    }
#pragma unroll
    for (int t = 0; t < kMassBatch; ++t) {
      float acc = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        // -inf: no allowed key of the tile in this row (or a row past N); NaN:
        // a tile the index never reached (the workspace was set to NaN first);
        // lse -inf: an empty row
        if (v[t][u] > -INFINITY && l2[u] > -INFINITY) acc += ex2_approx(v[t][u] - l2[u]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
      if (lane == j0 + t) keep = acc;
    }
  }
  if (lane < nkt) mass[(static_cast<size_t>(h) * nB + qb) * nB + kt0 + lane] = keep;
}

}  // namespace bsa
