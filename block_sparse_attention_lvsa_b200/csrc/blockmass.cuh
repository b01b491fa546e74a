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
// One warp per (head, key tile, query block), query blocks fastest so that
// neighbouring warps read neighbouring 512-byte runs of lpart.  Each lane
// adds its 4 rows in a fixed order, then a butterfly adds the lanes: the
// result does not depend on scheduling.
#pragma once
#include "ptx.cuh"

namespace bsa {

constexpr int kMassThreads = 256;

__global__ void __launch_bounds__(kMassThreads)
blockmass_reduce_kernel(const float* __restrict__ lpart, const float* __restrict__ lse, float* __restrict__ mass,
                        int N, int nB, int h_off, int hc) {
  const int lane = threadIdx.x & 31;
  const long long w = static_cast<long long>(blockIdx.x) * (kMassThreads / 32) + (threadIdx.x >> 5);
  const long long per_head = static_cast<long long>(nB) * nB;
  if (w >= per_head * hc) return;
  const int qb = static_cast<int>(w % nB);
  const int kt = static_cast<int>((w / nB) % nB);
  const int hl = static_cast<int>(w / per_head);
  const int h = hl + h_off;
  const float* lp = lpart + (static_cast<size_t>(hl) * nB + kt) * N;
  const float* ls = lse + static_cast<size_t>(h) * N;
  float acc = 0.f;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int q = qb * 128 + 32 * u + lane;
    if (q < N) {
      const float v = lp[q];
      const float l2 = ls[q] * 1.4426950408889634f;
      // -inf: no allowed key of the tile in this row; NaN: a tile the index
      // never reached (the workspace was set to NaN first); lse -inf: an empty row
      if (v > -INFINITY && l2 > -INFINITY) acc += ex2_approx(v - l2);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
  if (lane == 0) mass[(static_cast<size_t>(h) * nB + qb) * nB + kt] = acc;
}

}  // namespace bsa
