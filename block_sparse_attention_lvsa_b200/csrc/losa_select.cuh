// losa_select.cuh - LoSA minimal key-block set holding a fraction tau of
// the block attention mass, per (head, query block).
//
// Source: "LoSA (Near-Lossless Sparse Attention)" article (ai.ros.co.jp),
// sections "LoSA's innovative approach" (keep 99% of the attention mass) and
// "Balancing efficiency and quality" (per head and query block, the minimal
// key/value block set reaching that mass, measured once and frozen).
//
// Per row: Q_kb = floor(mass_kb * 2^33) (exact in double);  the kept set is
// the shortest prefix of the order (Q desc, kb asc) whose Q-sum reaches
// ceil(tau * (double)sum Q).  Instead of sorting the row, the kernel finds
// the last key of that prefix by a most-significant-digit radix select over
// the composite 64-bit key (Q << 16 | (65535 - kb)), whose descending order
// is exactly (Q desc, kb asc): 8 passes of a 256-bin histogram of Q sums and
// counts, each narrowing the key prefix to the digit where the running sum
// crosses the threshold.  Kept ids (key >= pivot) are then compacted in
// ascending kb order with warp ballots.  All sums are 64-bit integers, so
// the result does not depend on the order of accumulation.
#pragma once
#include "ptx.cuh"

namespace bsa {

constexpr int kSelectThreads = 256;
constexpr int kSelectMaxBlocks = 8192;

__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// grid: one CTA per row (h, qb); dynamic smem: nKB * 8 bytes of keys.
__global__ void __launch_bounds__(kSelectThreads)
losa_select_kernel(const float* __restrict__ mass, int nKB, double tau,
                   int32_t* __restrict__ idx, int32_t* __restrict__ cnt) {
  extern __shared__ unsigned long long s_key[];
  __shared__ unsigned long long s_hist[256];
  __shared__ unsigned int s_count[256];
  __shared__ unsigned long long s_red[kSelectThreads / 32];
  __shared__ unsigned long long s_prefix, s_above, s_thr;
  __shared__ int s_wcount[kSelectThreads / 32];

  const size_t row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* m = mass + row * nKB;

  // 1. exact quantisation and composite keys
  unsigned long long local = 0;
  for (int i = tid; i < nKB; i += kSelectThreads) {
    float x = m[i];
    if (!(x >= 0.0f && x < 16384.0f)) {       // NaN, negative, too large
      set_status(BSA_ERR_ARG);
      x = (x >= 16384.0f) ? 16383.999f : 0.0f;
    }
    const unsigned long long q = static_cast<unsigned long long>(static_cast<double>(x) * 8589934592.0);
    s_key[i] = (q << 16) | static_cast<unsigned long long>(65535 - i);
    local += q;
  }
  local = warp_sum_u64(local);
  if (lane == 0) s_red[warp] = local;
  __syncthreads();
  if (tid == 0) {
    unsigned long long total = 0;
    for (int w = 0; w < kSelectThreads / 32; ++w) total += s_red[w];
    const double t = __dmul_rn(tau, __ull2double_rn(total));
    s_thr = static_cast<unsigned long long>(ceil(t));
    s_prefix = 0;
    s_above = 0;
  }
  __syncthreads();
  const unsigned long long thr = s_thr;

  // 2. radix select of the pivot key (the last key of the kept prefix)
  for (int pass = 7; pass >= 0; --pass) {
    const int shift = pass * 8;
    s_hist[tid] = 0;          // 256 threads, 256 bins
    s_count[tid] = 0;
    __syncthreads();
    const unsigned long long prefix = s_prefix;
    const unsigned long long himask = (pass == 7) ? 0ull : (~0ull << (shift + 8));
    for (int i = tid; i < nKB; i += kSelectThreads) {
      const unsigned long long key = s_key[i];
      if (((key ^ prefix) & himask) == 0ull) {
        const int dgt = static_cast<int>((key >> shift) & 255ull);
        atomicAdd(&s_hist[dgt], key >> 16);
        atomicAdd(&s_count[dgt], 1u);
      }
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns digits 255-8l ... 248-8l (descending)
      unsigned long long lsum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) lsum += s_hist[255 - (8 * lane + j)];
      // exclusive prefix over lanes in lane order (= descending digits)
      unsigned long long incl = lsum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += v;
      }
      const unsigned long long excl = incl - lsum;
      const unsigned long long above = s_above;
      int found = -1;
      unsigned long long higher = 0, run = above + excl;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int dgt = 255 - (8 * lane + j);
        const unsigned long long hsum = s_hist[dgt];
        if (found < 0) {
          if (s_count[dgt] != 0u && run + hsum >= thr) {
            found = dgt;
            higher = run;
          }
          run += hsum;
        }
      }
      const unsigned int hit = __ballot_sync(0xFFFFFFFFu, found >= 0);
      // lowest lane with a hit holds the largest qualifying digit
      int winner = hit ? (__ffs(hit) - 1) : -1;
      if (winner < 0) {
        // cannot happen for tau <= 1; keep the smallest digit present
        int lowest = 256;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int dgt = 255 - (8 * lane + j);
          if (s_count[dgt] != 0u) lowest = min(lowest, dgt);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) lowest = min(lowest, __shfl_xor_sync(0xFFFFFFFFu, lowest, o));
        if (lane == 0) {
          s_prefix = prefix | (static_cast<unsigned long long>(lowest & 255) << shift);
        }
      } else if (lane == winner) {
        s_prefix = prefix | (static_cast<unsigned long long>(found) << shift);
        s_above = higher;
      }
    }
    __syncthreads();
  }
  const unsigned long long pivot = s_prefix;

  // 3. ascending compaction of kept ids (key >= pivot), then -1 padding
  int32_t* out = idx + row * nKB;
  int running = 0;
  for (int base = 0; base < nKB; base += kSelectThreads) {
    const int i = base + tid;
    const bool keep = (i < nKB) && (s_key[i] >= pivot);
    const unsigned int b = __ballot_sync(0xFFFFFFFFu, keep);
    if (lane == 0) s_wcount[warp] = __popc(b);
    __syncthreads();
    int off = running;
    int tot = 0;
#pragma unroll
    for (int w = 0; w < kSelectThreads / 32; ++w) {
      const int c = s_wcount[w];
      if (w < warp) off += c;
      tot += c;
    }
    if (keep) out[off + __popc(b & ((1u << lane) - 1u))] = i;
    running += tot;
    __syncthreads();
  }
  for (int i = running + tid; i < nKB; i += kSelectThreads) out[i] = -1;
  if (tid == 0) cnt[row] = running;
}

}  // namespace bsa
