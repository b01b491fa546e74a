// losa_select.cuh - LoSA minimal key-block set holding a fraction tau of
// the block attention mass, per (head, query block).
//
// Source: "LoSA (Near-Lossless Sparse Attention)" article (ai.ros.co.jp),
// sections "LoSA's innovative approach" (keep 99% of the attention mass) and
// "Balancing efficiency and quality" (per head and query block, the minimal
// key/value block set reaching that mass, measured once and frozen).
//
// Per row: Q_kb = floor(mass_kb * 2^33) (exact in double); the kept set is
// the shortest prefix of the order (Q desc, kb asc) whose Q-sum reaches
// ceil(tau * (double)sum Q).  With the composite 64-bit key
// key_kb = Q_kb << 16 | (65535 - kb), whose descending order is exactly
// (Q desc, kb asc), the prefix is {kb : key_kb >= pivot}, where pivot is the
// largest key x with S(x) = sum_{key >= x} Q >= threshold (S only drops at
// keys, so that x is itself a key).  One warp per row finds the pivot by
// bisection over the key bits: each step is a compare-and-sum over the row
// and a 64-bit warp-shuffle reduction - no sorting, no atomics, no block
// barriers.  The kept ids are then written in ascending kb order with warp
// ballots.  Every sum is a 64-bit integer, so the result does not depend on
// the order of accumulation.
#pragma once
#include "ptx.cuh"

namespace bsa {

constexpr int kSelectMaxBlocks = 8192;

__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}
__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long w = __shfl_xor_sync(0xFFFFFFFFu, v, o);
    v = w > v ? w : v;
  }
  return v;
}

// grid-stride over rows; each warp owns rows (warp id across the grid);
// dynamic smem: warps_per_cta * nKB * 8 bytes of keys
__global__ void losa_select_kernel(const float* __restrict__ mass, int rows, int nKB, double tau,
                                   int32_t* __restrict__ idx, int32_t* __restrict__ cnt) {
  extern __shared__ unsigned long long s_keys[];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int wpc = blockDim.x >> 5;
  unsigned long long* key = s_keys + static_cast<size_t>(wid) * nKB;
  for (int row = blockIdx.x * wpc + wid; row < rows; row += gridDim.x * wpc) {
    const float* m = mass + static_cast<size_t>(row) * nKB;
    // 1. exact quantisation and composite keys
    unsigned long long total = 0, kmax = 0;
    bool bad = false;
    for (int i = lane; i < nKB; i += 32) {
      float xv = m[i];
      if (!(xv >= 0.0f && xv < 16384.0f)) {       // NaN, negative, too large
        bad = true;
        xv = (xv >= 16384.0f) ? 16383.999f : 0.0f;
      }
      const unsigned long long q = static_cast<unsigned long long>(static_cast<double>(xv) * 8589934592.0);
      const unsigned long long k = (q << 16) | static_cast<unsigned long long>(65535 - i);
      key[i] = k;
      total += q;
      kmax = k > kmax ? k : kmax;
    }
    if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) set_status(BSA_ERR_ARG);
    total = warp_sum_u64(total);
    kmax = warp_max_u64(kmax);
    __syncwarp();
    const unsigned long long thr =
        static_cast<unsigned long long>(ceil(__dmul_rn(tau, __ull2double_rn(total))));
    // 2. pivot = largest key x with S(x) >= thr (thr == 0: the largest key)
    unsigned long long pivot = kmax;
    if (thr > 0) {
      unsigned long long prefix = 0;
      for (int b = 63 - __clzll(static_cast<long long>(kmax)); b >= 0; --b) {
        const unsigned long long c = prefix | (1ull << b);
        unsigned long long s = 0;
        for (int i = lane; i < nKB; i += 32) {
          const unsigned long long k = key[i];
          if (k >= c) s += k >> 16;
        }
        if (warp_sum_u64(s) >= thr) prefix = c;
      }
      pivot = prefix;
    }
    // 3. ascending compaction of kept ids (key >= pivot), then -1 padding
    int32_t* out = idx + static_cast<size_t>(row) * nKB;
    int running = 0;
    for (int base = 0; base < nKB; base += 32) {
      const int i = base + lane;
      const bool keep = (i < nKB) && (key[i] >= pivot);
      const unsigned int bmask = __ballot_sync(0xFFFFFFFFu, keep);
      if (keep) out[running + __popc(bmask & ((1u << lane) - 1u))] = i;
      running += __popc(bmask);
    }
    for (int i = running + lane; i < nKB; i += 32) out[i] = -1;
    if (lane == 0) cnt[row] = running;
    __syncwarp();
  }
}

// Same computation with the row's keys in registers (nKB <= 32 * KPL): lane
// l holds the keys of blocks l, l+32, ...; loads are unrolled, and the pivot
// search decides two key bits per round (three candidate thresholds, three
// independent warp reductions), halving the dependent rounds.
template <int KPL>
__global__ void losa_select_reg_kernel(const float* __restrict__ mass, int rows, int nKB, double tau,
                                       int32_t* __restrict__ idx, int32_t* __restrict__ cnt) {
  const int lane = threadIdx.x & 31;
  const int wpc = blockDim.x >> 5;
  for (int row = blockIdx.x * wpc + (threadIdx.x >> 5); row < rows; row += gridDim.x * wpc) {
    const float* m = mass + static_cast<size_t>(row) * nKB;
    unsigned long long key[KPL];
    float mv[KPL];
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
      const int i = lane + 32 * j;
      mv[j] = (i < nKB) ? m[i] : 0.0f;
    }
    unsigned long long total = 0, kmax = 0;
    bool bad = false;
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
      const int i = lane + 32 * j;
      float xv = mv[j];
      if (!(xv >= 0.0f && xv < 16384.0f)) {       // NaN, negative, too large
        bad = bad || (i < nKB);
        xv = (xv >= 16384.0f) ? 16383.999f : 0.0f;
      }
      const unsigned long long q = static_cast<unsigned long long>(static_cast<double>(xv) * 8589934592.0);
      // padding slots get key 0: below every real key (real keys carry 65535 - kb > 0)
      key[j] = (i < nKB) ? ((q << 16) | static_cast<unsigned long long>(65535 - i)) : 0ull;
      total += (i < nKB) ? q : 0ull;
      kmax = key[j] > kmax ? key[j] : kmax;
    }
    if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) set_status(BSA_ERR_ARG);
    total = warp_sum_u64(total);
    kmax = warp_max_u64(kmax);
    const unsigned long long thr =
        static_cast<unsigned long long>(ceil(__dmul_rn(tau, __ull2double_rn(total))));
    unsigned long long pivot = kmax;
    if (thr > 0) {
      unsigned long long prefix = 0;
      int b = 63 - __clzll(static_cast<long long>(kmax));   // highest bit that can be set
      if ((b & 1) == 0) {                                    // odd number of bits: one binary round
        const unsigned long long c = 1ull << b;
        unsigned long long s0 = 0;
#pragma unroll
        for (int j = 0; j < KPL; ++j) s0 += (key[j] >= c) ? (key[j] >> 16) : 0ull;
        if (warp_sum_u64(s0) >= thr) prefix = c;
        --b;
      }
      for (; b >= 1; b -= 2) {                               // bits b, b-1 per round
        const unsigned long long c1 = prefix | (1ull << (b - 1));
        const unsigned long long c2 = prefix | (2ull << (b - 1));
        const unsigned long long c3 = prefix | (3ull << (b - 1));
        unsigned long long s1 = 0, s2 = 0, s3 = 0;
#pragma unroll
        for (int j = 0; j < KPL; ++j) {
          const unsigned long long qj = key[j] >> 16;
          s1 += (key[j] >= c1) ? qj : 0ull;
          s2 += (key[j] >= c2) ? qj : 0ull;
          s3 += (key[j] >= c3) ? qj : 0ull;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          s1 += __shfl_xor_sync(0xFFFFFFFFu, s1, o);
          s2 += __shfl_xor_sync(0xFFFFFFFFu, s2, o);
          s3 += __shfl_xor_sync(0xFFFFFFFFu, s3, o);
        }
        // S is non-increasing: take the largest candidate that still reaches thr
        prefix = (s3 >= thr) ? c3 : (s2 >= thr) ? c2 : (s1 >= thr) ? c1 : prefix;
      }
      pivot = prefix;
    }
    int32_t* out = idx + static_cast<size_t>(row) * nKB;
    int running = 0;
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
      const int i = lane + 32 * j;
      const bool keep = (i < nKB) && (key[j] >= pivot);
      const unsigned int bmask = __ballot_sync(0xFFFFFFFFu, keep);
      if (keep) out[running + __popc(bmask & ((1u << lane) - 1u))] = i;
      running += __popc(bmask);
    }
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
      const int i = lane + 32 * j;
      if (i < nKB && i >= running) out[i] = -1;
    }
    if (lane == 0) cnt[row] = running;
  }
}

}  // namespace bsa
