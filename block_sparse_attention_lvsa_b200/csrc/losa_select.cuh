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
// bisection: each step is a compare-and-sum over the row and a 64-bit
// warp-shuffle reduction - no sorting, no atomics, no block barriers.  Rows
// of up to 2048 blocks (registers) bisect over the 31 bits of the mass
// instead of the 57-bit keys and settle ties in Q by kb afterwards (see
// losa_select_reg_kernel); longer rows (shared memory) bisect over the keys.
// The kept ids are then written in ascending kb order with warp ballots.
// Every sum is a 64-bit integer, so the result does not depend on the order
// of accumulation.
#pragma once
#include "ptx.cuh"

namespace bsa {

constexpr int kSelectMaxBlocks = 8192;

__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}
// ceil(tau * (double)total) with one IEEE double multiply, never above the
// total: for totals above 2^53 the conversion to double can round up, and a
// threshold the whole row cannot reach would make the kept set ill-defined
// (the shortest prefix reaching the total is then the answer).
__device__ __forceinline__ unsigned long long select_threshold(double tau, unsigned long long total) {
  const unsigned long long t = static_cast<unsigned long long>(ceil(__dmul_rn(tau, __ull2double_rn(total))));
  return t < total ? t : total;
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
    const unsigned long long thr = select_threshold(tau, total);
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

// Same result with the row in registers (nKB <= 32 * KPL; lane l holds
// blocks l, l+32, ...), found by a search over 32-bit values instead of the
// 64-bit keys.  Q is a non-decreasing function of the mass, and the bit
// pattern of a non-negative float orders like its value, so
// S(u) = sum of Q over blocks whose mass bits are >= u is non-increasing in
// u.  Bisection over the 31 bits gives the largest u with S(u) >= threshold
// (for rows of up to 512 blocks it stops early once the interval left to
// search holds one mass value);
// u is the mass bits of some block, and its Q is the pivot value Qp.  Every
// block with Q > Qp has a larger mass, so their Q-sum A stays below the
// threshold (else u + 1 would qualify), and the kept set is every block
// with Q > Qp plus the first ceil((threshold - A) / Qp) blocks with Q == Qp
// in ascending kb order: the shortest prefix of the (Q desc, kb asc) order.
// A zero threshold (all masses zero) keeps the first block of that order.
template <int KPL>
__global__ void losa_select_reg_kernel(const float* __restrict__ mass, int rows, int nKB, double tau,
                                       int32_t* __restrict__ idx, int32_t* __restrict__ cnt) {
  const int lane = threadIdx.x & 31;
  const int wpc = blockDim.x >> 5;
  for (int row = blockIdx.x * wpc + (threadIdx.x >> 5); row < rows; row += gridDim.x * wpc) {
    const float* m = mass + static_cast<size_t>(row) * nKB;
    unsigned long long q[KPL];
    uint32_t mb[KPL];
    float mv[KPL];
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
      const int i = lane + 32 * j;
      mv[j] = (i < nKB) ? m[i] : 0.0f;
    }
    unsigned long long total = 0, qmax = 0;
    bool bad = false;
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
      const int i = lane + 32 * j;
      float xv = mv[j];
      if (!(xv >= 0.0f && xv < 16384.0f)) {       // NaN, negative, too large
        bad = bad || (i < nKB);
        xv = (xv >= 16384.0f) ? 16383.999f : 0.0f;
      }
      // padding slots: Q = 0 and mass bits 0, never counted or kept
      q[j] = (i < nKB) ? static_cast<unsigned long long>(static_cast<double>(xv) * 8589934592.0) : 0ull;
      mb[j] = (i < nKB) ? (__float_as_uint(xv) & 0x7FFFFFFFu) : 0u;   // -0.0 orders as +0.0
      total += q[j];
      qmax = q[j] > qmax ? q[j] : qmax;
    }
    if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) set_status(BSA_ERR_ARG);
    total = warp_sum_u64(total);
    const unsigned long long thr = select_threshold(tau, total);
    unsigned long long qp, take;          // pivot value, blocks of Q == qp to keep
    if (thr == 0) {
      qp = warp_max_u64(qmax);
      take = 1;
    } else {
      uint32_t u = 0;
      for (int b = 30; b >= 0; --b) {
        const uint32_t c = u | (1u << b);
        unsigned long long sum = 0;
#pragma unroll
        for (int j = 0; j < KPL; ++j) sum += (mb[j] >= c) ? q[j] : 0ull;
        if (warp_sum_u64(sum) >= thr) u = c;
        // S(u) >= threshold > S(u + 2^b) now holds, so some block has mass
        // bits in [u, u + 2^b); when all of them share one value, that value
        // is the answer and the remaining rounds can be skipped (tried after
        // the rounds of bits 24, 21, ..., 3 for rows of up to 512 blocks;
        // longer rows keep all 31 rounds, where the check measured slower)
        if (KPL <= 16 && b > 0 && b <= 24 && (24 - b) % 3 == 0) {
          uint32_t lo = 0xFFFFFFFFu, hi = 0u;
#pragma unroll
          for (int j = 0; j < KPL; ++j) {
            if (lane + 32 * j < nKB && mb[j] >= u && mb[j] - u < (1u << b)) {
              lo = min(lo, mb[j]);
              hi = max(hi, mb[j]);
            }
          }
          lo = __reduce_min_sync(0xFFFFFFFFu, lo);
          hi = __reduce_max_sync(0xFFFFFFFFu, hi);
          if (lo == hi) {
            u = lo;
            break;
          }
        }
      }
      unsigned long long qu = 0;
#pragma unroll
      for (int j = 0; j < KPL; ++j) qu = (mb[j] == u && lane + 32 * j < nKB) ? q[j] : qu;
      qp = warp_max_u64(qu);
      unsigned long long above = 0;
#pragma unroll
      for (int j = 0; j < KPL; ++j) above += (q[j] > qp) ? q[j] : 0ull;
      above = warp_sum_u64(above);
      // thr > above and qp >= 1 here (see above); the guards only keep a
      // malformed row from dividing by zero
      const unsigned long long need = thr > above ? thr - above : 1ull;
      take = qp > 0 ? (need + qp - 1) / qp : 1ull;
    }
    int32_t* out = idx + static_cast<size_t>(row) * nKB;
    int running = 0;
    unsigned long long ties = 0;
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
      const int i = lane + 32 * j;
      const bool tie = (i < nKB) && (q[j] == qp);
      const unsigned int tmask = __ballot_sync(0xFFFFFFFFu, tie);
      const unsigned long long rank = ties + __popc(tmask & ((1u << lane) - 1u));
      ties += __popc(tmask);
      const bool keep = (i < nKB) && (q[j] > qp || (tie && rank < take));
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
