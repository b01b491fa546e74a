// lvsa_index.cuh - LVSA attended-frame sets and their expansion to the
// 128-token tile grid.
//
// Source: "LVSA: Training-Free Sparse Attention for Long Video Diffusion"
// (gist.science explainer), technical summary section 2 "Method": query
// frame t attends A(t) = G u W(t); the anchors G_s rotate by s mod T_per per
// denoising step; the local window is widened around anchors so that the
// budget |A(t)| stays at C.  Fill rule used here: A(t) = G_s u {t} plus the
// nearest non-anchor frames (distance |f - t|, earlier frame first at equal
// distance, clipped to [0, T)) until |A(t)| = C; nothing is dropped when
// |G_s u {t}| already exceeds C.
#pragma once
#include "ptx.cuh"

namespace bsa {

constexpr int kMaxFrames = 1024;            // T limit: one thread per frame, 32 bit-words
constexpr int kMaxFrameWords = kMaxFrames / 32;

// One thread per query frame t.  frames [T][T] (ascending, -1 padded), counts [T].
__global__ void lvsa_build_index_kernel(int T, int T_per, int C, int step,
                                        int32_t* __restrict__ frames, int32_t* __restrict__ counts) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  uint32_t bits[kMaxFrameWords];
  const int TW = (T + 31) / 32;
  for (int w = 0; w < kMaxFrameWords; ++w) bits[w] = 0u;
  const int s_mod = step % T_per;
  int have = 0;
  // anchors: (f - s) mod T_per == 0  <=>  f mod T_per == s mod T_per
  for (int f = s_mod; f < T; f += T_per) {
    bits[f >> 5] |= 1u << (f & 31);
    ++have;
  }
  if (!((bits[t >> 5] >> (t & 31)) & 1u)) {
    bits[t >> 5] |= 1u << (t & 31);
    ++have;
  }
  int need = C - have;
  for (int dist = 1; need > 0 && (t - dist >= 0 || t + dist < T); ++dist) {
    const int cand[2] = {t - dist, t + dist};   // earlier frame first at a tie
    for (int c = 0; c < 2; ++c) {
      const int f = cand[c];
      if (need > 0 && f >= 0 && f < T && !((bits[f >> 5] >> (f & 31)) & 1u)) {
        bits[f >> 5] |= 1u << (f & 31);
        --need;
      }
    }
  }
  int32_t* row = frames + static_cast<size_t>(t) * T;
  int n = 0;
  for (int w = 0; w < TW; ++w) {
    uint32_t b = bits[w];
    while (b) {
      const int i = __ffs(b) - 1;
      b &= b - 1;
      row[n++] = w * 32 + i;
    }
  }
  counts[t] = n;
  for (int i = n; i < T; ++i) row[i] = -1;
}

// Bit matrix fbits[t][w]: bit f of row t set iff f in A(t).  One thread per t.
__global__ void lvsa_frame_bits_kernel(int T, const int32_t* __restrict__ frames,
                                       const int32_t* __restrict__ counts, uint32_t* __restrict__ fbits) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  const int TW = (T + 31) / 32;
  uint32_t bits[kMaxFrameWords];
  for (int w = 0; w < kMaxFrameWords; ++w) bits[w] = 0u;
  int n = counts[t];
  if (n < 0 || n > T) {
    set_status(BSA_ERR_INDEX_RANGE);
    n = n < 0 ? 0 : T;
  }
  const int32_t* row = frames + static_cast<size_t>(t) * T;
  for (int i = 0; i < n; ++i) {
    const int f = row[i];
    if (f < 0 || f >= T) {
      set_status(BSA_ERR_INDEX_RANGE);
      continue;
    }
    bits[f >> 5] |= 1u << (f & 31);
  }
  for (int w = 0; w < TW; ++w) fbits[static_cast<size_t>(t) * TW + w] = bits[w];
}

// Per query tile qt (one warp): ascending kept key tiles on the 128 grid and
// a "partial" flag (some pair of the 128x128 block not allowed, or the key
// tile reaches past N).  Output rows are nB long; count[qt] entries valid.
// The frames spanned by a tile's rows (and columns) form a contiguous range,
// so "some pair allowed" is a test against the union of the rows' frame sets
// and "all pairs allowed" a test against their intersection.
__global__ void lvsa_tiles_kernel(int N, int T, int P, int nB, const uint32_t* __restrict__ fbits,
                                  int32_t* __restrict__ tile_cnt, int32_t* __restrict__ tile_idx,
                                  uint8_t* __restrict__ tile_flag) {
  __shared__ uint32_t s_union[4][kMaxFrameWords];
  __shared__ uint32_t s_inter[4][kMaxFrameWords];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x * 4 + warp;
  if (qt >= nB) return;
  const int TW = (T + 31) / 32;
  const int q_lo = qt * 128, q_hi = min(q_lo + 128, N) - 1;
  const int fq_lo = q_lo / P, fq_hi = q_hi / P;
  if (lane < TW) {
    uint32_t u = 0u, in = 0xFFFFFFFFu;
    for (int f = fq_lo; f <= fq_hi; ++f) {
      const uint32_t b = fbits[static_cast<size_t>(f) * TW + lane];
      u |= b;
      in &= b;
    }
    s_union[warp][lane] = u;
    s_inter[warp][lane] = in;
  }
  __syncwarp();
  int total = 0;
  for (int base = 0; base < nB; base += 32) {
    const int kt = base + lane;
    bool keep = false, partial = false;
    if (kt < nB) {
      const int k_lo = kt * 128, k_hi = min(k_lo + 128, N) - 1;
      bool any = false, all = true;
      for (int f = k_lo / P; f <= k_hi / P; ++f) {
        any |= (s_union[warp][f >> 5] >> (f & 31)) & 1u;
        all &= ((s_inter[warp][f >> 5] >> (f & 31)) & 1u) != 0u;
      }
      keep = any;
      partial = !all || (k_lo + 128 > N);
    }
    const uint32_t ballot = __ballot_sync(0xFFFFFFFFu, keep);
    if (keep) {
      const int pos = total + __popc(ballot & ((1u << lane) - 1u));
      tile_idx[static_cast<size_t>(qt) * nB + pos] = kt;
      tile_flag[static_cast<size_t>(qt) * nB + pos] = partial ? 1 : 0;
    }
    total += __popc(ballot);
  }
  if (lane == 0) tile_cnt[qt] = total;
}

// Per-entry partial flags of a block index intersected with LVSA frames.
// Entry (h, qb, j < cnt[h][qb]) keeps key tile kt = idx[h][qb][j].  Pairs of
// that tile stay subject to the LVSA element rule, so the tile is whole only
// if LVSA keeps it whole for query tile qb: its flag is the one in qb's LVSA
// tile list (found by binary search: the lists are ascending).  A tile the
// LVSA list does not hold is marked partial; its element mask then admits
// none of its pairs.  One block per (h, qb) row.
__global__ void compose_flags_kernel(int nB, const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt,
                                     const int32_t* __restrict__ tile_cnt, const int32_t* __restrict__ tile_idx,
                                     const uint8_t* __restrict__ tile_flag, uint8_t* __restrict__ flags) {
  const size_t row = blockIdx.x;                        // h * nB + qb
  const int qb = static_cast<int>(row % nB);
  const int c = min(max(cnt[row], 0), nB);
  const int n = min(max(tile_cnt[qb], 0), nB);
  const int32_t* lv = tile_idx + static_cast<size_t>(qb) * nB;
  for (int j = threadIdx.x; j < nB; j += blockDim.x) {
    uint8_t f = 0;
    if (j < c) {
      f = 1;
      const int kt = idx[row * nB + j];
      int lo = 0, hi = n;                               // first position with lv[pos] >= kt
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (lv[mid] < kt) lo = mid + 1; else hi = mid;
      }
      if (lo < n && lv[lo] == kt) f = tile_flag[static_cast<size_t>(qb) * nB + lo];
    }
    flags[row * nB + j] = f;
  }
}

}  // namespace bsa
