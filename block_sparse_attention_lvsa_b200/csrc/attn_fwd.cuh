// attn_fwd.cuh - block-sparse / dense softmax attention forward on sm_100a
// tensor cores (tcgen05 + TMEM + TMA), and the LoSA block-mass pass.
//
// Sources: "LVSA: Training-Free Sparse Attention for Long Video Diffusion"
// (gist.science explainer), technical summary section 2 (block-sparse
// attention restricted to A(t); cost |A(t)| * P * d per query) and section 4
// (block-sparse kernel against dense attention); "LoSA (Near-Lossless Sparse
// Attention)" article, section "Balancing efficiency and quality" (one dense
// step measuring exact inter-block mass, then the frozen block index).
//
// One CTA = one 128-row query tile of one head; it walks the key tiles its
// list holds.  Warp roles (256 threads):
//   warp 0      TMA producer: Q once, then K (and V) tiles into 2-deep rings
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer
//   warps 4..7  softmax warpgroup: thread r owns query row r (TMEM lane r)
// TMEM columns: S0 [0,128) and S1 [128,256) (double-buffered scores, f32),
// O [256, 256+d) (f32 accumulator).  S(j+1) = Q K(j+1)^T runs on the tensor
// core while the softmax of tile j runs; then O += P(j) V(j), with P(j) in
// shared memory (bf16, 128-byte swizzled, K-major).  The online softmax
// keeps a running row maximum in log2 units and rescales O (TMEM ld/st)
// only when the maximum grows by more than 2^8, which is exact after the
// final division by the row sum.  Tiles flagged partial (frame boundary or
// sequence end) get an element mask from the frame bit matrix.
//
// Mass mode (MASS = true) is the second pass of the dense measuring step:
// it recomputes S tile by tile, forms p = exp2(s*scale*log2e - lse*log2e)
// with the final row LSE of the forward pass and reduces p over the tile's
// 128 x 128 entries into mass[h][qt][kt] (fixed reduction order).
#pragma once
#include "ptx.cuh"

namespace bsa {

struct AttnParams {
  int N, H, nB;
  float sl2;                        // scale * log2(e)
  // key-tile lists: tile j of (h, qt) is list[h*lhs + qt*lrs + j], j < count[h*chs + qt]
  const int32_t* list;
  const int32_t* count;
  const uint8_t* flags;             // per list entry: 1 = partial tile (LVSA), or null
  long long lhs;                    // list head stride (elements)
  int lrs;                          // list row stride (elements)
  int chs;                          // count head stride
  int dense;                        // 1: tile j = j for j < nB, no list
  // element mask source (LVSA): bit f of fbits[fq*TW + f/32] = frame f allowed for frame fq
  const uint32_t* fbits;
  int TW, P;
  // outputs
  __nv_bfloat16* o;
  float* lse;
  // mass pass
  float* mass;
  const float* lse_in;
  long long wait_limit_ns;
};

constexpr int kAttnThreads = 256;
constexpr float kRescaleLog2 = 8.0f;

template <int D, bool MASS>
struct AttnSmem {
  static constexpr uint32_t kBox = 128 * 64 * 2;          // one 128-row x 64-col bf16 box
  static constexpr uint32_t kTile = (D / 64) * kBox;       // 128 x D tile
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK = kQ + kTile;               // 2 stages
  static constexpr uint32_t kV = kK + 2 * kTile;           // 2 stages (fwd only)
  static constexpr uint32_t kP = MASS ? kV : kV + 2 * kTile;   // 2 boxes (fwd only)
  static constexpr uint32_t kBar = MASS ? kP : kP + 2 * kBox;
  static constexpr uint32_t kNumBars = 20;
  static constexpr uint32_t kHolder = kBar + kNumBars * 8;
  static constexpr uint32_t kRed = kHolder + 16;           // 2 x 4 floats (mass reduction)
  static constexpr uint32_t kBytes = kRed + 64;
  static constexpr uint32_t kAlloc = kBytes + 1024;         // + alignment slack
  static constexpr uint32_t kTmemCols = MASS ? 256 : 512;
};

// barrier slots
enum : int { B_QFULL = 0, B_KFULL = 1, B_KEMPTY = 3, B_VFULL = 5, B_VEMPTY = 7, B_SFULL = 9,
             B_SEMPTY = 11, B_PFULL = 13, B_PVDONE = 14, B_FINAL = 15, B_RFULL = 16, B_REMPTY = 18 };

__device__ __forceinline__ void set_bit_range(uint32_t (&mw)[4], int a, int b) {
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const int lo = max(a, 32 * w), hi = min(b, 32 * w + 32);
    if (lo < hi) {
      const int n = hi - lo;
      const uint32_t bits = (n == 32) ? 0xFFFFFFFFu : ((1u << n) - 1u);
      mw[w] |= bits << (lo - 32 * w);
    }
  }
}

// Element mask of one key tile for query frame fq: bit c set iff key k0+c < N
// and frame(k0+c) is allowed for fq (all frames allowed when fbits is null).
__device__ __forceinline__ void tile_mask(const AttnParams& p, int fq, int k0, uint32_t (&mw)[4]) {
  mw[0] = mw[1] = mw[2] = mw[3] = 0u;
  const int kend = min(k0 + 128, p.N);
  if (p.fbits == nullptr) {
    set_bit_range(mw, 0, kend - k0);
    return;
  }
  const uint32_t* row = p.fbits + static_cast<size_t>(fq) * p.TW;
  for (int f = k0 / p.P; f * p.P < kend; ++f) {
    if ((__ldg(row + (f >> 5)) >> (f & 31)) & 1u) {
      set_bit_range(mw, max(f * p.P, k0) - k0, min((f + 1) * p.P, kend) - k0);
    }
  }
}

template <int D, bool MASS>
__global__ void __launch_bounds__(kAttnThreads, 1)
attn_tile_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using L = AttnSmem<D, MASS>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t bar0 = base + L::kBar;
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
  volatile uint32_t* holder = reinterpret_cast<volatile uint32_t*>(gbase + L::kHolder);

  const int qt = blockIdx.x, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long limit = p.wait_limit_ns;

  // ---- this CTA's key-tile list
  int n;
  const int32_t* list = nullptr;
  const uint8_t* flags = nullptr;
  if (p.dense) {
    n = p.nB;
  } else {
    n = p.count[static_cast<size_t>(h) * p.chs + qt];
    if (n < 0 || n > p.lrs) {
      if (threadIdx.x == 0) set_status(BSA_ERR_INDEX_RANGE);
      n = n < 0 ? 0 : p.lrs;
    }
    const size_t off = static_cast<size_t>(h) * p.lhs + static_cast<size_t>(qt) * p.lrs;
    list = p.list + off;
    if (p.flags) flags = p.flags + off;
  }
  auto tile_of = [&](int j) -> int { return p.dense ? j : __ldg(list + j); };
  auto valid = [&](int kt) -> bool { return kt >= 0 && kt < p.nB; };

  // ---- setup: barriers (thread 0), TMEM (warp 1)
  if (threadIdx.x == 0) {
    mbar_init(bar(B_QFULL), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(B_KFULL + s), 1);
      mbar_init(bar(B_KEMPTY + s), 1);
      mbar_init(bar(B_VFULL + s), 1);
      mbar_init(bar(B_VEMPTY + s), 1);
      mbar_init(bar(B_SFULL + s), 1);
      mbar_init(bar(B_SEMPTY + s), 128);
    }
    mbar_init(bar(B_PFULL), 128);
    mbar_init(bar(B_PVDONE), 1);
    mbar_init(bar(B_FINAL), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(B_RFULL + s), 4);
      mbar_init(bar(B_REMPTY + s), 1);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(base + L::kHolder, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *holder;

  constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, false, false);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, false, true);

  if (warp == 0) {
    // ================================================= TMA producer ====
    if (lane == 0 && n > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      if (!MASS) tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(bar(B_QFULL), L::kTile);
#pragma unroll
      for (int b = 0; b < D / 64; ++b)
        tma_load_3d(base + L::kQ + b * L::kBox, &tmQ, bar(B_QFULL), b * 64, h, qt * 128);
      int it = 0;
      bool ok = true;
      for (int j = 0; j < n && ok; ++j) {
        const int kt = tile_of(j);
        if (!valid(kt)) continue;
        const int slot = it & 1;
        if (it >= 2) ok = mbar_wait(bar(B_KEMPTY + slot), ((it - 2) >> 1) & 1, limit);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(B_KFULL + slot), L::kTile);
#pragma unroll
        for (int b = 0; b < D / 64; ++b)
          tma_load_3d(base + L::kK + slot * L::kTile + b * L::kBox, &tmK, bar(B_KFULL + slot), b * 64, h,
                      kt * 128);
        if (!MASS) {
          if (it >= 2) ok = mbar_wait(bar(B_VEMPTY + slot), ((it - 2) >> 1) & 1, limit);
          if (!ok) break;
          mbar_arrive_expect_tx(bar(B_VFULL + slot), L::kTile);
#pragma unroll
          for (int b = 0; b < D / 64; ++b)
            tma_load_3d(base + L::kV + slot * L::kTile + b * L::kBox, &tmV, bar(B_VFULL + slot), b * 64, h,
                        kt * 128);
        }
        ++it;
      }
      // drain: wait (bounded) for this thread's own copies still in flight
      mbar_wait(bar(B_QFULL), 0, limit);
      for (int u = max(0, it - 2); u < it; ++u) {
        mbar_wait(bar(B_KFULL + (u & 1)), (u >> 1) & 1, limit);
        if (!MASS) mbar_wait(bar(B_VFULL + (u & 1)), (u >> 1) & 1, limit);
      }
    }
  } else if (warp == 1) {
    // ================================================= MMA issuer ======
    if (lane == 0 && n > 0) {
      const uint32_t tS0 = tbase, tS1 = tbase + 128, tO = tbase + 256;
      bool ok = true;
      bool have_q = false;
      int it = 0;
      auto issue_pv = [&](int u) -> bool {
        if (!mbar_wait(bar(B_PFULL), u & 1, limit)) return false;
        if (!mbar_wait(bar(B_VFULL + (u & 1)), (u >> 1) & 1, limit)) return false;
        tc_fence_after();
        const uint32_t vbase = base + L::kV + (u & 1) * L::kTile;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {        // 16 keys per step
          const uint64_t da = sw128_desc(base + L::kP + (kk >> 2) * L::kBox + (kk & 3) * 32, 16, 1024);
          const uint64_t db = sw128_desc(vbase + kk * 2048, L::kBox, 1024);
          mma_bf16_ss(tO, da, db, kIdescPV, (u > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(bar(B_PVDONE));
        tc_commit(bar(B_VEMPTY + (u & 1)));
        return true;
      };
      for (int j = 0; j < n && ok; ++j) {
        const int kt = tile_of(j);
        if (!valid(kt)) continue;
        if (!have_q) {
          ok = mbar_wait(bar(B_QFULL), 0, limit);
          have_q = true;
          if (!ok) break;
        }
        const int b = it & 1;
        if (it >= 2) ok = mbar_wait(bar(B_SEMPTY + b), ((it - 2) >> 1) & 1, limit);
        if (!ok) break;
        ok = mbar_wait(bar(B_KFULL + b), (it >> 1) & 1, limit);
        if (!ok) break;
        tc_fence_after();
        const uint32_t kbase = base + L::kK + b * L::kTile;
        const uint32_t dS = b ? tS1 : tS0;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {     // 16 channels per step
          const uint32_t off = (kk >> 2) * L::kBox + (kk & 3) * 32;
          const uint64_t da = sw128_desc(base + L::kQ + off, 16, 1024);
          const uint64_t db = sw128_desc(kbase + off, 16, 1024);
          mma_bf16_ss(dS, da, db, kIdescQK, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(B_SFULL + b));
        tc_commit(bar(B_KEMPTY + b));
        if (!MASS && it >= 1) ok = issue_pv(it - 1);
        ++it;
      }
      if (!MASS && ok && it >= 1) issue_pv(it - 1);
      // all issued MMAs complete before the CTA may release TMEM
      tc_commit(bar(B_FINAL));
      mbar_wait(bar(B_FINAL), 0, limit);
    }
  } else if (warp >= 4) {
    // ================================================= softmax WG ======
    const int r = threadIdx.x - 128;                 // row within tile = TMEM lane
    const int q = qt * 128 + r;
    const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const uint32_t tS0 = tbase + lane_off, tS1 = tbase + lane_off + 128;
    const uint32_t tO = tbase + lane_off + 256;
    const int fq = (p.fbits != nullptr) ? (min(q, p.N - 1) / p.P) : 0;
    const uint32_t pbase = base + L::kP + static_cast<uint32_t>(r) * 128;
    const uint32_t rsw = static_cast<uint32_t>(r & 7);

    float m_run = -INFINITY, l_run = 0.f;
    float lse2 = 0.f;
    if (MASS) {
      const float v = (q < p.N) ? p.lse_in[static_cast<size_t>(h) * p.N + q] : -INFINITY;
      lse2 = isfinite(v) ? v * 1.4426950408889634f : INFINITY;   // rows without mass contribute 0
    }
    float* red = reinterpret_cast<float*>(gbase + L::kRed);
    bool ok = true;
    int it = 0;
    for (int j = 0; j < n && ok; ++j) {
      const int kt = tile_of(j);
      if (!valid(kt)) {
        if (threadIdx.x == 128) set_status(BSA_ERR_INDEX_RANGE);
        continue;
      }
      const int b = it & 1;
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar(B_SFULL + b), (it >> 1) & 1, limit));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld_x128(b ? tS1 : tS0, sr);
      tc_fence_before();
      mbar_arrive(bar(B_SEMPTY + b));
      float* s = reinterpret_cast<float*>(sr);

      const bool partial = p.dense ? (kt * 128 + 128 > p.N)
                                   : (flags ? (flags[j] != 0) : (kt * 128 + 128 > p.N));
      if (partial) {
        uint32_t mw[4];
        tile_mask(p, fq, kt * 128, mw);
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (!((mw[c >> 5] >> (c & 31)) & 1u)) s[c] = -INFINITY;
      }

      if (MASS) {
        float acc = 0.f;
#pragma unroll
        for (int c = 0; c < 128; ++c) acc += ex2_approx(fmaf(s[c], p.sl2, -lse2));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
        // hand the warp partial to row 0's thread through a 2-slot ring
        // guarded by mbarriers (bounded waits; no CTA-wide barrier in the loop)
        const int sl = it & 1;
        bool okw = true;
        if (lane == 0) {
          if (it >= 2) okw = mbar_wait(bar(B_REMPTY + sl), ((it - 2) >> 1) & 1, limit);
          if (okw) {
            red[sl * 4 + (warp & 3)] = acc;
            mbar_arrive(bar(B_RFULL + sl));
          }
        }
        if (r == 0 && okw) {
          okw = mbar_wait(bar(B_RFULL + sl), (it >> 1) & 1, limit);
          if (okw) {
            const volatile float* rr = red + sl * 4;
            const float tot = (rr[0] + rr[1]) + (rr[2] + rr[3]);
            p.mass[(static_cast<size_t>(h) * p.nB + qt) * p.nB + kt] = tot;
            mbar_arrive(bar(B_REMPTY + sl));
          }
        }
        ok = __shfl_sync(0xFFFFFFFFu, okw ? 1 : 0, 0) != 0;
        if (!ok) break;
      } else {
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 128; ++c) mx = fmaxf(mx, s[c]);
        const float mx2 = mx * p.sl2;
        const bool need = mx2 > m_run + kRescaleLog2;
        const float m_new = need ? mx2 : m_run;
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        float rs = 0.f;
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          s[c] = ex2_approx(fmaf(s[c], p.sl2, -m_use));
          rs += s[c];
        }
        const float alpha = need ? ((m_run == -INFINITY) ? 0.f : ex2_approx(m_run - m_new)) : 1.f;
        l_run = l_run * alpha + rs;
        m_run = m_new;
        if (it > 0) {
          // PV(it-1) must finish before O is rescaled and P is overwritten
          ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar(B_PVDONE), (it - 1) & 1, limit));
          if (!ok) break;
          tc_fence_after();
          if (__any_sync(0xFFFFFFFFu, alpha != 1.f)) {
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
              uint32_t ov[32];
              tmem_ld_x32(tO + c0, ov);
#pragma unroll
              for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
              tmem_st_x32(tO + c0, ov);
            }
          }
        }
        // P (bf16) into the 128B-swizzled K-major operand tile: row r, 16B chunk c
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const uint32_t addr = pbase + (c >> 3) * L::kBox + (((c & 7) ^ rsw) << 4);
          st_shared_v4(addr, pack_bf16x2(s[8 * c + 0], s[8 * c + 1]), pack_bf16x2(s[8 * c + 2], s[8 * c + 3]),
                       pack_bf16x2(s[8 * c + 4], s[8 * c + 5]), pack_bf16x2(s[8 * c + 6], s[8 * c + 7]));
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar(B_PFULL));
      }
      ++it;
    }

    if (!MASS) {
      // ---- epilogue: O / l (bf16) and LSE
      if (ok && it > 0) {
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar(B_PVDONE), (it - 1) & 1, limit));
        tc_fence_after();
      }
      const bool have = __all_sync(0xFFFFFFFFu, ok && it > 0);
      const float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
      __nv_bfloat16* orow = p.o + (static_cast<size_t>(q) * p.H + h) * D;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t ov[32];
        __syncwarp();
        if (have) {
          tmem_ld_x32(tO + c0, ov);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) ov[c] = 0u;
        }
        if (q < p.N) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(ov[8 * v4 + 0]) * inv, __uint_as_float(ov[8 * v4 + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(ov[8 * v4 + 2]) * inv, __uint_as_float(ov[8 * v4 + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(ov[8 * v4 + 4]) * inv, __uint_as_float(ov[8 * v4 + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(ov[8 * v4 + 6]) * inv, __uint_as_float(ov[8 * v4 + 7]) * inv);
            dst[v4] = w;
          }
        }
      }
      if (q < p.N) {
        p.lse[static_cast<size_t>(h) * p.N + q] =
            (l_run > 0.f) ? (m_run + __log2f(l_run)) * 0.6931471805599453f : -INFINITY;
      }
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tbase, L::kTmemCols);
  }
}

}  // namespace bsa
