// attn_fwd.cuh - block-sparse / dense softmax attention forward on sm_100a
// tensor cores (tcgen05 + TMEM + TMA), with a mode that also records what
// the LoSA block mass needs.
//
// Sources: "LVSA: Training-Free Sparse Attention for Long Video Diffusion"
// (gist.science explainer), technical summary section 2 (block-sparse
// attention restricted to A(t); cost |A(t)| * P * d per query) and section 4
// (block-sparse kernel against dense attention); "LoSA (Near-Lossless Sparse
// Attention)" article, section "Balancing efficiency and quality" (one dense
// step measuring exact inter-block mass, then the frozen block index).
//
// One CTA = two neighbouring 128-row query tiles (0 = 2x, 1 = 2x+1) of one
// head.  Every 128-key tile either of them keeps (the merge of their two
// sorted lists) is loaded once by TMA and used by both, which halves the
// bytes each SM pulls from L2 per FLOP.
//
// Warp roles (384 threads):
//   warp 0       TMA producer: Q_0, Q_1 once, then K tiles (2-deep ring)
//   warp 1       TMEM allocator and tcgen05.mma issuer (the whole warp runs
//                the loop, an elected lane issues)
//   warp 2       TMA producer: V tiles (3-deep ring)
//   warp 3       idle
//   warps 4..7   softmax group 0: thread r owns row r of query tile 0
//   warps 8..11  softmax group 1: thread r owns row r of query tile 1
// setmaxnreg moves registers from warps 0..3 (72 each) to the softmax
// warps (216 each), which hold a row's 128 scores in registers.
// TMEM columns: S_0 [0,128), S_1 [128,256) (f32 scores), O_0 [256,256+d),
// O_1 [256+d, 256+2d) (f32 accumulators).  The softmax writes P (bf16, two
// per 32-bit column) over the first 64 columns of its S tile and the PV
// product reads it from there as the A operand (tcgen05.mma with A in
// TMEM), so P never touches shared memory.
//
// Tensor-core order per key tile i (ping-pong between the two groups):
//   S_0(i) = Q_0 K_i^T,  O_1 += P_1(i-1) V_{i-1},  S_1(i) = Q_1 K_i^T,
//   O_0 += P_0(i) V_i
// Each PV goes out in two halves of 64 keys: the softmax signals once after
// storing P of the first 64 keys and again after the rest, so the first
// half of the product runs while the softmax still computes the second half
// of the exponentials.
// While group 0 turns S_0(i) into P_0(i) the tensor core runs O_1 and S_1,
// and the other way round.  MMAs issued by one thread execute in order, so
// S_x(i+1) (issued after O_x's PV) cannot overwrite P_x(i) before it is read,
// and when a group sees S_x(i) complete, O_x is idle (its previous PV was
// issued before S_x(i) and the completion barrier covers every earlier MMA):
// the group rescales O_x in place when its running max grows by more than
// 2^8 (exact after the final division).  Each thread reads its row's 128
// scores from TMEM once, takes the row max, then forms the exponentials and
// packs P over the same registers.  Tiles flagged partial (frame boundary or
// sequence end) get an element mask from the frame bit matrix.
//
// Mass mode (MASS = true) is LoSA's measuring step in one pass, on the dense
// index or any other: the same forward, which also writes, per query row
// and visited key tile, the log2 of that tile's share of the row's
// probability mass before normalisation,
// lpart = log2(sum_k exp2(s_k * scale * log2e - m)) + m with the stabiliser m
// the row used for the tile (tiles the index never reaches are not
// written).  The block mass of a (query block, key block) pair is then the
// sum over the block's rows of exp2(lpart - lse * log2e), which a separate
// reduction forms once the final LSE is known.
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
  // mass mode: lpart[(hl * nB + kt) * N + q] for local head hl = blockIdx.y
  float* lpart;
  int h_off;                        // head of blockIdx.y == 0
  long long wait_limit_ns;
};

constexpr int kAttnThreads = 384;
constexpr int kQTilesPerCta = 2;
constexpr float kRescaleLog2 = 8.0f;
constexpr int kKStages = 2;                        // K ring depth (128-key tiles)
constexpr int kVStages = 3;                        // V ring depth (a V tile lives until O_1's PV)
// setmaxnreg budgets (0 = off): warps 0..3 (producers, issuer, idle) and
// the two softmax warpgroups; at most the launch's 168 x 384 registers.
// Without the split the softmax spills ~100 bytes per thread inside its
// tile loop; measured 44.2 -> 40.0 ms per headline call with it.
constexpr int kRegsLow = 72;
constexpr int kRegsHigh = 216;
static_assert(kRegsLow * 128 + kRegsHigh * 256 <= 168 * kAttnThreads, "register split");

template <int D, bool MASS>
struct AttnSmem {
  static constexpr uint32_t kBox = 128 * 128;               // 128 rows x 64 bf16 (128 B) per box
  static constexpr uint32_t kTile = (D / 64) * kBox;        // one 128 x D tile
  static constexpr uint32_t kQ = 0;                         // Q_0, Q_1
  static constexpr uint32_t kK = kQ + 2 * kTile;
  static constexpr uint32_t kV = kK + kKStages * kTile;
  static constexpr uint32_t kBar = kV + kVStages * kTile;
  static constexpr uint32_t kNumBars = 32;
  static constexpr uint32_t kHolder = kBar + kNumBars * 8;
  static constexpr uint32_t kBytes = kHolder + 16;
  static constexpr uint32_t kAlloc = kBytes + 1024;          // + alignment slack
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kTmemO = 256;                    // O_0 at 256, O_1 at 256 + D
};

// barrier slots
enum : int {
  B_QFULL = 0,
  B_KFULL = 1,                        // kKStages
  B_KEMPTY = B_KFULL + kKStages,      // kKStages
  B_VFULL = B_KEMPTY + kKStages,      // kVStages
  B_VEMPTY = B_VFULL + kVStages,      // kVStages
  B_SFULL = B_VEMPTY + kVStages,      // [group]
  B_PFULL = B_SFULL + 2,              // [group]
  B_PVDONE = B_PFULL + 2,             // [group]
  B_PLO = B_PVDONE + 2,               // [group] first 64 keys of P stored
  B_FINAL = B_PLO + 2,
  B_COUNT = B_FINAL + 1
};
static_assert(B_COUNT <= 32, "barrier slots");

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

// Element mask of one 128-key tile for query frame fq: bit c set iff key
// k0+c < N and frame(k0+c) is allowed for fq (all frames when fbits is null).
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

// Merge walk over the key-tile lists of the CTA's two query tiles.  Every
// role runs its own copy over the same lists, so all of them see the same
// sequence of (tile, in list 0, in list 1).  Entries outside [0, nB) are
// skipped.
struct PairLists {
  const int32_t* l[2];
  int n[2];
  int dense, nB, N;
  int i[2];
  int cur[2];      // entry at i[x] (loaded one step ahead), 0x7FFFFFFF past the end

  __device__ __forceinline__ int load(int x, int j) const {
    return (j < n[x]) ? (dense ? j : ld_pinned_s32(l[x] + j)) : 0x7FFFFFFF;
  }
  __device__ __forceinline__ void start() {
    cur[0] = load(0, 0);
    cur[1] = load(1, 0);
  }
  // advance list x; the next entry's load is issued now and used a call later
  __device__ __forceinline__ void advance(int x) {
    ++i[x];
    cur[x] = load(x, i[x]);
  }
  // next kept tile: returns false at the end
  __device__ __forceinline__ bool next(int& kt, bool (&in)[2], bool& bad) {
    while (true) {
      bool skipped = false;
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        if (cur[x] != 0x7FFFFFFF && (cur[x] < 0 || cur[x] >= nB)) {   // out-of-range entry: skip
          bad = true;
          advance(x);
          skipped = true;
        }
      }
      if (skipped) continue;
      if (cur[0] == 0x7FFFFFFF && cur[1] == 0x7FFFFFFF) return false;
      kt = min(cur[0], cur[1]);
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        in[x] = (cur[x] == kt);
        if (in[x]) advance(x);
      }
      return true;
    }
  }
};

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ float max128(const float* s) {
  float a[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) a[k] = fmaxf(s[2 * k], s[2 * k + 1]);
#pragma unroll
  for (int j = 16; j < 128; j += 16)
#pragma unroll
    for (int k = 0; k < 8; ++k) a[k] = fmax3(a[k], s[j + 2 * k], s[j + 2 * k + 1]);
  return fmax3(fmax3(a[0], a[1], a[2]), fmax3(a[3], a[4], a[5]), fmaxf(a[6], a[7]));
}

__device__ __forceinline__ void apply_mask128(float* s, const uint32_t (&mw)[4]) {
#pragma unroll
  for (int c = 0; c < 128; ++c)
    if (!((mw[c >> 5] >> (c & 31)) & 1u)) s[c] = -INFINITY;
}

// exp2(s * sl2 - m) for one 128-score row; P (bf16 pairs) packed in place
// into sr[0..63] (pair j overwrites sr[j] only after elements 2j, 2j+1 >= j
// are read).  Returns the row sum of the float32 values.
// Packed float pairs (Blackwell f32x2 FMA-pipe ops): one instruction does two
// fmaf / two float adds with the same per-lane rounding.  The softmax uses
// them for the score scaling and the row sums, halving its FMA-pipe
// instructions; the pipe is shared with the MMA-issuing thread's
// sub-partition, where FMA-dense code slows the issue of tensor-core work.
__device__ __forceinline__ uint64_t f2pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// P of keys 0..63 (sr[0..31]) goes to TMEM as soon as it is formed and is
// signalled on `plo_bar` (the PV of those keys can start), keys 64..127 after
// the loop; the caller waits for that store (tmem_wait_st) before signalling
// the whole P ready.
__device__ __forceinline__ float row_exp_pack(const float* s, uint32_t* sr, float sl2, float m_use, uint32_t tP,
                                              uint32_t plo_bar, int lane) {
  const uint64_t sl2p = f2pack(sl2, sl2), nm = f2pack(-m_use, -m_use);
  uint64_t acc01 = f2pack(0.f, 0.f), acc23 = f2pack(0.f, 0.f);
#pragma unroll
  for (int c = 0; c < 128; c += 4) {
    const uint64_t x01 = ffma2(f2pack(s[c], s[c + 1]), sl2p, nm);
    const uint64_t x23 = ffma2(f2pack(s[c + 2], s[c + 3]), sl2p, nm);
    float x0, x1, x2, x3;
    f2unpack(x01, x0, x1);
    f2unpack(x23, x2, x3);
    const uint64_t e01 = f2pack(ex2_approx(x0), ex2_approx(x1));
    const uint64_t e23 = f2pack(ex2_approx(x2), ex2_approx(x3));
    acc01 = fadd2(acc01, e01);
    acc23 = fadd2(acc23, e23);
    float e0, e1, e2, e3;
    f2unpack(e01, e0, e1);
    f2unpack(e23, e2, e3);
    sr[c / 2] = pack_bf16x2(e0, e1);
    sr[c / 2 + 1] = pack_bf16x2(e2, e3);
    if (c == 60) {
      tmem_st_x32_async(tP, sr);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(plo_bar);
    }
  }
  tmem_st_x32_async(tP + 32, sr + 32);
  float r0, r1, r2, r3;
  f2unpack(acc01, r0, r1);
  f2unpack(acc23, r2, r3);
  return (r0 + r1) + (r2 + r3);
}

template <int D, bool MASS>
__global__ void __launch_bounds__(kAttnThreads, 1)
attn_tile_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                 const AttnParams p) {
  using L = AttnSmem<D, MASS>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t bar0 = base + L::kBar;
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
  volatile uint32_t* holder = reinterpret_cast<volatile uint32_t*>(gbase + L::kHolder);

  const int qt0 = blockIdx.x * kQTilesPerCta, h = blockIdx.y + p.h_off;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long limit = p.wait_limit_ns;

  // ---- the two query tiles' key-tile lists
  PairLists pl;
  const uint8_t* flg[2] = {nullptr, nullptr};     // per-entry partial flags (softmax only)
  pl.dense = p.dense;
  pl.nB = p.nB;
  pl.N = p.N;
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    const int qt = qt0 + x;
    pl.l[x] = nullptr;
    pl.i[x] = 0;
    if (qt >= p.nB) {
      pl.n[x] = 0;
    } else if (p.dense) {
      pl.n[x] = p.nB;
    } else {
      int n = p.count[static_cast<size_t>(h) * p.chs + qt];
      if (n < 0 || n > p.lrs) {
        if (threadIdx.x == 0) set_status(BSA_ERR_INDEX_RANGE);
        n = n < 0 ? 0 : p.lrs;
      }
      pl.n[x] = n;
      const size_t off = static_cast<size_t>(h) * p.lhs + static_cast<size_t>(qt) * p.lrs;
      pl.l[x] = p.list + off;
      if (p.flags) flg[x] = p.flags + off;
    }
  }
  pl.start();
  const bool active1 = (qt0 + 1) < p.nB;
  const bool any_work = pl.n[0] > 0 || pl.n[1] > 0;

  // ---- setup: barriers (thread 0), TMEM (warp 1)
  if (threadIdx.x == 0) {
    mbar_init(bar(B_QFULL), 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(bar(B_KFULL + s), 1);
      mbar_init(bar(B_KEMPTY + s), 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(bar(B_VFULL + s), 1);
      mbar_init(bar(B_VEMPTY + s), 1);
    }
    for (int x = 0; x < 2; ++x) mbar_init(bar(B_SFULL + x), 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar(B_PFULL + x), 4);
      mbar_init(bar(B_PLO + x), 4);
      mbar_init(bar(B_PVDONE + x), 1);
    }
    mbar_init(bar(B_FINAL), 1);
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
    // ============================================ TMA producer: Q, K ====
    if constexpr (kRegsLow > 0) regs_dec<kRegsLow>();
    if (lane == 0 && any_work) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      const int nq = active1 ? 2 : 1;
      mbar_arrive_expect_tx(bar(B_QFULL), nq * L::kTile);
      for (int x = 0; x < nq; ++x)
#pragma unroll
        for (int b = 0; b < D / 64; ++b)
          tma_load_3d(base + L::kQ + x * L::kTile + b * L::kBox, &tmQ, bar(B_QFULL), b * 64, h, (qt0 + x) * 128);
      int it = 0, kt;
      bool in[2], bad = false, ok = true;
      while (ok && pl.next(kt, in, bad)) {
        const int slot = it % kKStages;
        if (it >= kKStages) ok = mbar_wait(bar(B_KEMPTY + slot), ((it - kKStages) / kKStages) & 1, limit);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(B_KFULL + slot), L::kTile);
#pragma unroll
        for (int b = 0; b < D / 64; ++b)
          tma_load_3d(base + L::kK + slot * L::kTile + b * L::kBox, &tmK, bar(B_KFULL + slot), b * 64, h, kt * 128);
        ++it;
      }
      // drain: wait (bounded) for this thread's own copies still in flight
      mbar_wait(bar(B_QFULL), 0, limit);
      for (int u = max(0, it - kKStages); u < it; ++u)
        mbar_wait(bar(B_KFULL + u % kKStages), (u / kKStages) & 1, limit);
    }
  } else if (warp == 2) {
    // ============================================== TMA producer: V ====
    if constexpr (kRegsLow > 0) regs_dec<kRegsLow>();
    if (lane == 0 && any_work) {
      tma_prefetch_desc(&tmV);
      int it = 0, kt;
      bool in[2], bad = false, ok = true;
      while (ok && pl.next(kt, in, bad)) {
        const int slot = it % kVStages;
        if (it >= kVStages) ok = mbar_wait(bar(B_VEMPTY + slot), ((it - kVStages) / kVStages) & 1, limit);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(B_VFULL + slot), L::kTile);
#pragma unroll
        for (int b = 0; b < D / 64; ++b)
          tma_load_3d(base + L::kV + slot * L::kTile + b * L::kBox, &tmV, bar(B_VFULL + slot), b * 64, h, kt * 128);
        ++it;
      }
      for (int u = max(0, it - kVStages); u < it; ++u)
        mbar_wait(bar(B_VFULL + u % kVStages), (u / kVStages) & 1, limit);
    }
  } else if (warp == 1) {
    // ================================================= MMA issuer ======
    if constexpr (kRegsLow > 0) regs_dec<kRegsLow>();
    // The whole warp walks the lists and waits; one elected lane issues
    // (see mma4_ss_warp for why the issue is not done from a lane-0 branch).
    if (any_work) {
      bool ok = true, bad = false;
      const uint64_t dQ[2] = {desc64(sw128_desc(base + L::kQ, 16, 1024)),
                              desc64(sw128_desc(base + L::kQ + L::kTile, 16, 1024))};
      int cnt[2] = {0, 0};          // per query tile: key tiles processed
      int it = 0, kt;
      bool in[2];

      // S = Q_x K^T into TMEM column block `sb`, completion on SFULL + sb
      // (and, when given, on a second barrier)
      auto qk = [&](int x, int sb, int ks, int bar2) {
        const uint64_t dk = desc64(sw128_desc(base + L::kK + ks * L::kTile, 16, 1024));
        const uint32_t dS = tbase + sb * 128;
#pragma unroll
        for (int g = 0; g < D / 64; ++g)          // 64 channels (one 128-byte box) per group of 4
          mma4_ss_warp(dS, dQ[x] + g * (L::kBox >> 4), dk + g * (L::kBox >> 4), kIdescQK, g > 0 ? 1u : 0u);
        if (bar2 >= 0) tc_commit2_warp(bar(B_SFULL + sb), bar(bar2));
        else tc_commit_warp(bar(B_SFULL + sb));
      };
      // wait until V of key tile `vit` and P_x of the first 64 keys of the
      // group's c-th tile are in place
      auto pv_ready = [&](int x, int vit, int c) -> bool {
        if (!mbar_wait_warp(bar(B_VFULL + vit % kVStages), (vit / kVStages) & 1, limit)) return false;
        if (!mbar_wait_warp(bar(B_PLO + x), c & 1, limit)) return false;
        tc_fence_after();
        return true;
      };
      // O_x += P_x V (P_x from TMEM, V from shared memory, MN-major): the first
      // 64 keys at once, the other 64 once the softmax has stored them (an
      // expired wait skips them; the status word already says so); completion
      // on PVDONE + x (and, when given, on a second barrier)
      auto pv = [&](int x, int vit, int c, int bar2) {
        const uint64_t dv = desc64(sw128_desc(base + L::kV + (vit % kVStages) * L::kTile, L::kBox, 1024));
        const uint32_t tO = tbase + L::kTmemO + x * D;
        const uint32_t tP = tbase + x * 128;
        mma4_ts_warp(tO, tP, dv, kIdescPV, c > 0 ? 1u : 0u);     // keys 0..63
        const bool full = mbar_wait_warp(bar(B_PFULL + x), c & 1, limit);
        tc_fence_after();
        if (full) mma4_ts_warp(tO, tP + 32, dv + 512, kIdescPV, 1u);       // keys 64..127
        if (bar2 >= 0) tc_commit2_warp(bar(B_PVDONE + x), bar(bar2));
        else tc_commit_warp(bar(B_PVDONE + x));
      };

      if (!mbar_wait_warp(bar(B_QFULL), 0, limit)) ok = false;
      tc_fence_after();
      {
        // Issue order per key tile i: O_1 += P_1(i-1) V, S_1(i), [next tile
        // lookup and K wait], O_0 += P_0(i) V, S_0(i+1).  PV_0(i) and
        // S_0(i+1) go out back to back: any memory-pipe instruction issued
        // after queued MMAs (a list load, an mbarrier probe) waits for the
        // tensor core to take them, so the bookkeeping is done while the
        // queue still holds PV_1 and S_1.  In-order execution keeps S_x(i+1)
        // behind PV_x(i), which reads P_x(i) from the same TMEM columns.
        int pend_it = -1, pend_c = 0;       // O_1's PV of an earlier tile, not yet issued
        bool have = ok && pl.next(kt, in, bad);
        if (have) {
          ok = mbar_wait_warp(bar(B_KFULL), 0, limit);
          tc_fence_after();
          if (ok && in[0]) qk(0, 0, 0, -1);
        }
        while (ok && have) {
          const int ks = it % kKStages;
          if (pend_it >= 0) {
            ok = pv_ready(1, pend_it, pend_c);
            if (!ok) break;
            pv(1, pend_it, pend_c, B_VEMPTY + pend_it % kVStages);
            pend_it = -1;
          }
          if (in[1]) qk(1, 1, ks, B_KEMPTY + ks);
          else tc_commit_warp(bar(B_KEMPTY + ks));
          int nkt = 0;
          bool nin[2] = {false, false};
          const bool nhave = pl.next(nkt, nin, bad);
          if (nhave) {
            ok = mbar_wait_warp(bar(B_KFULL + (it + 1) % kKStages), ((it + 1) / kKStages) & 1, limit);
            if (!ok) break;
            tc_fence_after();
          }
          if (in[0]) {
            ok = pv_ready(0, it, cnt[0]);
            if (!ok) break;
            pv(0, it, cnt[0], in[1] ? -1 : B_VEMPTY + it % kVStages);
          }
          if (nhave && nin[0]) qk(0, 0, (it + 1) % kKStages, -1);
          if (in[1]) {
            pend_it = it;
            pend_c = cnt[1];
          }
          if (in[0]) ++cnt[0];
          if (in[1]) ++cnt[1];
          ++it;
          kt = nkt;
          in[0] = nin[0];
          in[1] = nin[1];
          have = nhave;
        }
        if (ok && pend_it >= 0 && pv_ready(1, pend_it, pend_c)) pv(1, pend_it, pend_c, B_VEMPTY + pend_it % kVStages);
      }
      if (bad && lane == 0) set_status(BSA_ERR_INDEX_RANGE);
      // all issued MMAs complete before the CTA may release TMEM
      tc_commit_warp(bar(B_FINAL));
      mbar_wait_warp(bar(B_FINAL), 0, limit);
    }
  } else if (warp == 3) {
    if constexpr (kRegsLow > 0) regs_dec<kRegsLow>();   // idle: its registers go to the softmax warps
  } else if (warp >= 4) {
    // ================================================= softmax groups ==
    if constexpr (kRegsLow > 0) regs_inc<kRegsHigh>();
    const int x = (threadIdx.x - 128) >> 7;           // query tile 0 or 1 of this CTA
    const int r = (threadIdx.x - 128) & 127;          // row within the tile = TMEM lane
    const int qt = qt0 + x;
    const int q = qt * 128 + r;
    const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const uint32_t tS = tbase + lane_off + x * 128;   // S_x; P_x over its first 64 columns
    const uint32_t tO = tbase + lane_off + L::kTmemO + x * D;
    const int fq = (p.fbits != nullptr) ? (min(q, p.N - 1) / p.P) : 0;

    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    int cnt = 0;

    // this group's tiles are its own list's in-range entries, in list order
    // (the merge walk of the producers visits exactly those, in that order)
    const int nx = x ? pl.n[1] : pl.n[0];
    const int32_t* lx = x ? pl.l[1] : pl.l[0];
    const uint8_t* fx = x ? flg[1] : flg[0];
    bool bad = false;
    const bool listed = !p.dense, flagged = !p.dense && fx != nullptr;
    // entry j + 1 (tile and flag) is loaded while tile j is processed
    int kt_next = (nx > 0) ? (listed ? ld_pinned_s32(lx) : 0) : 0;
    uint32_t f_next = (nx > 0 && flagged) ? ld_pinned_u8(fx) : 0u;
    for (int j = 0; ok && j < nx; ++j) {
      const int kt = kt_next;
      const uint32_t fl = f_next;
      if (j + 1 < nx) {
        kt_next = listed ? ld_pinned_s32(lx + j + 1) : (j + 1);
        if (flagged) f_next = ld_pinned_u8(fx + j + 1);
      }
      if (kt < 0 || kt >= p.nB) {
        bad = true;
        continue;
      }
      const bool part = flagged ? (fl != 0u) : (kt * 128 + 128 > p.N);
      uint32_t mw[4] = {0u, 0u, 0u, 0u};
      if (part) tile_mask(p, fq, kt * 128, mw);
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar(B_SFULL + x), cnt & 1, limit));
      if (!ok) break;
      tc_fence_after();
      {
        // one read of the 128 scores, then row max, exponentials, P in place
        uint32_t sr[128];
        tmem_ld_x128(tS, sr);
        float* s = reinterpret_cast<float*>(sr);
        if (part) apply_mask128(s, mw);
        const float mx = max128(s);
        const float mx2 = mx * p.sl2;
        const bool need = mx2 > m_run + kRescaleLog2;
        const float m_new = need ? mx2 : m_run;
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        float alpha = 1.f;
        if (__any_sync(0xFFFFFFFFu, need)) {
          alpha = need ? ((m_run == -INFINITY) ? 0.f : ex2_approx(m_run - m_new)) : 1.f;
          // O_x is idle here (its last PV completed before S_x(i)): rescale in place
          if (cnt > 0) {
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
        // p = exp2(s * scale * log2e - m), P packed in place
        const float rsum = row_exp_pack(s, sr, p.sl2, m_use, tS, bar(B_PLO + x), lane);
        tmem_wait_st();
        if constexpr (MASS) {
          // this tile's share of the row's mass, log2, before normalisation
          if (q < p.N)
            p.lpart[(static_cast<size_t>(blockIdx.y) * p.nB + kt) * p.N + q] =
                (rsum > 0.f) ? (log2f(rsum) + m_use) : -INFINITY;
        }
        l_run = l_run * alpha + rsum;
        m_run = m_new;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_PFULL + x));
      }
      ++cnt;
    }
    if (bad && r == 0) set_status(BSA_ERR_INDEX_RANGE);

    {
      // ---- epilogue: O / l (bf16) and LSE for this group's query tile.  The
      // group's Q tile in shared memory is idle now (its last QK^T completed
      // before its last PV, which PVDONE covers; with no tile at all, once its
      // load has landed): each thread writes its
      // row of O there in the 128-byte-swizzled layout of the TMA box (16-byte
      // chunk c of row r at chunk position c ^ (r & 7), so the eight rows of
      // every quarter warp hit distinct banks), and one thread stores the
      // whole tile with TMA (rows past N are clipped by the tensor map):
      // global writes are whole 128-byte rows instead of 16 bytes in each of
      // 32 rows per warp store.
      if (ok && cnt > 0) {
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar(B_PVDONE + x), (cnt - 1) & 1, limit));
        tc_fence_after();
      }
      const bool have = __all_sync(0xFFFFFFFFu, ok && cnt > 0);
      // a group that processed no tile (empty list) may get here before the
      // TMA load of its Q tile has landed: wait for it before reusing the buffer
      if (cnt == 0 && any_work) __all_sync(0xFFFFFFFFu, mbar_wait(bar(B_QFULL), 0, limit));
      const float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
      const uint32_t sO = base + L::kQ + x * L::kTile;
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
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          const int col = c0 + 8 * v4;                  // first of 8 channels in this 16-byte chunk
          const uint32_t dst = sO + (col / 64) * L::kBox + r * 128 + ((((col % 64) / 8) ^ (r & 7)) * 16);
          st_shared_v4(dst,
                       pack_bf16x2(__uint_as_float(ov[8 * v4 + 0]) * inv, __uint_as_float(ov[8 * v4 + 1]) * inv),
                       pack_bf16x2(__uint_as_float(ov[8 * v4 + 2]) * inv, __uint_as_float(ov[8 * v4 + 3]) * inv),
                       pack_bf16x2(__uint_as_float(ov[8 * v4 + 4]) * inv, __uint_as_float(ov[8 * v4 + 5]) * inv),
                       pack_bf16x2(__uint_as_float(ov[8 * v4 + 6]) * inv, __uint_as_float(ov[8 * v4 + 7]) * inv));
        }
      }
      fence_proxy_async_smem();
      named_barrier_sync(1 + x, 128);                   // the group's 128 rows are in shared memory
      if (r == 0 && qt < p.nB) {
#pragma unroll
        for (int b = 0; b < D / 64; ++b) tma_store_3d(&tmO, sO + b * L::kBox, b * 64, h, qt * 128);
        bulk_commit();
        bulk_wait_read_all();                           // shared memory read before the CTA may exit
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
