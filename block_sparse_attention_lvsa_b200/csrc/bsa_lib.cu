// bsa_lib.cu - C ABI of libbsa.so (declared in include/bsa.h).
//
// Host side of every call: argument validation (before anything is
// enqueued), TMA tensor-map encoding, workspace carving and kernel launches
// on the caller's stream.  The library allocates no memory and never
// synchronises except in bsa_get_device_status.  Everything is one
// translation unit so the per-device status word is a single symbol.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <mutex>

#include "ptx.cuh"
#include "lvsa_index.cuh"
#include "losa_select.cuh"
#include "attn_fwd.cuh"
#include "blockmass.cuh"

namespace {

using namespace bsa;

constexpr long long kWaitLimitNs = 1500000000LL;   // 1.5 s per device-side wait
constexpr int kMaxDevices = 64;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D view (d, H, N) of a bf16 [N, H, d] tensor; box (64, 1, rows), 128B swizzle.
bool make_qkv_map(CUtensorMap* m, const void* ptr, int N, int H, int d, int rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(N)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(H) * d * 2};
  cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(rows)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
int n_tiles(int N) { return (N + 127) / 128; }

int check_qkv(const void* q, const void* k, const void* v, int N, int H, int d, const void* o, const float* lse) {
  if (!q || !k || !v || !o || !lse) return BSA_ERR_ARG;
  if (N < 1 || H < 1 || H > 65535) return BSA_ERR_ARG;
  if (d != 64 && d != 128) return BSA_ERR_UNSUPPORTED;
  if (static_cast<long long>(N) * H * d >= (1LL << 31)) return BSA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
    return BSA_ERR_ARG;
  return BSA_OK;
}

// grid over query-tile pairs x `grid_heads` heads, from head prm.h_off
template <int D, bool MASS>
int launch_attn(const void* q, const void* k, const void* v, int N, int H, int grid_heads, const AttnParams& prm,
                cudaStream_t st) {
  using L = AttnSmem<D, MASS>;
  // set once per device; concurrent first calls may both set it (idempotent)
  static std::atomic<bool> attr_set[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BSA_ERR_CUDA;
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(attn_tile_kernel<D, MASS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(L::kAlloc)) != cudaSuccess)
      return BSA_ERR_CUDA;
    attr_set[dev].store(true, std::memory_order_release);
  }
  CUtensorMap mq, mk, mv, mo;
  // query, key, value and output tiles are all 128 rows (boxes of 128 rows x 64 channels)
  if (!make_qkv_map(&mq, q, N, H, D, 128) || !make_qkv_map(&mk, k, N, H, D, 128) ||
      !make_qkv_map(&mv, v, N, H, D, 128) || !make_qkv_map(&mo, prm.o, N, H, D, 128))
    return BSA_ERR_CUDA;
  dim3 grid((prm.nB + kQTilesPerCta - 1) / kQTilesPerCta, grid_heads);
  attn_tile_kernel<D, MASS><<<grid, kAttnThreads, L::kAlloc, st>>>(mq, mk, mv, mo, prm);
  return cudaGetLastError() == cudaSuccess ? BSA_OK : BSA_ERR_CUDA;
}

int launch_attn_any(int d, bool mass, const void* q, const void* k, const void* v, int N, int H, int grid_heads,
                    const AttnParams& prm, cudaStream_t st) {
  if (d == 128) return mass ? launch_attn<128, true>(q, k, v, N, H, grid_heads, prm, st)
                            : launch_attn<128, false>(q, k, v, N, H, grid_heads, prm, st);
  return mass ? launch_attn<64, true>(q, k, v, N, H, grid_heads, prm, st)
              : launch_attn<64, false>(q, k, v, N, H, grid_heads, prm, st);
}

AttnParams base_params(int N, int H, float scale, void* o, float* lse) {
  AttnParams p;
  std::memset(&p, 0, sizeof(p));
  p.N = N;
  p.H = H;
  p.nB = n_tiles(N);
  p.sl2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.wait_limit_ns = kWaitLimitNs;
  return p;
}

// Workspace of the one-pass dense measuring step, per head: log2 partial
// sums [nB key tiles][N rows] float32.
size_t dense_mass_head_bytes(int N) { return static_cast<size_t>(n_tiles(N)) * static_cast<size_t>(N) * 4; }

// Forward in mass mode over head passes of `hc` heads, each followed by the
// block-mass reduction.  With `unvisited`, the log partial sums are first
// set to NaN (all bytes 0xFF): entries of tiles the index never reaches keep
// it and the reduction counts them as no mass.
int blockmass_passes(const void* q, const void* k, const void* v, int N, int H, int d, AttnParams p, float* lpart,
                     int hc, bool unvisited, const float* lse, float* mass, cudaStream_t st) {
  const int nB = n_tiles(N);
  const size_t per_head = dense_mass_head_bytes(N);
  for (int h0 = 0; h0 < H; h0 += hc) {
    const int hn = std::min(hc, H - h0);
    if (unvisited && cudaMemsetAsync(lpart, 0xFF, per_head * hn, st) != cudaSuccess) return BSA_ERR_CUDA;
    p.lpart = lpart;
    p.h_off = h0;
    int rc = launch_attn_any(d, true, q, k, v, N, H, hn, p, st);
    if (rc != BSA_OK) return rc;
    const dim3 grid((nB + kMassWarps - 1) / kMassWarps, (nB + kMassKt - 1) / kMassKt, hn);
    blockmass_reduce_kernel<<<grid, kMassThreads, 0, st>>>(lpart, lse, mass, N, nB, h0);
    if (cudaGetLastError() != cudaSuccess) return BSA_ERR_CUDA;
  }
  return BSA_OK;
}

// Workspace layout for LVSA frame indexes.
struct LvsaWs {
  size_t fbits, cnt, idx, flag, total;
};
LvsaWs lvsa_ws_layout(int N, int T) {
  const size_t nB = static_cast<size_t>(n_tiles(N));
  const size_t TW = static_cast<size_t>((T + 31) / 32);
  LvsaWs w;
  w.fbits = 0;
  w.cnt = round_up(w.fbits + static_cast<size_t>(T) * TW * 4, 256);
  w.idx = round_up(w.cnt + nB * 4, 256);
  w.flag = round_up(w.idx + nB * nB * 4, 256);
  w.total = round_up(w.flag + nB * nB, 256);
  return w;
}

// Workspace bytes an index needs (LVSA tile lists; for the intersection also
// its per-entry flags [H][nB][nB]); (size_t)-1 for an invalid index.
size_t index_ws_bytes(const bsa_index* index, int N, int H) {
  if (!index) return static_cast<size_t>(-1);
  if (index->kind == BSA_INDEX_BLOCKS) return 0;
  if (index->kind != BSA_INDEX_LVSA_FRAMES && index->kind != BSA_INDEX_LVSA_BLOCKS) return static_cast<size_t>(-1);
  if (index->T < 1 || index->T > kMaxFrames || N % index->T) return static_cast<size_t>(-1);
  const size_t nB = static_cast<size_t>(n_tiles(N));
  size_t t = lvsa_ws_layout(N, index->T).total;
  if (index->kind == BSA_INDEX_LVSA_BLOCKS) t += round_up(static_cast<size_t>(H) * nB * nB, 256);
  return t;
}

// Validates `index`, enqueues its expansion (LVSA frame sets -> tile lists,
// flags of the intersection) and fills the list fields of `p`; *used = the
// workspace bytes taken from its start.
int setup_index(const bsa_index* index, int N, int H, void* workspace, size_t ws_bytes, AttnParams& p,
                size_t* used, cudaStream_t st) {
  const int nB = p.nB;
  *used = 0;
  const bool lvsa = index->kind == BSA_INDEX_LVSA_FRAMES || index->kind == BSA_INDEX_LVSA_BLOCKS;
  const bool blocks = index->kind == BSA_INDEX_BLOCKS || index->kind == BSA_INDEX_LVSA_BLOCKS;
  if (!lvsa && !blocks) return BSA_ERR_ARG;
  if (blocks) {
    if (index->block != 128) return BSA_ERR_UNSUPPORTED;
    if (index->H != H || index->nQB != nB || index->nKB != nB) return BSA_ERR_SHAPE;
    if (!index->idx || !index->cnt) return BSA_ERR_ARG;
    p.list = index->idx;
    p.count = index->cnt;
    p.flags = nullptr;
    p.lhs = static_cast<long long>(index->nQB) * index->nKB;
    p.lrs = index->nKB;
    p.chs = index->nQB;
  }
  if (lvsa) {
    const int T = index->T;
    if (T < 1 || T > kMaxFrames) return BSA_ERR_ARG;
    if (N % T) return BSA_ERR_SHAPE;
    if (!index->frames || !index->counts) return BSA_ERR_ARG;
    const LvsaWs w = lvsa_ws_layout(N, T);
    const size_t need = index_ws_bytes(index, N, H);
    if (!workspace || ws_bytes < need || !aligned(workspace, 256)) return BSA_ERR_WORKSPACE;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint32_t* fbits = reinterpret_cast<uint32_t*>(ws + w.fbits);
    int32_t* tcnt = reinterpret_cast<int32_t*>(ws + w.cnt);
    int32_t* tidx = reinterpret_cast<int32_t*>(ws + w.idx);
    uint8_t* tflag = ws + w.flag;
    lvsa_frame_bits_kernel<<<(T + 127) / 128, 128, 0, st>>>(T, index->frames, index->counts, fbits);
    lvsa_tiles_kernel<<<(nB + 3) / 4, 128, 0, st>>>(N, T, N / T, nB, fbits, tcnt, tidx, tflag);
    p.fbits = fbits;
    p.TW = (T + 31) / 32;
    p.P = N / T;
    if (blocks) {
      uint8_t* cflag = ws + w.total;
      compose_flags_kernel<<<static_cast<unsigned>(H) * nB, 256, 0, st>>>(nB, index->idx, index->cnt, tcnt, tidx,
                                                                        tflag, cflag);
      p.flags = cflag;
    } else {
      p.list = tidx;
      p.count = tcnt;
      p.flags = tflag;
      p.lhs = 0;
      p.lrs = nB;
      p.chs = 0;
    }
    if (cudaGetLastError() != cudaSuccess) return BSA_ERR_CUDA;
    *used = need;
  }
  return BSA_OK;
}

}  // namespace

extern "C" {

const char* bsa_version(void) { return "bsa-b200 0.1 (sm_100a)"; }

const char* bsa_status_string(int s) {
  switch (s) {
    case BSA_OK: return "BSA_OK";
    case BSA_WARN_OVER_BUDGET: return "BSA_WARN_OVER_BUDGET";
    case BSA_ERR_ARG: return "BSA_ERR_ARG";
    case BSA_ERR_SHAPE: return "BSA_ERR_SHAPE";
    case BSA_ERR_CUDA: return "BSA_ERR_CUDA";
    case BSA_ERR_INDEX_RANGE: return "BSA_ERR_INDEX_RANGE";
    case BSA_ERR_TIMEOUT: return "BSA_ERR_TIMEOUT";
    case BSA_ERR_UNSUPPORTED: return "BSA_ERR_UNSUPPORTED";
    case BSA_ERR_WORKSPACE: return "BSA_ERR_WORKSPACE";
    default: return "BSA_UNKNOWN_STATUS";
  }
}

int lvsa_build_index(int T, int T_per, int W, int C, int step, int32_t* frames, int32_t* counts, void* stream) {
  if (T < 1 || T > kMaxFrames || T_per < 1 || W < 1 || C < 1 || step < 0) return BSA_ERR_ARG;
  if (!frames || !counts || !aligned(frames, 4) || !aligned(counts, 4)) return BSA_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int threads = 128;
  lvsa_build_index_kernel<<<(T + threads - 1) / threads, threads, 0, st>>>(T, T_per, C, step, frames, counts);
  if (cudaGetLastError() != cudaSuccess) return BSA_ERR_CUDA;
  // over budget iff some t has |G_s u {t}| > C (pure function of the scalars)
  const int s_mod = step % T_per;
  const int nG = (s_mod < T) ? (T - 1 - s_mod) / T_per + 1 : 0;
  const bool has_non_anchor = nG < T;
  const bool over = (nG > C) || (has_non_anchor && nG + 1 > C);
  return over ? BSA_WARN_OVER_BUDGET : BSA_OK;
}

int lvsa_build_index_window(int T, int T_per, int W, int step, int32_t* frames, int32_t* counts, void* stream) {
  if (T < 1 || T > kMaxFrames || T_per < 1 || W < 1 || step < 0) return BSA_ERR_ARG;
  // |G_s| = number of f in [0, T) with f = step mod T_per (mod T_per)
  const int s_mod = step % T_per;
  const int nG = (s_mod < T) ? (T - 1 - s_mod) / T_per + 1 : 0;
  const int C = static_cast<int>(std::min<long long>(T, static_cast<long long>(nG) + W));
  // |G_s u {t}| <= min(T, nG + 1) <= C, so the fill never reports over budget
  return lvsa_build_index(T, T_per, W, C, step, frames, counts, stream);
}

size_t bsa_workspace_bytes(int op, int N, int H, int d, const bsa_index* index) {
  if (N < 1 || H < 1 || (d != 64 && d != 128)) return static_cast<size_t>(-1);
  const size_t per_head = dense_mass_head_bytes(N);
  // head shares of log partial sums: every head in one pass, up to 4 GiB
  const size_t heads = std::max<size_t>(1, std::min<size_t>(static_cast<size_t>(H), (size_t(4) << 30) / per_head));
  if (op == BSA_OP_DENSE_BLOCKMASS) return per_head * heads;
  if (op != BSA_OP_BLOCKSPARSE_FWD && op != BSA_OP_BLOCKMASS) return static_cast<size_t>(-1);
  const size_t ix = index_ws_bytes(index, N, H);
  if (ix == static_cast<size_t>(-1)) return ix;
  return op == BSA_OP_BLOCKSPARSE_FWD ? ix : round_up(ix, 256) + per_head * heads;
}

int blocksparse_attn_fwd(const void* q, const void* k, const void* v, int N, int H, int d, float scale,
                         const bsa_index* index, void* o, float* lse, void* workspace, size_t ws_bytes,
                         void* stream) {
  int rc = check_qkv(q, k, v, N, H, d, o, lse);
  if (rc != BSA_OK) return rc;
  if (!index || !std::isfinite(scale)) return BSA_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  AttnParams p = base_params(N, H, scale, o, lse);
  size_t used = 0;
  rc = setup_index(index, N, H, workspace, ws_bytes, p, &used, st);
  if (rc != BSA_OK) return rc;
  return launch_attn_any(d, false, q, k, v, N, H, H, p, st);
}

int attn_blockmass(const void* q, const void* k, const void* v, int N, int H, int d, float scale,
                   const bsa_index* index, void* o, float* lse, float* mass, void* workspace, size_t ws_bytes,
                   void* stream) {
  int rc = check_qkv(q, k, v, N, H, d, o, lse);
  if (rc != BSA_OK) return rc;
  if (!index || !mass || !aligned(mass, 4) || !std::isfinite(scale)) return BSA_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  AttnParams p = base_params(N, H, scale, o, lse);
  size_t used = 0;
  rc = setup_index(index, N, H, workspace, ws_bytes, p, &used, st);
  if (rc != BSA_OK) return rc;
  const size_t off = round_up(used, 256);
  const size_t per_head = dense_mass_head_bytes(N);
  if (!workspace || ws_bytes < off || ws_bytes - off < per_head) return BSA_ERR_WORKSPACE;
  float* lpart = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + off);
  const int hc = static_cast<int>(std::min<size_t>(static_cast<size_t>(H), (ws_bytes - off) / per_head));
  return blockmass_passes(q, k, v, N, H, d, p, lpart, hc, /*unvisited=*/true, lse, mass, st);
}

int attn_dense_blockmass(const void* q, const void* k, const void* v, int N, int H, int d, int block, float scale,
                         void* o, float* lse, float* mass, void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_qkv(q, k, v, N, H, d, o, lse);
  if (rc != BSA_OK) return rc;
  if (!mass || !aligned(mass, 4) || !std::isfinite(scale)) return BSA_ERR_ARG;
  if (block != 128) return BSA_ERR_UNSUPPORTED;
  const size_t per_head = dense_mass_head_bytes(N);
  if (!workspace || !aligned(workspace, 256) || ws_bytes < per_head) return BSA_ERR_WORKSPACE;
  AttnParams p = base_params(N, H, scale, o, lse);
  p.dense = 1;
  const int hc = static_cast<int>(std::min<size_t>(static_cast<size_t>(H), ws_bytes / per_head));
  // every (row, key tile) is visited: no need to mark the workspace first
  return blockmass_passes(q, k, v, N, H, d, p, static_cast<float*>(workspace), hc, false, lse, mass,
                          static_cast<cudaStream_t>(stream));
}

int losa_select(const float* mass, int H, int nQB, int nKB, double tau, int32_t* idx, int32_t* cnt, void* stream) {
  if (!mass || !idx || !cnt || !aligned(mass, 4) || !aligned(idx, 4) || !aligned(cnt, 4)) return BSA_ERR_ARG;
  if (H < 1 || nQB < 1 || nKB < 1) return BSA_ERR_ARG;
  if (nKB > kSelectMaxBlocks) return BSA_ERR_UNSUPPORTED;
  if (!(tau > 0.0 && tau <= 1.0)) return BSA_ERR_ARG;
  const long long rows = static_cast<long long>(H) * nQB;
  if (rows > 0x7FFFFFFFLL) return BSA_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // rows of up to 2048 blocks: keys in registers, 8 warps (one row each) per CTA
  if (nKB <= 2048) {
    const int wpc = 8;
    const long long ctas = std::min<long long>((rows + wpc - 1) / wpc, 1LL << 20);
    const dim3 grid(static_cast<unsigned>(ctas)), block(wpc * 32);
    const int r = static_cast<int>(rows);
    if (nKB <= 256)
      losa_select_reg_kernel<8><<<grid, block, 0, st>>>(mass, r, nKB, tau, idx, cnt);
    else if (nKB <= 512)
      losa_select_reg_kernel<16><<<grid, block, 0, st>>>(mass, r, nKB, tau, idx, cnt);
    else if (nKB <= 1024)
      losa_select_reg_kernel<32><<<grid, block, 0, st>>>(mass, r, nKB, tau, idx, cnt);
    else
      losa_select_reg_kernel<64><<<grid, block, 0, st>>>(mass, r, nKB, tau, idx, cnt);
    return cudaGetLastError() == cudaSuccess ? BSA_OK : BSA_ERR_CUDA;
  }
  // longer rows: keys in shared memory, warps per CTA sized to <= 96 KB
  const size_t row_bytes = static_cast<size_t>(nKB) * 8;
  const int wpc = static_cast<int>(std::min<size_t>(8, std::max<size_t>(1, (96 * 1024) / row_bytes)));
  const size_t smem = row_bytes * wpc;
  static std::atomic<bool> attr_set[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BSA_ERR_CUDA;
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    // largest request: 96 KB (several warps) or one row of kSelectMaxBlocks keys (64 KB)
    if (cudaFuncSetAttribute(losa_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 96 * 1024) !=
        cudaSuccess)
      return BSA_ERR_CUDA;
    attr_set[dev].store(true, std::memory_order_release);
  }
  const long long ctas = std::min<long long>((rows + wpc - 1) / wpc, 1LL << 20);
  losa_select_kernel<<<static_cast<unsigned>(ctas), wpc * 32, smem, st>>>(mass, static_cast<int>(rows), nKB, tau,
                                                                         idx, cnt);
  return cudaGetLastError() == cudaSuccess ? BSA_OK : BSA_ERR_CUDA;
}

int bsa_get_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return BSA_ERR_CUDA;
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_bsa_status, sizeof(int)) != cudaSuccess) return BSA_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_bsa_status, &zero, sizeof(int)) != cudaSuccess) return BSA_ERR_CUDA;
  return v;
}

}  // extern "C"

namespace {
__global__ void debug_expired_wait_kernel(long long limit_ns, int form) {
  __shared__ alignas(8) unsigned long long bar;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    fence_mbar_init();
  }
  __syncthreads();
  // nothing ever arrives on this barrier: the wait must give up by itself
  if (form == 0) {
    if (threadIdx.x == 0) mbar_wait(b, 0, limit_ns);
  } else {
    // the whole-warp form: every lane must see the same (false) result
    const bool ok = mbar_wait_warp(b, 0, limit_ns);
    if (__any_sync(0xFFFFFFFFu, ok) && threadIdx.x == 0) atomicExch(&g_bsa_status, BSA_ERR_ARG);
  }
}
}  // namespace

extern "C" int bsa_debug_expired_wait(long long limit_ns, int form, void* stream) {
  if (limit_ns < 100000LL || limit_ns > 10000000000LL || form < 0 || form > 1) return BSA_ERR_ARG;
  debug_expired_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, form);
  return cudaGetLastError() == cudaSuccess ? BSA_OK : BSA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// blocksparse_attn_fwd_noalloc: the workspace of blocksparse_attn_fwd placed in
// a file-scope device array, for callers that cannot allocate device memory.
// Host code must not use the array's name as a device address: the address
// is looked up once per device with cudaGetSymbolAddress (that device
// current) and passed on like a caller-owned workspace.
namespace {
constexpr size_t kNoAllocScratchBytes = BSA_NOALLOC_SCRATCH_BYTES;
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
void* g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mu;
}  // namespace

extern "C" int blocksparse_attn_fwd_noalloc(const void* q, const void* k, const void* v, int N, int H, int d,
                                            float scale, const bsa_index* index, void* o, float* lse,
                                            void* stream) {
  if (!index || N < 1 || H < 1) return BSA_ERR_ARG;
  if (index->kind == BSA_INDEX_LVSA_FRAMES || index->kind == BSA_INDEX_LVSA_BLOCKS) {
    // frame lists need the tile lists; the intersection also H * nB * nB flag bytes
    if (index->T < 1 || index->T > kMaxFrames) return BSA_ERR_ARG;
    if (N % index->T) return BSA_ERR_SHAPE;
    if (index_ws_bytes(index, N, H) > kNoAllocScratchBytes) return BSA_ERR_WORKSPACE;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BSA_ERR_CUDA;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return BSA_ERR_CUDA;
      g_noalloc_ptr[dev] = p;
    }
    scratch = g_noalloc_ptr[dev];
  }
  return blocksparse_attn_fwd(q, k, v, N, H, d, scale, index, o, lse, scratch, kNoAllocScratchBytes, stream);
}
