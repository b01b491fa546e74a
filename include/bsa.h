/*
 * bsa.h - C ABI of libbsa.so: frame/block-sparse self-attention for long
 * video diffusion-transformer token sequences on NVIDIA B200 (sm_100a).
 *
 * Two sources of sparsity are supported:
 *
 *  LVSA  "LVSA: Training-Free Sparse Attention for Long Video Diffusion"
 *        (gist.science explainer of arXiv 2605.31057), technical summary,
 *        section 2 "Method": query frame t attends the frame set
 *        A(t) = G u W(t) made of rotating global anchor frames G_s (shifted
 *        by s mod T_per at denoising step s; every frame is an anchor once
 *        per T_per steps) and a local window W(t) widened around anchors so
 *        that |A(t)| stays at the budget C.
 *
 *  LoSA  "LoSA (Near-Lossless Sparse Attention)" article (ai.ros.co.jp),
 *        section "Balancing efficiency and quality": one dense attention
 *        step measures the exact attention mass between blocks; per head and
 *        query block the minimal key-block set holding 99% of the mass is
 *        kept, and that index is frozen for every later denoising step.
 *
 * Conventions common to every call
 *  - Tensors are row-major.  q, k, v and o are bfloat16 [N, H, d]
 *    (token-major, then head, then channel; batch 1).  lse is float32
 *    [H, N] (natural log).  Integer index arrays are int32.
 *  - Every pointer argument is a DEVICE pointer unless stated otherwise.
 *    The caller owns all memory, including the workspace; the library
 *    allocates nothing and frees nothing.
 *  - Work is enqueued asynchronously on the caller's stream (cudaStream_t
 *    passed as void*; NULL = legacy default stream).  No call synchronises
 *    except bsa_get_device_status.
 *  - Return value: BSA_OK (0) or a positive warning on success; a negative
 *    bsa_status on error.  Argument errors are detected on the host before
 *    anything is enqueued, and then no output is touched.  Errors found by a
 *    kernel while it runs (index out of range, a bounded wait that expired)
 *    are recorded in a per-device status word read by bsa_get_device_status.
 *  - No C++ exception crosses this interface.
 *  - Supported: batch 1, bfloat16 inputs, d in {64, 128}, N >= 1,
 *    N * H * d < 2^31, 16-byte aligned q/k/v/o.  Anything else returns
 *    BSA_ERR_UNSUPPORTED or BSA_ERR_ARG.
 */
#ifndef BSA_H_
#define BSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum bsa_status {
  BSA_OK = 0,
  BSA_WARN_OVER_BUDGET = 1,   /* some |A(t)| > C because |G_s u {t}| > C  */
  BSA_ERR_ARG = -1,           /* null pointer, bad scalar, misalignment    */
  BSA_ERR_SHAPE = -2,         /* inconsistent sizes (e.g. T does not divide N) */
  BSA_ERR_CUDA = -3,          /* a CUDA runtime/driver call failed         */
  BSA_ERR_INDEX_RANGE = -4,   /* an index entry out of range (kernel-detected) */
  BSA_ERR_TIMEOUT = -5,       /* a bounded device-side wait expired        */
  BSA_ERR_UNSUPPORTED = -6,   /* valid request outside the supported set   */
  BSA_ERR_WORKSPACE = -7      /* workspace missing or smaller than needed  */
} bsa_status;

/* Index kinds accepted by blocksparse_attn_fwd. */
enum {
  BSA_INDEX_LVSA_FRAMES = 1,  /* frame lists from lvsa_build_index          */
  BSA_INDEX_BLOCKS = 2,       /* key-block lists from losa_select           */
  BSA_INDEX_LVSA_BLOCKS = 3   /* both: LVSA frames within selected blocks   */
};

/*
 * Sparse index handed to blocksparse_attn_fwd (host struct; the arrays it
 * points to are device memory owned by the caller).
 *
 * kind == BSA_INDEX_LVSA_FRAMES (fields T, frames, counts):
 *   frames [T][T] int32: row t holds A(t) ascending in its first counts[t]
 *   entries (the rest is ignored); counts [T] int32.  Every listed frame
 *   must lie in [0, T).  Token i belongs to frame i / P with P = N / T;
 *   query token q may attend key token k iff frame(k) is in A(frame(q)).
 *   The same frame lists serve every head.
 * kind == BSA_INDEX_BLOCKS (fields block, H, nQB, nKB, idx, cnt):
 *   block must be 128 and nQB == nKB == ceil(N / 128).  idx [H][nQB][nKB]
 *   int32: row (h, qb) lists its kept key blocks in its first cnt[h][qb]
 *   entries, ascending (the rest is ignored); cnt [H][nQB] int32.  Query
 *   token q of head h may attend key token k iff k / 128 is listed in row
 *   (h, q / 128).  Entries outside [0, nKB) are skipped and reported as
 *   BSA_ERR_INDEX_RANGE through the device status word; a count outside
 *   [0, nKB] is clamped and reported the same way.
 * kind == BSA_INDEX_LVSA_BLOCKS (all fields of kinds 1 and 2): the
 *   intersection - query token q of head h may attend key token k iff
 *   frame(k) is in A(frame(q)) and k / 128 is listed in row (h, q / 128).
 *   This runs LoSA's per-head block selection inside LVSA's frame sets; the
 *   pages never combine the two methods, so it is offered as a variant.
 */
typedef struct bsa_index {
  int kind;
  /* kind 1 */
  int T;
  const int32_t* frames;
  const int32_t* counts;
  /* kind 2 */
  int block, H, nQB, nKB;
  const int32_t* idx;
  const int32_t* cnt;
} bsa_index;

/*
 * lvsa_build_index - LVSA attended-frame sets for denoising step `step`.
 *
 * Source: [LVSA] section 2 (core mechanism; rotating global anchors;
 * expanded adaptive window).  Computes G_s = {f in [0,T): (f - step) mod
 * T_per == 0} and, per query frame t, A(t) = G_s u {t} plus the non-anchor
 * frames nearest to t (distance |f - t|; at equal distance the earlier frame
 * first; clipped to [0, T)) until |A(t)| = C.  If |G_s u {t}| > C then
 * A(t) = G_s u {t} and the call returns BSA_WARN_OVER_BUDGET (anchors and t
 * are never dropped).  C >= T gives every frame (dense attention).  W, the
 * nominal window size, must be >= 1; with the fill-to-budget rule it does
 * not change the sets.
 *
 * frames: out, device int32 [T][T]; row t = A(t) ascending, padded with -1.
 * counts: out, device int32 [T]; counts[t] = |A(t)|.
 * Limits: 1 <= T <= 1024, T_per >= 1, W >= 1, C >= 1, step >= 0.
 * Returns BSA_OK, BSA_WARN_OVER_BUDGET, or BSA_ERR_ARG / BSA_ERR_CUDA.
 */
int lvsa_build_index(int T, int T_per, int W, int C, int step,
                     int32_t* frames, int32_t* counts, void* stream);

/*
 * lvsa_build_index_window - LVSA attended-frame sets under the fixed-window
 * reading of the same passage.
 *
 * Source: [LVSA] section 2 (A(t) = G u W(t) with a local window of size W).
 * Where lvsa_build_index fills each set to the budget C, this call reads
 * the window as holding W non-anchor frames: W(t) = the W non-anchor frames
 * nearest to t (t itself first when it is not an anchor, then by distance
 * |f - t|, the earlier frame first at a tie, clipped to [0, T)), or every
 * non-anchor frame when there are fewer; A(t) = G_s u {t} u W(t), so
 * |A(t)| = |G_s| + min(W, T - |G_s|).  The sets equal lvsa_build_index's
 * with C = min(T, |G_s| + W), which is how they are computed.
 *
 * frames, counts: as for lvsa_build_index.
 * Limits: 1 <= T <= 1024, T_per >= 1, W >= 1, step >= 0.
 * Returns BSA_OK, or BSA_ERR_ARG / BSA_ERR_CUDA.
 */
int lvsa_build_index_window(int T, int T_per, int W, int step,
                            int32_t* frames, int32_t* counts, void* stream);

/*
 * attn_dense_blockmass - dense attention forward that also emits LoSA block mass.
 *
 * Source: [LoSA] section "Balancing efficiency and quality" (one dense
 * step measures the exact inter-block attention mass).  Computes, for
 * every head h and query token q (all N keys visible, no causal mask):
 *   o[q,h,:]  = sum_k softmax_k(scale * <q,k>) v[k,h,:]      (bfloat16 out)
 *   lse[h,q]  = log sum_k exp(scale * <q,k>)                 (float32 out)
 *   mass[h,qb,kb] = sum_{q in qb} sum_{k in kb} p_h(q,k)     (float32 out)
 * where qb, kb are 128-token blocks (the last one may be short) and p the
 * float32 softmax probabilities (not their bf16 rounding).  Sum over kb of
 * mass[h,qb,:] = number of tokens in qb.
 *
 * One pass: the forward also writes, per head, key tile kt and row q, the
 * log2 of the tile's share of the row's unnormalised mass (with the row's
 * running stabiliser); a reduction then divides by the final row sum and
 * adds the rows of each query block.  The probabilities are never
 * recomputed.
 *
 * q, k, v: in, bf16 [N,H,d].  block: must be 128.  scale: softmax scale
 * (normally d^-1/2).  o: out, bf16 [N,H,d].  lse: out, float32 [H,N].
 * mass: out, float32 [H][nB][nB], nB = ceil(N/128).
 * workspace, ws_bytes: device scratch, 256-byte aligned, owned by the
 * caller, at least one head's share (nB * N * 4 bytes); heads are processed
 * in passes of floor(ws_bytes / share) (bsa_workspace_bytes gives all heads
 * in one pass up to 4 GiB).  Too small or misaligned: BSA_ERR_WORKSPACE.
 * Returns BSA_OK or a negative bsa_status.
 */
int attn_dense_blockmass(const void* q, const void* k, const void* v,
                         int N, int H, int d, int block, float scale,
                         void* o, float* lse, float* mass,
                         void* workspace, size_t ws_bytes, void* stream);

/*
 * attn_blockmass - attention restricted to an index that also emits the
 * LoSA block mass of that restricted attention.
 *
 * Source: [LoSA] section "Balancing efficiency and quality" (the measuring
 * step records the attention mass between blocks), applied to attention
 * already restricted by `index` (e.g. LVSA frames, [LVSA] section 2), so
 * that a LoSA selection can be made inside the LVSA sets.  o and lse are
 * those of blocksparse_attn_fwd with the same index; mass[h,qb,kb] sums the
 * restricted float32 probabilities over the (qb, kb) rectangle (0 for
 * blocks the index does not reach).  attn_dense_blockmass is the case of
 * the full index.
 *
 * index: any kind accepted by blocksparse_attn_fwd.  workspace: device,
 * 256-byte aligned, at least bsa_workspace_bytes(BSA_OP_BLOCKSPARSE_FWD,
 * ...) rounded up to 256 plus one head's share of log partial sums
 * (ceil(N/128) * N * 4 bytes); heads are processed in passes of as many
 * shares as fit.  bsa_workspace_bytes(BSA_OP_BLOCKMASS, ...) gives all heads
 * in one pass up to 4 GiB.  Other arguments as for attn_dense_blockmass.
 * Returns BSA_OK or a negative bsa_status (BSA_ERR_WORKSPACE when the
 * workspace is too small or misaligned).
 */
int attn_blockmass(const void* q, const void* k, const void* v,
                   int N, int H, int d, float scale, const bsa_index* index,
                   void* o, float* lse, float* mass,
                   void* workspace, size_t ws_bytes, void* stream);

/*
 * losa_select - per (head, query block) minimal key-block set holding
 * fraction tau of the block mass.
 *
 * Source: [LoSA] sections "LoSA's innovative approach" (99% mass
 * constraint) and "Balancing efficiency and quality" (minimal set per head
 * and query block, frozen for later steps).  Per row (h, qb):
 *   Q_kb = floor(mass[h,qb,kb] * 2^33) (exact integer);
 *   order key blocks by Q descending, equal Q by kb ascending;
 *   threshold = ceil(tau * (double)sum_kb Q_kb) (one IEEE double multiply);
 *   keep the shortest prefix of that order whose sum reaches the threshold
 *   (at least one block); write the kept ids ascending.
 * The result depends only on the mass values (integer arithmetic), so it
 * is reproducible bit for bit.
 *
 * mass: in, float32 [H][nQB][nKB]; entries finite, >= 0 and < 2^14
 *   (violations are clamped to [0, 2^14) and reported as BSA_ERR_ARG
 *   through the device status word).
 * tau: in (0, 1].
 * idx: out, int32 [H][nQB][nKB]: kept ids ascending, then -1 padding.
 * cnt: out, int32 [H][nQB].
 * Limits: 1 <= nKB <= 8192.
 * Returns BSA_OK or a negative bsa_status.
 */
int losa_select(const float* mass, int H, int nQB, int nKB, double tau,
                int32_t* idx, int32_t* cnt, void* stream);

/*
 * blocksparse_attn_fwd - exact masked softmax attention restricted to an
 * LVSA frame index or a LoSA block index.
 *
 * Source: [LVSA] section 2 (block-sparse attention over A(t); cost
 * |A(t)| * P * d per query, linear in T) and section 4 (block-sparse kernel
 * speed-up over dense); [LoSA] "Balancing efficiency and quality" (the
 * frozen block index reused at every later step).  For every head h and
 * query token q with allowed key set K(q) (defined by `index`, see
 * bsa_index):
 *   o[q,h,:] = sum_{k in K(q)} softmax(scale * <q,k>) v[k,h,:]  (bf16 out)
 *   lse[h,q] = log sum_{k in K(q)} exp(scale * <q,k>)          (f32 out)
 * An empty K(q) gives o = 0 and lse = -inf.
 *
 * q, k, v: in, bf16 [N,H,d].  scale: softmax scale.  index: host pointer
 * to a bsa_index (read during the call only).  o: out, bf16 [N,H,d].
 * lse: out, float32 [H,N].
 * workspace: device scratch of at least
 *   bsa_workspace_bytes(BSA_OP_BLOCKSPARSE_FWD, N, H, d, index) bytes,
 *   256-byte aligned; it is overwritten.  For LVSA frame indexes it holds
 *   the frame-pair bit matrix and the per-query-tile key-tile lists built
 *   on the device by this call; block indexes need none (NULL, 0 allowed).
 * Returns BSA_OK or a negative bsa_status.
 */
int blocksparse_attn_fwd(const void* q, const void* k, const void* v,
                         int N, int H, int d, float scale,
                         const bsa_index* index, void* o, float* lse,
                         void* workspace, size_t ws_bytes, void* stream);

/*
 * blocksparse_attn_fwd_noalloc - the same computation as blocksparse_attn_fwd,
 * for callers that cannot allocate device memory.
 *
 * The pages have no counterpart to this call; it exists for integration.
 * Some callers cannot hand the library a workspace: plug-in hosts that own
 * all device memory and give a plug-in no allocator, or latency-critical
 * loops where a cudaMalloc (which may synchronise the device, or fail at run
 * time) is not acceptable.  This entry point takes no workspace and
 * allocates nothing: its scratch (the LVSA frame-pair bit matrix and key-tile
 * lists) lives in one file-scope device array of BSA_NOALLOC_SCRATCH_BYTES
 * bytes that every GPU loading the library holds until the process exits.
 *
 * Arguments, layouts and results are those of blocksparse_attn_fwd, and all
 * three index kinds are accepted.  Block indexes (BSA_INDEX_BLOCKS) need no
 * scratch.  LVSA frame indexes (BSA_INDEX_LVSA_FRAMES) need the frame-pair
 * bit matrix and the key-tile lists, about 5 * ceil(N/128)^2 bytes: up to
 * about N = 234,000 tokens fits.  The intersection (BSA_INDEX_LVSA_BLOCKS)
 * needs H * ceil(N/128)^2 bytes more for its per-head flags, so it fits only
 * small shapes (N = 32,760 with up to 250 heads; not the 14B-head 720p shape).
 * The need is bsa_workspace_bytes(BSA_OP_BLOCKSPARSE_FWD, ...); when it is
 * larger than BSA_NOALLOC_SCRATCH_BYTES the call returns BSA_ERR_WORKSPACE
 * before anything is enqueued.
 *
 * The first call on a device looks up the device address of the array on
 * that device (cudaGetSymbolAddress, with that device current); make that
 * first call before any stream capture.  All calls on a device share the one
 * array, and each call overwrites what the previous one left there before
 * reading it (nothing has to start at zero).  Calls that overlap on the GPU
 * (other streams, other host threads) race on the array: serialise them.
 */
#define BSA_NOALLOC_SCRATCH_BYTES (16u << 20)
int blocksparse_attn_fwd_noalloc(const void* q, const void* k, const void* v,
                                 int N, int H, int d, float scale,
                                 const bsa_index* index, void* o, float* lse,
                                 void* stream);

/* Operation codes for bsa_workspace_bytes. */
enum {
  BSA_OP_BLOCKSPARSE_FWD = 1,
  BSA_OP_DENSE_BLOCKMASS = 2,
  BSA_OP_BLOCKMASS = 3
};

/*
 * bsa_workspace_bytes - scratch bytes the operation `op` needs for these
 * sizes (0 if none).  index may be NULL for BSA_OP_DENSE_BLOCKMASS.  For
 * BSA_OP_DENSE_BLOCKMASS the answer is the share of as many heads as fit in
 * 4 GiB (at least one, at most H), share = ceil(N/128) * N * 4 bytes; any
 * workspace of at least one share is accepted by attn_dense_blockmass.
 * Returns (size_t)-1 for invalid arguments.
 */
size_t bsa_workspace_bytes(int op, int N, int H, int d, const bsa_index* index);

/*
 * bsa_get_device_status - synchronise `stream`, then return and clear the
 * current device's status word: BSA_OK, or the first kernel-detected error
 * since the last call (BSA_ERR_INDEX_RANGE, BSA_ERR_TIMEOUT, BSA_ERR_ARG).
 * Returns BSA_ERR_CUDA if the synchronisation itself failed.
 */
int bsa_get_device_status(void* stream);

/* bsa_status_string - static, human-readable name of a status code. */
const char* bsa_status_string(int status);

/*
 * bsa_debug_expired_wait - diagnostic for the bounded-wait machinery.
 * Enqueues one tiny kernel (one warp) that waits on a barrier that nothing
 * ever signals, giving up after 2 * `limit_ns` SM clock cycles (`limit_ns`
 * nanoseconds at 2 GHz; `limit_ns` in 1e5..1e10) and recording
 * BSA_ERR_TIMEOUT in the status word.  `form` 0: one thread waits (the
 * producers' and softmax warps' form); 1: the whole warp waits and must get
 * the same failed result in every lane (the MMA issuer's form; a lane that
 * saw the wait succeed records BSA_ERR_ARG instead).  Lets tests check that
 * an expired wait ends the kernel and leaves the context usable.  Returns
 * BSA_ERR_ARG for an out-of-range `limit_ns` or `form`.  No part of the
 * pages corresponds to it.
 */
int bsa_debug_expired_wait(long long limit_ns, int form, void* stream);

/* bsa_version - library version string. */
const char* bsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BSA_H_ */
