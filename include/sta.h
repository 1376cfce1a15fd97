/*
 * sta.h -- C ABI of the sparse spatiotemporal attention library (libsta.so).
 *
 * Content-adaptive sparse self-attention over a video latent grid of
 * F frames x H x W tokens, for B200 (sm_100a).  Two stages:
 *
 *   sta_build_blocks     selector: Q, K (or geometry) -> integer KV-unit lists
 *   sta_sparse_attn_fwd  exact softmax attention over the kept units only
 *   sta_dense_attn_fwd   the same kernel over every key (the denominator of
 *                        the speedup metric)
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Tensors q, k, v, o are [heads][N][d], N = F*H*W, tokens in raster order
 *   (frame-major, then row h, then column w), d contiguous.  Element type is
 *   sta_problem.dtype (bf16, or fp32 which is rounded to bf16 on the device
 *   before the tensor cores; o then is fp32).
 * - Every pointer argument that names tensor data is a DEVICE pointer owned
 *   by the caller.  The library never allocates, frees or retains memory and
 *   keeps no state between calls.  Scratch space, where needed, is passed in
 *   as `workspace` after querying its size.  (The one exception is
 *   sta_sparse_attn_fwd_noalloc, which uses a fixed array of its own.)
 * - Every call only enqueues work on `stream` (a cudaStream_t; NULL is the
 *   legacy default stream) and returns.  Results are valid once the caller
 *   has synchronised the stream.
 * - The host return value reports argument errors and launch failures.
 *   In-kernel errors are OR-ed into the caller's device word `dev_status`
 *   (an int32 in device memory, may be NULL) as STA_DEV_* bits; decode it
 *   after synchronising with sta_dev_status_string().
 * - Each call that enqueues selector, attention or permutation work is
 *   wrapped in an NVTX range named after the call (seen by profilers that
 *   trace NVTX; free otherwise).
 * - Shapes supported: d in {64, 128}; block_q in {16, 32, 64, 128};
 *   kv_unit in {16, 32, 64, 128}.  Anything else returns STA_ERR_UNSUPPORTED.
 *   There is no CPU path.
 *
 * Page references are to the pages this library restates:
 *   [TRA]   "Token Radius Attention for Efficient Video Generation"
 *   [RAD]   "Radial Attention to Accelerate Video Generation"
 *   [HETA]  "Where Compute Matters: Heterogeneous Attention for Efficient
 *            Video Diffusion"
 *   [AB]    "AB-Attention speeds up video diffusion transformers up to 2.23x,
 *            no training"
 *   [DYN]   "DynamicRad: Content-Adaptive Sparse Attention for Long Video
 *            Diffusion"
 */
#ifndef STA_H
#define STA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Opaque CUDA stream handle (binary-compatible with cudaStream_t). */
typedef struct CUstream_st* sta_stream_t;

typedef enum {
  STA_OK = 0,
  STA_ERR_ARG = -1,          /* null pointer, bad dimension, inconsistent sizes */
  STA_ERR_UNSUPPORTED = -2,  /* valid request outside the supported shapes     */
  STA_ERR_CAPACITY = -3,     /* a list row needs more than `cap` entries       */
  STA_ERR_CUDA = -4,         /* a CUDA runtime/driver call or launch failed    */
  STA_ERR_WORKSPACE = -5     /* workspace pointer NULL or smaller than needed  */
} sta_status;

/* Bits OR-ed into *dev_status by kernels. */
#define STA_DEV_TIMEOUT   0x1  /* a bounded wait ran out; the CTA abandoned its work */
#define STA_DEV_CAPACITY  0x2  /* a list row was truncated at `cap`                  */
#define STA_DEV_EMPTY_ROW 0x4  /* a query row had no kept key; its output is 0      */
#define STA_DEV_BAD_INDEX 0x8  /* a list entry was out of range and was skipped     */
#define STA_DEV_RANGE     0x10 /* an importance operand exceeded the fp16 range     */
#define STA_DEV_DEBUG     0x20 /* debug build only: an index check failed and the
                                  access it guarded was skipped                    */

typedef enum { STA_BF16 = 0, STA_F32 = 1 } sta_dtype;

typedef enum {
  STA_SEL_RADIAL = 0,    /* static radial window         [RAD] The idea behind Radial Attention */
  STA_SEL_ENTROPY = 1,   /* pooled entropy -> radius     [TRA] 2. Methodology, The TRA Pipeline */
  STA_SEL_IBCS_SIP = 2,  /* k-means importance + Philox inclusion-probability sampling  [AB]   */
  STA_SEL_ROUTED = 3,    /* difficulty routing: dense for the top fraction, local window [HETA] */
  STA_SEL_TRA_TOKEN = 4, /* per-query entropy -> budget -> disk radius -> token voting  [TRA]  */
  STA_SEL_DYNRAD = 5     /* static-ratio / dynamic-threshold selection in the radial prior [DYN] */
} sta_selector;

/* Problem geometry.  N = F*H*W tokens per head. */
typedef struct {
  int heads, F, H, W, d;
  sta_dtype dtype;
} sta_problem;

/*
 * Selector parameters.  Only the group of the chosen kind is read.
 *
 * radial   [RAD]: window at frame distance df (tokens):
 *            w(df) = H*W                                  if df <= full_df
 *                  = w0 >> floor(log2(df + w_off))         otherwise
 *          query token i and key token j are related iff |s_i - s_j| < w(|f_i - f_j|)
 *          (s = h*W + w inside a frame); a block pair is kept iff any of its
 *          token pairs is related.  Lists are shared by all heads.
 * entropy  [TRA]: pooled block means, H_b = entropy of softmax_c(Qbar_b.Kbar_c/sqrt(d)),
 *          radius r_b = clamp(floor(alpha + beta*H_b), r_lo, r_hi) (fp32),
 *          key block kept iff the Chebyshev distance of block cells
 *          (f, h/tile_h, w/tile_w) of the blocks' centre tokens is <= r_b.
 * ibcs_sip [AB]: k-means (km_k centroids, km_iters iterations) of each query
 *          block's queries; importance p_j of kv_unit-token sub-blocks;
 *          pi_j = min(1, lambda p_j), sum pi = ceil(sample_frac * n_sub);
 *          keep j iff u_j < pi_j with u_j from Philox4x32-10 (key = seed,
 *          counter = (j/4, 0, head*n_qblocks + qblock, 0)); logw_j = -ln pi_j.
 * routed   [HETA]: the ceil(dense_frac*N) tokens of highest difficulty (fp32,
 *          ties to the lower index) attend to all keys; every other token
 *          attends to keys with |df| <= win_f, dh in [-win_h, win_h),
 *          dw in [-win_w, win_w).  `difficulty` is a device pointer [N].
 * tra_token [TRA] 2. Methodology (Insight I, Insight II, The TRA Pipeline):
 *          tra_entropy is a device pointer [heads][N] of per-query attention
 *          entropies in nats (from sta_dense_attn_entropy_fwd, the dense
 *          warm-up).  Query i keeps about n_i = tau * exp(H_i) keys, laid out
 *          as a disk per frame: r0^2 = n_i / (pi * sum_f exp(-2 gamma |f - f_i|)),
 *          r_f^2 = r0^2 * exp(-2 gamma |f - f_i|) (fp32); frame f holds
 *          pi * r_f^2 tokens of the budget and keeps nothing when that is
 *          below 1; otherwise key j is kept iff
 *          (h_j - h_i)^2 + (w_j - w_i)^2 <= r_{f_j}^2.  A key block is listed
 *          for a query block iff at least tra_vote kept (query, key) pairs fall
 *          in the pair (token voting).  block_q == kv_unit; lists per head.
 *          Blocks are runs of block_q sequence positions: raster order, or
 *          with layout_tile_h, layout_tile_w > 0 the tile-major order of
 *          sta_permute_tokens (2. Methodology, The TRA Pipeline, Efficient
 *          Execution); tra_entropy is then indexed by tile-major position.
 * dynrad   [DYN] Abstract: the radial lists (radial_* parameters) are the
 *          candidates; p_c = softmax over the candidates of the pooled
 *          scores Qbar_b.Kbar_c/sqrt(d) (fp32); candidates ranked by score
 *          (ties to the lower block id).  dyn_mode 0 (static ratio) keeps the
 *          ceil(dyn_ratio * n) best (relative slack 1e-6, at least 1);
 *          dyn_mode 1 (dynamic threshold) keeps the shortest best-first
 *          prefix whose p mass reaches dyn_threshold.  block_q == kv_unit,
 *          at most 1024 blocks; lists per head, ascending.
 */
typedef struct {
  sta_selector kind;
  int block_q;   /* query block size in tokens                          */
  int kv_unit;   /* key/value unit size in tokens (list entries)        */
  /* radial */
  int radial_w0, radial_w_off, radial_full_df;
  /* entropy */
  float ent_alpha, ent_beta;
  int ent_r_lo, ent_r_hi, ent_tile_h, ent_tile_w;
  /* ibcs_sip */
  int km_k, km_iters;
  float sample_frac;
  uint64_t seed;
  /* routed */
  float dense_frac;
  int win_f, win_h, win_w;
  const float* difficulty;
  /* tra_token */
  float tra_tau, tra_gamma;
  int tra_vote;
  const float* tra_entropy;
  /* dynrad (and the radial_* fields for its prior) */
  int dyn_mode;
  float dyn_ratio, dyn_threshold;
  /* token order of the sequence the lists index (tra_token): 0, 0 = raster;
   * tile_h x tile_w = tile-major (see sta_permute_tokens) */
  int layout_tile_h, layout_tile_w;
} sta_selector_params;

/*
 * Block lists (ELL layout), all device memory owned by the caller.
 *   rows      = n_qblocks (head_shared = 1) or heads * n_qblocks, with
 *               n_qblocks = ceil(N / block_q)
 *   idx       [rows][cap] int32 unit ids, ascending; unit u covers tokens
 *             [u*kv_unit, min((u+1)*kv_unit, N))
 *   cnt       [rows] int32 number of valid entries per row
 *   logw      [rows][cap] float, -ln(pi) per entry (ibcs_sip) or NULL
 *   required_cap  device int32, written with the largest row length seen
 *             (may be NULL).  Rows longer than cap are truncated and
 *             STA_DEV_CAPACITY is raised.
 * Routed extras (STA_SEL_ROUTED; the local lists above then hold the
 * kv_unit units touched by each query block's local windows):
 *   routed_ids   [n_routed] int32 ascending routed token ids
 *   routed_flag  [N] uint8, 1 if the token is routed
 *   n_routed     host field, set by sta_build_blocks
 * Entropy extras (STA_SEL_ENTROPY, optional):
 *   entropy [heads][n_qblocks] float, radius [heads][n_qblocks] int32
 */
typedef struct {
  int32_t* idx;
  int32_t* cnt;
  float* logw;
  int32_t cap;
  int32_t head_shared;
  int32_t* required_cap;
  int32_t* routed_ids;
  uint8_t* routed_flag;
  int32_t n_routed;
  float* entropy;
  int32_t* radius;
} sta_block_lists;

/* Workspace bytes sta_build_blocks needs for this problem and selector.
 * The workspace must start on a 256-byte boundary (cudaMalloc and torch
 * allocations do); any other start is STA_ERR_WORKSPACE. */
size_t sta_build_blocks_workspace(const sta_problem* prob, const sta_selector_params* sel);

/* Rows of the lists the selector writes (n_qblocks, or heads*n_qblocks). */
int sta_build_blocks_rows(const sta_problem* prob, const sta_selector_params* sel);

/*
 * Stage (a): selector.  Each kind restates one page's block selection:
 *   STA_SEL_RADIAL    [RAD] The idea behind Radial Attention (static mask,
 *                     window shrinking with frame distance);
 *   STA_SEL_ENTROPY   [TRA] 2. Methodology, Insight I and The TRA Pipeline
 *                     (entropy -> radius -> block mask), on pooled blocks;
 *   STA_SEL_TRA_TOKEN [TRA] 2. Methodology, Insight II and The TRA Pipeline
 *                     (budget tau*exp(H), decaying disks, token voting);
 *   STA_SEL_IBCS_SIP  [AB] method paragraph (intra-block clustering
 *                     importance, inclusion-probability sampling, 1/pi);
 *   STA_SEL_ROUTED    [HETA] Abstract (uncertain tokens dense, rest local);
 *   STA_SEL_DYNRAD    [DYN] Abstract (static-ratio / dynamic-threshold
 *                     selection inside a radial prior).
 * The formulas of each kind are in the sta_selector_params comment above.
 * q, k: device tensors [heads][N][d] (may be NULL for
 * the radial, routed and tra_token kinds, which read only geometry,
 * difficulty or the entropies).  The kinds that read q and k (entropy,
 * ibcs_sip, dynrad) take bf16 only.  Writes `out` (see sta_block_lists).
 * Asynchronous on `stream`.
 * Errors: STA_ERR_ARG (null/inconsistent, a parameter out of range),
 * STA_ERR_UNSUPPORTED (shape, dtype or a size beyond a selector's limit),
 * STA_ERR_WORKSPACE (workspace missing, short or misaligned), STA_ERR_CUDA.
 */
sta_status sta_build_blocks(const sta_problem* prob, const sta_selector_params* sel,
                            const void* q, const void* k, sta_block_lists* out,
                            void* workspace, size_t workspace_bytes,
                            int32_t* dev_status, sta_stream_t stream);

/* Attention modes. */
typedef enum {
  STA_ATTN_LISTS = 0,   /* per (head, query block) rows of `lists`                  */
  STA_ATTN_ROUTED = 1   /* routed rows dense over all keys + local lists w/ window  */
} sta_attn_mode;

typedef struct {
  sta_attn_mode mode;
  int block_q;       /* query block of the lists (tokens)                   */
  int kv_unit;       /* unit size of the list entries (tokens)              */
  float scale;       /* logit scale; <= 0 selects 1/sqrt(d)                 */
  int win_f, win_h, win_w;  /* STA_ATTN_ROUTED local window                 */
} sta_attn_params;

/* Workspace bytes of the attention calls (0 for bf16 inputs). */
size_t sta_attn_workspace(const sta_problem* prob);

/*
 * Stage (b): exact attention over the kept units.
 * [TRA] 1. Problem Statement (block-level sparsity) and The TRA Pipeline;
 * [AB] method paragraph (pruned blocks vanish from the softmax; sampled
 * units weighted by 1/pi; small units packed into full tensor-core tiles).
 * For query i with kept key set K_i and weights w (1, or exp(logw)):
 *   O_i = sum_k w_k exp(s_ik - m_i) v_k / sum_k w_k exp(s_ik - m_i),
 *   s_ik = scale * q_i.k_k.  Rows with no kept key get O_i = 0.
 * o: device [heads][N][d] (bf16, or fp32 when dtype is STA_F32).  Rows not
 * covered by any list row are left untouched.
 */
sta_status sta_sparse_attn_fwd(const sta_problem* prob, const sta_attn_params* prm,
                               const void* q, const void* k, const void* v,
                               const sta_block_lists* lists, void* o,
                               void* workspace, size_t workspace_bytes,
                               int32_t* dev_status, sta_stream_t stream);

/*
 * Dense softmax attention over all N keys ([TRA] 1. Problem Statement),
 * the same kernel with an implicit full list of 128-key units.
 */
sta_status sta_dense_attn_fwd(const sta_problem* prob, const void* q, const void* k,
                              const void* v, float scale, void* o,
                              void* workspace, size_t workspace_bytes,
                              int32_t* dev_status, sta_stream_t stream);

/*
 * Dense attention that also writes each query's attention entropy
 * ([TRA] 2. Methodology, The TRA Pipeline: entropy is taken during a dense
 * warm-up pass and feeds the STA_SEL_TRA_TOKEN selector):
 *   entropy[h][i] = -sum_j p_ij ln p_ij,  p_ij = softmax_j(scale * q_i.k_j)
 * in nats, accumulated in fp32 from the unrounded probabilities.  entropy:
 * device float [heads][N], caller-owned.  Other arguments, results and
 * errors as sta_dense_attn_fwd.
 */
sta_status sta_dense_attn_entropy_fwd(const sta_problem* prob, const void* q, const void* k,
                                      const void* v, float scale, void* o, float* entropy,
                                      void* workspace, size_t workspace_bytes,
                                      int32_t* dev_status, sta_stream_t stream);

/*
 * sta_sparse_attn_fwd with no workspace argument, for callers that cannot
 * allocate device memory: a plugin that its host framework hands only the
 * input and output buffers, or a pipeline that bans cudaMalloc after
 * start-up because it can synchronise the device.  (The pages have no
 * counterpart: this is a deployment convenience of this library.)
 *
 * Same arguments and results as sta_sparse_attn_fwd.  bf16 inputs need no
 * scratch.  fp32 inputs are rounded to bf16 into one fixed 12 MiB device
 * array inside the library (never cudaMalloc), so 3 * heads*N*d bf16
 * copies, each rounded up to 256 bytes, must fit in 12 MiB: at most
 * 2,097,152 elements per tensor; larger problems return STA_ERR_WORKSPACE
 * and enqueue nothing.  Each device the library is used on holds the array
 * until the process exits.
 * The first call on a device looks the array's device address up (with that
 * device current) and caches it; make that first call before any stream
 * capture.  A reset of the device (cudaDeviceReset) unloads the array and
 * leaves the cached address stale: do not use this entry point on a device
 * after resetting it.  Argument errors (STA_ERR_ARG, STA_ERR_UNSUPPORTED)
 * are checked before the size limit, as by sta_sparse_attn_fwd.  Every call on every stream shares the one array and leaves its
 * contents behind: two fp32 calls that may overlap on the GPU (different
 * streams, no ordering between them) race on it.  Calls on one stream are
 * ordered and safe.
 */
sta_status sta_sparse_attn_fwd_noalloc(const sta_problem* prob, const sta_attn_params* prm,
                                       const void* q, const void* k, const void* v,
                                       const sta_block_lists* lists, void* o,
                                       int32_t* dev_status, sta_stream_t stream);

/*
 * Token permutation between the raster order and a tile-major order
 * ([TRA] 2. Methodology, The TRA Pipeline, Efficient Execution: tokens are
 * reordered tile by tile so that a query's spatial neighbours are
 * contiguous).  Within each frame, positions run over spatial tiles of
 * tile_h x tile_w tokens: tile row, tile column, row inside the tile, column
 * inside the tile.  Tiles on the bottom and right edges are cut by the grid
 * (no padding), so the order is a permutation of the N tokens of each frame.
 * tile_h = 1, tile_w = W is the raster order.
 *   inverse = 0: out[h][j] = in[h][perm(j)]   (raster -> tile-major)
 *   inverse = 1: out[h][perm(j)] = in[h][j]   (tile-major -> raster)
 * with perm(j) the raster token at tile-major position j.  in, out: device
 * tensors [heads][N][d] of prob->dtype, caller-owned, not overlapping.
 * Attention in the tile-major order is the same attention: permute q, k, v,
 * run the selector (layout_tile_h/w set) and sta_sparse_attn_fwd, and permute
 * o back.  Errors: STA_ERR_ARG (null, overlap, tile_h or tile_w outside
 * [1, H] x [1, W]), STA_ERR_CUDA.
 */
sta_status sta_permute_tokens(const sta_problem* prob, int tile_h, int tile_w, int inverse,
                              const void* in, void* out, sta_stream_t stream);

/* Static description of a status code / of the device status bits. */
const char* sta_status_string(sta_status s);
const char* sta_dev_status_string(int32_t bits);

/*
 * Description of the last CUDA error an entry point of this library ran into
 * on the calling thread (the reason behind a STA_ERR_CUDA return), or "no CUDA
 * error".  The string is static; the record persists until the next failure.
 */
const char* sta_last_cuda_error(void);

/*
 * Self-test of the bounded waits that every kernel of this library uses (no
 * counterpart on the pages; it supports failure detection).  One CTA waits on
 * a barrier phase that nothing completes, with a limit of limit_ns
 * nanoseconds of GPU global time (0 < limit_ns <= 2e9).  When the limit runs
 * out the kernel gives up, ORs STA_DEV_TIMEOUT into *dev_status, writes 0 to
 * *waited_ok (1 would mean the wait completed) and returns; it never traps,
 * so the context stays usable.  dev_status and waited_ok: device int32.
 * Errors: STA_ERR_ARG, STA_ERR_CUDA.
 */
sta_status sta_selftest_bounded_wait(uint64_t limit_ns, int32_t* dev_status, int32_t* waited_ok,
                                     sta_stream_t stream);

/*
 * Debug build (no counterpart on the pages; it stands in for a memory
 * checker).  libsta_debug.so is this library compiled with STA_DEBUG=1 and
 * exports the same calls.  Its kernels check every list entry, token index
 * and TMEM column they touch; a failed check ORs STA_DEV_DEBUG into
 * *dev_status and skips the access instead of trapping.  Results are those of
 * the release build; the checks cost a few percent.
 * sta_debug_build() returns 1 in libsta_debug.so and 0 in libsta.so.
 */
int sta_debug_build(void);

/*
 * Self-test of the debug build's index checks: one thread stores 1 into
 * buf[index] through the checked path, where buf is a device int32 array of
 * n elements (n >= 1).  An index outside [0, n) raises STA_DEV_DEBUG in
 * *dev_status and stores nothing.  Only the debug build runs it: libsta.so
 * has no checks and returns STA_ERR_UNSUPPORTED without launching anything.
 * Errors: STA_ERR_ARG (null pointer, n < 1), STA_ERR_UNSUPPORTED, STA_ERR_CUDA.
 */
sta_status sta_selftest_index_check(int32_t* buf, int n, int index, int32_t* dev_status,
                                    sta_stream_t stream);

/* Library version (major*10000 + minor*100 + patch). */
int sta_version(void);

#ifdef __cplusplus
}
#endif

#endif /* STA_H */
