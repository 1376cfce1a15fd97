// common.cuh -- internal declarations shared by the library's translation
// units (not part of the C ABI).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <atomic>

#include "sta.h"

namespace sta {

// Key/value tile width and query tile height of the attention kernel.
constexpr int kTileQ = 128;
constexpr int kTileK = 128;

// Bounded-wait budget of every in-kernel wait (global-timer nanoseconds).
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ void raise_status(int32_t* dev_status, int32_t bits) {
  if (dev_status) atomicOr(dev_status, bits);
}

// Index checks of the STA_DEBUG build (libsta_debug.so): dcheck(ok, st)
// returns ok and, when ok is false, raises STA_DEV_DEBUG; the caller skips
// the guarded access.  In the release build it is `true` and the condition
// is compiled away.
#ifndef STA_DEBUG
#define STA_DEBUG 0
#endif
__device__ __forceinline__ bool dcheck(bool ok, int32_t* dev_status) {
#if STA_DEBUG
  if (!ok) raise_status(dev_status, STA_DEV_DEBUG);
  return ok;
#else
  (void)ok;
  (void)dev_status;
  return true;
#endif
}
// TMEM address (lane << 16 | column) of an access of `cols` columns by a
// warp's 32 lanes inside the `alloc` columns allocated at `base`.
__device__ __forceinline__ bool tmem_in_range(uint32_t addr, uint32_t base, uint32_t cols,
                                              uint32_t alloc = 512) {
  const uint32_t col = (addr & 0xffffu) - (base & 0xffffu);
  const uint32_t lane = addr >> 16;
  return col + cols <= alloc && lane + 32u <= 128u;
}

// Token layout of a sequence ("Token Radius Attention for Efficient Video
// Generation", 2. Methodology, The TRA Pipeline, Efficient Execution: tokens
// reordered tile by tile).  Within a frame, positions run over spatial tiles
// of th x tw tokens: tile row, tile column, row in the tile, column in the
// tile; tiles on the bottom and right edges are cut by the grid (no padding).
// th = 1, tw = W is the raster order.
struct TokLayout {
  int H, W, th, tw;
};

// Grid coordinates (f, h, w) of the token at sequence position t, and the
// number of positions from t on that continue along the same grid row (to
// the end of the tile's row).
__device__ __forceinline__ void layout_coords(const TokLayout& L, int t, int& f, int& h, int& w,
                                              int& run) {
  const int S = L.H * L.W;
  f = t / S;
  const int j = t - f * S;
  const int tr = j / (L.th * L.W);       // tile row (every earlier one is full height)
  const int rem = j - tr * L.th * L.W;
  const int thr = min(L.th, L.H - tr * L.th);  // height of this tile row
  const int tc = rem / (thr * L.tw);     // tile column (every earlier one is full width)
  const int rem2 = rem - tc * thr * L.tw;
  const int twc = min(L.tw, L.W - tc * L.tw);  // width of this tile
  const int i = rem2 / twc;
  const int c = rem2 - i * twc;
  h = tr * L.th + i;
  w = tc * L.tw + c;
  run = twc - c;
}

enum AttnKind : int {
  kItemList = 0,       // raster query block, keys from a list row
  kItemDense = 1,      // raster query block, every key
  kItemGatherDense = 2,  // gathered (routed) query rows, every key
  kItemLocal = 3       // raster query block, list row + local window predicate
};

enum AttnMode : int { kModeLists = 0, kModeDense = 1, kModeRouted = 2 };

struct AttnArgs {
  int heads, N, F, H, W;
  float scale_log2;  // logit scale * log2(e)
  int mode;
  int block_q;       // raster query block (tokens)
  int unit;          // list unit size (tokens)
  int n_qb;          // ceil(N / block_q)
  int n_items;
  // lists
  const int32_t* idx;
  const int32_t* cnt;
  const float* logw;
  int cap;
  int head_shared;
  // routed
  const int32_t* routed_ids;
  const uint8_t* routed_flag;
  int n_routed;
  int n_dense_items;  // per head = ceil(n_routed / kTileQ)
  int win_f, win_h, win_w;
  // tensors
  const __nv_bfloat16* q;  // for gathered query rows
  void* o;
  int out_f32;
  int32_t* dev_status;
  float* entropy;  // dense mode: per-query attention entropy [heads][N] (nats), or null
};

// Launchers (attn_fwd.cu).  With d = 128 and 16-key units the
// unit maps have 8-row boxes and tm_k_il / tm_v_il are the interleaved
// five-dimensional views (see interleaved_unit_map); otherwise those two are
// unused.
cudaError_t launch_attention(int d, const AttnArgs& a, const CUtensorMap& tm_q,
                             const CUtensorMap& tm_k_unit, const CUtensorMap& tm_v_unit,
                             const CUtensorMap& tm_k_full, const CUtensorMap& tm_v_full,
                             const CUtensorMap& tm_k_il, const CUtensorMap& tm_v_il,
                             int num_sms, cudaStream_t stream);
cudaError_t launch_f32_to_bf16(const float* src, __nv_bfloat16* dst, size_t n, cudaStream_t s);

// Row permutation between the raster and a tile-major layout (layout.cu):
// out[h][j] = in[h][perm(j)] (inverse = 0) or out[h][perm(j)] = in[h][j]
// (inverse = 1), rows of row_bytes (a multiple of 16).
cudaError_t launch_permute_rows(const void* in, void* out, int heads, int N, int row_bytes,
                                const TokLayout& L, int inverse, cudaStream_t s);

// Radial selector (sel_radial.cu).
cudaError_t launch_radial_lists(int F, int H, int W, int B, int w0, int w_off, int full_df,
                                int32_t* idx, int32_t* cnt, int cap, int32_t* required_cap,
                                int32_t* dev_status, cudaStream_t stream);

// Raises kernel Fn's dynamic shared memory limit to at least `bytes` on the
// current device, calling cudaFuncSetAttribute only when the limit grows (the
// attribute is per device, and the call costs host time on every launch).
template <auto Fn>
cudaError_t set_dyn_smem(int bytes) {
  static std::atomic<int> done[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool cached = dev >= 0 && dev < 64;
  if (cached && done[dev].load(std::memory_order_acquire) >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(Fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && cached) {
    int prev = done[dev].load(std::memory_order_relaxed);
    while (prev < bytes && !done[dev].compare_exchange_weak(prev, bytes)) {
    }
  }
  return e;
}

// Block means (sel_pool.cu): out_i[h][b][d] = mean of the rows of block b of
// x_i (fp32); x1/out1 may be null.  The _f16x2 form writes each mean as the
// fp16 pair hi = fp16(m), lo = fp16(m - hi) instead (STA_DEV_RANGE beyond
// the fp16 range).
cudaError_t launch_block_means(const __nv_bfloat16* x0, const __nv_bfloat16* x1, float* out0,
                               float* out1, int heads, int N, int d, int U, cudaStream_t s);
cudaError_t launch_block_means_f16x2(const __nv_bfloat16* x, __half* hi, __half* lo, int heads,
                                     int N, int d, int U, int32_t* dev_status, cudaStream_t s);

// Entropy-radius selector (sel_entropy.cu).
int entropy_max_blocks(int d);
cudaError_t launch_entropy_lists(const float* qbar, const float* kbar, float* scores, int heads,
                                 int F, int H, int W, int d, int B, float scale, float alpha,
                                 float beta, int r_lo, int r_hi, int tile_h, int tile_w,
                                 int32_t* idx, int32_t* cnt, int cap, int32_t* required_cap,
                                 float* entropy, int32_t* radius, int32_t* dev_status,
                                 cudaStream_t s);

// Token-level entropy -> disk radius -> token voting (sel_tra.cu).
int tra_max_frames();
int tra_max_block();
cudaError_t launch_tra_token_lists(const float* entropy, int heads, int F, int H, int W, int B,
                                   int tile_h, int tile_w, float tau, float gamma, int vote,
                                   int32_t* idx, int32_t* cnt, int cap, int32_t* required_cap,
                                   int32_t* dev_status, cudaStream_t s);

// Dual-mode selection in the radial prior (sel_dynrad.cu).
int dynrad_max_candidates();
cudaError_t launch_dynrad_lists(const float* qbar, const float* kbar, const int32_t* prior_idx,
                                const int32_t* prior_cnt, int prior_cap, int heads, int nb, int d,
                                float scale, int mode, float ratio, float threshold, int32_t* idx,
                                int32_t* cnt, int cap, int32_t* required_cap,
                                int32_t* dev_status, cudaStream_t s);

// Difficulty routing (sel_routed.cu).
cudaError_t launch_routed_select(const float* difficulty, int N, int n_routed,
                                 int32_t* routed_ids, uint8_t* routed_flag, cudaStream_t s);
cudaError_t launch_routed_local_lists(int F, int H, int W, int B, int U, int win_f, int win_h,
                                      int win_w, int32_t* idx, int32_t* cnt, int cap,
                                      int32_t* required_cap, int32_t* dev_status,
                                      cudaStream_t s);

// Clustering importance + inclusion-probability sampling (sel_ibcs.cu,
// sel_importance.cu).
int ibcs_max_subblocks();
cudaError_t launch_kmeans(const __nv_bfloat16* q, __half* cent_hi, __half* cent_lo, float* wts,
                          int heads, int N, int d, int B, int km_k, int iters,
                          int32_t* dev_status, cudaStream_t s);
cudaError_t launch_importance_tc(const float* wts, float* p, int heads, int n_rows, int nqb,
                                 int km, int n_sub, int N, int U, float scale,
                                 const CUtensorMap& ch,
                                 const CUtensorMap& cl, const CUtensorMap& kh,
                                 const CUtensorMap& kl, int32_t* dev_status, cudaStream_t s);
cudaError_t launch_sip_sample(const float* p, int rows, int n_sub, int m, uint64_t seed,
                              int32_t* idx, float* logw, int32_t* cnt, int cap,
                              int32_t* required_cap, int32_t* dev_status, cudaStream_t s);

// Self-test of the bounded wait (selftest.cu).
cudaError_t launch_index_check_selftest(int32_t* buf, int n, int index, int32_t* dev_status,
                                        cudaStream_t s);
cudaError_t launch_bounded_wait_selftest(uint64_t limit_ns, int32_t* dev_status,
                                         int32_t* waited_ok, cudaStream_t s);

}  // namespace sta
