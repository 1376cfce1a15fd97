// sel_radial.cu -- static radial block lists.
//
// "Radial Attention to Accelerate Video Generation", The idea behind Radial
// Attention: a static mask keeps token pairs whose spatial distance is
// within a window that shrinks as the frame distance grows (O(N log N)
// pairs); the mask is shared by every head.  Window at frame distance df:
//   w(df) = S                                  if df <= full_df
//         = w0 >> floor(log2(df + w_off))       otherwise      (S = H*W)
// Tokens i, j are related iff |s_i - s_j| < w(|f_i - f_j|), s = h*W + w.
// Block pair (qb, kb) is kept iff some token pair in it is related: each
// block is a union of per-frame runs of flattened spatial indices, and two
// runs [a1, a2] (frame fa) and [b1, b2] (frame fb) contain a related pair
// iff max(0, b1 - a2, a1 - b2) < w(|fa - fb|).
//
// One CTA per query block; threads test key blocks in chunks, and a
// warp-ballot prefix sum writes the kept ids in ascending order.
#include <cuda_runtime.h>

#include "common.cuh"

namespace sta {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxRuns = 8;  // a block spans at most ceil(B/S)+1 frames

__device__ __forceinline__ int radial_window(int df, int S, int w0, int w_off, int full_df) {
  if (df <= full_df) return S;
  const int n = df + w_off;
  if (n < 1) return 0;
  const int e = 31 - __clz(n);
  return w0 >> e;
}

struct Runs {
  int n;
  int f[kMaxRuns], lo[kMaxRuns], hi[kMaxRuns];
};

__device__ __forceinline__ void block_runs(int b, int B, int N, int S, Runs& r) {
  const int t0 = b * B;
  const int t1 = min(t0 + B, N);  // exclusive
  r.n = 0;
  for (int t = t0; t < t1 && r.n < kMaxRuns;) {
    const int f = t / S;
    const int end = min(t1, (f + 1) * S);
    r.f[r.n] = f;
    r.lo[r.n] = t - f * S;
    r.hi[r.n] = end - 1 - f * S;
    ++r.n;
    t = end;
  }
}

__global__ void __launch_bounds__(kThreads) radial_lists_kernel(
    int F, int H, int W, int B, int w0, int w_off, int full_df, int32_t* __restrict__ idx,
    int32_t* __restrict__ cnt, int cap, int32_t* required_cap, int32_t* dev_status) {
  const int S = H * W;
  const int N = F * S;
  const int nb = (N + B - 1) / B;
  const int qb = blockIdx.x;
  __shared__ int warp_counts[kThreads / 32];
  __shared__ int running;
  Runs rq;
  block_runs(qb, B, N, S, rq);
  if (threadIdx.x == 0) running = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int base = 0; base < nb; base += kThreads) {
    const int kb = base + threadIdx.x;
    bool keep = false;
    if (kb < nb) {
      Runs rk;
      block_runs(kb, B, N, S, rk);
      for (int i = 0; i < rq.n && !keep; ++i) {
        for (int j = 0; j < rk.n && !keep; ++j) {
          const int gap = max(0, max(rk.lo[j] - rq.hi[i], rq.lo[i] - rk.hi[j]));
          const int df = abs(rq.f[i] - rk.f[j]);
          if (gap < radial_window(df, S, w0, w_off, full_df)) keep = true;
        }
      }
    }
    const unsigned ballot = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) warp_counts[warp] = __popc(ballot);
    __syncthreads();
    int before = running;
    for (int w = 0; w < warp; ++w) before += warp_counts[w];
    const int pos = before + __popc(ballot & ((1u << lane) - 1u));
    if (keep && pos < cap && dcheck(kb < nb && qb < nb, dev_status))
      idx[static_cast<size_t>(qb) * cap + pos] = kb;
    __syncthreads();
    if (threadIdx.x == 0) {
      int tot = 0;
      for (int w = 0; w < kThreads / 32; ++w) tot += warp_counts[w];
      running += tot;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const int total = running;
    cnt[qb] = min(total, cap);
    if (required_cap) atomicMax(required_cap, total);
    if (total > cap) raise_status(dev_status, STA_DEV_CAPACITY);
  }
}

}  // namespace

cudaError_t launch_radial_lists(int F, int H, int W, int B, int w0, int w_off, int full_df,
                                int32_t* idx, int32_t* cnt, int cap, int32_t* required_cap,
                                int32_t* dev_status, cudaStream_t stream) {
  const int N = F * H * W;
  const int nb = (N + B - 1) / B;
  radial_lists_kernel<<<nb, kThreads, 0, stream>>>(F, H, W, B, w0, w_off, full_df, idx, cnt, cap,
                                                  required_cap, dev_status);
  return cudaGetLastError();
}

}  // namespace sta
