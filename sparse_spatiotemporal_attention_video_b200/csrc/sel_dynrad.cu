// sel_dynrad.cu -- dual-mode adaptive selection inside the radial prior.
//
// "DynamicRad: Content-Adaptive Sparse Attention for Long Video Diffusion"
// (Abstract): adaptive selection grounded in a radial locality prior, in a
// static-ratio mode (speed first) and a dynamic-threshold mode (quality
// first).  With the static radial list of query block b as its candidates:
//
//   s_c = scale * Qbar_b . Kbar_c     (block means, fp32)
//   p_c = softmax over the candidates of s_c
//   rank: candidates ordered by s descending, ties to the lower block id
//   static-ratio rho:      keep rank < k, k = ceil(rho * n * (1 - 1e-6)) in [1, n]
//   dynamic-threshold th:  keep c iff the p mass of the ranks before c is
//                          below th (the shortest prefix whose mass reaches th)
//
// One CTA per (query block, head).  Each warp scores whole candidates: the
// lanes split d (4 or 2 floats each, so one Kbar row is one coalesced 512- or
// 256-byte read), four candidates are in flight per warp, and a butterfly
// reduction leaves the dot product in every lane.  The ranks come from a pairwise count
// (n <= kDynMaxCand candidates), the prefix masses from a double-precision
// scan of p in rank order, and the kept ids, already in ascending block
// order, are compacted with warp ballots and a block-wide scan.
#include <cuda_runtime.h>
#include <math.h>

#include <type_traits>

#include "common.cuh"

namespace sta {
namespace {

constexpr int kDynThreads = 256;
constexpr int kDynMaxCand = 1024;

struct DynArgs {
  const float* qbar;  // [heads][nb][d]
  const float* kbar;  // [heads][nb][d]
  const int32_t* prior_idx;  // [nb][prior_cap] radial candidates, ascending
  const int32_t* prior_cnt;  // [nb]
  int prior_cap;
  int heads, nb, d;
  float scale;
  int mode;  // 0 static ratio, 1 dynamic threshold
  float ratio, threshold;
  int32_t* idx;
  int32_t* cnt;
  int cap;
  int32_t* required_cap;
  int32_t* dev_status;
};

// Scores s_j of the n candidates into cand[] / sc[] (one warp per candidate).
template <int D>
__device__ __forceinline__ void dyn_scores(const DynArgs& a, const float* qb, const float* kh,
                                           int b, int n, int* cand, float* sc) {
  constexpr int V = D / 32;  // floats per lane: 4 (d = 128) or 2 (d = 64)
  constexpr int U = 4;       // candidates in flight per warp
  constexpr int kWarps = kDynThreads / 32;
  using Vec = typename std::conditional<V == 4, float4, float2>::type;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Vec qv = __ldg(reinterpret_cast<const Vec*>(qb) + lane);
  const int32_t* prow = a.prior_idx + static_cast<size_t>(b) * a.prior_cap;
  for (int j0 = warp * U; j0 < n; j0 += kWarps * U) {
    int c[U];
    Vec kv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {  // j0 + u < n is the same in every lane
      c[u] = 0;
      kv[u] = Vec{};
      if (j0 + u < n) {
        c[u] = __ldg(prow + j0 + u);
        kv[u] = __ldg(reinterpret_cast<const Vec*>(kh + static_cast<size_t>(c[u]) * D) + lane);
      }
    }
    float acc[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      acc[u] = qv.x * kv[u].x;
      acc[u] = fmaf(qv.y, kv[u].y, acc[u]);
      if constexpr (V == 4) {
        acc[u] = fmaf(qv.z, kv[u].z, acc[u]);
        acc[u] = fmaf(qv.w, kv[u].w, acc[u]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int u = 0; u < U; ++u) acc[u] += __shfl_xor_sync(0xffffffffu, acc[u], o);
    // lane u stores candidate j0 + u
    float mine = acc[0];
    int mc = c[0];
#pragma unroll
    for (int u = 1; u < U; ++u) {
      mine = lane == u ? acc[u] : mine;
      mc = lane == u ? c[u] : mc;
    }
    if (lane < U && j0 + lane < n) {
      cand[j0 + lane] = mc;
      sc[j0 + lane] = mine * a.scale;
    }
  }
}

__global__ void __launch_bounds__(kDynThreads) dynrad_lists_kernel(const DynArgs a) {
  __shared__ int cand[kDynMaxCand];
  __shared__ float sc[kDynMaxCand];
  __shared__ int rank[kDynMaxCand];
  __shared__ double scan[kDynMaxCand];
  __shared__ float red[kDynThreads / 32];
  __shared__ double redd[kDynThreads / 32];
  __shared__ int warp_tot[kDynThreads / 32];
  __shared__ int running;
  const int b = blockIdx.x, head = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = min(__ldg(a.prior_cnt + b), kDynMaxCand);
  const float* qb = a.qbar + (static_cast<size_t>(head) * a.nb + b) * a.d;
  const float* kh = a.kbar + static_cast<size_t>(head) * a.nb * a.d;
  if (threadIdx.x == 0) running = 0;
  // scores of the candidates
  if (a.d == 128)
    dyn_scores<128>(a, qb, kh, b, n, cand, sc);
  else
    dyn_scores<64>(a, qb, kh, b, n, cand, sc);
  __syncthreads();
  float lmax = -INFINITY;
  for (int j = threadIdx.x; j < n; j += kDynThreads) lmax = fmaxf(lmax, sc[j]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
  if (lane == 0) red[warp] = lmax;
  __syncthreads();
  float m = red[0];
  for (int w = 1; w < kDynThreads / 32; ++w) m = fmaxf(m, red[w]);
  // ranks (ties to the lower block id) and the softmax normaliser
  double lz = 0.0;
  for (int j = threadIdx.x; j < n; j += kDynThreads) {
    int r = 0;
    const float sj = sc[j];
    for (int i = 0; i < n; ++i) {
      const float si = sc[i];
      r += (si > sj || (si == sj && cand[i] < cand[j])) ? 1 : 0;
    }
    rank[j] = r;
    lz += static_cast<double>(expf(sj - m));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lz += __shfl_xor_sync(0xffffffffu, lz, o);
  __syncthreads();  // every warp is done with red[] before it is reused
  if (lane == 0) redd[warp] = lz;
  __syncthreads();
  double Z = 0.0;
  for (int w = 0; w < kDynThreads / 32; ++w) Z += redd[w];
  // p in rank order, then an inclusive scan (Hillis-Steele, doubles)
  for (int j = threadIdx.x; j < n; j += kDynThreads)
    scan[rank[j]] = static_cast<double>(expf(sc[j] - m)) / Z;
  __syncthreads();
  if (a.mode == 1) {
    for (int off = 1; off < n; off <<= 1) {
      double v[kDynMaxCand / kDynThreads];
      int q = 0;
      for (int i = threadIdx.x; i < n; i += kDynThreads, ++q)
        v[q] = i >= off ? scan[i - off] : 0.0;
      __syncthreads();
      q = 0;
      for (int i = threadIdx.x; i < n; i += kDynThreads, ++q) scan[i] += v[q];
      __syncthreads();
    }
  }
  int k = 0;
  if (a.mode == 0) {
    k = static_cast<int>(ceil(static_cast<double>(a.ratio) * n * (1.0 - 1e-6)));
    k = max(1, min(n, k));
  }
  // keep flags in candidate (ascending block) order, compacted
  const size_t row = static_cast<size_t>(head) * a.nb + b;
  int32_t* out = a.idx + row * a.cap;
  for (int c0 = 0; c0 < n; c0 += kDynThreads) {
    const int j = c0 + threadIdx.x;
    bool keep = false;
    if (j < n) {
      const int r = rank[j];
      if (a.mode == 0) {
        keep = r < k;
      } else {
        const double before = r > 0 ? scan[r - 1] : 0.0;
        keep = before < static_cast<double>(a.threshold);
      }
    }
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) warp_tot[warp] = __popc(bal);
    __syncthreads();
    int pos = running;
    for (int w = 0; w < warp; ++w) pos += warp_tot[w];
    pos += __popc(bal & ((1u << lane) - 1u));
    if (keep && pos < a.cap && dcheck(cand[j] >= 0 && cand[j] < a.nb, a.dev_status))
      out[pos] = cand[j];
    __syncthreads();
    if (threadIdx.x == 0)
      for (int w = 0; w < kDynThreads / 32; ++w) running += warp_tot[w];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const int total = running;
    a.cnt[row] = min(total, a.cap);
    if (a.required_cap) atomicMax(a.required_cap, total);
    if (total > a.cap) raise_status(a.dev_status, STA_DEV_CAPACITY);
  }
}

}  // namespace

int dynrad_max_candidates() { return kDynMaxCand; }

cudaError_t launch_dynrad_lists(const float* qbar, const float* kbar, const int32_t* prior_idx,
                                const int32_t* prior_cnt, int prior_cap, int heads, int nb, int d,
                                float scale, int mode, float ratio, float threshold, int32_t* idx,
                                int32_t* cnt, int cap, int32_t* required_cap,
                                int32_t* dev_status, cudaStream_t s) {
  DynArgs a;
  a.qbar = qbar;
  a.kbar = kbar;
  a.prior_idx = prior_idx;
  a.prior_cnt = prior_cnt;
  a.prior_cap = prior_cap;
  a.heads = heads;
  a.nb = nb;
  a.d = d;
  a.scale = scale;
  a.mode = mode;
  a.ratio = ratio;
  a.threshold = threshold;
  a.idx = idx;
  a.cnt = cnt;
  a.cap = cap;
  a.required_cap = required_cap;
  a.dev_status = dev_status;
  if (nb <= 0 || heads <= 0) return cudaSuccess;
  dynrad_lists_kernel<<<dim3(static_cast<unsigned>(nb), static_cast<unsigned>(heads)),
                        kDynThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace sta
