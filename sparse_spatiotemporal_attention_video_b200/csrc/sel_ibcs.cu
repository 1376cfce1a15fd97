// sel_ibcs.cu -- intra-block query clustering, block importance and
// inclusion-probability sampling of key/value sub-blocks.
//
// "AB-Attention speeds up video diffusion transformers up to 2.23x, no
// training", method paragraph and Key facts: importance of key/value blocks
// is estimated by clustering the queries of each query block (no token
// permutation); blocks are sampled in proportion to the estimate and every
// kept block is reweighted by its inverse inclusion probability, so that one
// pass gives an estimate of dense attention; small sampled blocks are packed
// into full tensor-core tiles.  The page gives no formulas; the
// importance-sampled workload fixes k = 4 centroids, 5 iterations, 128-query
// blocks, 16-key sub-blocks, ~10% of sub-blocks per query block and a Philox
// stream per (seed, head, query block).  Steps, in that order:
//
//  1. Kbar_j = mean of the keys of sub-block j (n_j = its true count);
//     block_means in sel_pool.cu.
//  2. k-means on the n_b queries of a block: centroid c starts at the query
//     with local offset floor(c * n_b / k); one iteration assigns each query
//     to the nearest centroid in squared L2 distance (ties to the lower
//     centroid index) and moves each centroid to the mean of its members (an
//     empty cluster keeps its centroid); n_c = member counts of the last
//     assignment.                                           (kmeans_kernel)
//  3. p_j = sum_c (n_c / n_b) softmax_j(c_c . Kbar_j * scale + ln n_j)
//                          (importance_tc_kernel in sel_importance.cu)
//  4. m = ceil(frac * n_sub) (host); pi_j = min(1, lambda p_j) with
//     sum_j pi_j = m by water filling: repeatedly set lambda = (m - #capped)
//     / (sum of uncapped p) and cap every j with lambda p_j >= 1.
//  5. keep j iff u_j < pi_j, u_j = (x_j >> 8) * 2^-24, x_j = word j%4 of
//     Philox4x32-10(key = seed, counter = (j/4, 0, head*n_qb + qb, 0));
//     logw_j = -ln pi_j.                                  (sip_sample_kernel)
//
// Precision: the sampling decisions compare u_j with pi_j, so p is computed
// to fp32 accuracy: the importance scores on the tensor cores from fp16
// hi/lo operand splits (sel_importance.cu), fp64 sums of the softmax
// normaliser and of the water-filling sums.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"

namespace sta {
namespace {

// ------------------------------------------------------------------ k-means
// One CTA of 512 threads per (head, query block).  Assignment: thread
// (g, r) = (tid / 128, tid % 128) sums the squared distance of query r over
// dimension quarter g; the four partials are added in order g = 0..3.
// Update: thread (g, r) sums dimension r over queries [32g, 32g+32) per
// cluster; the four partials are added in order.  Rows of the staged block
// have an odd stride (D+1 floats), so the 32 lanes of a warp (consecutive r)
// hit distinct banks.
constexpr int kKmThreads = 512;
constexpr int kKmRows = 128;  // largest query block

template <int D, int KM>
__global__ void __launch_bounds__(kKmThreads) kmeans_kernel(
    const __nv_bfloat16* __restrict__ q, int N, int B, int nqb, int iters,
    float* __restrict__ cent, float* __restrict__ wts) {
  constexpr int QS = D + 1;
  constexpr int DQ = D / 4;  // dimensions per quarter
  extern __shared__ float km_smem[];
  float* sq = km_smem;                       // [128][QS]
  float* sc = sq + kKmRows * QS;             // [KM][D]
  float* part = sc + KM * D;                 // [4][128][KM] distances / [4][KM][D] sums
  int* sassign = reinterpret_cast<int*>(part + 4 * kKmRows * KM);  // [128]
  int* pcount = sassign + kKmRows;           // [4][KM]
  __shared__ int scount[KM];
  const int row = blockIdx.x;  // head * nqb + qb
  const int head = row / nqb;
  const int qb = row - head * nqb;
  const int q0 = qb * B;
  const int nb = min(B, N - q0);
  const int g = threadIdx.x / kKmRows;
  const int r = threadIdx.x - g * kKmRows;
  const __nv_bfloat16* qh = q + (static_cast<size_t>(head) * N + q0) * D;
  // stage the block as fp32 (rows >= nb are never read)
  for (int i = threadIdx.x; i < nb * D / 8; i += kKmThreads) {
    const int rr = (i * 8) / D;
    const int c = i * 8 - rr * D;
    const uint4 v = __ldcs(reinterpret_cast<const uint4*>(qh) + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      sq[rr * QS + c + 2 * t] = __uint_as_float(w[t] << 16);
      sq[rr * QS + c + 2 * t + 1] = __uint_as_float(w[t] & 0xffff0000u);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < KM * D; i += kKmThreads) {
    const int c = i / D, col = i - c * D;
    sc[i] = sq[((c * nb) / KM) * QS + col];
  }
  __syncthreads();
  for (int it = 0; it < iters; ++it) {
    // assignment: partial squared distances over one quarter of the dims
    if (r < nb) {
      float d2[KM];
#pragma unroll
      for (int c = 0; c < KM; ++c) d2[c] = 0.f;
#pragma unroll 8
      for (int i = 0; i < DQ; ++i) {
        const int col = g * DQ + i;
        const float x = sq[r * QS + col];
#pragma unroll
        for (int c = 0; c < KM; ++c) {
          const float t = x - sc[c * D + col];
          d2[c] = fmaf(t, t, d2[c]);
        }
      }
#pragma unroll
      for (int c = 0; c < KM; ++c) part[(g * kKmRows + r) * KM + c] = d2[c];
    }
    __syncthreads();
    if (g == 0 && r < nb) {
      int best = 0;
      float bd = 0.f;
#pragma unroll
      for (int c = 0; c < KM; ++c) {
        float d = part[r * KM + c];
#pragma unroll
        for (int gg = 1; gg < 4; ++gg) d += part[(gg * kKmRows + r) * KM + c];
        if (c == 0 || d < bd) {
          bd = d;
          best = c;
        }
      }
      sassign[r] = best;
    }
    __syncthreads();
    // update: partial member sums of dimension r over one quarter of the queries
    if (r < D) {
      float acc[KM];
      int n[KM];
#pragma unroll
      for (int c = 0; c < KM; ++c) {
        acc[c] = 0.f;
        n[c] = 0;
      }
      const int t1 = min(nb, (g + 1) * (kKmRows / 4));
      for (int t = g * (kKmRows / 4); t < t1; ++t) {
        const int as = sassign[t];
        const float x = sq[t * QS + r];
#pragma unroll
        for (int c = 0; c < KM; ++c) {
          if (as == c) {
            acc[c] += x;
            ++n[c];
          }
        }
      }
#pragma unroll
      for (int c = 0; c < KM; ++c) part[(g * KM + c) * D + r] = acc[c];
      if (r == 0) {
#pragma unroll
        for (int c = 0; c < KM; ++c) pcount[g * KM + c] = n[c];
      }
    }
    __syncthreads();
    if (g == 0 && r < D) {
#pragma unroll
      for (int c = 0; c < KM; ++c) {
        const int n = pcount[c] + pcount[KM + c] + pcount[2 * KM + c] + pcount[3 * KM + c];
        float acc = part[c * D + r];
#pragma unroll
        for (int gg = 1; gg < 4; ++gg) acc += part[(gg * KM + c) * D + r];
        if (n > 0) sc[c * D + r] = acc / static_cast<float>(n);
        if (r == 0) scount[c] = n;
      }
    }
    __syncthreads();
  }
  float* co = cent + static_cast<size_t>(row) * KM * D;
  for (int i = threadIdx.x; i < KM * D; i += kKmThreads) co[i] = sc[i];
  if (threadIdx.x < KM) {
    const int n = iters > 0 ? scount[threadIdx.x] : 0;
    wts[static_cast<size_t>(row) * KM + threadIdx.x] =
        static_cast<float>(n) / static_cast<float>(nb);
  }
}

// ------------------------------------------------------------ SIP sampling
constexpr int kSipThreads = 256;
constexpr int kSipWarps = kSipThreads / 32;

// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as
// easy as 1, 2, 3", SC'11): ten rounds of two 32x32->64-bit multiplies whose
// high halves are XOR-ed with the other two counter words and the key, with
// the key bumped by two Weyl constants between rounds.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
  constexpr uint32_t kM0 = 0xD2511F53u, kM1 = 0xCD9E8D57u;
  constexpr uint32_t kW0 = 0x9E3779B9u, kW1 = 0xBB67AE85u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t hi0 = __umulhi(kM0, c.x), lo0 = kM0 * c.x;
    const uint32_t hi1 = __umulhi(kM1, c.z), lo1 = kM1 * c.z;
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
    k0 += kW0;
    k1 += kW1;
  }
  return c;
}

__device__ __forceinline__ double block_sum_d(double v, double* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double t = 0.0;
#pragma unroll
  for (int w = 0; w < kSipWarps; ++w) t += red[w];
  __syncthreads();
  return t;
}

__device__ __forceinline__ int block_sum_i(int v, int* red, int& excl) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  if (lane == 31) red[warp] = inc;
  __syncthreads();
  int before = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kSipWarps; ++w) {
    if (w < warp) before += red[w];
    tot += red[w];
  }
  excl = before + inc - v;
  __syncthreads();
  return tot;
}

__global__ void __launch_bounds__(kSipThreads) sip_sample_kernel(
    const float* __restrict__ p, int n_sub, int m, uint32_t seed_lo, uint32_t seed_hi,
    int32_t* __restrict__ idx, float* __restrict__ logw, int32_t* __restrict__ cnt, int cap,
    int32_t* required_cap, int32_t* dev_status) {
  extern __shared__ float sip_smem[];
  float* sp = sip_smem;                                    // [n_sub]
  uint8_t* capped = reinterpret_cast<uint8_t*>(sp + n_sub);  // [n_sub]
  __shared__ double redd[kSipWarps];
  __shared__ int redi[kSipWarps];
  const int row = blockIdx.x;  // head * nqb + qb
  const float* pr = p + static_cast<size_t>(row) * ((n_sub + 3) & ~3);  // 16-byte rows
  for (int j = threadIdx.x; j < n_sub; j += kSipThreads) {
    sp[j] = __ldcs(pr + j);
    capped[j] = 0;
  }
  __syncthreads();
  // water filling
  int ncap = 0;
  double lam = 0.0;
  for (int iter = 0; iter <= n_sub; ++iter) {
    double part = 0.0;
    for (int j = threadIdx.x; j < n_sub; j += kSipThreads)
      if (!capped[j]) part += static_cast<double>(sp[j]);
    const double rest = block_sum_d(part, redd);
    if (!(rest > 0.0)) break;
    lam = static_cast<double>(m - ncap) / rest;
    int newc = 0;
    for (int j = threadIdx.x; j < n_sub; j += kSipThreads) {
      if (!capped[j] && lam * static_cast<double>(sp[j]) >= 1.0) {
        capped[j] = 1;
        ++newc;
      }
    }
    int dummy;
    const int tot = block_sum_i(newc, redi, dummy);
    if (tot == 0) break;
    ncap += tot;
  }
  // Poisson sampling over a contiguous chunk per thread, ascending output
  const int chunk = (n_sub + kSipThreads - 1) / kSipThreads;
  const int j_lo = min(n_sub, threadIdx.x * chunk);
  const int j_hi = min(n_sub, j_lo + chunk);
  auto pi_of = [&](int j) -> double {
    if (capped[j]) return 1.0;
    return fmin(1.0, lam * static_cast<double>(sp[j]));
  };
  auto keep_of = [&](int j, uint4& words, int& group) -> bool {
    if ((j >> 2) != group) {
      group = j >> 2;
      words = philox4x32_10(make_uint4(static_cast<uint32_t>(group), 0u,
                                       static_cast<uint32_t>(row), 0u),
                            seed_lo, seed_hi);
    }
    const uint32_t x = (j & 3) == 0 ? words.x : (j & 3) == 1 ? words.y : (j & 3) == 2 ? words.z : words.w;
    const double u = static_cast<double>(x >> 8) * (1.0 / 16777216.0);
    return u < pi_of(j);
  };
  int mine = 0;
  {
    uint4 w = make_uint4(0, 0, 0, 0);
    int g = -1;
    for (int j = j_lo; j < j_hi; ++j) mine += keep_of(j, w, g) ? 1 : 0;
  }
  int before;
  const int total = block_sum_i(mine, redi, before);
  {
    uint4 w = make_uint4(0, 0, 0, 0);
    int g = -1;
    int pos = before;
    int32_t* out = idx + static_cast<size_t>(row) * cap;
    float* lw = logw ? logw + static_cast<size_t>(row) * cap : nullptr;
    for (int j = j_lo; j < j_hi; ++j) {
      if (keep_of(j, w, g)) {
        if (pos < cap) {
          out[pos] = j;
          if (lw) lw[pos] = static_cast<float>(-log(pi_of(j)));
        }
        ++pos;
      }
    }
  }
  if (threadIdx.x == 0) {
    cnt[row] = min(total, cap);
    if (required_cap) atomicMax(required_cap, total);
    if (total > cap) raise_status(dev_status, STA_DEV_CAPACITY);
  }
}

template <int D, int KM>
cudaError_t launch_kmeans_t(const __nv_bfloat16* q, float* cent, float* wts, int heads, int N,
                            int B, int iters, cudaStream_t s) {
  const int nqb = (N + B - 1) / B;
  const size_t km_smem =
      sizeof(float) * (static_cast<size_t>(kKmRows) * (D + 1) + KM * D + 4 * kKmRows * KM) +
      sizeof(int) * (kKmRows + 4 * KM);
  cudaError_t e = set_dyn_smem<kmeans_kernel<D, KM>>(static_cast<int>(km_smem));
  if (e != cudaSuccess) return e;
  kmeans_kernel<D, KM><<<heads * nqb, kKmThreads, km_smem, s>>>(q, N, B, nqb, iters, cent, wts);
  return cudaGetLastError();
}

}  // namespace

int ibcs_max_subblocks() { return static_cast<int>((200 * 1024) / (sizeof(float) + 1)); }

cudaError_t launch_kmeans(const __nv_bfloat16* q, float* cent, float* wts, int heads, int N,
                          int d, int B, int km_k, int iters, cudaStream_t s) {
#define STA_KM_CASE(DD, KK) \
  if (d == DD && km_k == KK) return launch_kmeans_t<DD, KK>(q, cent, wts, heads, N, B, iters, s);
  STA_KM_CASE(128, 4)
  STA_KM_CASE(128, 2)
  STA_KM_CASE(128, 1)
  STA_KM_CASE(128, 8)
  STA_KM_CASE(64, 4)
  STA_KM_CASE(64, 2)
  STA_KM_CASE(64, 1)
  STA_KM_CASE(64, 8)
#undef STA_KM_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_sip_sample(const float* p, int rows, int n_sub, int m, uint64_t seed,
                              int32_t* idx, float* logw, int32_t* cnt, int cap,
                              int32_t* required_cap, int32_t* dev_status, cudaStream_t s) {
  const size_t smem = static_cast<size_t>(n_sub) * (sizeof(float) + 1);
  cudaError_t e = set_dyn_smem<sip_sample_kernel>(static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  sip_sample_kernel<<<rows, kSipThreads, smem, s>>>(
      p, n_sub, m, static_cast<uint32_t>(seed & 0xffffffffu), static_cast<uint32_t>(seed >> 32),
      idx, logw, cnt, cap, required_cap, dev_status);
  return cudaGetLastError();
}

}  // namespace sta
