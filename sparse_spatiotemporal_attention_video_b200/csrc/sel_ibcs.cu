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
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"

namespace sta {
namespace {

// ------------------------------------------------------------------ k-means
// One CTA of 128 threads per (head, query block); thread r owns query r.
//
// The block is staged once in shared memory as bf16 (exact), with a row
// pitch that makes each thread's 8-byte reads of its own row conflict-free.
// Assignment: thread r forms the squared distances to every centroid over
// the 128 dimensions itself (packed f32x2 subtract / fused multiply-add,
// even and odd dimensions in the two halves, added at the end; centroids are
// warp-uniform shared-memory broadcasts) and takes the argmin, ties to the
// lower index.  The direct form sum (x - c)^2 is kept (not |c|^2 - 2 x.c):
// it has no cancellation, so a distance carries fp32 rounding relative to
// itself.
// Update: the members are counting-sorted by cluster (warp ballots), then
// thread t sums dimension pair t % 64 over the members of clusters
// t / 64, t / 64 + 2, ... in sorted order (runs of plain adds) and writes the
// mean.  An empty cluster keeps its centroid.  Three barriers per iteration.
constexpr int kKmThreads = 128;
constexpr int kKmWarps = kKmThreads / 32;
constexpr int kKmRows = 128;           // largest query block
constexpr int kKmRowPitch = 128 + 8;   // bf16 per staged row (272 B: conflict-free 16 B reads)

template <int KM>
struct KmSmem {
  __nv_bfloat16 q[kKmRows * kKmRowPitch];  // staged block, rows >= nb zero
  float negc[KM * 128];                    // -centroid
  int perm[kKmRows];                       // members sorted by cluster
  int wcount[kKmWarps][KM];                // per-warp member counts
  int start[KM + 1];                       // first sorted position of each cluster
};

// The centroids are written as the fp16 pair hi = fp16(c), lo = fp16(c - hi),
// the tensor-core operands of the importance scores (a centroid beyond the
// fp16 range raises STA_DEV_RANGE).
template <int KM>
__global__ void __launch_bounds__(kKmThreads, KM >= 8 ? 4 : 6) kmeans_kernel(
    const __nv_bfloat16* __restrict__ q, int N, int B, int nqb, int iters,
    __half* __restrict__ cent_hi, __half* __restrict__ cent_lo, float* __restrict__ wts,
    int32_t* dev_status) {
  constexpr int D = 128;
  extern __shared__ __align__(16) uint8_t km_raw[];
  KmSmem<KM>& sm = *reinterpret_cast<KmSmem<KM>*>(km_raw);
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int row = blockIdx.x;  // head * nqb + qb
  const int head = row / nqb;
  const int qb = row - head * nqb;
  const int q0 = qb * B;
  const int nb = min(B, N - q0);
  const __nv_bfloat16* qh = q + (static_cast<size_t>(head) * N + q0) * D;

  // stage the block (16-byte loads, 16 per row); rows >= nb are zero
  for (int i = tid; i < kKmRows * (D / 8); i += kKmThreads) {
    const int r = i >> 4, c8 = (i & 15) * 8;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (r < nb) v = __ldcs(reinterpret_cast<const uint4*>(qh) + i);
    *reinterpret_cast<uint4*>(&sm.q[r * kKmRowPitch + c8]) = v;
  }
  __syncthreads();
  for (int i = tid; i < KM * D; i += kKmThreads) {
    const int c = i / D, col = i - c * D;
    sm.negc[i] = -__bfloat162float(sm.q[((c * nb) / KM) * kKmRowPitch + col]);
  }
  __syncthreads();
  const __nv_bfloat16* xrow = &sm.q[tid * kKmRowPitch];  // this thread's query

  for (int it = 0; it < iters; ++it) {
    // ---- assignment (thread = query) and per-warp cluster counts
    int best = -1, rank = 0;
    {
      float2 acc[KM];
#pragma unroll
      for (int c = 0; c < KM; ++c) acc[c] = make_float2(0.f, 0.f);
#pragma unroll
      for (int j4 = 0; j4 < D / 4; ++j4) {  // 4 dimensions per step
        const uint2 w = *reinterpret_cast<const uint2*>(xrow + 4 * j4);
        const float2 x0 = make_float2(__uint_as_float(w.x << 16),
                                      __uint_as_float(w.x & 0xffff0000u));
        const float2 x1 = make_float2(__uint_as_float(w.y << 16),
                                      __uint_as_float(w.y & 0xffff0000u));
#pragma unroll
        for (int c = 0; c < KM; ++c) {
          const float4 nc = *reinterpret_cast<const float4*>(&sm.negc[c * D + 4 * j4]);
          const float2 t0 = __fadd2_rn(x0, make_float2(nc.x, nc.y));
          acc[c] = __ffma2_rn(t0, t0, acc[c]);
          const float2 t1 = __fadd2_rn(x1, make_float2(nc.z, nc.w));
          acc[c] = __ffma2_rn(t1, t1, acc[c]);
        }
      }
      if (tid < nb) {
        float bd = 0.f;
#pragma unroll
        for (int c = 0; c < KM; ++c) {
          const float d = acc[c].x + acc[c].y;
          if (c == 0 || d < bd) {
            bd = d;
            best = c;
          }
        }
      }
#pragma unroll
      for (int c = 0; c < KM; ++c) {
        const unsigned bal = __ballot_sync(0xffffffffu, best == c);
        if (best == c) rank = __popc(bal & ((1u << lane) - 1u));
        if (lane == 0) sm.wcount[warp][c] = __popc(bal);
      }
    }
    __syncthreads();
    // ---- counting sort: members of cluster 0, then 1, ...
    if (best >= 0) {
      int pos = rank;
      for (int c = 0; c < best; ++c)
#pragma unroll
        for (int w = 0; w < kKmWarps; ++w) pos += sm.wcount[w][c];
      for (int w = 0; w < warp; ++w) pos += sm.wcount[w][best];
      sm.perm[pos] = tid;
    }
    if (tid <= KM) {
      int s0 = 0;
      for (int c = 0; c < tid; ++c)
#pragma unroll
        for (int w = 0; w < kKmWarps; ++w) s0 += sm.wcount[w][c];
      sm.start[tid] = s0;
    }
    __syncthreads();
    // ---- update: mean of the members, dimension pair j of cluster c
    {
      const int j = tid & 63;
#pragma unroll
      for (int c = tid >> 6; c < KM; c += kKmThreads / 64) {
        const int a = sm.start[c], b = sm.start[c + 1];
        if (b > a) {
          float2 acc = make_float2(0.f, 0.f);
          for (int t = a; t < b; ++t) {
            const uint32_t w =
                *reinterpret_cast<const uint32_t*>(&sm.q[sm.perm[t] * kKmRowPitch + 2 * j]);
            acc = __fadd2_rn(acc, make_float2(__uint_as_float(w << 16),
                                              __uint_as_float(w & 0xffff0000u)));
          }
          const float n = static_cast<float>(b - a);
          *reinterpret_cast<float2*>(&sm.negc[c * D + 2 * j]) = make_float2(-(acc.x / n),
                                                                            -(acc.y / n));
        }
      }
    }
    __syncthreads();
  }
  const size_t co = static_cast<size_t>(row) * KM * D;
  bool bad = false;
  for (int i = tid; i < KM * D; i += kKmThreads) {
    const float v = -sm.negc[i];
    const __half h = __float2half_rn(v);
    cent_hi[co + i] = h;
    cent_lo[co + i] = __float2half_rn(v - __half2float(h));
    if (!(fabsf(v) < 65504.f)) bad = true;
  }
  if (bad) raise_status(dev_status, STA_DEV_RANGE);
  if (tid < KM) {
    const int n = iters > 0 ? sm.start[tid + 1] - sm.start[tid] : 0;
    wts[static_cast<size_t>(row) * KM + tid] = static_cast<float>(n) / static_cast<float>(nb);
  }
}

// ------------------------------------------------------------ SIP sampling
constexpr int kSipThreads = 256;
constexpr int kSipWarps = kSipThreads / 32;

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

// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as
// easy as 1, 2, 3", SC'11): ten rounds of two 32x32->64-bit multiplies whose
// high halves are XOR-ed with the other two counter words and the key, with
// the key bumped by two Weyl constants between rounds.  Two counter blocks
// are advanced in lockstep (independent chains: the multiplies of one overlap
// the dependent steps of the other).
__device__ __forceinline__ void philox4x32_10_x2(uint4& a, uint4& b, uint32_t k0, uint32_t k1) {
  constexpr uint32_t kM0 = 0xD2511F53u, kM1 = 0xCD9E8D57u;
  constexpr uint32_t kW0 = 0x9E3779B9u, kW1 = 0xBB67AE85u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t ah0 = __umulhi(kM0, a.x), al0 = kM0 * a.x;
    const uint32_t ah1 = __umulhi(kM1, a.z), al1 = kM1 * a.z;
    const uint32_t bh0 = __umulhi(kM0, b.x), bl0 = kM0 * b.x;
    const uint32_t bh1 = __umulhi(kM1, b.z), bl1 = kM1 * b.z;
    a = make_uint4(ah1 ^ a.y ^ k0, al1, ah0 ^ a.w ^ k1, al0);
    b = make_uint4(bh1 ^ b.y ^ k0, bl1, bh0 ^ b.w ^ k1, bl0);
    k0 += kW0;
    k1 += kW1;
  }
}

// Sum of an int and a double over the CTA with one barrier: the partials go
// to slot `slot` of double-buffered shared arrays, so that consecutive calls
// alternate slots and a slot is rewritten only after every thread has passed
// the barrier of the call in between.
__device__ __forceinline__ void block_sum2(int& c, double& d, int slot, int (*rc)[kSipWarps],
                                           double (*rd)[kSipWarps]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    c += __shfl_xor_sync(0xffffffffu, c, o);
    d += __shfl_xor_sync(0xffffffffu, d, o);
  }
  if (lane == 0) {
    rc[slot][warp] = c;
    rd[slot][warp] = d;
  }
  __syncthreads();
  c = 0;
  d = 0.0;
#pragma unroll
  for (int w = 0; w < kSipWarps; ++w) {
    c += rc[slot][w];
    d += rd[slot][w];
  }
}

// One CTA per (head, query block) row of p.  Thread t owns the Philox groups
// (4 consecutive sub-blocks each) t, t + T, ..., t + (G-1) T and keeps their
// p in registers for every pass:
//  - Water filling: each round caps every uncapped j with lambda p_j >= 1
//    and, in the same pass, sums the p of the sub-blocks that stay uncapped,
//    the next round's denominator; one barrier per round.
//  - Draws: one Philox block per group (two groups in lockstep); j is kept
//    where u_j < pi_j, with pi_j = 1 for capped j, else min(1, lambda p_j).
//  - Output: ids in ascending order are groups in (k, t) order; an exclusive
//    block scan of the per-group kept counts over t, offset by the totals of
//    the earlier k, places them; logw = -ln pi.
// Precision: lambda and the sums across threads are fp64; a thread's own
// sums are pairwise in fp32 (relative error ~3e-7), and the per-element
// comparisons use lambda rounded to fp32.  A decision can then differ from
// an fp64 evaluation only where lambda p_j or u_j lies within ~1e-6 of the
// threshold, inside the 1e-5 band in which sampling decisions are reported
// as near-threshold; a cap decision that differs there moves pi_j by less
// than 1e-6 and lambda by far less.
template <int G>
__global__ void __launch_bounds__(kSipThreads, G <= 8 ? 4 : 1) sip_sample_kernel(
    const float* __restrict__ p, int n_sub, int m, uint32_t seed_lo, uint32_t seed_hi,
    int32_t* __restrict__ idx, float* __restrict__ logw, int32_t* __restrict__ cnt, int cap,
    int32_t* required_cap, int32_t* dev_status) {
  constexpr int MW = (4 * G + 31) / 32;  // words of the per-thread bit masks
  __shared__ int rc[2][kSipWarps];
  __shared__ double rd[2][kSipWarps];
  __shared__ int tab[kSipWarps][G];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row = blockIdx.x;  // head * nqb + qb
  const int ld = (n_sub + 3) & ~3;
  const int n_grp = ld / 4;
  const float4* pr = reinterpret_cast<const float4*>(p + static_cast<size_t>(row) * ld);
  float pv[4 * G];
#pragma unroll
  for (int k = 0; k < G; ++k) {
    const int g = tid + k * kSipThreads;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (g < n_grp) v = __ldcs(pr + g);  // padding columns hold 0
    pv[4 * k] = v.x;
    pv[4 * k + 1] = v.y;
    pv[4 * k + 2] = v.z;
    pv[4 * k + 3] = v.w;
  }
  // elements past n_sub (padding) are 0 and are never capped or kept
  uint32_t valid[MW];
#pragma unroll
  for (int w = 0; w < MW; ++w) valid[w] = 0u;
#pragma unroll
  for (int i = 0; i < 4 * G; ++i)
    if (4 * (tid + (i >> 2) * kSipThreads) + (i & 3) < n_sub) valid[i >> 5] |= 1u << (i & 31);
  // pairwise sum of the thread's uncapped p (capped elements masked out)
  auto thread_sum = [&](const uint32_t (&capped)[MW]) -> double {
    float t[4 * G];
#pragma unroll
    for (int i = 0; i < 4 * G; ++i) t[i] = (capped[i >> 5] >> (i & 31)) & 1u ? 0.f : pv[i];
#pragma unroll
    for (int w = 2 * G; w >= 1; w >>= 1)
#pragma unroll
      for (int i = 0; i < w; ++i) t[i] += t[i + w];
    return static_cast<double>(t[0]);
  };
  uint32_t capped[MW];
#pragma unroll
  for (int w = 0; w < MW; ++w) capped[w] = ~valid[w];  // padding counts as capped, not in any sum
  int slot = 0;
  int dummy = 0;
  double rest = thread_sum(capped);
  block_sum2(dummy, rest, slot, rc, rd);
  // water filling
  int ncap = 0;
  double lam = 0.0;
  for (int round = 0; round <= n_sub && rest > 0.0; ++round) {
    lam = static_cast<double>(m - ncap) / rest;
    const float lamf = static_cast<float>(lam);
    int newc = 0;
#pragma unroll
    for (int i = 0; i < 4 * G; ++i) {
      const uint32_t bit = 1u << (i & 31);
      if (!(capped[i >> 5] & bit) && lamf * pv[i] >= 1.f) {
        capped[i >> 5] |= bit;
        ++newc;
      }
    }
    double part = thread_sum(capped);
    slot ^= 1;
    block_sum2(newc, part, slot, rc, rd);
    if (newc == 0) break;
    ncap += newc;
    rest = part;
  }
  const float lamf = static_cast<float>(lam);
  // pi as fp32: 1 for capped, else min(1, lambda p)
  auto pi_of = [&](int i) -> float {
    if ((capped[i >> 5] >> (i & 31)) & 1u) return 1.f;
    return fminf(1.f, lamf * pv[i]);
  };
  // draws
  uint32_t kept[MW];
#pragma unroll
  for (int w = 0; w < MW; ++w) kept[w] = 0u;
  const uint32_t ctr = static_cast<uint32_t>(row);
#pragma unroll
  for (int k = 0; k < G; k += 2) {
    const int g0 = tid + k * kSipThreads, g1 = g0 + kSipThreads;
    uint4 a = make_uint4(static_cast<uint32_t>(g0), 0u, ctr, 0u);
    uint4 b = make_uint4(static_cast<uint32_t>(g1), 0u, ctr, 0u);
    if (g0 < n_grp) philox4x32_10_x2(a, b, seed_lo, seed_hi);
    const uint32_t xa[4] = {a.x, a.y, a.z, a.w}, xb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      // u = (x >> 8) * 2^-24, exact in fp32
      const int i0 = 4 * k + e, i1 = 4 * (k + 1) + e;
      if (((valid[i0 >> 5] >> (i0 & 31)) & 1u) &&
          static_cast<float>(xa[e] >> 8) * (1.f / 16777216.f) < pi_of(i0))
        kept[i0 >> 5] |= 1u << (i0 & 31);
      if (k + 1 < G && ((valid[i1 >> 5] >> (i1 & 31)) & 1u) &&
          static_cast<float>(xb[e] >> 8) * (1.f / 16777216.f) < pi_of(i1))
        kept[i1 >> 5] |= 1u << (i1 & 31);
    }
  }
  // ascending output: exclusive scan of the kept counts of group k over the
  // threads, offset by the totals of groups k' < k
  int inc[G];
#pragma unroll
  for (int k = 0; k < G; ++k) {
    inc[k] = __popc((kept[(4 * k) >> 5] >> ((4 * k) & 31)) & 0xfu);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, inc[k], o);
      if (lane >= o) inc[k] += t;
    }
    if (lane == 31) tab[warp][k] = inc[k];
  }
  __syncthreads();
  int base = 0;
  int32_t* out = idx + static_cast<size_t>(row) * cap;
  float* lw = logw ? logw + static_cast<size_t>(row) * cap : nullptr;
#pragma unroll
  for (int k = 0; k < G; ++k) {
    int before = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < kSipWarps; ++w) {
      const int c = tab[w][k];
      if (w < warp) before += c;
      tot += c;
    }
    const uint32_t bits = (kept[(4 * k) >> 5] >> ((4 * k) & 31)) & 0xfu;
    int pos = base + before + inc[k] - __popc(bits);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (bits & (1u << e)) {
        if (pos < cap && dcheck(4 * (tid + k * kSipThreads) + e < n_sub, dev_status)) {
          out[pos] = 4 * (tid + k * kSipThreads) + e;
          if (lw) lw[pos] = -logf(pi_of(4 * k + e));
        }
        ++pos;
      }
    }
    base += tot;
  }
  if (tid == 0) {
    cnt[row] = min(base, cap);
    if (required_cap) atomicMax(required_cap, base);
    if (base > cap) raise_status(dev_status, STA_DEV_CAPACITY);
  }
}

template <int KM>
cudaError_t launch_kmeans_t(const __nv_bfloat16* q, __half* cent_hi, __half* cent_lo, float* wts,
                            int heads, int N, int B, int iters, int32_t* dev_status,
                            cudaStream_t s) {
  const int nqb = (N + B - 1) / B;
  const int smem = static_cast<int>(sizeof(KmSmem<KM>));
  cudaError_t e = set_dyn_smem<kmeans_kernel<KM>>(smem);
  if (e != cudaSuccess) return e;
  kmeans_kernel<KM><<<heads * nqb, kKmThreads, smem, s>>>(q, N, B, nqb, iters, cent_hi, cent_lo,
                                                          wts, dev_status);
  return cudaGetLastError();
}

}  // namespace

// Sub-blocks per row the sampler holds in registers: 4 per group, up to 40
// groups per thread.
int ibcs_max_subblocks() { return 4 * 40 * kSipThreads; }

cudaError_t launch_kmeans(const __nv_bfloat16* q, __half* cent_hi, __half* cent_lo, float* wts,
                          int heads, int N, int d, int B, int km_k, int iters,
                          int32_t* dev_status, cudaStream_t s) {
#define STA_KM_CASE(KK)                                                                    \
  if (km_k == KK)                                                                          \
    return launch_kmeans_t<KK>(q, cent_hi, cent_lo, wts, heads, N, B, iters, dev_status, s);
  if (d != 128 || B < 1 || B > kKmRows) return cudaErrorInvalidValue;
  STA_KM_CASE(4)
  STA_KM_CASE(2)
  STA_KM_CASE(1)
  STA_KM_CASE(8)
#undef STA_KM_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_sip_sample(const float* p, int rows, int n_sub, int m, uint64_t seed,
                              int32_t* idx, float* logw, int32_t* cnt, int cap,
                              int32_t* required_cap, int32_t* dev_status, cudaStream_t s) {
  const int n_grp = (n_sub + 3) / 4;
  const uint32_t lo = static_cast<uint32_t>(seed & 0xffffffffu);
  const uint32_t hi = static_cast<uint32_t>(seed >> 32);
#define STA_SIP_CASE(GG)                                                                   \
  if (n_grp <= GG * kSipThreads) {                                                         \
    sip_sample_kernel<GG><<<rows, kSipThreads, 0, s>>>(p, n_sub, m, lo, hi, idx, logw, cnt, \
                                                       cap, required_cap, dev_status);     \
    return cudaGetLastError();                                                             \
  }
  STA_SIP_CASE(8)
  STA_SIP_CASE(16)
  STA_SIP_CASE(40)
#undef STA_SIP_CASE
  return cudaErrorInvalidValue;
}

}  // namespace sta
