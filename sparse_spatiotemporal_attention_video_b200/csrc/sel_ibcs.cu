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
// One CTA of 256 threads per (head, query block), the block staged once in
// shared memory as bf16 (exact) and its fp32 values held in registers.
//
// Assignment: thread (g, p) = (tid / 64, tid % 64) owns queries p and p + 64
// over dimension quarter g (32 fp32 values each, in registers for all
// iterations) and forms the partial squared distances to every centroid
// with packed f32x2 subtract / fused multiply-add (even and odd dimensions
// in the two halves, added at the end); the centroids are read from shared
// memory as warp-uniform 16-byte broadcasts.  The four quarter partials of a
// query are added in order g = 0..3 and the argmin keeps the lower index on
// ties.  The direct form sum (x - c)^2 is kept (not |c|^2 - 2 x.c): it has no
// cancellation, so the distance carries fp32 rounding relative to itself.
//
// Update: the members are counting-sorted by cluster (warp ballots), so the
// member sum of dimension pair j over cluster c is a run of plain adds; thread
// (s, j) = (tid / 64, tid % 64) sums dimension pair j over the quarter s of
// the sorted members, cut at cluster boundaries, and the four partials are
// added in order.  An empty cluster keeps its centroid.
constexpr int kKmThreads = 256;
constexpr int kKmRows = 128;           // largest query block
constexpr int kKmRowPitch = 128 + 8;   // bf16 per staged row (272 B: conflict-free 16 B reads)

template <int KM>
struct KmSmem {
  __nv_bfloat16 q[kKmRows * kKmRowPitch];  // staged block, rows >= nb zero
  float negc[KM * 128];                    // -centroid
  float part[4 * KM * kKmRows];            // [g][c][r] distances / [s][c][dim] sums
  int perm[kKmRows];                       // members sorted by cluster
  int wcount[4][KM];                       // per-warp member counts (warps 0-3)
  int start[KM + 1];                       // first sorted position of each cluster
};

template <int KM>
__global__ void __launch_bounds__(kKmThreads, KM >= 8 ? 1 : 2) kmeans_kernel(
    const __nv_bfloat16* __restrict__ q, int N, int B, int nqb, int iters,
    float* __restrict__ cent, float* __restrict__ wts) {
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
  // registers: queries p and p + 64, dimensions [32g, 32g + 32) as 16 pairs
  const int g = tid >> 6, p = tid & 63;
  float2 x[2][16];
#pragma unroll
  for (int qi = 0; qi < 2; ++qi) {
#pragma unroll
    for (int v8 = 0; v8 < 4; ++v8) {
      const uint4 w =
          *reinterpret_cast<const uint4*>(&sm.q[(p + 64 * qi) * kKmRowPitch + 32 * g + 8 * v8]);
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int t = 0; t < 4; ++t)
        x[qi][4 * v8 + t] = make_float2(__uint_as_float(ww[t] << 16),
                                        __uint_as_float(ww[t] & 0xffff0000u));
    }
  }
  __syncthreads();

  for (int it = 0; it < iters; ++it) {
    // ---- assignment: partial distances over quarter g
    {
      float2 acc[2][KM];
#pragma unroll
      for (int qi = 0; qi < 2; ++qi)
#pragma unroll
        for (int c = 0; c < KM; ++c) acc[qi][c] = make_float2(0.f, 0.f);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
#pragma unroll
        for (int c = 0; c < KM; ++c) {
          const float4 nc = *reinterpret_cast<const float4*>(&sm.negc[c * D + 32 * g + 4 * i]);
          const float2 n0 = make_float2(nc.x, nc.y), n1 = make_float2(nc.z, nc.w);
#pragma unroll
          for (int qi = 0; qi < 2; ++qi) {
            const float2 t0 = __fadd2_rn(x[qi][2 * i], n0);
            acc[qi][c] = __ffma2_rn(t0, t0, acc[qi][c]);
            const float2 t1 = __fadd2_rn(x[qi][2 * i + 1], n1);
            acc[qi][c] = __ffma2_rn(t1, t1, acc[qi][c]);
          }
        }
      }
#pragma unroll
      for (int qi = 0; qi < 2; ++qi)
#pragma unroll
        for (int c = 0; c < KM; ++c)
          sm.part[(g * KM + c) * kKmRows + p + 64 * qi] = acc[qi][c].x + acc[qi][c].y;
    }
    __syncthreads();
    // ---- argmin and counting sort (warps 0-3: thread r = query r)
    int best = -1, rank = 0;
    if (tid < kKmRows) {
      const int r = tid;
      if (r < nb) {
        float bd = 0.f;
#pragma unroll
        for (int c = 0; c < KM; ++c) {
          float d = sm.part[c * kKmRows + r];
#pragma unroll
          for (int gg = 1; gg < 4; ++gg) d += sm.part[(gg * KM + c) * kKmRows + r];
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
    if (tid < kKmRows) {
      if (best >= 0) {
        int pos = rank;
        for (int c = 0; c < best; ++c)
#pragma unroll
          for (int w = 0; w < 4; ++w) pos += sm.wcount[w][c];
        for (int w = 0; w < warp; ++w) pos += sm.wcount[w][best];
        sm.perm[pos] = tid;
      }
      if (tid <= KM) {
        int s0 = 0;
        for (int c = 0; c < tid; ++c)
#pragma unroll
          for (int w = 0; w < 4; ++w) s0 += sm.wcount[w][c];
        sm.start[tid] = s0;
      }
    }
    __syncthreads();
    // ---- update: member sums of dimension pair j over sorted quarter s
    {
      const int s = tid >> 6, j = tid & 63;
      const int lo = (s * nb) >> 2, hi = ((s + 1) * nb) >> 2;
#pragma unroll
      for (int c = 0; c < KM; ++c) {
        const int a = max(lo, sm.start[c]), b = min(hi, sm.start[c + 1]);
        float2 acc = make_float2(0.f, 0.f);
        for (int t = a; t < b; ++t) {
          const uint32_t w =
              *reinterpret_cast<const uint32_t*>(&sm.q[sm.perm[t] * kKmRowPitch + 2 * j]);
          acc = __fadd2_rn(acc, make_float2(__uint_as_float(w << 16),
                                            __uint_as_float(w & 0xffff0000u)));
        }
        *reinterpret_cast<float2*>(&sm.part[(s * KM + c) * D + 2 * j]) = acc;
      }
    }
    __syncthreads();
    for (int i = tid; i < KM * D; i += kKmThreads) {
      const int c = i / D, col = i - c * D;
      const int n = sm.start[c + 1] - sm.start[c];
      if (n > 0) {
        float acc = sm.part[c * D + col];
#pragma unroll
        for (int s = 1; s < 4; ++s) acc += sm.part[(s * KM + c) * D + col];
        sm.negc[i] = -(acc / static_cast<float>(n));
      }
    }
    __syncthreads();
  }
  float* co = cent + static_cast<size_t>(row) * KM * D;
  for (int i = tid; i < KM * D; i += kKmThreads) co[i] = -sm.negc[i];
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

// One CTA per (head, query block) row of p.  Shared memory: p of the row
// (ld = n_sub rounded up to 4 floats) and one flag byte per sub-block
// (bit 0 capped, bit 1 kept).
//  - Water filling: each round caps every uncapped j with lambda p_j >= 1
//    and, in the same pass, sums (fp64) the p of the sub-blocks that stay
//    uncapped, which is the next round's denominator.
//  - Draws: thread t takes the Philox groups t, t + T, ... two at a time and
//    sets the kept bit where u_j < pi_j; pi_j = 1 for capped j, else
//    min(1, lambda p_j) in fp64.
//  - Output: thread t owns a contiguous chunk of sub-blocks (a multiple of 4),
//    counts its kept bits, and an exclusive block scan places its ids in
//    ascending order, with logw = -ln pi.
__global__ void __launch_bounds__(kSipThreads) sip_sample_kernel(
    const float* __restrict__ p, int n_sub, int m, uint32_t seed_lo, uint32_t seed_hi,
    int32_t* __restrict__ idx, float* __restrict__ logw, int32_t* __restrict__ cnt, int cap,
    int32_t* required_cap, int32_t* dev_status) {
  extern __shared__ __align__(16) float sip_smem[];
  const int ld = (n_sub + 3) & ~3;
  float* sp = sip_smem;                                          // [ld]
  uint8_t* flag = reinterpret_cast<uint8_t*>(sp + ld);           // [ld]
  __shared__ double redd[kSipWarps];
  __shared__ int redi[kSipWarps];
  const int tid = threadIdx.x;
  const int row = blockIdx.x;  // head * nqb + qb
  const float4* pr = reinterpret_cast<const float4*>(p + static_cast<size_t>(row) * ld);
  double part = 0.0;
  for (int i = tid; i < ld / 4; i += kSipThreads) {
    const float4 v = __ldcs(pr + i);  // padding columns hold 0
    reinterpret_cast<float4*>(sp)[i] = v;
    reinterpret_cast<uint32_t*>(flag)[i] = 0u;
    part += (static_cast<double>(v.x) + static_cast<double>(v.y)) +
            (static_cast<double>(v.z) + static_cast<double>(v.w));
  }
  double rest = block_sum_d(part, redd);  // its barriers also publish sp / flag
  // water filling
  int ncap = 0;
  double lam = 0.0;
  for (int round = 0; round <= n_sub && rest > 0.0; ++round) {
    lam = static_cast<double>(m - ncap) / rest;
    int newc = 0;
    part = 0.0;
    for (int j = tid; j < n_sub; j += kSipThreads) {
      if (!flag[j]) {
        const double pj = static_cast<double>(sp[j]);
        if (lam * pj >= 1.0) {
          flag[j] = 1;
          ++newc;
        } else {
          part += pj;
        }
      }
    }
    int dummy;
    const int tot = block_sum_i(newc, redi, dummy);
    if (tot == 0) break;
    ncap += tot;
    rest = block_sum_d(part, redd);
  }
  auto pi_of = [&](int j) -> double {
    if (flag[j] & 1) return 1.0;
    return fmin(1.0, lam * static_cast<double>(sp[j]));
  };
  // draws
  const int n_grp = ld / 4;
  const uint32_t ctr = static_cast<uint32_t>(row);
  auto mark = [&](int g, uint4 w) {
    const uint32_t x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = 4 * g + e;
      if (j < n_sub && static_cast<double>(x[e] >> 8) * (1.0 / 16777216.0) < pi_of(j))
        flag[j] |= 2;
    }
  };
  for (int g = tid; g < n_grp; g += 2 * kSipThreads) {
    const int g2 = g + kSipThreads;
    uint4 a = make_uint4(static_cast<uint32_t>(g), 0u, ctr, 0u);
    uint4 b = make_uint4(static_cast<uint32_t>(g2), 0u, ctr, 0u);
    philox4x32_10_x2(a, b, seed_lo, seed_hi);
    mark(g, a);
    if (g2 < n_grp) mark(g2, b);
  }
  __syncthreads();
  // ascending output
  const int chunk = ((n_grp + kSipThreads - 1) / kSipThreads) * 4;
  const int j_lo = min(ld, tid * chunk);
  const int j_hi = min(ld, j_lo + chunk);
  int mine = 0;
  for (int j = j_lo; j < j_hi; j += 4)
    mine += __popc(reinterpret_cast<const uint32_t*>(flag)[j >> 2] & 0x02020202u);
  int before;
  const int total = block_sum_i(mine, redi, before);
  int pos = before;
  int32_t* out = idx + static_cast<size_t>(row) * cap;
  float* lw = logw ? logw + static_cast<size_t>(row) * cap : nullptr;
  for (int j = j_lo; j < j_hi; ++j) {
    if (flag[j] & 2) {
      if (pos < cap) {
        out[pos] = j;
        if (lw) lw[pos] = static_cast<float>(-log(pi_of(j)));
      }
      ++pos;
    }
  }
  if (tid == 0) {
    cnt[row] = min(total, cap);
    if (required_cap) atomicMax(required_cap, total);
    if (total > cap) raise_status(dev_status, STA_DEV_CAPACITY);
  }
}

template <int KM>
cudaError_t launch_kmeans_t(const __nv_bfloat16* q, float* cent, float* wts, int heads, int N,
                            int B, int iters, cudaStream_t s) {
  const int nqb = (N + B - 1) / B;
  const int smem = static_cast<int>(sizeof(KmSmem<KM>));
  cudaError_t e = set_dyn_smem<kmeans_kernel<KM>>(smem);
  if (e != cudaSuccess) return e;
  kmeans_kernel<KM><<<heads * nqb, kKmThreads, smem, s>>>(q, N, B, nqb, iters, cent, wts);
  return cudaGetLastError();
}

}  // namespace

int ibcs_max_subblocks() { return static_cast<int>((200 * 1024) / (sizeof(float) + 1)); }

cudaError_t launch_kmeans(const __nv_bfloat16* q, float* cent, float* wts, int heads, int N,
                          int d, int B, int km_k, int iters, cudaStream_t s) {
#define STA_KM_CASE(KK) \
  if (km_k == KK) return launch_kmeans_t<KK>(q, cent, wts, heads, N, B, iters, s);
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
  const size_t smem = static_cast<size_t>((n_sub + 3) & ~3) * (sizeof(float) + 1);
  cudaError_t e = set_dyn_smem<sip_sample_kernel>(static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  sip_sample_kernel<<<rows, kSipThreads, smem, s>>>(
      p, n_sub, m, static_cast<uint32_t>(seed & 0xffffffffu), static_cast<uint32_t>(seed >> 32),
      idx, logw, cnt, cap, required_cap, dev_status);
  return cudaGetLastError();
}

}  // namespace sta
