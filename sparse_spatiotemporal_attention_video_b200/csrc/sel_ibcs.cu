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
//                                                       (importance_kernel)
//  4. m = ceil(frac * n_sub) (host); pi_j = min(1, lambda p_j) with
//     sum_j pi_j = m by water filling: repeatedly set lambda = (m - #capped)
//     / (sum of uncapped p) and cap every j with lambda p_j >= 1.
//  5. keep j iff u_j < pi_j, u_j = (x_j >> 8) * 2^-24, x_j = word j%4 of
//     Philox4x32-10(key = seed, counter = (j/4, 0, head*n_qb + qb, 0));
//     logw_j = -ln pi_j.                                  (sip_sample_kernel)
//
// Precision: the sampling decisions compare u_j with pi_j, so p is computed
// to fp32 accuracy (fp32 scores on the FMA pipe, fp64 sums of the softmax
// normaliser and of the water-filling sums) rather than on the bf16 tensor
// cores, whose logit error would move pi by ~1e-3.
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

// --------------------------------------------------------------- importance
// CTA tile: 128 centroid rows (128/KM query blocks of one head) x 128
// sub-blocks, K = D in chunks of 32.  The centroid tile is staged once,
// transposed (As[k][row]); sub-block-mean chunks are double-buffered through
// registers (Bs[k][j]).  Thread (ty, tx) owns rows ty*8..ty*8+7 (8/KM whole
// query blocks) and columns tx*4..tx*4+3 and 64+tx*4..64+tx*4+3 (two float4
// reads per k that fall on distinct banks).  One sweep over all sub-blocks
// stores the scores z_cj and keeps an online max and an fp64 sum of exp per
// row; the 16 threads of a row group then merge them into (w_c / Z_c, M_c).
// Storing z (4 B per score, written and read once) is cheaper than a second
// sweep of the GEMM; sip_sample_kernel forms p from it.
constexpr int kImpThreads = 256;
constexpr int kImpRows = 128;
constexpr int kImpCols = 128;
constexpr int kImpKc = 32;
constexpr int kImpPad = 4;
constexpr int kImpStride = kImpCols + kImpPad;

template <int D>
constexpr size_t imp_smem_bytes() {
  return sizeof(float) * (static_cast<size_t>(D) * (kImpRows + kImpPad) +
                          2ull * kImpKc * kImpStride);
}

template <int D, int KM>
__global__ void __launch_bounds__(kImpThreads, 1) importance_kernel(
    const float* __restrict__ cent, const float* __restrict__ wts,
    const float* __restrict__ kbar, int nqb, int n_sub, int N, int U, float scale,
    float* __restrict__ zout, float* __restrict__ stats) {
  static_assert(8 % KM == 0, "centroids per query block must divide 8");
  constexpr int NCH = D / kImpKc;
  extern __shared__ float4 imp_smem4[];
  float* As = reinterpret_cast<float*>(imp_smem4);     // [D][kImpRows + pad]
  float* Bs = As + D * (kImpRows + kImpPad);           // [2][kImpKc][kImpStride]
  const int head = blockIdx.y;
  const int row0 = blockIdx.x * kImpRows;              // first centroid row (per head)
  const int n_rows = nqb * KM;
  const int tid = threadIdx.x;
  const int ty = tid >> 4, tx = tid & 15;
  const float* ch = cent + static_cast<size_t>(head) * n_rows * D;
  const float* kh = kbar + static_cast<size_t>(head) * n_sub * D;

  for (int i = tid; i < kImpRows * (D / 4); i += kImpThreads) {
    const int r = i % kImpRows, k4 = i / kImpRows;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (row0 + r < n_rows) v = reinterpret_cast<const float4*>(ch + static_cast<size_t>(row0 + r) * D)[k4];
    As[(4 * k4 + 0) * (kImpRows + kImpPad) + r] = v.x;
    As[(4 * k4 + 1) * (kImpRows + kImpPad) + r] = v.y;
    As[(4 * k4 + 2) * (kImpRows + kImpPad) + r] = v.z;
    As[(4 * k4 + 3) * (kImpRows + kImpPad) + r] = v.w;
  }

  // B chunk loader: 32 k x 128 j = 1024 float4, 4 per thread
  auto load_chunk = [&](int j0, int ch_i, float4 (&reg)[4]) {
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int i = tid + t * kImpThreads;
      const int j = i % kImpCols, k4 = i / kImpCols;
      reg[t] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j0 + j < n_sub)
        reg[t] = reinterpret_cast<const float4*>(kh + static_cast<size_t>(j0 + j) * D +
                                                 ch_i * kImpKc)[k4];
    }
  };
  auto store_chunk = [&](int buf, const float4 (&reg)[4]) {
    float* b = Bs + buf * kImpKc * kImpStride;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int i = tid + t * kImpThreads;
      const int j = i % kImpCols, k4 = i / kImpCols;
      b[(4 * k4 + 0) * kImpStride + j] = reg[t].x;
      b[(4 * k4 + 1) * kImpStride + j] = reg[t].y;
      b[(4 * k4 + 2) * kImpStride + j] = reg[t].z;
      b[(4 * k4 + 3) * kImpStride + j] = reg[t].w;
    }
  };
  // z[8][8] = scores of this thread's rows x columns for sub-block tile j0
  auto tile_scores = [&](int j0, float (&z)[8][8]) {
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
      for (int b = 0; b < 8; ++b) z[a][b] = 0.f;
    float4 reg[4];
    load_chunk(j0, 0, reg);
    __syncthreads();  // previous users of Bs are done
    store_chunk(0, reg);
    __syncthreads();
#pragma unroll 1
    for (int c = 0; c < NCH; ++c) {
      if (c + 1 < NCH) load_chunk(j0, c + 1, reg);
      const float* b = Bs + (c & 1) * kImpKc * kImpStride;
#pragma unroll 4
      for (int kk = 0; kk < kImpKc; ++kk) {
        const float* ar = As + (c * kImpKc + kk) * (kImpRows + kImpPad) + ty * 8;
        const float4 a0 = *reinterpret_cast<const float4*>(ar);
        const float4 a1 = *reinterpret_cast<const float4*>(ar + 4);
        const float4 b0 = *reinterpret_cast<const float4*>(b + kk * kImpStride + tx * 4);
        const float4 b1 = *reinterpret_cast<const float4*>(b + kk * kImpStride + 64 + tx * 4);
        const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int x = 0; x < 8; ++x)
#pragma unroll
          for (int y = 0; y < 8; ++y) z[x][y] = fmaf(av[x], bv[y], z[x][y]);
      }
      if (c + 1 < NCH) {
        store_chunk((c + 1) & 1, reg);
        __syncthreads();
      }
    }
    // scale and ln n_j; columns past n_sub are -inf
#pragma unroll
    for (int y = 0; y < 8; ++y) {
      const int j = j0 + (y < 4 ? tx * 4 + y : 64 + tx * 4 + (y - 4));
      float lnn = -INFINITY;
      if (j < n_sub) lnn = logf(static_cast<float>(min(U, N - j * U)));
#pragma unroll
      for (int x = 0; x < 8; ++x) z[x][y] = (j < n_sub) ? fmaf(z[x][y], scale, lnn) : -INFINITY;
    }
  };

  // ---- sweep 1: per-row max and sum of exp
  float m[8];
  double s[8];
#pragma unroll
  for (int x = 0; x < 8; ++x) {
    m[x] = -INFINITY;
    s[x] = 0.0;
  }
  for (int j0 = 0; j0 < n_sub; j0 += kImpCols) {
    float z[8][8];
    tile_scores(j0, z);
    // keep the scores: p is formed from them once the normalisers are known
#pragma unroll
    for (int x = 0; x < 8; ++x) {
      const int r = row0 + ty * 8 + x;
      if (r >= n_rows) continue;
      float* zr = zout + (static_cast<size_t>(head) * n_rows + r) * n_sub + j0;
#pragma unroll
      for (int y = 0; y < 8; ++y) {
        const int c = y < 4 ? tx * 4 + y : 64 + tx * 4 + (y - 4);
        if (j0 + c < n_sub) zr[c] = z[x][y];
      }
    }
#pragma unroll
    for (int x = 0; x < 8; ++x) {
      float t = z[x][0];
#pragma unroll
      for (int y = 1; y < 8; ++y) t = fmaxf(t, z[x][y]);
      if (t == -INFINITY) continue;
      if (t > m[x]) {
        if (m[x] != -INFINITY) s[x] *= exp(static_cast<double>(m[x]) - static_cast<double>(t));
        m[x] = t;
      }
      double acc = 0.0;
#pragma unroll
      for (int y = 0; y < 8; ++y) acc += static_cast<double>(expf(z[x][y] - m[x]));
      s[x] += acc;
    }
  }
  // merge the 16 column groups of each row group (lanes with equal ty)
#pragma unroll
  for (int x = 0; x < 8; ++x) {
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) {
      const float mo = __shfl_xor_sync(0xffffffffu, m[x], o);
      const double so = __shfl_xor_sync(0xffffffffu, s[x], o);
      const float mn = fmaxf(m[x], mo);
      double acc = 0.0;
      if (m[x] != -INFINITY) acc += s[x] * exp(static_cast<double>(m[x]) - static_cast<double>(mn));
      if (mo != -INFINITY) acc += so * exp(static_cast<double>(mo) - static_cast<double>(mn));
      m[x] = mn;
      s[x] = acc;
    }
  }
  // per centroid row: coefficient w_c / Z_c and the maximum M_c
  if (tx == 0) {
#pragma unroll
    for (int x = 0; x < 8; ++x) {
      const int r = row0 + ty * 8 + x;
      if (r >= n_rows) continue;
      float coef = 0.f;
      if (s[x] > 0.0)
        coef = static_cast<float>(
            static_cast<double>(__ldg(wts + static_cast<size_t>(head) * n_rows + r)) / s[x]);
      float2* st = reinterpret_cast<float2*>(stats) + static_cast<size_t>(head) * n_rows + r;
      *st = make_float2(coef, m[x]);
    }
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

template <int KM>
__global__ void __launch_bounds__(kSipThreads) sip_sample_kernel(
    const float* __restrict__ z, const float* __restrict__ stats, int n_sub, int m,
    uint32_t seed_lo, uint32_t seed_hi, int32_t* __restrict__ idx, float* __restrict__ logw,
    int32_t* __restrict__ cnt, int cap, int32_t* required_cap, int32_t* dev_status) {
  extern __shared__ float sip_smem[];
  float* sp = sip_smem;                                    // [n_sub]
  uint8_t* capped = reinterpret_cast<uint8_t*>(sp + n_sub);  // [n_sub]
  __shared__ double redd[kSipWarps];
  __shared__ int redi[kSipWarps];
  __shared__ float2 cs[KM];
  const int row = blockIdx.x;  // head * nqb + qb
  if (threadIdx.x < KM)
    cs[threadIdx.x] = reinterpret_cast<const float2*>(stats)[static_cast<size_t>(row) * KM + threadIdx.x];
  __syncthreads();
  // p_j = sum_c (w_c / Z_c) exp(z_cj - M_c), centroids in order; the scores
  // of four j per thread are loaded before any is used
  const float* zr = z + static_cast<size_t>(row) * KM * n_sub;
  for (int j0 = threadIdx.x; j0 < n_sub; j0 += 4 * kSipThreads) {
    float zv[4][KM];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = j0 + u * kSipThreads;
#pragma unroll
      for (int c = 0; c < KM; ++c)
        zv[u][c] = j < n_sub ? __ldcs(zr + static_cast<size_t>(c) * n_sub + j) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = j0 + u * kSipThreads;
      if (j >= n_sub) break;
      float acc = 0.f;
#pragma unroll
      for (int c = 0; c < KM; ++c) {
        const float2 cm = cs[c];
        if (cm.x != 0.f) acc = fmaf(cm.x, expf(zv[u][c] - cm.y), acc);
      }
      sp[j] = acc;
      capped[j] = 0;
    }
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
cudaError_t launch_ibcs_t(const __nv_bfloat16* q, const float* kbar, float* cent, float* wts,
                          float* z, float* stats, int heads, int N, int B, int U, int iters, int m,
                          uint64_t seed, float scale, int32_t* idx, float* logw, int32_t* cnt,
                          int cap, int32_t* required_cap, int32_t* dev_status, cudaStream_t s) {
  const int nqb = (N + B - 1) / B;
  const int n_sub = (N + U - 1) / U;
  const size_t km_smem =
      sizeof(float) * (static_cast<size_t>(kKmRows) * (D + 1) + KM * D + 4 * kKmRows * KM) +
      sizeof(int) * (kKmRows + 4 * KM);
  cudaError_t e = set_dyn_smem<kmeans_kernel<D, KM>>(static_cast<int>(km_smem));
  if (e != cudaSuccess) return e;
  kmeans_kernel<D, KM><<<heads * nqb, kKmThreads, km_smem, s>>>(q, N, B, nqb, iters, cent, wts);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  const size_t imp_smem = imp_smem_bytes<D>();
  e = set_dyn_smem<importance_kernel<D, KM>>(static_cast<int>(imp_smem));
  if (e != cudaSuccess) return e;
  dim3 gi((nqb * KM + kImpRows - 1) / kImpRows, heads);
  importance_kernel<D, KM><<<gi, kImpThreads, imp_smem, s>>>(cent, wts, kbar, nqb, n_sub, N, U,
                                                             scale, z, stats);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  const size_t sip_smem = static_cast<size_t>(n_sub) * (sizeof(float) + 1);
  e = set_dyn_smem<sip_sample_kernel<KM>>(static_cast<int>(sip_smem));
  if (e != cudaSuccess) return e;
  sip_sample_kernel<KM><<<heads * nqb, kSipThreads, sip_smem, s>>>(
      z, stats, n_sub, m, static_cast<uint32_t>(seed & 0xffffffffu), static_cast<uint32_t>(seed >> 32),
      idx, logw, cnt, cap, required_cap, dev_status);
  return cudaGetLastError();
}

}  // namespace

int ibcs_max_subblocks() { return static_cast<int>((200 * 1024) / (sizeof(float) + 1)); }

cudaError_t launch_ibcs_sip(const __nv_bfloat16* q, const float* kbar, float* cent, float* wts,
                            float* z, float* stats, int heads, int N, int d, int B, int U, int km_k, int iters,
                            int m, uint64_t seed, float scale, int32_t* idx, float* logw,
                            int32_t* cnt, int cap, int32_t* required_cap, int32_t* dev_status,
                            cudaStream_t s) {
#define STA_IBCS_CASE(DD, KK)                                                                   \
  if (d == DD && km_k == KK)                                                                    \
    return launch_ibcs_t<DD, KK>(q, kbar, cent, wts, z, stats, heads, N, B, U, iters, m, seed, scale, \
                                 idx, logw, cnt, cap, required_cap, dev_status, s);
  STA_IBCS_CASE(128, 4)
  STA_IBCS_CASE(128, 2)
  STA_IBCS_CASE(128, 1)
  STA_IBCS_CASE(128, 8)
  STA_IBCS_CASE(64, 4)
  STA_IBCS_CASE(64, 2)
  STA_IBCS_CASE(64, 1)
  STA_IBCS_CASE(64, 8)
#undef STA_IBCS_CASE
  return cudaErrorInvalidValue;
}

}  // namespace sta
