// sel_entropy.cu -- pooled entropy -> radius -> Chebyshev block lists.
//
// "Token Radius Attention for Efficient Video Generation", 2. Methodology:
// Insight I (the entropy of a query's attention distribution says how
// diffuse it is, so diffuse queries need a larger budget), Insight II (the
// budget becomes the radius of a query-centred spatiotemporal neighbourhood)
// and The TRA Pipeline (entropy -> budget -> radius -> block-sparse mask).
// The block form computed here (pooled blocks, a linear map, a 3D Chebyshev
// cube of block cells) is the one the entropy-radius workload states:
//
//   s_bc = Qbar_b . Kbar_c * scale,  p_b = softmax_c(s_b.)    (all key blocks)
//   H_b  = -sum_c p_bc ln p_bc = ln Z - (sum_c e_c (s_bc - m)) / Z,
//          e_c = exp(s_bc - m), Z = sum_c e_c, m = max_c s_bc
//   r_b  = clamp(floor(fl32(alpha + fl32(beta * fl32(H_b)))), r_lo, r_hi)
//   keep key block c iff max(|df|, |dcell_h|, |dcell_w|) <= r_b, where a
//   block's cell is (f, h / tile_h, w / tile_w) of its centre token
//   c = b*B + (len_b - 1) / 2.
//
// Scores and exponentials are fp32; Z and the weighted sum are accumulated
// in fp64 and the entropy is rounded to fp32 once, so the fp32 radius
// decision sees the entropy to within a few fp32 ulps.  The two fp32 steps of
// the radius map use explicit round-to-nearest operations (no FMA
// contraction), as the decision is defined on them.
//
// Two kernels.  entropy_scores_kernel is a tiled fp32 GEMM per head:
// 64 x 64 tiles of s = Qbar Kbar^T * scale, the pooled rows staged in shared
// memory (rows padded to D+4 floats; thread (ty, tx) owns rows ty+16i and
// columns tx+16j, so float4 reads of neighbouring threads hit distinct banks),
// each score accumulated over the d dimensions in order.  entropy_rows_kernel
// gives one warp to each query block: it stages the row's scores and the
// block cells in shared memory, reduces the scores to the entropy, maps it
// to the radius and compacts the kept key blocks with warp ballots in
// ascending order.
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"

namespace sta {
namespace {

constexpr int kEntThreads = 256;
constexpr int kScoreTile = 64;  // query x key blocks per scores CTA
constexpr int kScoreT = kScoreTile / 16;  // rows (and columns) per thread
constexpr int kRowWarps = 8;    // query blocks per rows CTA

struct EntArgs {
  const float* scores;  // [heads][nb][nb]
  int heads, nb, F, H, W, B;
  float alpha, beta;
  int r_lo, r_hi, tile_h, tile_w;
  int32_t* idx;
  int32_t* cnt;
  int cap;
  int32_t* required_cap;
  float* entropy;   // [heads][nb] or null
  int32_t* radius;  // [heads][nb] or null
  int32_t* dev_status;
};

__device__ __forceinline__ void block_cell(int b, int B, int N, int H, int W, int tile_h,
                                           int tile_w, int& cf, int& ch, int& cw) {
  const int lo = b * B;
  const int len = min(B, N - lo);
  const int c = lo + (len - 1) / 2;
  const int S = H * W;
  cf = c / S;
  const int rem = c - cf * S;
  const int h = rem / W;
  ch = h / tile_h;
  cw = (rem - h * W) / tile_w;
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// s[h][b][c] = (Qbar_b . Kbar_c) * scale for a 64 x 64 tile of (b, c).
template <int D>
__global__ void __launch_bounds__(kEntThreads) entropy_scores_kernel(
    const float* __restrict__ qbar, const float* __restrict__ kbar, int nb, float scale,
    float* __restrict__ scores) {
  constexpr int KS = D + 4;
  extern __shared__ float4 ssm4[];
  float* sa = reinterpret_cast<float*>(ssm4);  // [64][KS] query rows
  float* sb = sa + kScoreTile * KS;              // [64][KS] key rows
  const int head = blockIdx.z;
  const int b0 = blockIdx.y * kScoreTile, c0 = blockIdx.x * kScoreTile;
  const float* qh = qbar + static_cast<size_t>(head) * nb * D;
  const float* kh = kbar + static_cast<size_t>(head) * nb * D;
  constexpr int PER = kScoreTile * D / 4 / kEntThreads;  // float4 per thread per operand
  float4 va[PER], vb[PER];
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int i = threadIdx.x + u * kEntThreads;
    const int r = (i * 4) / D, col = i * 4 - r * D;
    va[u] = b0 + r < nb ? __ldg(reinterpret_cast<const float4*>(qh + static_cast<size_t>(b0 + r) * D + col))
                        : make_float4(0.f, 0.f, 0.f, 0.f);
    vb[u] = c0 + r < nb ? __ldg(reinterpret_cast<const float4*>(kh + static_cast<size_t>(c0 + r) * D + col))
                        : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int i = threadIdx.x + u * kEntThreads;
    const int r = (i * 4) / D, col = i * 4 - r * D;
    *reinterpret_cast<float4*>(sa + r * KS + col) = va[u];
    *reinterpret_cast<float4*>(sb + r * KS + col) = vb[u];
  }
  __syncthreads();
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
  float acc[kScoreT][kScoreT];
#pragma unroll
  for (int i = 0; i < kScoreT; ++i)
#pragma unroll
    for (int j = 0; j < kScoreT; ++j) acc[i][j] = 0.f;
#pragma unroll 8
  for (int k = 0; k < D; k += 4) {
    float4 x[kScoreT], y[kScoreT];
#pragma unroll
    for (int i = 0; i < kScoreT; ++i)
      x[i] = *reinterpret_cast<const float4*>(sa + (ty + 16 * i) * KS + k);
#pragma unroll
    for (int j = 0; j < kScoreT; ++j)
      y[j] = *reinterpret_cast<const float4*>(sb + (tx + 16 * j) * KS + k);
#pragma unroll
    for (int i = 0; i < kScoreT; ++i)
#pragma unroll
      for (int j = 0; j < kScoreT; ++j) {
        acc[i][j] = fmaf(x[i].x, y[j].x, acc[i][j]);
        acc[i][j] = fmaf(x[i].y, y[j].y, acc[i][j]);
        acc[i][j] = fmaf(x[i].z, y[j].z, acc[i][j]);
        acc[i][j] = fmaf(x[i].w, y[j].w, acc[i][j]);
      }
  }
#pragma unroll
  for (int i = 0; i < kScoreT; ++i) {
    const int b = b0 + ty + 16 * i;
    if (b >= nb) continue;
    float* out = scores + (static_cast<size_t>(head) * nb + b) * nb;
#pragma unroll
    for (int j = 0; j < kScoreT; ++j) {
      const int c = c0 + tx + 16 * j;
      if (c < nb) out[c] = acc[i][j] * scale;
    }
  }
}

// One warp per query block: entropy of softmax over its scores, radius,
// Chebyshev list.  Cells are packed as f << 20 | cell_h << 10 | cell_w.
__global__ void __launch_bounds__(kRowWarps * 32) entropy_rows_kernel(const EntArgs a) {
  extern __shared__ float rsm[];
  const int nb = a.nb;
  float* ss = rsm;                                             // [8][nb]
  int* scell = reinterpret_cast<int*>(ss + kRowWarps * nb);    // [nb]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = a.F * a.H * a.W;
  for (int b = threadIdx.x; b < nb; b += kRowWarps * 32) {
    int cf, ch, cw;
    block_cell(b, a.B, N, a.H, a.W, a.tile_h, a.tile_w, cf, ch, cw);
    scell[b] = (cf << 20) | (ch << 10) | cw;
  }
  const int row = blockIdx.x * kRowWarps + warp;  // head*nb + qb (< 2^31: checked on the host)
  const bool live = row < a.heads * nb;
  float* s = ss + warp * nb;
  if (live) {
    const float* src = a.scores + static_cast<size_t>(row) * nb;
    for (int c = lane; c < nb; c += 32) s[c] = __ldg(src + c);
  }
  __syncthreads();
  if (!live) return;
  const int qb = row % nb;
  float m = -INFINITY;
  for (int c = lane; c < nb; c += 32) m = fmaxf(m, s[c]);
  m = warp_max_f(m);
  double z = 0.0, wsum = 0.0;
  for (int c = lane; c < nb; c += 32) {
    const float t = s[c] - m;
    const float e = expf(t);
    z += static_cast<double>(e);
    wsum += static_cast<double>(e) * static_cast<double>(t);
  }
  z = warp_sum_d(z);
  wsum = warp_sum_d(wsum);
  const float h32 = static_cast<float>(log(z) - wsum / z);
  const float t = __fadd_rn(a.alpha, __fmul_rn(a.beta, h32));
  const float tf = floorf(t);
  int r;
  if (!(tf == tf)) r = a.r_lo;  // NaN entropy: smallest radius
  else if (tf <= static_cast<float>(a.r_lo)) r = a.r_lo;
  else if (tf >= static_cast<float>(a.r_hi)) r = a.r_hi;
  else r = static_cast<int>(tf);

  const int qc = scell[qb];
  const int qf = qc >> 20, qh = (qc >> 10) & 1023, qw = qc & 1023;
  int32_t* out = a.idx + static_cast<size_t>(row) * a.cap;
  int total = 0;
  for (int c0 = 0; c0 < nb; c0 += 32) {
    const int kb = c0 + lane;
    bool keep = false;
    if (kb < nb) {
      const int kc = scell[kb];
      const int kf = kc >> 20, kh = (kc >> 10) & 1023, kw = kc & 1023;
      keep = max(abs(kf - qf), max(abs(kh - qh), abs(kw - qw))) <= r;
    }
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    const int pos = total + __popc(bal & ((1u << lane) - 1u));
    if (keep && pos < a.cap && dcheck(kb < nb, a.dev_status)) out[pos] = kb;
    total += __popc(bal);
  }
  if (lane == 0) {
    a.cnt[row] = min(total, a.cap);
    if (a.required_cap) atomicMax(a.required_cap, total);
    if (total > a.cap) raise_status(a.dev_status, STA_DEV_CAPACITY);
    if (a.entropy) a.entropy[row] = h32;
    if (a.radius) a.radius[row] = r;
  }
}

size_t rows_smem(int nb) {
  return sizeof(float) * static_cast<size_t>(kRowWarps) * nb + sizeof(int) * static_cast<size_t>(nb);
}

template <int D>
cudaError_t launch_scores_t(const float* qbar, const float* kbar, int heads, int nb, float scale,
                            float* scores, cudaStream_t s) {
  const int smem = static_cast<int>(sizeof(float) * 2 * kScoreTile * (D + 4));
  cudaError_t e = set_dyn_smem<entropy_scores_kernel<D>>(smem);
  if (e != cudaSuccess) return e;
  const int nt = (nb + kScoreTile - 1) / kScoreTile;
  entropy_scores_kernel<D><<<dim3(nt, nt, heads), kEntThreads, smem, s>>>(qbar, kbar, nb, scale,
                                                                          scores);
  return cudaGetLastError();
}

}  // namespace

int entropy_max_blocks(int d) {
  (void)d;
  // the rows kernel stages 8 score rows and the cells of all blocks
  return static_cast<int>((227 * 1024) / (sizeof(float) * kRowWarps + sizeof(int)));
}

cudaError_t launch_entropy_lists(const float* qbar, const float* kbar, float* scores, int heads,
                                 int F, int H, int W, int d, int B, float scale, float alpha,
                                 float beta, int r_lo, int r_hi, int tile_h, int tile_w,
                                 int32_t* idx, int32_t* cnt, int cap, int32_t* required_cap,
                                 float* entropy, int32_t* radius, int32_t* dev_status,
                                 cudaStream_t s) {
  const int N = F * H * W;
  const int nb = (N + B - 1) / B;
  cudaError_t e = d == 128   ? launch_scores_t<128>(qbar, kbar, heads, nb, scale, scores, s)
                  : d == 64 ? launch_scores_t<64>(qbar, kbar, heads, nb, scale, scores, s)
                            : cudaErrorInvalidValue;
  if (e != cudaSuccess) return e;
  EntArgs a;
  a.scores = scores;
  a.heads = heads;
  a.nb = nb;
  a.F = F;
  a.H = H;
  a.W = W;
  a.B = B;
  a.alpha = alpha;
  a.beta = beta;
  a.r_lo = r_lo;
  a.r_hi = r_hi;
  a.tile_h = tile_h;
  a.tile_w = tile_w;
  a.idx = idx;
  a.cnt = cnt;
  a.cap = cap;
  a.required_cap = required_cap;
  a.entropy = entropy;
  a.radius = radius;
  a.dev_status = dev_status;
  const int smem = static_cast<int>(rows_smem(nb));
  e = set_dyn_smem<entropy_rows_kernel>(smem);
  if (e != cudaSuccess) return e;
  const long long rows = static_cast<long long>(heads) * nb;
  entropy_rows_kernel<<<static_cast<unsigned>((rows + kRowWarps - 1) / kRowWarps),
                        kRowWarps * 32, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace sta
