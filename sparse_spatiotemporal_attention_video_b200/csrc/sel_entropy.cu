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
// One CTA of 8 warps handles 8 query blocks of one head: pooled key blocks
// are staged in shared memory in chunks of 64 (rows padded to D+4 floats so
// that 32 lanes reading 32 different rows hit distinct banks), lane i scores
// key blocks i and i+32 of the chunk against the warp's query block, and the
// list is compacted with warp ballots in ascending key-block order.
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"

namespace sta {
namespace {

constexpr int kEntWarps = 8;
constexpr int kEntThreads = kEntWarps * 32;
constexpr int kEntChunk = 64;

struct EntArgs {
  const float* qbar;  // [heads][nb][D]
  const float* kbar;  // [heads][nb][D]
  int heads, nb, F, H, W, B;
  float scale, alpha, beta;
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

template <int D>
__global__ void __launch_bounds__(kEntThreads) entropy_lists_kernel(const EntArgs a) {
  constexpr int KS = D + 4;  // padded row stride of the staged key blocks
  extern __shared__ float4 smem4[];
  float* sm = reinterpret_cast<float*>(smem4);
  float* sq = sm;                                  // [8][D]
  float* sk = sq + kEntWarps * D;                  // [64][KS]
  float* ss = sk + kEntChunk * KS;                 // [8][nb]
  const int head = blockIdx.y;
  const int qb0 = blockIdx.x * kEntWarps;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb = a.nb;
  const float* qh = a.qbar + static_cast<size_t>(head) * nb * D;
  const float* kh = a.kbar + static_cast<size_t>(head) * nb * D;

  for (int i = threadIdx.x; i < kEntWarps * D / 4; i += kEntThreads) {
    const int r = (i * 4) / D;
    const int qb = min(qb0 + r, nb - 1);
    reinterpret_cast<float4*>(sq)[i] =
        reinterpret_cast<const float4*>(qh + static_cast<size_t>(qb) * D)[(i * 4 - r * D) / 4];
  }
  for (int c0 = 0; c0 < nb; c0 += kEntChunk) {
    __syncthreads();
    for (int i = threadIdx.x; i < kEntChunk * D / 4; i += kEntThreads) {
      const int r = (i * 4) / D;
      const int col = i * 4 - r * D;
      const int kb = c0 + r;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (kb < nb) v = *reinterpret_cast<const float4*>(kh + static_cast<size_t>(kb) * D + col);
      *reinterpret_cast<float4*>(sk + r * KS + col) = v;
    }
    __syncthreads();
    const float4* qv = reinterpret_cast<const float4*>(sq + warp * D);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int r = lane + 32 * half;
      const float4* kv = reinterpret_cast<const float4*>(sk + r * KS);
      float acc = 0.f;
#pragma unroll 8
      for (int i = 0; i < D / 4; ++i) {
        const float4 x = qv[i], y = kv[i];
        acc = fmaf(x.x, y.x, acc);
        acc = fmaf(x.y, y.y, acc);
        acc = fmaf(x.z, y.z, acc);
        acc = fmaf(x.w, y.w, acc);
      }
      if (c0 + r < nb) ss[warp * nb + c0 + r] = acc * a.scale;
    }
  }
  __syncthreads();

  const int qb = qb0 + warp;
  if (qb >= nb) return;
  const float* s = ss + warp * nb;
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

  const int N = a.F * a.H * a.W;
  int qf, qh_, qw;
  block_cell(qb, a.B, N, a.H, a.W, a.tile_h, a.tile_w, qf, qh_, qw);
  const size_t row = static_cast<size_t>(head) * nb + qb;
  int32_t* out = a.idx + row * a.cap;
  int total = 0;
  for (int c0 = 0; c0 < nb; c0 += 32) {
    const int kb = c0 + lane;
    bool keep = false;
    if (kb < nb) {
      int kf, kh2, kw;
      block_cell(kb, a.B, N, a.H, a.W, a.tile_h, a.tile_w, kf, kh2, kw);
      const int dist = max(abs(kf - qf), max(abs(kh2 - qh_), abs(kw - qw)));
      keep = dist <= r;
    }
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    const int pos = total + __popc(bal & ((1u << lane) - 1u));
    if (keep && pos < a.cap) out[pos] = kb;
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

template <int D>
size_t ent_smem(int nb) {
  return sizeof(float) * (static_cast<size_t>(kEntWarps) * D + kEntChunk * (D + 4) +
                          static_cast<size_t>(kEntWarps) * nb);
}

template <int D>
cudaError_t launch_ent_t(const EntArgs& a, cudaStream_t s) {
  const size_t smem = ent_smem<D>(a.nb);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(entropy_lists_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 g((a.nb + kEntWarps - 1) / kEntWarps, a.heads);
  entropy_lists_kernel<D><<<g, kEntThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

int entropy_max_blocks(int d) {
  // key blocks whose scores fit the CTA's shared memory
  const size_t fixed = sizeof(float) * (static_cast<size_t>(kEntWarps) * d + kEntChunk * (d + 4));
  return static_cast<int>((227 * 1024 - fixed) / (sizeof(float) * kEntWarps));
}

cudaError_t launch_entropy_lists(const float* qbar, const float* kbar, int heads, int F, int H,
                                 int W, int d, int B, float scale, float alpha, float beta,
                                 int r_lo, int r_hi, int tile_h, int tile_w, int32_t* idx,
                                 int32_t* cnt, int cap, int32_t* required_cap, float* entropy,
                                 int32_t* radius, int32_t* dev_status, cudaStream_t s) {
  EntArgs a;
  a.qbar = qbar;
  a.kbar = kbar;
  a.heads = heads;
  a.F = F;
  a.H = H;
  a.W = W;
  a.B = B;
  const int N = F * H * W;
  a.nb = (N + B - 1) / B;
  a.scale = scale;
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
  if (d == 128) return launch_ent_t<128>(a, s);
  if (d == 64) return launch_ent_t<64>(a, s);
  return cudaErrorInvalidValue;
}

}  // namespace sta
