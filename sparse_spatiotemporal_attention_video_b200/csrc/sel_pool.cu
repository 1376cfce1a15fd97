// sel_pool.cu -- block means of a [heads][N][d] bf16 tensor (fp32 out).
//
// "Token Radius Attention for Efficient Video Generation", 2. Methodology,
// The TRA Pipeline: the selector works on pooled query and key blocks (the
// entropy-radius workload pools 128 x 128 blocks); "AB-Attention ...",
// method paragraph: importance is scored against small key sub-blocks
// (16 keys).  Both need xbar_b = mean of the rows of block b, over its true
// row count (the last block of a head may be partial).
//
// Bandwidth-bound: every input byte is read once.  A thread owns one 16-byte
// column group (8 bf16) and 8 rows of one block (rows phase, phase+P, ...,
// so a warp reads whole consecutive rows), keeps 8 fp32 partial sums, and
// the P partials of a column group are added in shared memory.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace sta {
namespace {

constexpr int kPoolThreads = 256;
constexpr int kRowsPerThread = 8;

template <int D, int U>
struct PoolShape {
  static constexpr int CG = D / 8;                    // 16-byte column groups per row
  static constexpr int P = U / kRowsPerThread;        // row phases per block
  static constexpr int TPU = CG * P;                  // threads per block
  static constexpr int UPC = kPoolThreads / TPU;      // blocks per CTA
  static_assert(U % kRowsPerThread == 0, "unit must be a multiple of 8 rows");
  static_assert(kPoolThreads % TPU == 0, "threads per unit must divide the CTA");
};

__device__ __forceinline__ void add_bf16x8(float (&acc)[8], const uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[2 * i] += __uint_as_float(w[i] << 16);
    acc[2 * i + 1] += __uint_as_float(w[i] & 0xffff0000u);
  }
}

// blockIdx.y selects the tensor (x0 or x1) so that Q and K pool in one launch.
template <int D, int U>
__global__ void __launch_bounds__(kPoolThreads) block_means_kernel(
    const __nv_bfloat16* __restrict__ x0, const __nv_bfloat16* __restrict__ x1,
    float* __restrict__ out0, float* __restrict__ out1, int heads, int N) {
  using S = PoolShape<D, U>;
  __shared__ float part[kPoolThreads][9];  // 9: odd stride, conflict-free column reads
  const __nv_bfloat16* x = blockIdx.y ? x1 : x0;
  float* out = blockIdx.y ? out1 : out0;
  const int nb = (N + U - 1) / U;
  const int tid = threadIdx.x;
  const int ul = tid / S::TPU;
  const int rem = tid - ul * S::TPU;
  const int phase = rem / S::CG;
  const int cg = rem - phase * S::CG;
  const long long unit = static_cast<long long>(blockIdx.x) * S::UPC + ul;
  const bool valid = unit < static_cast<long long>(heads) * nb;
  int n = 0;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  if (valid) {
    const int h = static_cast<int>(unit / nb);
    const int b = static_cast<int>(unit - static_cast<long long>(h) * nb);
    n = min(U, N - b * U);
    const uint4* base = reinterpret_cast<const uint4*>(
        x + (static_cast<size_t>(h) * N + static_cast<size_t>(b) * U) * D);
    uint4 v[kRowsPerThread];
#pragma unroll
    for (int i = 0; i < kRowsPerThread; ++i) {
      const int r = phase + S::P * i;
      v[i] = (r < n) ? __ldcs(base + static_cast<size_t>(r) * S::CG + cg) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < kRowsPerThread; ++i) add_bf16x8(acc, v[i]);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) part[tid][i] = acc[i];
  __syncthreads();
  if (valid && phase == 0) {
    float s[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i] = 0.f;
    for (int p = 0; p < S::P; ++p) {
      const int t = ul * S::TPU + p * S::CG + cg;
#pragma unroll
      for (int i = 0; i < 8; ++i) s[i] += part[t][i];
    }
    const float inv = 1.0f / static_cast<float>(n);
    float4* o = reinterpret_cast<float4*>(out + static_cast<size_t>(unit) * D + cg * 8);
    o[0] = make_float4(s[0] * inv, s[1] * inv, s[2] * inv, s[3] * inv);
    o[1] = make_float4(s[4] * inv, s[5] * inv, s[6] * inv, s[7] * inv);
  }
}

template <int D, int U>
cudaError_t launch_pool_t(const __nv_bfloat16* x0, const __nv_bfloat16* x1, float* out0,
                          float* out1, int heads, int N, cudaStream_t s) {
  using S = PoolShape<D, U>;
  const long long units = static_cast<long long>(heads) * ((N + U - 1) / U);
  const long long grid = (units + S::UPC - 1) / S::UPC;
  if (grid <= 0) return cudaSuccess;
  if (grid > 0x7fffffffll) return cudaErrorInvalidValue;
  dim3 g(static_cast<unsigned>(grid), x1 ? 2 : 1);
  block_means_kernel<D, U><<<g, kPoolThreads, 0, s>>>(x0, x1, out0, out1, heads, N);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_block_means(const __nv_bfloat16* x0, const __nv_bfloat16* x1, float* out0,
                               float* out1, int heads, int N, int d, int U, cudaStream_t s) {
#define STA_POOL_CASE(DD, UU) \
  if (d == DD && U == UU) return launch_pool_t<DD, UU>(x0, x1, out0, out1, heads, N, s);
  STA_POOL_CASE(128, 128)
  STA_POOL_CASE(128, 64)
  STA_POOL_CASE(128, 32)
  STA_POOL_CASE(128, 16)
  STA_POOL_CASE(64, 128)
  STA_POOL_CASE(64, 64)
  STA_POOL_CASE(64, 32)
  STA_POOL_CASE(64, 16)
#undef STA_POOL_CASE
  return cudaErrorInvalidValue;
}

}  // namespace sta
