// sel_pool.cu -- block means of a [heads][N][d] bf16 tensor (fp32 out, or
// the fp16 hi/lo operand pair of the importance scores).
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
#include "pool_dev.cuh"

namespace sta {
namespace {

// blockIdx.y selects the tensor (x0 or x1) so that Q and K pool in one launch.
template <int D, int U>
__global__ void __launch_bounds__(kPoolThreads) block_means_kernel(
    const __nv_bfloat16* __restrict__ x0, const __nv_bfloat16* __restrict__ x1,
    float* __restrict__ out0, float* __restrict__ out1, int heads, int N) {
  __shared__ float part[kPoolThreads][9];  // 9: odd stride, conflict-free column reads
  pool_pass<D, U>(blockIdx.y ? x1 : x0, blockIdx.y ? out1 : out0, heads, N,
                  static_cast<long long>(blockIdx.x) * PoolShape<D, U>::UPC, part);
}

// The same means as the fp16 hi/lo pair (no fp32 copy).
template <int D, int U>
__global__ void __launch_bounds__(kPoolThreads) block_means_f16x2_kernel(
    const __nv_bfloat16* __restrict__ x, __half* __restrict__ hi, __half* __restrict__ lo,
    int heads, int N, int32_t* dev_status) {
  __shared__ float part[kPoolThreads][9];
  bool bad = false;
  pool_pass<D, U>(x, nullptr, heads, N, static_cast<long long>(blockIdx.x) * PoolShape<D, U>::UPC,
                  part, hi, lo, &bad);
  if (bad) raise_status(dev_status, STA_DEV_RANGE);
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

template <int D, int U>
cudaError_t launch_pool_f16x2_t(const __nv_bfloat16* x, __half* hi, __half* lo, int heads, int N,
                                int32_t* dev_status, cudaStream_t s) {
  using S = PoolShape<D, U>;
  const long long units = static_cast<long long>(heads) * ((N + U - 1) / U);
  const long long grid = (units + S::UPC - 1) / S::UPC;
  if (grid <= 0) return cudaSuccess;
  if (grid > 0x7fffffffll) return cudaErrorInvalidValue;
  block_means_f16x2_kernel<D, U><<<static_cast<unsigned>(grid), kPoolThreads, 0, s>>>(
      x, hi, lo, heads, N, dev_status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_block_means_f16x2(const __nv_bfloat16* x, __half* hi, __half* lo, int heads,
                                     int N, int d, int U, int32_t* dev_status, cudaStream_t s) {
#define STA_POOL_CASE(DD, UU) \
  if (d == DD && U == UU) return launch_pool_f16x2_t<DD, UU>(x, hi, lo, heads, N, dev_status, s);
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
