// layout.cu -- token permutation between the raster order and a tile-major
// order.
//
// "Token Radius Attention for Efficient Video Generation", 2. Methodology,
// The TRA Pipeline, Efficient Execution: the tokens are reordered tile by
// tile, so that the spatial neighbours a query's radius reaches are
// contiguous and the token-level masks become block-sparse over few blocks.
// Attention in that order is attention over the permuted Q, K and V, with
// the output permuted back.  The position -> token map is computed from the
// grid and tile shape (layout_coords in common.cuh); no table is stored.
//
// HBM-bound: one read and one write of every row.  Each row (d elements) is
// moved by rows_bytes / 16 lanes with 16-byte accesses; the lane that starts
// a row computes its source (or destination) token and passes it on by
// shuffle.  Reads and writes of a row are contiguous.
#include <cuda_runtime.h>

#include "common.cuh"

namespace sta {
namespace {

constexpr int kPermThreads = 256;

__global__ void __launch_bounds__(kPermThreads) permute_rows_kernel(
    const uint4* __restrict__ in, uint4* __restrict__ out, int heads, int N, int vpr,
    TokLayout L, int inverse) {
  const int lane = threadIdx.x & 31;
  const long long total = static_cast<long long>(heads) * N * vpr;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  // every lane of a warp runs the same number of iterations (the shuffle
  // below needs the whole warp): the loop bound is rounded up to the stride
  const long long base0 = static_cast<long long>(blockIdx.x) * blockDim.x + (threadIdx.x - lane);
  for (long long b = base0; b < total; b += stride) {
    const long long i = b + lane;
    const bool act = i < total;
    const long long row = act ? i / vpr : 0;
    const int v = act ? static_cast<int>(i - row * vpr) : 0;
    int t = 0;
    if (act && v == 0) {
      const int j = static_cast<int>(row % N);
      int f, h, w, run;
      layout_coords(L, j, f, h, w, run);
      t = (f * L.H + h) * L.W + w;
    }
    // the row's first lane sits v lanes below: rows start at multiples of
    // vpr, which divides 32, and b is a multiple of 32
    t = __shfl_sync(0xffffffffu, t, lane - v);
    if (act) {
      const long long head = row / N;
      const long long src = inverse ? row : head * N + t;
      const long long dst = inverse ? head * N + t : row;
      out[dst * vpr + v] = __ldcs(in + src * vpr + v);
    }
  }
}

}  // namespace

cudaError_t launch_permute_rows(const void* in, void* out, int heads, int N, int row_bytes,
                                const TokLayout& L, int inverse, cudaStream_t s) {
  if (row_bytes % 16 != 0) return cudaErrorInvalidValue;
  const int vpr = row_bytes / 16;
  if (vpr < 1 || 32 % vpr != 0) return cudaErrorInvalidValue;
  const long long total = static_cast<long long>(heads) * N * vpr;
  if (total <= 0) return cudaSuccess;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  long long grid = (total + kPermThreads - 1) / kPermThreads;
  const long long cap = static_cast<long long>(sms) * 8;  // 8 resident CTAs per SM
  if (grid > cap) grid = cap;
  permute_rows_kernel<<<static_cast<unsigned>(grid), kPermThreads, 0, s>>>(
      static_cast<const uint4*>(in), static_cast<uint4*>(out), heads, N, vpr, L, inverse);
  return cudaGetLastError();
}

}  // namespace sta
