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
// HBM-bound: one read and one write of every row.  A warp takes 32 rows at a
// time: lane l decodes row l's token (32-bit arithmetic, once per row), then
// the warp copies the rows 32 / vpr at a time with 16-byte accesses, vpr =
// row bytes / 16 lanes per row, the token passed by shuffle.  Reads and
// writes of a row are contiguous.
#include <cuda_runtime.h>

#include "common.cuh"

namespace sta {
namespace {

constexpr int kPermThreads = 256;

__global__ void __launch_bounds__(kPermThreads) permute_rows_kernel(
    const uint4* __restrict__ in, uint4* __restrict__ out, int rows, int N, int vpr,
    TokLayout L, int inverse) {
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  const int rpi = 32 / vpr;  // rows copied per warp instruction
  for (int r0 = ((blockIdx.x * blockDim.x + threadIdx.x) >> 5) * 32; r0 < rows;
       r0 += warps * 32) {
    // lane l: the token of row r0 + l (its raster index within the head)
    int tok = 0;
    const int rl = r0 + lane;
    if (rl < rows) {
      const int head = rl / N;
      const int j = rl - head * N;
      int f, h, w, run;
      layout_coords(L, j, f, h, w, run);
      tok = head * N + (f * L.H + h) * L.W + w;
    }
    const int n = min(32, rows - r0);
    for (int k = 0; k < n; k += rpi) {
      const int kr = k + lane / vpr;  // this lane's row within the 32
      const int v = lane % vpr;
      const int t = __shfl_sync(0xffffffffu, tok, kr & 31);
      // (no status word here: a failed debug check only skips the row)
      if (kr < n && dcheck(t >= 0 && t < rows, nullptr)) {
        const long long row = r0 + kr;
        const long long src = inverse ? row : t;
        const long long dst = inverse ? t : row;
        out[dst * vpr + v] = __ldcs(in + src * vpr + v);
      }
    }
  }
}

}  // namespace

cudaError_t launch_permute_rows(const void* in, void* out, int heads, int N, int row_bytes,
                                const TokLayout& L, int inverse, cudaStream_t s) {
  if (row_bytes % 16 != 0) return cudaErrorInvalidValue;
  const int vpr = row_bytes / 16;
  if (vpr < 1 || 32 % vpr != 0) return cudaErrorInvalidValue;
  const long long rows = static_cast<long long>(heads) * N;
  if (rows <= 0) return cudaSuccess;
  if (rows > (1ll << 30)) return cudaErrorInvalidValue;  // 32-bit row indices
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long warps_needed = (rows + 31) / 32;
  long long grid = (warps_needed * 32 + kPermThreads - 1) / kPermThreads;
  const long long cap = static_cast<long long>(sms) * 8;  // 8 resident CTAs per SM
  if (grid > cap) grid = cap;
  permute_rows_kernel<<<static_cast<unsigned>(grid), kPermThreads, 0, s>>>(
      static_cast<const uint4*>(in), static_cast<uint4*>(out), static_cast<int>(rows), N, vpr,
      L, inverse);
  return cudaGetLastError();
}

}  // namespace sta
