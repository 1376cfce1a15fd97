// pool_dev.cuh -- device code of the block means (one pass of a 256-thread
// CTA over up to 256 / (d/8 * U/8) blocks), shared by the standalone pooling
// kernel and the fused entropy selector.
//
// A thread owns one 16-byte column group (8 bf16) and 8 rows of one block
// (rows phase, phase+P, ..., so a warp reads whole consecutive rows), keeps 8
// fp32 partial sums, and the P partials of a column group are added in
// shared memory in phase order; the mean divides by the block's true row
// count (the last block of a head may be partial).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace sta {

constexpr int kPoolThreads = 256;
constexpr int kPoolRowsPerThread = 8;

template <int D, int U>
struct PoolShape {
  static constexpr int CG = D / 8;                    // 16-byte column groups per row
  static constexpr int P = U / kPoolRowsPerThread;    // row phases per block
  static constexpr int TPU = CG * P;                  // threads per block
  static constexpr int UPC = kPoolThreads / TPU;      // blocks per CTA pass
  static_assert(U % kPoolRowsPerThread == 0, "unit must be a multiple of 8 rows");
  static_assert(kPoolThreads % TPU == 0, "threads per unit must divide the CTA");
};

__device__ __forceinline__ void pool_add_bf16x8(float (&acc)[8], const uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[2 * i] += __uint_as_float(w[i] << 16);
    acc[2 * i + 1] += __uint_as_float(w[i] & 0xffff0000u);
  }
}

// Means of blocks first_unit .. first_unit + UPC - 1 (unit = head * nb + b)
// of x [heads][N][D] into out [heads][nb][D] (fp32), or, when out is null,
// as the fp16 pair hi = fp16(mean), lo = fp16(mean - hi) into hi/lo (the
// tensor-core operands of the importance scores; a mean beyond the fp16
// range sets *range_bad).  part: 256 x 9 floats of shared memory; the caller
// synchronises the CTA before reusing it.
template <int D, int U>
__device__ __forceinline__ void pool_pass(const __nv_bfloat16* __restrict__ x,
                                          float* __restrict__ out, int heads, int N,
                                          long long first_unit, float (*part)[9],
                                          __half* hi = nullptr, __half* lo = nullptr,
                                          bool* range_bad = nullptr) {
  using S = PoolShape<D, U>;
  const int nb = (N + U - 1) / U;
  const int tid = threadIdx.x;
  const int ul = tid / S::TPU;
  const int rem = tid - ul * S::TPU;
  const int phase = rem / S::CG;
  const int cg = rem - phase * S::CG;
  const long long unit = first_unit + ul;
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
    uint4 v[kPoolRowsPerThread];
#pragma unroll
    for (int i = 0; i < kPoolRowsPerThread; ++i) {
      const int r = phase + S::P * i;
      v[i] = (r < n) ? __ldcs(base + static_cast<size_t>(r) * S::CG + cg) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < kPoolRowsPerThread; ++i) pool_add_bf16x8(acc, v[i]);
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
    if (out) {
      float4* o = reinterpret_cast<float4*>(out + static_cast<size_t>(unit) * D + cg * 8);
      o[0] = make_float4(s[0] * inv, s[1] * inv, s[2] * inv, s[3] * inv);
      o[1] = make_float4(s[4] * inv, s[5] * inv, s[6] * inv, s[7] * inv);
    } else {
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float v0 = s[2 * i] * inv, v1 = s[2 * i + 1] * inv;
        const __half h0 = __float2half_rn(v0), h1 = __float2half_rn(v1);
        const __half l0 = __float2half_rn(v0 - __half2float(h0));
        const __half l1 = __float2half_rn(v1 - __half2float(h1));
        hw[i] = static_cast<uint32_t>(__half_as_ushort(h0)) |
                (static_cast<uint32_t>(__half_as_ushort(h1)) << 16);
        lw[i] = static_cast<uint32_t>(__half_as_ushort(l0)) |
                (static_cast<uint32_t>(__half_as_ushort(l1)) << 16);
        if (!(fabsf(v0) < 65504.f) || !(fabsf(v1) < 65504.f)) *range_bad = true;
      }
      const size_t at = static_cast<size_t>(unit) * D + cg * 8;
      *reinterpret_cast<uint4*>(hi + at) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4*>(lo + at) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
  }
}

}  // namespace sta
