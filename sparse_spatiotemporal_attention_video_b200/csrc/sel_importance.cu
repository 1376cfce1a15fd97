// sel_importance.cu -- block importance of the clustering selector on the
// tensor cores:
//
//   p_j = sum_c (n_c / n_b) softmax_j(c_c . Kbar_j * scale + ln n_j)
//
// ("AB-Attention speeds up video diffusion transformers up to 2.23x, no
// training", method paragraph: importance of key/value blocks from the
// clustered queries of each query block; the workload fixes k = 4 centroids
// and 16-key sub-blocks.)
//
// Precision.  Sampling decisions compare u_j with pi_j = min(1, lambda p_j),
// so p must be close to fp32 accuracy.  Each fp32 operand x (a sub-block
// mean or a centroid) is written by its producer (block means, k-means) as
// two fp16 values, x = hi + lo with hi = fp16(x) and lo = fp16(x - hi) (22
// significant bits together), and every score is accumulated in fp32 on the
// tensor cores as hi_c.hi_k + hi_c.lo_k + lo_c.hi_k (the lo.lo term is below
// fp32 rounding).  Against fp64 this moves pi by < 3e-7 on the workload's
// data, far inside the 1e-5 band where decisions may legitimately differ;
// bf16 halves (8 + 8 bits) moved it by up to 1.3e-5.  fp16 limits the
// operands to |x| < 65504 (pooled keys and query centroids are O(1)); values
// beyond it raise STA_DEV_RANGE.
//
// Kernel.  One CTA per (head, 128 centroid rows = 32 query blocks x 4).
//   warp 0      TMA: the centroid tile (hi, lo) once, then for each 128-wide
//               tile of sub-blocks the Kbar tile (hi, lo) into a 2-stage ring.
//   warp 1      MMA issuer: per tile 8 K-steps x 3 products, M=128 N=128
//               K=16 (tcgen05.mma kind::f16, fp16 operands K-major in shared
//               memory, fp32 accumulator in TMEM, double-buffered).
//   warps 2-9   epilogue, two groups of 4 warps: group J reads columns
//               [64J, 64J+64) of each accumulator row r (TMEM lane r = the
//               centroid row).  Sweep 1 over all tiles keeps an online max
//               and an fp64 sum of exp per row; the two groups then merge
//               them into M_c and coef_c = w_c / Z_c.  Sweep 2 recomputes
//               the scores and forms e = coef_c exp(z - M_c); the 4 centroid
//               rows of a query block are 4 neighbouring lanes, which sum
//               their e by a two-step reduce-scatter (each lane ends with 16
//               of the 64 columns) and store p.
// Every wait is bounded (STA_DEV_TIMEOUT, abort flag, no trap).
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "sm100.cuh"

namespace sta {
namespace {

constexpr int kImpTcThreads = 320;
constexpr int kImpTile = 128;                    // rows and columns of a tile
constexpr int kImpHalf = 128 * 128;              // bytes of one 64-column half (fp16)
constexpr int kImpTileBytes = 2 * kImpHalf;      // one 128 x 128 fp16 tile
constexpr int kImpStages = 2;
constexpr float kLog2eImp = 1.4426950408889634f;

struct ImpSmem {
  static constexpr int OFF_AH = 0;
  static constexpr int OFF_AL = OFF_AH + kImpTileBytes;
  static constexpr int OFF_B = OFF_AL + kImpTileBytes;            // [stage][hi, lo]
  static constexpr int OFF_BAR = OFF_B + kImpStages * 2 * kImpTileBytes;
  // a_full, b_full[2], b_empty[2], acc_full[2], acc_empty[2], mma_done, xbar[4]
  static constexpr int NBAR = 1 + 2 * kImpStages + 4 + 1 + 4;
  static constexpr int OFF_RED = OFF_BAR + NBAR * 8;                // m, s (double) x 2 x 128
  static constexpr int OFF_MISC = OFF_RED + 2 * 128 * (4 + 8);
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;
};

struct ImpArgs {
  const float* wts;  // [heads][n_rows] n_c / n_b
  float* p;          // [heads][nqb][ld], ld = n_sub rounded up to 4 (16-byte rows)
  int n_rows, nqb, n_sub, ld, N, U, tiles;
  float scale;
  int32_t* dev_status;
};

__device__ __forceinline__ void imp_fail(volatile int* abort, int32_t* st) {
  *abort = 1;
  raise_status(st, STA_DEV_TIMEOUT);
}

// f16 x f16 -> f32, both operands K-major.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
  return (1u << 4)                                 // D format: f32
         | (static_cast<uint32_t>(N >> 3) << 17)   // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);  // M / 16
}

template <int KM>
__global__ void __launch_bounds__(kImpTcThreads, 1)
    importance_tc_kernel(const __grid_constant__ ImpArgs a,
                         const __grid_constant__ CUtensorMap tm_ch,
                         const __grid_constant__ CUtensorMap tm_cl,
                         const __grid_constant__ CUtensorMap tm_kh,
                         const __grid_constant__ CUtensorMap tm_kl) {
  extern __shared__ uint8_t imp_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(imp_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sAh = smem + ImpSmem::OFF_AH;
  uint8_t* sAl = smem + ImpSmem::OFF_AL;
  uint8_t* sB = smem + ImpSmem::OFF_B;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + ImpSmem::OFF_BAR);
  uint64_t* a_full = bars;
  uint64_t* b_full = a_full + 1;
  uint64_t* b_empty = b_full + kImpStages;
  uint64_t* acc_full = b_empty + kImpStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* mma_done = acc_empty + 2;
  uint64_t* xbar = mma_done + 1;  // [4 quadrants], 64 arrivals
  float* red_m = reinterpret_cast<float*>(smem + ImpSmem::OFF_RED);           // [2][128]
  double* red_s = reinterpret_cast<double*>(smem + ImpSmem::OFF_RED + 2 * 128 * 4);  // [2][128]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + ImpSmem::OFF_MISC);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + ImpSmem::OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int head = blockIdx.y;
  const int row0 = blockIdx.x * kImpTile;
  const int tiles = a.tiles;
  const uint64_t limit = kWaitLimitNs;
  int no_abort_storage = 0;
  volatile int* no_abort = &no_abort_storage;

  if (threadIdx.x == 0) {
    mbar_init(a_full, 1);
    for (int i = 0; i < kImpStages; ++i) {
      mbar_init(b_full + i, 1);
      mbar_init(b_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(acc_full + i, 1);
      mbar_init(acc_empty + i, 256);
    }
    mbar_init(mma_done, 1);
    for (int i = 0; i < 4; ++i) mbar_init(xbar + i, 64);
    *abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_ch);
    tma_prefetch_desc(&tm_cl);
    tma_prefetch_desc(&tm_kh);
    tma_prefetch_desc(&tm_kl);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_arrive_expect_tx(a_full, 2 * kImpTileBytes);
      for (int h = 0; h < 2; ++h) {
        tma_load_3d(sAh + h * kImpHalf, &tm_ch, a_full, h * 64, row0, head);
        tma_load_3d(sAl + h * kImpHalf, &tm_cl, a_full, h * 64, row0, head);
      }
      int g = 0;
      for (; g < 2 * tiles; ++g) {
        if (*abort) break;
        const int st = g % kImpStages;
        const uint32_t use = static_cast<uint32_t>(g / kImpStages);
        if (!mbar_wait(b_empty + st, (use & 1) ^ 1, abort, limit)) {
          imp_fail(abort, a.dev_status);
          break;
        }
        const int j = g % tiles;
        uint8_t* dst = sB + st * 2 * kImpTileBytes;
        mbar_arrive_expect_tx(b_full + st, 2 * kImpTileBytes);
        for (int h = 0; h < 2; ++h) {
          tma_load_3d(dst + h * kImpHalf, &tm_kh, b_full + st, h * 64, j * kImpTile, head);
          tma_load_3d(dst + kImpTileBytes + h * kImpHalf, &tm_kl, b_full + st, h * 64,
                      j * kImpTile, head);
        }
      }
      // let every copy issued here land before the CTA can exit
      mbar_wait(a_full, 0, no_abort, limit);
      for (int i = (g > kImpStages ? g - kImpStages : 0); i < g; ++i)
        mbar_wait(b_full + (i % kImpStages), (i / kImpStages) & 1, no_abort, limit);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_f16_f32(kImpTile, kImpTile);
      const uint32_t aH = smem_u32(sAh), aL = smem_u32(sAl), bBase = smem_u32(sB);
      bool ok = mbar_wait(a_full, 0, abort, limit);
      tc_fence_after();
      for (int g = 0; ok && g < 2 * tiles; ++g) {
        const int st = g % kImpStages;
        const int acc = g & 1;
        if (!mbar_wait(b_full + st, (g / kImpStages) & 1, abort, limit) ||
            !mbar_wait(acc_empty + acc, ((g >> 1) & 1) ^ 1, abort, limit)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tAcc = tmem + acc * kImpTile;
        if (!dcheck(tmem_in_range(tAcc, tmem, kImpTile, 2 * kImpTile), a.dev_status)) {
          ok = false;
          break;
        }
        const uint32_t bH = bBase + st * 2 * kImpTileBytes, bL = bH + kImpTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kImpHalf + (kk & 3) * 32;
          const uint64_t dah = smem_desc_sw128(aH + off, 16, 1024);
          const uint64_t dal = smem_desc_sw128(aL + off, 16, 1024);
          const uint64_t dbh = smem_desc_sw128(bH + off, 16, 1024);
          const uint64_t dbl = smem_desc_sw128(bL + off, 16, 1024);
          mma_bf16_ss(tAcc, dah, dbh, IDESC, kk > 0 ? 1u : 0u);
          mma_bf16_ss(tAcc, dah, dbl, IDESC, 1u);
          mma_bf16_ss(tAcc, dal, dbh, IDESC, 1u);
        }
        mma_commit(b_empty + st);
        mma_commit(acc_full + acc);
      }
      if (!ok) imp_fail(abort, a.dev_status);
      mma_commit(mma_done);
      mbar_wait(mma_done, 0, no_abort, limit);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int J = (warp - 2) >> 2;  // column half of every tile
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // centroid row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const int grow = row0 + r;       // centroid row within the head
    const bool row_ok = grow < a.n_rows;
    // scores in log2 units (z * log2(e)), so that exp2 (MUFU ex2) replaces expf:
    // relative error ~1e-6 on p, against the 1e-4 that would reach the
    // sampling band
    const float scale2 = a.scale * kLog2eImp;
    const float ln_full = log2f(static_cast<float>(a.U));
    const float ln_last = log2f(static_cast<float>(a.N - (a.n_sub - 1) * a.U));
    bool ok = true;
    float m = -INFINITY;
    double ssum = 0.0;
    float coef = 0.f;
    for (int g = 0; ok && g < 2 * tiles; ++g) {
      const int acc = g & 1;
      if (!mbar_wait(acc_full + acc, (g >> 1) & 1, abort, limit)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float x[64];
      {
        uint32_t v0[32], v1[32];
        const uint32_t ta = tmem + lane_off + acc * kImpTile + J * 64;
        if (!dcheck(tmem_in_range(ta, tmem, 64, 2 * kImpTile), a.dev_status)) {
          ok = false;
          break;
        }
        tmem_ld32(ta, v0);
        tmem_ld32(ta + 32, v1);
        tmem_wait_ld();
        tmem_regs_ready(v0);
        tmem_regs_ready(v1);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          x[i] = __uint_as_float(v0[i]);
          x[32 + i] = __uint_as_float(v1[i]);
        }
      }
      tc_fence_before();
      mbar_arrive(acc_empty + acc);
      const int j = g % tiles;
      const int c0 = j * kImpTile + J * 64;  // first sub-block of this thread's columns
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const int col = c0 + c;
        x[c] = col < a.n_sub ? fmaf(x[c], scale2, col == a.n_sub - 1 ? ln_last : ln_full)
                             : -INFINITY;
      }
      if (g < tiles) {
        // sweep 1: online max and fp64 sum of exp over this row's columns
        float t = x[0];
#pragma unroll
        for (int c = 1; c < 64; ++c) t = fmaxf(t, x[c]);
        if (t != -INFINITY) {
          if (t > m) {
            if (m != -INFINITY) ssum *= exp2(static_cast<double>(m) - static_cast<double>(t));
            m = t;
          }
          float part[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) part[i] = 0.f;
#pragma unroll
          for (int c = 0; c < 64; ++c) part[c & 7] += fast_exp2(x[c] - m);
          ssum += static_cast<double>(((part[0] + part[1]) + (part[2] + part[3])) +
                                      ((part[4] + part[5]) + (part[6] + part[7])));
        }
        if (g == tiles - 1) {
          // merge the two column halves of the row: M_c and coef_c = w_c / Z_c
          red_m[J * 128 + r] = m;
          red_s[J * 128 + r] = ssum;
          mbar_arrive(xbar + quad);
          if (!mbar_wait(xbar + quad, 0, abort, limit)) {
            ok = false;
            break;
          }
          const float mo = red_m[(1 - J) * 128 + r];
          const double so = red_s[(1 - J) * 128 + r];
          const float mm = fmaxf(m, mo);
          double z = 0.0;
          if (m != -INFINITY) z += ssum * exp2(static_cast<double>(m) - static_cast<double>(mm));
          if (mo != -INFINITY) z += so * exp2(static_cast<double>(mo) - static_cast<double>(mm));
          m = mm;
          coef = (row_ok && z > 0.0)
                     ? static_cast<float>(
                           static_cast<double>(__ldg(a.wts + static_cast<size_t>(head) * a.n_rows + grow)) / z)
                     : 0.f;
        }
      } else {
        // sweep 2: e = coef exp(z - M); the KM centroid rows of a query
        // block are KM neighbouring lanes, which sum their e by a butterfly
        // reduce-scatter: at each step a lane keeps half of its current
        // columns and receives the partner's partial sums of that half
#pragma unroll
        for (int c = 0; c < 64; ++c) x[c] = coef != 0.f ? coef * fast_exp2(x[c] - m) : 0.f;
        int base = 0;
#pragma unroll
        for (int mask = KM / 2; mask >= 1; mask /= 2) {
          const int half = 32 * mask * 2 / KM;  // columns kept after this step
          const bool up = (lane & mask) != 0;
#pragma unroll
          for (int i = 0; i < half; ++i) {
            const float send = up ? x[i] : x[half + i];
            const float got = __shfl_xor_sync(0xffffffffu, send, mask);
            x[i] = (up ? x[half + i] : x[i]) + got;
          }
          if (up) base += half;
        }
        const int qb = grow / KM;  // rows are query block * KM + centroid
        if (row_ok && qb < a.nqb) {
          const int col0 = c0 + base;  // a multiple of 64 / KM >= 8
          float* pr = a.p + (static_cast<size_t>(head) * a.nqb + qb) * a.ld + col0;
          // whole float4s up to ld (padding columns beyond n_sub hold 0)
#pragma unroll
          for (int i = 0; i < 64 / KM; i += 4)
            if (col0 + i < a.ld)
              *reinterpret_cast<float4*>(pr + i) = make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
        }
      }
    }
    if (!ok) imp_fail(abort, a.dev_status);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 256);
}

// hi = fp16(x), lo = fp16(x - hi) of an fp32 array (n elements).
}  // namespace

cudaError_t launch_importance_tc(const float* wts, float* p, int heads, int n_rows, int nqb,
                                 int km, int n_sub, int N, int U, float scale,
                                 const CUtensorMap& ch,
                                 const CUtensorMap& cl, const CUtensorMap& kh,
                                 const CUtensorMap& kl, int32_t* dev_status, cudaStream_t s) {
  ImpArgs a;
  a.wts = wts;
  a.p = p;
  a.n_rows = n_rows;
  a.nqb = nqb;
  a.n_sub = n_sub;
  a.ld = (n_sub + 3) & ~3;
  a.N = N;
  a.U = U;
  a.tiles = (n_sub + kImpTile - 1) / kImpTile;
  a.scale = scale;
  a.dev_status = dev_status;
  dim3 g((n_rows + kImpTile - 1) / kImpTile, heads);
  cudaError_t e;
#define STA_IMP_CASE(KK)                                                            \
  if (km == KK) {                                                                   \
    e = set_dyn_smem<importance_tc_kernel<KK>>(ImpSmem::ALLOC);                     \
    if (e != cudaSuccess) return e;                                                 \
    importance_tc_kernel<KK><<<g, kImpTcThreads, ImpSmem::ALLOC, s>>>(a, ch, cl, kh, kl); \
    return cudaGetLastError();                                                      \
  }
  STA_IMP_CASE(4)
  STA_IMP_CASE(2)
  STA_IMP_CASE(1)
  STA_IMP_CASE(8)
#undef STA_IMP_CASE
  return cudaErrorInvalidValue;
}

}  // namespace sta
