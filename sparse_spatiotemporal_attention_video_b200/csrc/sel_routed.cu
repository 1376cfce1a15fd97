// sel_routed.cu -- difficulty routing (dense for the hardest tokens, a
// local window for the rest).
//
// "Where Compute Matters: Heterogeneous Attention for Efficient Video
// Diffusion", Abstract: a token-wise difficulty estimate sends uncertain
// tokens through dense global attention and the others through efficient
// local attention; about 20% of tokens take the dense path.  The routed
// workload fixes the rule computed here:
//   * R = the n_routed tokens of highest fp32 difficulty, ties broken towards
//     the lower token index (n_routed = ceil(frac * N), from the host);
//   * a routed query attends to all N keys;
//   * a local query at (f, h, w) attends to keys with |f' - f| <= win_f,
//     h' in [h - win_h, h + win_h), w' in [w - win_w, w + win_w), clipped at
//     the grid edges.
//
// routed_select_kernel (one CTA): radix select on order-preserving 32-bit
// keys of the scores (8 bits per pass, most significant first) finds the
// key T of the n_routed-th largest score and how many tokens equal to T are
// still needed; a final pass in token order flags every token above T and
// the first `need` tokens equal to T, and compacts the flagged ids
// (ascending) with block-wide scans (8 consecutive tokens per thread).
//
// routed_local_lists_kernel: for each query block, the kv units (kv_unit
// consecutive tokens) holding at least one key inside the window of at least
// one query of the block.  Query and key tokens are split into runs of one
// grid row (fixed f, h; w in [w1, w2]); a query run (f, h, [w1, w2]) and a
// key run (f', h', [a, b]) hold a windowed pair iff |f' - f| <= win_f,
// h' - h in [-win_h, win_h) and [a - w2, b - w1] meets [-win_w, win_w - 1].
// The lists depend on geometry only (shared by all heads); queries routed to
// the dense path are still counted, so a list may hold units that only a
// routed query reaches -- the attention applies the window per element and
// writes local outputs only for non-routed queries, so this is exact.
#include <cuda_runtime.h>

#include "common.cuh"

namespace sta {
namespace {

constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelPer = 8;  // tokens per thread in the final pass

// Order-preserving map fp32 -> uint32 (larger float -> larger key); -0 and
// +0 map to the same key.
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t b = __float_as_uint(f);
  if ((b & 0x7fffffffu) == 0) b = 0;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Exclusive block-wide scan of one int per thread; returns the total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot, int& excl) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int w = (lane < kSelWarps) ? warp_tot[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += t;
    }
    if (lane < kSelWarps) warp_tot[lane] = wi - w;  // exclusive warp offsets
    if (lane == 31) warp_tot[kSelWarps] = wi;       // total
  }
  __syncthreads();
  excl = warp_tot[warp] + inc - v;
  const int total = warp_tot[kSelWarps];
  __syncthreads();
  return total;
}

__global__ void __launch_bounds__(kSelThreads) routed_select_kernel(
    const float* __restrict__ dif, int N, int n_routed, int32_t* __restrict__ routed_ids,
    uint8_t* __restrict__ routed_flag) {
  __shared__ int hist[256];
  __shared__ int warp_tot[kSelWarps + 1];
  __shared__ uint32_t s_prefix;
  __shared__ int s_need;
  if (threadIdx.x == 0) {
    s_prefix = 0;
    s_need = n_routed;
  }
  uint32_t mask = 0;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += kSelThreads) hist[i] = 0;
    __syncthreads();
    const uint32_t prefix = s_prefix;
    if (s_need > 0) {
      for (int i = threadIdx.x; i < N; i += kSelThreads) {
        const uint32_t k = order_key(__ldg(dif + i));
        if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 0xff], 1);
      }
    }
    __syncthreads();
    if (threadIdx.x == 0 && s_need > 0) {
      // walk digits from the top until the running count reaches `need`
      int need = s_need, digit = 255;
      for (; digit > 0; --digit) {
        if (hist[digit] >= need) break;
        need -= hist[digit];
      }
      s_need = need;
      s_prefix = prefix | (static_cast<uint32_t>(digit) << shift);
    }
    mask |= 0xffu << shift;
    __syncthreads();
  }
  const uint32_t T = s_prefix;
  const int need_eq = s_need;  // tokens equal to T still to take (lowest ids)
  const bool none = n_routed <= 0;
  // Final pass in token order, kSelPer consecutive tokens per thread (two
  // block scans per kSelThreads * kSelPer tokens): the eq tokens before this
  // thread's run decide which of its own eq tokens are taken.
  int eq_before = 0, out_before = 0;
  for (int base = 0; base < N; base += kSelThreads * kSelPer) {
    const int i0 = base + threadIdx.x * kSelPer;
    uint32_t k[kSelPer];
    int n_eq = 0;
#pragma unroll
    for (int j = 0; j < kSelPer; ++j) {
      k[j] = (i0 + j < N) ? order_key(__ldg(dif + i0 + j)) : 0u;
      n_eq += (i0 + j < N && k[j] == T) ? 1 : 0;
    }
    int eq_excl;
    const int eq_tot = block_exclusive_scan(n_eq, warp_tot, eq_excl);
    int eq_seen = eq_before + eq_excl;
    uint32_t take_bits = 0;
#pragma unroll
    for (int j = 0; j < kSelPer; ++j) {
      if (i0 + j >= N || none) continue;
      bool take = k[j] > T;
      if (k[j] == T) {
        take = eq_seen < need_eq;
        ++eq_seen;
      }
      if (take) take_bits |= 1u << j;
    }
    int out_excl;
    const int out_tot = block_exclusive_scan(__popc(take_bits), warp_tot, out_excl);
    int pos = out_before + out_excl;
#pragma unroll
    for (int j = 0; j < kSelPer; ++j) {
      if (i0 + j >= N) continue;
      const bool take = (take_bits >> j) & 1u;
      routed_flag[i0 + j] = take ? 1 : 0;
      if (take) routed_ids[pos++] = i0 + j;
    }
    eq_before += eq_tot;
    out_before += out_tot;
  }
}

// Calls fn(f, h, w_lo, w_hi) for the row runs of tokens [t0, t1).
template <typename Fn>
__device__ __forceinline__ bool for_runs(int t0, int t1, int H, int W, Fn fn) {
  const int S = H * W;
  for (int t = t0; t < t1;) {
    const int f = t / S;
    const int rem = t - f * S;
    const int h = rem / W;
    const int w = rem - h * W;
    const int len = min(t1 - t, W - w);
    if (fn(f, h, w, w + len - 1)) return true;
    t += len;
  }
  return false;
}

__global__ void __launch_bounds__(256) routed_local_lists_kernel(
    int F, int H, int W, int B, int U, int win_f, int win_h, int win_w,
    int32_t* __restrict__ idx, int32_t* __restrict__ cnt, int cap, int32_t* required_cap,
    int32_t* dev_status) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = H * W;
  const int N = F * S;
  const int nqb = (N + B - 1) / B;
  const int qb = blockIdx.x * 8 + warp;
  if (qb >= nqb) return;
  const int q0 = qb * B, q1 = min(N, q0 + B);
  const int fq0 = q0 / S, fq1 = (q1 - 1) / S;
  // keys can only lie in frames [fq0 - win_f, fq1 + win_f]
  const int k_lo = max(0, fq0 - win_f) * S;
  const int k_hi = min(F, fq1 + win_f + 1) * S;  // exclusive
  const int u_lo = k_lo / U, u_hi = (k_hi + U - 1) / U;
  int32_t* out = idx + static_cast<size_t>(qb) * cap;
  int total = 0;
  for (int u0 = u_lo; u0 < u_hi; u0 += 32) {
    const int u = u0 + lane;
    bool keep = false;
    if (u < u_hi) {
      const int t0 = u * U, t1 = min(N, t0 + U);
      keep = for_runs(t0, t1, H, W, [&](int fk, int hk, int a, int b) {
        return for_runs(q0, q1, H, W, [&](int fq, int hq, int w1, int w2) {
          const int df = fk - fq, dh = hk - hq;
          return df <= win_f && df >= -win_f && dh >= -win_h && dh < win_h &&
                 a - w2 <= win_w - 1 && b - w1 >= -win_w;
        });
      });
    }
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    const int pos = total + __popc(bal & ((1u << lane) - 1u));
    if (keep && pos < cap && dcheck(u * U < N, dev_status)) out[pos] = u;
    total += __popc(bal);
  }
  if (lane == 0) {
    cnt[qb] = min(total, cap);
    if (required_cap) atomicMax(required_cap, total);
    if (total > cap) raise_status(dev_status, STA_DEV_CAPACITY);
  }
}

}  // namespace

cudaError_t launch_routed_select(const float* difficulty, int N, int n_routed,
                                 int32_t* routed_ids, uint8_t* routed_flag, cudaStream_t s) {
  routed_select_kernel<<<1, kSelThreads, 0, s>>>(difficulty, N, n_routed, routed_ids,
                                                 routed_flag);
  return cudaGetLastError();
}

cudaError_t launch_routed_local_lists(int F, int H, int W, int B, int U, int win_f, int win_h,
                                      int win_w, int32_t* idx, int32_t* cnt, int cap,
                                      int32_t* required_cap, int32_t* dev_status,
                                      cudaStream_t s) {
  const int N = F * H * W;
  const int nqb = (N + B - 1) / B;
  routed_local_lists_kernel<<<(nqb + 7) / 8, 256, 0, s>>>(F, H, W, B, U, win_f, win_h, win_w,
                                                          idx, cnt, cap, required_cap,
                                                          dev_status);
  return cudaGetLastError();
}

}  // namespace sta
