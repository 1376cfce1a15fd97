// sel_tra.cu -- token-level entropy -> budget -> disk radius -> token voting.
//
// "Token Radius Attention for Efficient Video Generation", 2. Methodology:
// Insight I (the token budget follows the query's attention entropy,
// B ~ tau * exp(H) / N, so query i keeps about n_i = tau * exp(H_i) keys),
// Insight II (the kept keys form a query-centred spatial disk whose radius
// shrinks with temporal distance by exp(-gamma * delta)) and The TRA Pipeline
// (entropy from a dense warm-up -> budget -> base radius -> per-frame 2D disk
// -> token voting into block-sparse lists):
//
//   r0^2  = tau * exp(H_i) / (pi * G(f_i)),  G(f) = sum_f' exp(-2 gamma |f' - f|)
//   r_f^2 = r0^2 * exp(-2 gamma |f - f_i|)                          (fp32)
//   frame f's share of the budget is n_f = pi * r_f^2 tokens; a frame with
//   n_f < 1 keeps no key, otherwise
//   key j kept for query i  iff  (h_j - h_i)^2 + (w_j - w_i)^2 <= r_{f_j}^2
//   key block kb listed for query block qb iff at least `vote` kept pairs
//   (i in qb, j in kb).
//
// Blocks are runs of B consecutive sequence positions, in the raster order or
// in a tile-major order (tokens reordered tile by tile, The TRA Pipeline,
// Efficient Execution); a position's grid coordinates come from
// layout_coords.  One CTA per (query block, head).  The block's queries
// (coordinates and r0^2) and the per-distance decay table are staged in
// shared memory; thread t then takes key blocks t, t + 256, ...: it splits
// the block's positions into grid-row segments [w0, w1] of one (f, h) (in a
// tile-major order a segment ends at the tile's edge) and, per query, counts
// the keys
// of each segment inside the query's disk: with rest = r_f^2 - dh^2 >= 0
// (exact in fp32: dh^2 is an integer below 2^24) and dw = floor(sqrt(rest))
// (corrected so that dw^2 <= rest < (dw+1)^2 exactly), the row's kept
// columns are [w_i - dw, w_i + dw].  A segment is skipped without visiting
// the queries when no query can reach it: per frame, the largest r_f^2 over
// the block's queries (frames whose share is below one token excluded)
// against the squared row distance from the block's row span.  With vote 1
// (any kept pair lists the block) the segments are merged into maximal
// rectangles and each (rectangle, query) pair takes one test of its nearest
// key: for a 16 x 8 tile block that is one test per query instead of 16.
// Key blocks are decided into a shared bitmask (no barriers between a
// thread's blocks, whose costs differ widely) and compacted in ascending
// order with one block-wide scan per 8,192 blocks.
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"

namespace sta {
namespace {

constexpr int kTraThreads = 256;
constexpr int kTraMaxQ = 128;   // query block size limit
constexpr int kTraMaxF = 1024;  // frame count limit (decay table)
constexpr int kTraChunk = 32 * kTraThreads;  // key blocks decided per compaction

struct TraArgs {
  const float* entropy;  // [heads][N], indexed by sequence position
  int heads, F, H, W, B, nb;
  TokLayout L;           // token order of the sequence (raster or tile-major)
  float tau, gamma;
  int vote;
  int32_t* idx;
  int32_t* cnt;
  int cap;
  int32_t* required_cap;
  int32_t* dev_status;
};

// Largest integer dw >= 0 with dw^2 <= t, for 0 <= t < W^2 (the squares
// are compared in double, exactly).
__device__ __forceinline__ int floor_sqrt(float t) {
  long long dw = static_cast<long long>(sqrtf(t));
  while (static_cast<double>((dw + 1) * (dw + 1)) <= static_cast<double>(t)) ++dw;
  while (dw > 0 && static_cast<double>(dw * dw) > static_cast<double>(t)) --dw;
  return static_cast<int>(dw);
}

__global__ void __launch_bounds__(kTraThreads) tra_token_lists_kernel(const TraArgs a) {
  __shared__ float decay[kTraMaxF];    // exp(-2 gamma delta), delta = |f - f_i|
  __shared__ float qr0[kTraMaxQ];      // r0^2 of each query of the block
  __shared__ int qf[kTraMaxQ], qh[kTraMaxQ], qw[kTraMaxQ];
  __shared__ float reach[kTraMaxF];   // per frame: max r_f^2 over the block's queries
  __shared__ int warp_tot[kTraThreads / 32];
  __shared__ uint32_t keepbits[kTraChunk / 32];  // decided key blocks of a chunk
  __shared__ int running, hmin, hmax;
  const int qb = blockIdx.x, head = blockIdx.y;
  const int S = a.H * a.W;
  const int N = a.F * S;
  const int q0 = qb * a.B;
  const int nq = min(a.B, N - q0);
  for (int dlt = threadIdx.x; dlt < a.F; dlt += kTraThreads)
    decay[dlt] = expf(-2.0f * a.gamma * static_cast<float>(dlt));
  if (threadIdx.x == 0) {
    running = 0;
    hmin = a.H;
    hmax = -1;
  }
  __syncthreads();
  const float* Hh = a.entropy + static_cast<size_t>(head) * N;
  for (int r = threadIdx.x; r < nq; r += kTraThreads) {
    const int t = q0 + r;  // sequence position
    int f, h, w, run;
    layout_coords(a.L, t, f, h, w, run);
    if (!dcheck(f < a.F && h < a.H && w < a.W, a.dev_status)) {
      qr0[r] = 0.f;  // the query is dropped (it reaches no key)
      qf[r] = qh[r] = qw[r] = 0;
      continue;
    }
    qf[r] = f;
    qh[r] = h;
    qw[r] = w;
    float G = 0.f;  // frames in order: the same sum on every query of frame f
    for (int f2 = 0; f2 < a.F; ++f2) G += decay[abs(f2 - f)];
    const float n = a.tau * expf(__ldg(Hh + t));
    qr0[r] = n / (3.14159265358979f * G);
    atomicMin(&hmin, qh[r]);
    atomicMax(&hmax, qh[r]);
  }
  __syncthreads();
  for (int f = threadIdx.x; f < a.F; f += kTraThreads) {
    float m = -1.f;
    for (int r = 0; r < nq; ++r) {
      const float rf = qr0[r] * decay[abs(f - qf[r])];
      if (rf * 3.14159265358979f >= 1.f) m = fmaxf(m, rf);
    }
    reach[f] = m;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t row = static_cast<size_t>(head) * a.nb + qb;
  int32_t* out = a.idx + row * a.cap;
  // Is key block kb listed?  (No barriers inside: threads take their key
  // blocks at their own pace.)
  auto decide = [&](int kb) -> bool {
    bool keep = false;
    if (a.vote == 1) {
      // vote 1: the block is kept iff one of its maximal key rectangles
      // (grid-row segments of one frame, vertically merged when consecutive
      // rows span the same columns) has its key nearest to some query inside
      // that query's disk; the nearest key minimises the squared distance
      // over the rectangle, so one integer test per (rectangle, query)
      // decides it
      const int t0 = kb * a.B, t1 = min(N, t0 + a.B);
      auto test_rect = [&](int f, int h0, int h1, int w0, int w1) -> bool {
        const int drow = max(0, max(h0 - hmax, hmin - h1));
        if (static_cast<float>(drow * drow) > reach[f]) return false;  // no query reaches it
        for (int r = 0; r < nq; ++r) {
          const float rf = qr0[r] * decay[abs(f - qf[r])];
          if (rf * 3.14159265358979f < 1.f) continue;  // share below one token
          const int dh = max(0, max(h0 - qh[r], qh[r] - h1));
          const int dw = max(0, max(w0 - qw[r], qw[r] - w1));
          if (static_cast<float>(dh * dh + dw * dw) <= rf) return true;  // exact integers
        }
        return false;
      };
      bool have = false;
      int cf = 0, ch0 = 0, ch1 = 0, cw0 = 0, cw1 = 0;  // rectangle being grown
      for (int t = t0; t < t1 && !keep;) {
        int f, h, w0, run;
        layout_coords(a.L, t, f, h, w0, run);
        const int len = min(run, t1 - t);
        const int w1 = w0 + len - 1;
        t += len;
        if (have && f == cf && h == ch1 + 1 && w0 == cw0 && w1 == cw1) {
          ch1 = h;
          continue;
        }
        if (have) keep = test_rect(cf, ch0, ch1, cw0, cw1);
        have = true;
        cf = f;
        ch0 = ch1 = h;
        cw0 = w0;
        cw1 = w1;
      }
      if (!keep && have) keep = test_rect(cf, ch0, ch1, cw0, cw1);
    } else {
      const int t0 = kb * a.B, t1 = min(N, t0 + a.B);  // [t0, t1)
      const float wsq = static_cast<float>(a.W) * static_cast<float>(a.W);
      int votes = 0;
      // grid-row segments [w0, w1] of one (f, h) of the key block
      for (int t = t0; t < t1 && votes < a.vote;) {
        int f, h, w0, run;
        layout_coords(a.L, t, f, h, w0, run);
        const int len = min(run, t1 - t);
        const int w1 = w0 + len - 1;  // inclusive
        t += len;
        const int drow = max(0, max(hmin - h, h - hmax));
        if (static_cast<float>(drow * drow) > reach[f]) continue;  // no query reaches it
        for (int r = 0; r < nq && votes < a.vote; ++r) {
          const float rf = qr0[r] * decay[abs(f - qf[r])];
          if (rf * 3.14159265358979f < 1.f) continue;  // share below one token
          const int dh = h - qh[r];
          const float rest = rf - static_cast<float>(dh * dh);
          if (rest < 0.f) continue;
          // rest >= W^2: the disk spans the whole row
          const int dw = rest >= wsq ? a.W : floor_sqrt(rest);
          const int lo = max(w0, qw[r] - dw), hi_w = min(w1, qw[r] + dw);
          if (hi_w >= lo) votes += hi_w - lo + 1;
        }
      }
      keep = votes >= a.vote;
    }
    return keep;
  };
  // Key blocks are decided kTraChunk at a time into a bitmask, then
  // compacted in ascending order: thread t takes word t of the mask, an
  // exclusive block scan of the words' bit counts places their ids.
  for (int c0 = 0; c0 < a.nb; c0 += kTraChunk) {
    const int c1 = min(a.nb, c0 + kTraChunk);
    for (int wd = threadIdx.x; wd < kTraChunk / 32; wd += kTraThreads) keepbits[wd] = 0u;
    __syncthreads();
    for (int kb = c0 + threadIdx.x; kb < c1; kb += kTraThreads)
      if (decide(kb)) atomicOr(&keepbits[(kb - c0) >> 5], 1u << ((kb - c0) & 31));
    __syncthreads();
    const int nwords = (c1 - c0 + 31) >> 5;  // <= kTraChunk / 32 <= kTraThreads
    const uint32_t bits = threadIdx.x < nwords ? keepbits[threadIdx.x] : 0u;
    const int cntw = __popc(bits);
    int inc = cntw;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += t;
    }
    if (lane == 31) warp_tot[warp] = inc;
    __syncthreads();
    int before = running;
    for (int wd = 0; wd < warp; ++wd) before += warp_tot[wd];
    int pos = before + inc - cntw;
    for (uint32_t b = bits; b; b &= b - 1u) {
      const int kb = c0 + threadIdx.x * 32 + (__ffs(b) - 1);
      if (pos < a.cap && dcheck(kb < a.nb, a.dev_status)) out[pos] = kb;
      ++pos;
    }
    __syncthreads();
    if (threadIdx.x == 0)
      for (int wd = 0; wd < kTraThreads / 32; ++wd) running += warp_tot[wd];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const int total = running;
    a.cnt[row] = min(total, a.cap);
    if (a.required_cap) atomicMax(a.required_cap, total);
    if (total > a.cap) raise_status(a.dev_status, STA_DEV_CAPACITY);
  }
}

}  // namespace

int tra_max_frames() { return kTraMaxF; }
int tra_max_block() { return kTraMaxQ; }

cudaError_t launch_tra_token_lists(const float* entropy, int heads, int F, int H, int W, int B,
                                   int tile_h, int tile_w, float tau, float gamma, int vote,
                                   int32_t* idx, int32_t* cnt, int cap, int32_t* required_cap,
                                   int32_t* dev_status, cudaStream_t s) {
  TraArgs a;
  a.entropy = entropy;
  a.heads = heads;
  a.F = F;
  a.H = H;
  a.W = W;
  a.L = TokLayout{H, W, tile_h, tile_w};
  a.B = B;
  const long long N = static_cast<long long>(F) * H * W;
  a.nb = static_cast<int>((N + B - 1) / B);
  a.tau = tau;
  a.gamma = gamma;
  a.vote = vote;
  a.idx = idx;
  a.cnt = cnt;
  a.cap = cap;
  a.required_cap = required_cap;
  a.dev_status = dev_status;
  if (a.nb <= 0 || heads <= 0) return cudaSuccess;
  tra_token_lists_kernel<<<dim3(static_cast<unsigned>(a.nb), static_cast<unsigned>(heads)),
                           kTraThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace sta
