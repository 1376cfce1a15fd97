// attn_fwd.cu -- exact block-sparse softmax attention on sm_100a.
//
// What it computes ("Token Radius Attention for Efficient Video Generation",
// 1. Problem Statement and The TRA Pipeline; "AB-Attention ..." method
// paragraph): for every query row i of a work item and the key units listed
// for it, O_i = sum_k w_k exp(s_ik - m_i) v_k / sum_k w_k exp(s_ik - m_i)
// with s_ik = scale * q_i.k_k; keys outside the listed units never enter the
// softmax; w_k = 1/pi of the key's sampled unit (stored as -ln pi) or 1.
//
// How (one persistent CTA per SM, 12 warps):
//   warp 0      producer: TMA loads of the 128-row Q tile and, per 128-key
//               tile, of the listed key/value units (kv_unit rows each,
//               128-byte swizzle) into a K ring and a V ring; gathered query
//               rows (routed items) are copied by the warp and swizzled by
//               hand.  With d = 128, a 16-key unit is one copy of both
//               halves through a five-dimensional view, and its tile is laid
//               out [8-row group][half][8 rows][128 B]: a 128-key tile then
//               takes 8 copies per operand instead of 16 of 2 KB, which the
//               copy engine serves too slowly to keep the tensor core busy.
//   warp 1      QK issuer (one thread): S = Q K^T of tile t into TMEM S
//               buffer t%2 (tcgen05.mma, M=128 N=128 K=16 steps, both
//               operands K-major in shared memory), once the PV of tile t-2
//               (which reads P from that buffer) has completed.
//   warp 11     PV issuer (one thread): O_0 += P[:, 0:64] V[0:64] and
//               O_1 += P[:, 64:128] V[64:128] with P read from TMEM (bf16,
//               aliased onto the S buffer) and V MN-major in shared memory.
//               The two issuers feed one tensor pipe: while one waits on a
//               barrier or commits, the other's products keep it busy (one
//               thread issuing both streams left the pipe idle for about
//               800 cycles per tile).
//               TMEM: S_0 | S_1 | O_0 | O_1 (512 columns).
//   warps 2-9   softmax, two groups of 4 warps.  Group J owns keys
//               [64J, 64J+64) of every tile and the accumulator O_J: thread r
//               of the group holds query row r (TMEM lane r), reads its 64
//               logits, masks partial units / the local window, adds
//               log-weights, keeps its own running max m_J and sum l_J in
//               registers (max updates that move by <= 16 in log2 units are
//               deferred, so O_J is rescaled only on large jumps) and writes
//               P as bf16 into TMEM.  The two groups never wait on each other
//               inside an item: each is an independent online softmax over its
//               half of the keys.  At the end of an item the two (m, l) of a
//               row are exchanged once through shared memory and each group
//               writes half of the output columns:
//                 O = (O_0 2^(m_0-m) + O_1 2^(m_1-m)) / (l_0 2^(m_0-m) + l_1 2^(m_1-m)).
//               The row sum adds the bf16-rounded P the tensor core
//               multiplies, not the fp32 values: numerator and denominator
//               then carry the same weights, so a dominant key's rounding
//               error scales with (v - O) instead of v (with a deferred
//               maximum its weight is not exactly 1, and summing fp32 P
//               doubled the output error).
// Every wait is bounded; a timeout raises STA_DEV_TIMEOUT, sets a CTA-wide
// abort flag and unwinds without trapping.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "sm100.cuh"

namespace sta {
namespace {

// Warp 0 Q/K producer, warp 1 QK issuer, warps 2-9 two softmax groups,
// warp 10 V producer, warp 11 PV issuer.
constexpr int kWarpV = 10;
constexpr int kWarpPV = 11;
constexpr int kThreads = 384;
constexpr int kHalfBytes = 128 * 128;  // 128 rows x 128 bytes: one 64-column half of a tile
constexpr float kLog2e = 1.4426950408889634f;

// Tuning constants (compile-time).
// Deferred rescale: the running row maximum moves (and O is rescaled) only
// when a tile's maximum exceeds it by more than this many log2 units.  P
// then stays below 2^16 (bf16 and the fp32 sums have the range to spare);
// 16 measured 2% faster than 8 on every workload (fewer waits for the
// previous tile's PV before a rescale).
#ifndef STA_RESCALE_THRESHOLD
#define STA_RESCALE_THRESHOLD 16.0f
#endif
constexpr float kRescaleThreshold = STA_RESCALE_THRESHOLD;
// Speculative row maximum (see softmax_role); 0 finds each tile's maximum
// before its exponentials.
#ifndef STA_SPEC_MAX
#define STA_SPEC_MAX 0
#endif
// K/V ring depths: two stages each, one per S buffer, so that a ring slot
// is free exactly when the MMA that read it has been committed (see the
// producers); deeper rings measured no faster.
#ifndef STA_KSTAGES
#define STA_KSTAGES 2
#endif
#ifndef STA_VSTAGES
#define STA_VSTAGES 2
#endif

template <int D, int KS, int VS>
struct Layout {
  static constexpr int DH = D / 64;
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + TILE_BYTES;
  static constexpr int OFF_V = OFF_K + KS * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_V + VS * TILE_BYTES;
  // barriers: q_full, q_empty, k_full[KS], v_full[VS], s_full[2],
  // p_full[2], o_done[2], o_free, mma_done, and the
  // (m, l) exchange barriers of the two softmax groups: lbar[4]
  static constexpr int NBAR = 2 + KS + VS + 8 + 4;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;  // room to align the base to 1024
};

struct Item {
  int head, kind, q_start, q_len, row, gbase, ntiles, unit, upt, cnt;
};

__device__ __forceinline__ Item decode_item(const AttnArgs& a, int it) {
  Item I;
  I.gbase = 0;
  I.row = -1;
  I.cnt = 0;
  if (a.mode == kModeRouted) {
    const int nd = a.heads * a.n_dense_items;
    if (it < nd) {
      I.head = it / a.n_dense_items;
      const int j = it - I.head * a.n_dense_items;
      I.kind = kItemGatherDense;
      I.gbase = j * kTileQ;
      I.q_start = 0;
      I.q_len = min(kTileQ, a.n_routed - I.gbase);
      I.unit = kTileK;
      I.upt = 1;
      I.ntiles = (a.N + kTileK - 1) / kTileK;
      return I;
    }
    it -= nd;
    I.kind = kItemLocal;
  } else {
    I.kind = (a.mode == kModeDense) ? kItemDense : kItemList;
  }
  I.head = it / a.n_qb;
  const int qb = it - I.head * a.n_qb;
  I.q_start = qb * a.block_q;
  I.q_len = min(a.block_q, a.N - I.q_start);
  if (I.kind == kItemDense) {
    I.unit = kTileK;
    I.upt = 1;
    I.ntiles = (a.N + kTileK - 1) / kTileK;
  } else {
    I.row = a.head_shared ? qb : I.head * a.n_qb + qb;
    I.unit = a.unit;
    I.upt = kTileK / a.unit;
    int c = __ldg(a.cnt + I.row);
    c = max(0, min(c, a.cap));
    I.cnt = c;
    I.ntiles = (c + I.upt - 1) / I.upt;
  }
  return I;
}

// Unit loaded into slot s of tile t of item I.  Returns the unit id to load
// (always a valid unit), the number of valid keys in the slot (0 for an
// empty slot or a bad list entry) and the entry's log-weight.
__device__ __forceinline__ int slot_unit(const AttnArgs& a, const Item& I, int t, int s,
                                         int& nvalid, float& lw, bool& bad) {
  lw = 0.f;
  bad = false;
  if (I.kind == kItemDense || I.kind == kItemGatherDense) {
    nvalid = min(kTileK, a.N - t * kTileK);
    return t;
  }
  const int pos = t * I.upt + s;
  if (pos >= I.cnt) {
    nvalid = 0;
    return 0;
  }
  const size_t off = static_cast<size_t>(I.row) * a.cap + pos;
  const int u = __ldg(a.idx + off);
  const int n_units = (a.N + I.unit - 1) / I.unit;
  if (u < 0 || u >= n_units) {
    nvalid = 0;
    bad = true;
    return 0;
  }
  nvalid = min(I.unit, a.N - u * I.unit);
  if (a.logw) lw = __ldg(a.logw + off);
  return u;
}

__device__ __forceinline__ void fail(volatile int* abort, int32_t* st) {
  *abort = 1;
  raise_status(st, STA_DEV_TIMEOUT);
}

// One softmax group's 64 logit columns of a tile, as SLOTS runs of
// W = min(UNIT, 64) columns; a 128-key unit contributes the half the group
// owns.  All per-column indices below are compile-time.
template <int UNIT>
struct HalfInfo {
  static constexpr int W = UNIT < 64 ? UNIT : 64;
  static constexpr int SLOTS = 64 / W;
  int lim[SLOTS];     // valid columns of the slot (keys past N / empty slots masked)
  float braw[SLOTS];  // log-weight / scale: added to raw logits
  int tok0[SLOTS];    // key token of the slot's first column
  bool full, bias;
};

template <int UNIT>
__device__ __forceinline__ void load_half_info(const AttnArgs& a, const Item& I, int t, int J,
                                               float inv_scale, HalfInfo<UNIT>& hi) {
  constexpr int W = HalfInfo<UNIT>::W;
  hi.full = true;
  hi.bias = (a.logw != nullptr) && (I.kind == kItemList || I.kind == kItemLocal);
#pragma unroll
  for (int s = 0; s < HalfInfo<UNIT>::SLOTS; ++s) {
    const int col = J * 64 + s * W;  // first tile column of the slot
    const int gs = col / UNIT;       // the tile's slot (list position)
    const int off = col - gs * UNIT;  // column offset inside that unit
    int nv;
    float lw;
    bool bad;
    const int u = slot_unit(a, I, t, gs, nv, lw, bad);
    const int lim = min(max(nv - off, 0), W);
    hi.lim[s] = lim;
    hi.braw[s] = lw * inv_scale;
    hi.tok0[s] = u * UNIT + off;
    if (lim < W) hi.full = false;
  }
}

// The list entries (unit id, log-weight) of one group's slots of a tile,
// loaded one tile ahead so that their latency hides behind the current tile.
template <int UNIT>
struct HalfRaw {
  int u[HalfInfo<UNIT>::SLOTS];  // unit id, or -1 past the end of the row
  float lw[HalfInfo<UNIT>::SLOTS];
};

template <int UNIT>
__device__ __forceinline__ void load_half_raw(const AttnArgs& a, const Item& I, int t, int J,
                                              HalfRaw<UNIT>& hr) {
  constexpr int W = HalfInfo<UNIT>::W;
#pragma unroll
  for (int s = 0; s < HalfInfo<UNIT>::SLOTS; ++s) {
    const int gs = (J * 64 + s * W) / UNIT;
    const int pos = t * I.upt + gs;
    hr.u[s] = -1;
    hr.lw[s] = 0.f;
    if (t < I.ntiles && pos < I.cnt) {
      const size_t off = static_cast<size_t>(I.row) * a.cap + pos;
      hr.u[s] = __ldg(a.idx + off);
      if (a.logw) hr.lw[s] = __ldg(a.logw + off);
    }
  }
}

// HalfInfo of a list tile from its prefetched entries (same rules as
// load_half_info: out-of-range ids mask their slot).
template <int UNIT>
__device__ __forceinline__ void half_info_from_raw(const AttnArgs& a, const Item& I, int J,
                                                   float inv_scale, const HalfRaw<UNIT>& hr,
                                                   HalfInfo<UNIT>& hi) {
  constexpr int W = HalfInfo<UNIT>::W;
  const int n_units = (a.N + UNIT - 1) / UNIT;
  hi.full = true;
  hi.bias = (a.logw != nullptr) && (I.kind == kItemList || I.kind == kItemLocal);
#pragma unroll
  for (int s = 0; s < HalfInfo<UNIT>::SLOTS; ++s) {
    const int col = J * 64 + s * W;
    const int off = col - (col / UNIT) * UNIT;
    const int u = hr.u[s];
    const bool ok = u >= 0 && u < n_units;
    const int nv = ok ? min(UNIT, a.N - u * UNIT) : 0;
    const int lim = min(max(nv - off, 0), W);
    hi.lim[s] = lim;
    hi.braw[s] = ok ? hr.lw[s] * inv_scale : 0.f;
    hi.tok0[s] = (ok ? u : 0) * UNIT + off;
    if (lim < W) hi.full = false;
  }
}

// The local window of one query row ("Where Compute Matters: Heterogeneous
// Attention for Efficient Video Diffusion", Abstract: easy tokens attend to a
// spatiotemporal neighbourhood): key (f, h, w) is inside iff |f - fq| <=
// win_f, -win_h <= h - hq < win_h and -win_w <= w - wq < win_w, with
// (fq, hq, wq) the query's grid position.
struct WinGeom {
  int fq, hq, wq;
};

// Bit c (c < n <= 64) set iff the key c places after grid position (f, h,
// w) in raster order lies in the window.  The keys are walked as runs
// within one grid row, one column interval per run: a run ends at the row's
// end, so a slot of n <= W keys is one or two runs.
__device__ __forceinline__ uint64_t window_bits(int f, int h, int w, int n, const AttnArgs& a,
                                                const WinGeom& g) {
  uint64_t bits = 0;
  for (int c0 = 0; c0 < n;) {
    const int run = min(a.W - w, n - c0);
    const int df = f - g.fq, dh = h - g.hq;
    if (df <= a.win_f && df >= -a.win_f && dh >= -a.win_h && dh < a.win_h) {
      // run columns [lo, hi): keys w + lo .. w + hi - 1 of this row
      const int lo = max(g.wq - a.win_w - w, 0);
      const int hi = min(g.wq + a.win_w - w, run);
      if (hi > lo) {
        const int len = hi - lo;
        const uint64_t ones = len >= 64 ? ~0ull : ((1ull << len) - 1ull);
        bits |= ones << (c0 + lo);
      }
    }
    c0 += run;
    w = 0;
    if (++h == a.H) {
      h = 0;
      ++f;
    }
  }
  return bits;
}

// Masks (partial units, key tokens past N) and the local window on one
// group's 64 logit columns.  Log-weights are not added here: they are
// constant per slot, so the caller folds them into the per-slot maxima and
// into the exponent's offset.
template <int UNIT>
__device__ __forceinline__ void mask_half(float (&x)[64], const HalfInfo<UNIT>& hi, bool window,
                                          const uint64_t* wbits) {
  constexpr int W = HalfInfo<UNIT>::W;
  if (!hi.full) {
#pragma unroll
    for (int c = 0; c < 64; ++c)
      if ((c % W) >= hi.lim[c / W]) x[c] = -INFINITY;
  }
  if (window) {
    // Per slot: the bit set of the columns whose keys lie in the query's
    // window (window_bits, formed by the caller), applied column by column.
#pragma unroll
    for (int sl = 0; sl < HalfInfo<UNIT>::SLOTS; ++sl) {
      const uint64_t bits = wbits[sl];
#pragma unroll
      for (int c = 0; c < W; ++c)
        if (!((bits >> c) & 1ull)) x[sl * W + c] = -INFINITY;
    }
  }
}

struct SoftmaxShared {
  uint64_t* s_full;  // [2]: S buffer J holds the logits of the current tile of parity J
  uint64_t* p_full;  // [2]: 8 arrivals (one per softmax warp), P of the tile in
                     // S buffer J is in TMEM
  uint64_t* o_done;  // [2]: the PV into O_J of the last committed tile has completed
  uint64_t* o_free;  // 8 arrivals: both O accumulators have been read out
  uint64_t* lbar;    // [4 quadrants], 2 arrivals: (m, l) exchange of an item
  volatile int* abort;
};

__device__ __forceinline__ float nan_flag() { return __int_as_float(0x7fc00000); }

// Exponentials of one 64-column half: p = 2^(x*scale_log2 + off[s]) with the
// offset off[s] = log-weight - m of the column's slot (W columns each), packed
// to bf16 pairs; the row sum adds the rounded values.  The scale-and-shift and
// the running sums use the paired fp32 instructions (two lanes of work per
// instruction).  The packed pairs are stored into TMEM at taddr (this
// thread's lane) in two 16-word chunks as they are formed, so that the first
// chunk's store overlaps the second chunk's arithmetic.  Also returns, in
// amax, the largest exponent argument: the tile's maximum relative to the
// maximum the offsets were formed with (-inf when every column is masked).
template <int W, bool ENT = false>
__device__ __forceinline__ float exp_store_half(const float (&x)[64], float scale_log2,
                                                const float (&off)[64 / W], bool simple,
                                                uint32_t taddr, float& amax, float& zt,
                                                float& at) {
  const float2 sl = make_float2(scale_log2, scale_log2);
  float2 acc[4];
  float mx[4];
  float2 ez = make_float2(0.f, 0.f), ea = make_float2(0.f, 0.f);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    acc[j] = make_float2(0.f, 0.f);
    mx[j] = -INFINITY;
  }
#pragma unroll
  for (int ch = 0; ch < 2; ++ch) {
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int c = ch * 32 + 2 * i;
      const float o = off[c / W];
      const float2 arg = __ffma2_rn(make_float2(x[c], x[c + 1]), sl, make_float2(o, o));
      mx[i & 3] = fmax3(mx[i & 3], arg.x, arg.y);
      (void)simple;
      const float p0 = fast_exp2(arg.x);
      const float p1 = fast_exp2(arg.y);
      pk[i] = pack_bf16x2(p0, p1);
      acc[i & 3] = __fadd2_rn(acc[i & 3], make_float2(bf16_lo(pk[i]), bf16_hi(pk[i])));
      if constexpr (ENT) {
        // entropy terms from the unrounded p: sum p and sum p * (y - m) (log2
        // units; masked columns have p = 0 and a clamped argument)
        const float2 pp = make_float2(p0, p1);
        ez = __fadd2_rn(ez, pp);
        ea = __ffma2_rn(pp, make_float2(fmaxf(arg.x, -256.f), fmaxf(arg.y, -256.f)), ea);
      }
    }
    tmem_st16(taddr + ch * 16, pk);
  }
  zt = ez.x + ez.y;
  at = ea.x + ea.y;
  amax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
  const float2 s01 = __fadd2_rn(acc[0], acc[1]), s23 = __fadd2_rn(acc[2], acc[3]);
  const float2 t = __fadd2_rn(s01, s23);
  return t.x + t.y;
}

// O_J *= f (this thread's row): D/32 chunks of 32 columns through registers.
template <int D>
__device__ __forceinline__ void rescale_o(uint32_t tO, float f) {
#pragma unroll
  for (int ch = 0; ch < D / 32; ++ch) {
    uint32_t v[32];
    tmem_ld32(tO + ch * 32, v);
    tmem_wait_ld();
    tmem_regs_ready(v);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * f);
    tmem_st32(tO + ch * 32, v);
  }
}

// Largest logit of each W-column slot.
template <int W>
__device__ __forceinline__ void slot_max(const float (&x)[64], float (&ms)[64 / W]) {
  constexpr int A = W >= 32 ? 8 : 4;  // independent max chains per slot
#pragma unroll
  for (int s = 0; s < 64 / W; ++s) {
    float mv[A];
#pragma unroll
    for (int j = 0; j < A; ++j) mv[j] = x[s * W + j];
#pragma unroll
    for (int c = A; c < W; ++c) mv[c % A] = fmaxf(mv[c % A], x[s * W + c]);
#pragma unroll
    for (int j = A / 2; j > 0; j /= 2)
#pragma unroll
      for (int i = 0; i < j; ++i) mv[i] = fmaxf(mv[i], mv[i + j]);
    ms[s] = mv[0];
  }
}

// Loads 64 consecutive TMEM columns starting at taddr (this thread's lane).
__device__ __forceinline__ void load_cols64(uint32_t taddr, float (&x)[64]) {
  uint32_t v0[32], v1[32];
  tmem_ld32(taddr, v0);
  tmem_ld32(taddr + 32, v1);
  tmem_wait_ld();
  tmem_regs_ready(v0);
  tmem_regs_ready(v1);
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    x[i] = __uint_as_float(v0[i]);
    x[32 + i] = __uint_as_float(v1[i]);
  }
}

// Softmax warpgroup J (4 warps): keys [64J, 64J+64) of every tile, query
// row r = 32*quadrant + lane per thread, accumulator O_J (see the file
// comment).
template <int D, int UNIT, bool ENT, bool WIN>
__device__ __forceinline__ void softmax_role(const AttnArgs& a, const SoftmaxShared& sh,
                                             uint32_t tmem, int warp, int lane, int J) {
  constexpr int OH = D / 2;     // output columns per group
  const int OB = J * OH;        // first output column of this group
  const int quad = warp & 3;
  const int r = quad * 32 + lane;
  const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
  const uint32_t tO = tmem + lane_off + 256 + J * D;
  const float scale_log2 = a.scale_log2;
  const float inv_scale = kLog2e / scale_log2;  // natural-log weight -> raw logit units
  const uint64_t limit = kWaitLimitNs;
  volatile int* abort = sh.abort;
  // (m, l) of each row exchanged by the two groups at the end of an item
  // (with the entropy terms z, a): [group][row]
  __shared__ __align__(16) float4 xch4[ENT ? 256 : 1];
  __shared__ __align__(16) float2 xch2[ENT ? 1 : 256];
  uint32_t g = 0, nitem = 0;
  bool ok = true;
  for (int it = blockIdx.x; it < a.n_items && ok; it += gridDim.x) {
    if (__any_sync(0xffffffffu, *abort != 0)) break;
    const Item I = decode_item(a, it);
    int tok = -1;
    if (I.kind == kItemGatherDense) {
      // caller-supplied routed ids: an id outside [0, N) is skipped (its row
      // neither read nor written) and reported
      if (r < I.q_len) {
        tok = __ldg(a.routed_ids + I.gbase + r);
        if (tok < 0 || tok >= a.N) {
          if (J == 0) raise_status(a.dev_status, STA_DEV_BAD_INDEX);
          tok = -1;
        }
      }
    } else if (r < I.q_len) {
      tok = I.q_start + r;
    }
    bool active = tok >= 0;
    if (active && !dcheck(tok < a.N, a.dev_status)) active = false;
    if (active && I.kind == kItemLocal && __ldg(a.routed_flag + tok)) active = false;
    const size_t orow = static_cast<size_t>(I.head) * a.N + (tok < 0 ? 0 : tok);
    if (I.ntiles == 0) {
      if (active) {
        if (a.out_f32) {
          float4* op = reinterpret_cast<float4*>(static_cast<float*>(a.o) + orow * D + OB);
          for (int i = 0; i < OH / 4; ++i) op[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        } else {
          uint4* op =
              reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.o) + orow * D + OB);
          for (int i = 0; i < OH / 8; ++i) op[i] = make_uint4(0, 0, 0, 0);
        }
        raise_status(a.dev_status, STA_DEV_EMPTY_ROW);
      }
      continue;
    }
    // the local-window code exists only in the routed kernels (WIN)
    const bool window = WIN && (I.kind == kItemLocal);
    WinGeom wg{0, 0, 0};
    if (window && tok >= 0) {
      const int S = a.H * a.W;
      wg.fq = tok / S;
      const int rem = tok - wg.fq * S;
      wg.hq = rem / a.W;
      wg.wq = rem - wg.hq * a.W;
    }
    const bool dense_like = (I.kind == kItemDense || I.kind == kItemGatherDense);
    const bool weighted = !dense_like && a.logw != nullptr;
    const int n_full = a.N / UNIT;  // units whose keys all lie below N
    const int n_units = (a.N + UNIT - 1) / UNIT;
    float m_run = -INFINITY, l_run = 0.f;
    float z_run = 0.f, a_run = 0.f;  // entropy terms (ENT): sum p, sum p (y - m)
    HalfRaw<UNIT> raw_next;
    if (!dense_like) load_half_raw<UNIT>(a, I, 0, J, raw_next);
    for (int t = 0; t < I.ntiles; ++t) {
      const uint32_t gg = g + t;
      const uint32_t sb = gg & 1;
      const uint32_t tS = tmem + lane_off + sb * 128;
      if (!dcheck(tmem_in_range(tS + J * 64, tmem, 64) && tmem_in_range(tO, tmem, D),
                  a.dev_status)) {
        ok = false;
        break;
      }
      // Only the raw entries stay live across the tile; the per-slot masks
      // are derived from them on the (rare) masked path.
      HalfRaw<UNIT> raw = {};
      bool full;  // every column of the group's half is a valid key
      if (dense_like) {
        full = (t * kTileK + J * 64 + 64 <= a.N);
      } else {
        raw = raw_next;
        full = true;
#pragma unroll
        for (int q = 0; q < HalfInfo<UNIT>::SLOTS; ++q)
          full = full && (static_cast<unsigned>(raw.u[q]) < static_cast<unsigned>(n_full));
        load_half_raw<UNIT>(a, I, t + 1, J, raw_next);  // next tile's entries
      }
      const bool simple = full && !weighted && !window;  // no mask, no weight
      constexpr int SW = HalfInfo<UNIT>::W, NS = HalfInfo<UNIT>::SLOTS;
      // Local items: this row's window columns of each slot.  The grid
      // position of slot q's first key is the same for every row: lane q
      // forms it (one division sequence for all slots) and the warp reads
      // it by shuffle; each row then walks the slot's row runs.
      uint64_t wbits[NS];
      if (window) {
        int t0_mine = 0;
#pragma unroll
        for (int q = 0; q < NS; ++q) {
          const int col = J * 64 + q * SW;
          const int u = static_cast<unsigned>(raw.u[q]) < static_cast<unsigned>(n_units)
                            ? raw.u[q] : 0;
          if (lane == q) t0_mine = u * UNIT + (col - (col / UNIT) * UNIT);
        }
        const int S = a.H * a.W;
        const int f_m = t0_mine / S;
        const int rem = t0_mine - f_m * S;
        const int h_m = rem / a.W;
        const int w_m = rem - h_m * a.W;
#pragma unroll
        for (int q = 0; q < NS; ++q)
          wbits[q] = window_bits(__shfl_sync(0xffffffffu, f_m, q),
                                 __shfl_sync(0xffffffffu, h_m, q),
                                 __shfl_sync(0xffffffffu, w_m, q), SW, a, wg);
      }
      if (!__all_sync(0xffffffffu,
                      mbar_wait(sh.s_full + sb, (gg >> 1) & 1, abort, limit))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float x[64];
      load_cols64(tS + J * 64, x);
      if (!full || window) {
        if (dense_like) {
          HalfInfo<kTileK> td;
          load_half_info<kTileK>(a, I, t, J, inv_scale, td);  // geometry only, no loads
          mask_half<kTileK>(x, td, false, nullptr);
        } else {
          HalfInfo<UNIT> ti;
          half_info_from_raw<UNIT>(a, I, J, inv_scale, raw, ti);
          mask_half<UNIT>(x, ti, window, wbits);
        }
      }
      // per-slot log-weights (raw logit units), 0 without weights (a masked
      // slot's value does not matter: its logits are -inf)
      float bias[NS];
#pragma unroll
      for (int q = 0; q < NS; ++q)
        bias[q] = (weighted && static_cast<unsigned>(raw.u[q]) < static_cast<unsigned>(n_units))
                      ? raw.lw[q] * inv_scale
                      : 0.f;
#if STA_SPEC_MAX
      // Speculative maximum: once every row of the warp has a finite running
      // maximum, the exponentials are formed against it straight away and
      // the tile's maximum comes out of the same pass; a row whose maximum
      // rose by more than the deferral threshold (the condition under which
      // O_J is rescaled) forms them again after the rescale.
      const bool spec = __all_sync(0xffffffffu, m_run != -INFINITY);
#else
      const bool spec = false;
#endif
      if (!spec) {
        float ms[NS];
        slot_max<SW>(x, ms);
        float mraw = ms[0] + bias[0];
#pragma unroll
        for (int q = 1; q < NS; ++q) mraw = fmaxf(mraw, ms[q] + bias[q]);
        const float m_tile = mraw * scale_log2;  // -inf if all masked
        const float m_new = fmaxf(m_run, m_tile);
        const bool need = (m_run != -INFINITY) && (m_new > m_run + kRescaleThreshold);
        if (__any_sync(0xffffffffu, need)) {
          // O_J holds tiles < t of this item; the last of them (tile gg - 1)
          // must be accumulated before O_J is rescaled.
          const uint32_t gp = gg - 1;
          if (!__all_sync(0xffffffffu,
                          mbar_wait(sh.o_done + (gp & 1), (gp >> 1) & 1, abort, limit))) {
            ok = false;
            break;
          }
          tc_fence_after();
          rescale_o<D>(tO, need ? fast_exp2(m_run - m_new) : 1.f);
          tmem_wait_st();
          if (need) {
            const float f = fast_exp2(m_run - m_new);
            l_run *= f;
            if constexpr (ENT) {
              a_run = f * fmaf(m_run - m_new, z_run, a_run);
              z_run *= f;
            }
            m_run = m_new;
          }
        }
        if (m_run == -INFINITY) m_run = m_new;
      }
      const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
      // P of this group's 64 keys, packed over the first 32 of its (already
      // read) logit columns
      float off[NS];
#pragma unroll
      for (int q = 0; q < NS; ++q) off[q] = fmaf(bias[q], scale_log2, -m_use);
      float amax, zt, at;
      float lsum = exp_store_half<SW, ENT>(x, scale_log2, off, simple, tS + J * 64, amax, zt, at);
      if (spec) {
        const bool redo = amax > kRescaleThreshold;
        if (__any_sync(0xffffffffu, redo)) {
          const uint32_t gp = gg - 1;  // as above: t >= 1 here
          if (!__all_sync(0xffffffffu,
                          mbar_wait(sh.o_done + (gp & 1), (gp >> 1) & 1, abort, limit))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float f = redo ? fast_exp2(-amax) : 1.f;
          rescale_o<D>(tO, f);
          tmem_wait_st();  // also orders the first pass's P stores before the second's
          if (redo) {
            l_run *= f;
            if constexpr (ENT) {
              a_run = f * fmaf(-amax, z_run, a_run);
              z_run *= f;
            }
            m_run += amax;
#pragma unroll
            for (int q = 0; q < NS; ++q) off[q] -= amax;
          }
          lsum = exp_store_half<SW, ENT>(x, scale_log2, off, simple, tS + J * 64, amax, zt, at);
        }
      }
      l_run += lsum;
      if constexpr (ENT) {
        z_run += zt;
        a_run += at;
      }
      // One arrival per warp, after every lane's stores have completed (a
      // barrier word takes its arrivals one at a time).
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sh.p_full + sb);
    }
    if (!ok) break;
    // ------------------------------------------------------------ epilogue
    const uint32_t gl = g + I.ntiles - 1;  // last tile of the item
    // The two groups exchange (m, l) of each row through shared memory, so
    // that no S buffer is held by the epilogue and the next item's QK
    // products need not wait for it.  A group rewrites its slot only at the
    // end of its next item, after the other group has read this one (it
    // took part in every tile of that item).
    if constexpr (ENT)
      xch4[J * 128 + r] = make_float4(m_run, l_run, z_run, a_run);
    else
      xch2[J * 128 + r] = make_float2(m_run, l_run);
    __syncwarp();
    if (lane == 0) mbar_arrive(sh.lbar + quad);
    bool okw = __all_sync(0xffffffffu, mbar_wait(sh.lbar + quad, nitem & 1, abort, limit));
    float mo = 0.f, lo = 0.f, zo = 0.f, ao = 0.f;
    if (okw) {
      if constexpr (ENT) {
        const float4 xo = xch4[(1 - J) * 128 + r];
        mo = xo.x;
        lo = xo.y;
        zo = xo.z;
        ao = xo.w;
      } else {
        const float2 xo = xch2[(1 - J) * 128 + r];
        mo = xo.x;
        lo = xo.y;
      }
    }
    // the commit after the item's last PV covers every earlier MMA
    if (okw)
      okw = __all_sync(0xffffffffu,
                       mbar_wait(sh.o_done + (gl & 1), (gl >> 1) & 1, abort, limit));
    g += I.ntiles;
    ++nitem;
    if (!okw) {
      ok = false;
      break;
    }
    tc_fence_after();
    const float m0 = J == 0 ? m_run : mo, m1 = J == 0 ? mo : m_run;
    const float l0 = J == 0 ? l_run : lo, l1 = J == 0 ? lo : l_run;
    const float m = fmaxf(m0, m1);
    const float f0 = (m0 != -INFINITY) ? fast_exp2(m0 - m) : 0.f;
    const float f1 = (m1 != -INFINITY) ? fast_exp2(m1 - m) : 0.f;
    const float l_tot = l0 * f0 + l1 * f1;
    const bool empty = !(l_tot > 0.f);
    const float inv_l = empty ? 0.f : 1.f / l_tot;
    const float c0 = f0 * inv_l, c1 = f1 * inv_l;
    if (J == 0 && active && empty) raise_status(a.dev_status, STA_DEV_EMPTY_ROW);
    if constexpr (ENT) {
      // H = ln Z - ln 2 * A / Z over both groups' keys, with Z = sum p and
      // A = sum p (y - m) brought to the common maximum m (log2 units)
      if (J == 0 && active && a.entropy) {
        const float z0 = J == 0 ? z_run : zo, z1 = J == 0 ? zo : z_run;
        const float a0 = J == 0 ? a_run : ao, a1 = J == 0 ? ao : a_run;
        float Z = 0.f, A = 0.f;
        if (f0 > 0.f) {
          Z = fmaf(f0, z0, Z);
          A = fmaf(f0, fmaf(m0 - m, z0, a0), A);
        }
        if (f1 > 0.f) {
          Z = fmaf(f1, z1, Z);
          A = fmaf(f1, fmaf(m1 - m, z1, a1), A);
        }
        const float H = Z > 0.f ? logf(Z) - 0.6931471805599453f * (A / Z) : 0.f;
        a.entropy[orow] = H;
      }
    }
    if (!dcheck(tmem_in_range(tmem + lane_off + 256 + OB, tmem, OH) &&
                    tmem_in_range(tmem + lane_off + 256 + D + OB, tmem, OH),
                a.dev_status)) {
      ok = false;
      break;
    }
#pragma unroll
    for (int ch = 0; ch < OH / 32; ++ch) {
      const uint32_t col = tmem + lane_off + 256 + OB + ch * 32;
      float o[32];
      uint32_t v[32];
      tmem_ld32(col, v);
      tmem_wait_ld();
      tmem_regs_ready(v);
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] = __uint_as_float(v[i]) * c0;
      tmem_ld32(col + D, v);
      tmem_wait_ld();
      tmem_regs_ready(v);
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] = fmaf(__uint_as_float(v[i]), c1, o[i]);
      if (active) {
        const size_t gcol = orow * D + OB + ch * 32;
        if (a.out_f32) {
          float4* op = reinterpret_cast<float4*>(static_cast<float*>(a.o) + gcol);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            __stcs(op + i, make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]));
        } else {
          uint4* op = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.o) + gcol);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            __stcs(op + i, make_uint4(pack_bf16x2(o[8 * i], o[8 * i + 1]),
                                      pack_bf16x2(o[8 * i + 2], o[8 * i + 3]),
                                      pack_bf16x2(o[8 * i + 4], o[8 * i + 5]),
                                      pack_bf16x2(o[8 * i + 6], o[8 * i + 7])));
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(sh.o_free);
  }
  if (!ok) fail(abort, a.dev_status);
}

// Slot s of a K or V tile in the interleaved layout ([8-row group][half]
// [8 rows][128 B]): one copy through the five-dimensional view when the
// unit lies in whole 8-row groups below N & ~7 (u < n_il), else 8-row copies
// per half through the three-dimensional map, which zero-fills rows past N.
template <int UNIT>
__device__ __forceinline__ void load_unit_il(uint8_t* tile, const CUtensorMap* m_il,
                                             const CUtensorMap* m8, uint64_t* bar, int s, int u,
                                             int n_il, int head, uint64_t pol) {
  constexpr int G = UNIT / 8;  // 8-row groups per unit
  uint8_t* dst = tile + s * G * 2048;
  if (u < n_il) {
    tma_load_5d_hint(dst, m_il, bar, 0, 0, 0, u * G, head, pol);
  } else {
#pragma unroll
    for (int j = 0; j < G; ++j)
#pragma unroll
      for (int h = 0; h < 2; ++h)
        tma_load_3d_hint(dst + j * 2048 + h * 1024, m8, bar, h * 64, u * UNIT + 8 * j, head, pol);
  }
}

template <int D, int KS, int VS, int UNIT, bool ENT, bool WIN>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ AttnArgs a, const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k_u,
                    const __grid_constant__ CUtensorMap tm_v_u,
                    const __grid_constant__ CUtensorMap tm_k_f,
                    const __grid_constant__ CUtensorMap tm_v_f,
                    const __grid_constant__ CUtensorMap tm_k_il,
                    const __grid_constant__ CUtensorMap tm_v_il) {
  using L = Layout<D, KS, VS>;
  static_assert(KS == 2 && VS == 2, "ring slots are released by the S-full / O-done commits");
  // d = 128 with 16-key units: list tiles use the interleaved layout
  // [8-row group][half][8 rows][128 B], one TMA copy per unit (two 2 KB
  // copies per unit, one per half, measured 18% slower; from 32 keys up the
  // per-half copies are the faster form)
  constexpr bool kInterleaved = (D == 128 && UNIT < 32);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  uint8_t* sQ = smem + L::OFF_Q;
  uint8_t* sK = smem + L::OFF_K;
  uint8_t* sV = smem + L::OFF_V;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;
  uint64_t* v_full = k_full + KS;
  uint64_t* s_full = v_full + VS;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_done = p_full + 2;
  uint64_t* o_free = o_done + 2;
  uint64_t* mma_done = o_free + 1;
  uint64_t* lbar = mma_done + 1;  // [4]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < KS; ++i) {
      mbar_init(k_full + i, 1);
    }
    for (int i = 0; i < VS; ++i) {
      mbar_init(v_full + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(p_full + i, 8);  // both softmax groups write P of every tile
      mbar_init(o_done + i, 1);
    }
    mbar_init(o_free, 8);
    mbar_init(mma_done, 2);  // one commit from each issuer
    for (int i = 0; i < 4; ++i) mbar_init(lbar + i, 2);
    *abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k_u);
    tma_prefetch_desc(&tm_v_u);
    tma_prefetch_desc(&tm_k_f);
    tma_prefetch_desc(&tm_v_f);
    if (kInterleaved) {
      tma_prefetch_desc(&tm_k_il);
      tma_prefetch_desc(&tm_v_il);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint64_t limit = kWaitLimitNs;
  int dummy_abort_storage = 0;
  volatile int* no_abort = &dummy_abort_storage;

  if (warp == 0 || warp == kWarpV) {
    // ----------------------------------------------------------- producers
    // Warp 0 loads the Q tile of each item and the K tiles, warp kWarpV the
    // V tiles, each into its own ring, so that a V copy never waits behind
    // a K slot.  K/V tiles are read by every query block of a head: keep
    // them in L2 ahead of the Q tiles, which are read once.
    const bool is_v = (warp == kWarpV);
    const uint64_t pol_kv = l2_policy_evict_last();
    const uint64_t pol_q = l2_policy_evict_first();
    const uint32_t RS = is_v ? VS : KS;
    uint64_t* ring_full = is_v ? v_full : k_full;
    // Slot n % 2 of the K ring is free once the QK of tile n-2 has
    // completed, which is the S-full commit of that tile (S buffer n % 2);
    // likewise the V ring's slot once the PV of tile n-2 has completed (its
    // O-done commit).  The next phase of either barrier needs tile n's copy,
    // so a wait can never see a phase further on.  Sharing the commits
    // halves the tcgen05.commit count per tile.
    uint64_t* ring_empty = is_v ? o_done : s_full;
    uint8_t* ring = is_v ? sV : sK;
    const CUtensorMap* m_il = is_v ? &tm_v_il : &tm_k_il;
    uint32_t n = 0, qn = 0;  // tiles issued into the ring, items
    int ok = 1;
    for (int it = blockIdx.x; it < a.n_items; it += gridDim.x) {
      if (__any_sync(0xffffffffu, *abort != 0)) break;
      const Item I = decode_item(a, it);
      if (I.ntiles == 0) continue;
      if (!is_v) {
        if (lane == 0) ok = mbar_wait(q_empty, (qn & 1) ^ 1, abort, limit);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
          if (lane == 0) fail(abort, a.dev_status);
          break;
        }
        if (I.kind == kItemGatherDense) {
          // Gather the routed query rows and store them in the 128-byte
          // swizzled layout TMA would produce (16-byte chunk c of row r sits
          // at chunk c ^ (r % 8) of the row).
          const __nv_bfloat16* qh = a.q + static_cast<size_t>(I.head) * a.N * D;
          for (int r = lane; r < kTileQ; r += 32) {
            const int src_r = (r < I.q_len) ? r : 0;
            int tok = __ldg(a.routed_ids + I.gbase + src_r);
            // an out-of-range id (reported by the softmax warps, which skip
            // its row) reads token 0 instead
            if (tok < 0 || tok >= a.N) tok = 0;
            const uint4* src = reinterpret_cast<const uint4*>(qh + static_cast<size_t>(tok) * D);
#pragma unroll
            for (int c = 0; c < D / 8; ++c) {
              const int h = c >> 3, cc = c & 7;
              uint4 val = __ldg(src + c);
              *reinterpret_cast<uint4*>(sQ + h * kHalfBytes + r * 128 + ((cc ^ (r & 7)) << 4)) =
                  val;
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(q_full);
        } else if (lane == 0) {
          mbar_arrive_expect_tx(q_full, L::TILE_BYTES);
#pragma unroll
          for (int h = 0; h < L::DH; ++h)
            tma_load_3d_hint(sQ + h * kHalfBytes, &tm_q, q_full, h * 64, I.q_start, I.head,
                             pol_q);
        }
        ++qn;
      }
      const bool dense_like = (I.kind == kItemDense || I.kind == kItemGatherDense);
      const CUtensorMap* mt =
          dense_like ? (is_v ? &tm_v_f : &tm_k_f) : (is_v ? &tm_v_u : &tm_k_u);
      const int unit = I.unit;
      const bool il = kInterleaved && !dense_like;
      const int nops = il ? I.upt : I.upt * L::DH;
      const int n_il = (a.N & ~7) / UNIT;  // units the interleaved view covers
      const int n_units = (a.N + unit - 1) / unit;
      // one lane per (slot, half) copy, or per slot in the interleaved layout
      const int s = il ? lane : lane / L::DH, h = il ? 0 : lane % L::DH;
      // List entries are fetched one tile ahead, so that their load latency
      // is not on the path from a free ring slot to the copies into it.
      auto fetch = [&](int t, int& e, bool& present) {
        present = false;
        e = 0;
        if (!dense_like && lane < nops && t < I.ntiles) {
          const int pos = t * I.upt + s;
          if (pos < I.cnt) {
            present = true;
            e = __ldg(a.idx + static_cast<size_t>(I.row) * a.cap + pos);
          }
        }
      };
      int e_next;
      bool p_next;
      fetch(0, e_next, p_next);
      for (int t = 0; t < I.ntiles; ++t) {
        int u = 0;
        if (lane < nops) {
          if (dense_like) {
            u = t;
          } else {
            const int e = e_next;
            const bool present = p_next;
            fetch(t + 1, e_next, p_next);
            // an out-of-range entry loads unit 0 (the softmax masks its slot)
            const bool valid = present && e >= 0 && e < n_units &&
                               dcheck(e * unit < a.N, a.dev_status);
            if (present && !valid && !is_v) raise_status(a.dev_status, STA_DEV_BAD_INDEX);
            u = valid ? e : 0;
          }
        }
        const uint32_t st = n % RS;
        if (lane == 0) ok = mbar_wait(ring_empty + st, ((n / RS) & 1) ^ 1, abort, limit);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (lane == 0) mbar_arrive_expect_tx(ring_full + st, L::TILE_BYTES);
        __syncwarp();
        if (il) {
          if (lane < nops)
            load_unit_il<UNIT>(ring + st * L::TILE_BYTES, m_il, mt, ring_full + st, s, u, n_il,
                               I.head, pol_kv);
        } else if (lane < nops) {
          tma_load_3d_hint(ring + st * L::TILE_BYTES + h * kHalfBytes + s * unit * 128, mt,
                           ring_full + st, h * 64, u * unit, I.head, pol_kv);
        }
        ++n;
      }
      if (!ok) {
        if (lane == 0) fail(abort, a.dev_status);
        break;
      }
    }
    // Let every copy this warp issued land before the CTA can exit.
    if (lane == 0)
      for (uint32_t i = (n > RS ? n - RS : 0); i < n; ++i)
        mbar_wait(ring_full + (i % RS), (i / RS) & 1, no_abort, limit);
    __syncwarp();
  } else if (warp == 1) {
    // ----------------------------------------------------------- QK issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK);
      uint32_t kt = 0, qn = 0, g = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < a.n_items && ok; it += gridDim.x) {
        if (*abort) break;
        const Item I = decode_item(a, it);
        if (I.ntiles == 0) continue;
        if (!mbar_wait(q_full, qn & 1, abort, limit)) {
          ok = false;
          break;
        }
        // K tiles of the current item are in the interleaved layout: 8-row
        // groups 2048 bytes apart, halves 1024 apart (else 1024 and 16384)
        const bool il = kInterleaved && (I.kind == kItemList || I.kind == kItemLocal);
        for (int t = 0; t < I.ntiles; ++t) {
          const uint32_t gg = g + t;
          const uint32_t sb = gg & 1;
          const int st = kt % KS;
          if (!mbar_wait(k_full + st, (kt / KS) & 1, abort, limit)) {
            ok = false;
            break;
          }
          // S buffer sb holds P of tile gg - 2 until the PV that reads it
          // has completed (the PV issuer commits o_done[sb] after it; that
          // PV cannot complete twice before this QK, which its successor
          // needs, is issued)
          if (gg >= 2 && !mbar_wait(o_done + sb, ((gg - 2) >> 1) & 1, abort, limit)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t tS = tmem + sb * 128;
          if (!dcheck(tmem_in_range(tS, tmem, 128), a.dev_status)) {
            ok = false;
            break;
          }
          const uint32_t kbase = aK + st * L::TILE_BYTES;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
            const uint64_t adesc = smem_desc_sw128(aQ + off, 16, 1024);
            const uint64_t bdesc =
                il ? smem_desc_sw128(kbase + (kk >> 2) * 1024 + (kk & 3) * 32, 16, 2048)
                   : smem_desc_sw128(kbase + off, 16, 1024);
            mma_bf16_ss(tS, adesc, bdesc, IDESC_QK, kk > 0 ? 1u : 0u);
          }
          ++kt;
          mma_commit(s_full + sb);
          if (t == I.ntiles - 1) mma_commit(q_empty);
        }
        if (!ok) break;
        ++qn;
        g += I.ntiles;
      }
      if (!ok) fail(abort, a.dev_status);
      // all issued MMAs (of both issuers) complete before TMEM is released
      mma_commit(mma_done);
      mbar_wait(mma_done, 0, no_abort, limit);
    }
    __syncwarp();
  } else if (warp == kWarpPV) {
    // ----------------------------------------------------------- PV issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t aV = smem_u32(sV);
      uint32_t vt = 0, qn = 0, g = 0;
      bool ok = true;
      // O_0/O_1 stay in use until both softmax groups have finished the
      // item's epilogue (o_free, one phase per item): nfree counts the
      // phases seen.  The first PV of item qn waits for epilogues 0..qn-1.
      uint32_t nfree = 0;
      auto ensure_free = [&](uint32_t k) -> bool {
        while (nfree < k) {
          if (!mbar_wait(o_free, nfree & 1, abort, limit)) return false;
          ++nfree;
        }
        return true;
      };
      for (int it = blockIdx.x; it < a.n_items && ok; it += gridDim.x) {
        if (*abort) break;
        const Item I = decode_item(a, it);
        if (I.ntiles == 0) continue;
        // V tiles in the interleaved layout as the K tiles above
        const bool il = kInterleaved && (I.kind == kItemList || I.kind == kItemLocal);
        for (int t = 0; t < I.ntiles; ++t) {
          const uint32_t gg = g + t;
          const uint32_t sb = gg & 1;
          if (!mbar_wait(p_full + sb, (gg >> 1) & 1, abort, limit) ||
              (t == 0 && !ensure_free(qn))) {
            ok = false;
            break;
          }
          const int st = vt % VS;
          if (!mbar_wait(v_full + st, (vt / VS) & 1, abort, limit)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t tS = tmem + sb * 128;
          // O_1, the accumulator PV reaches last
          if (!dcheck(tmem_in_range(tmem + 256 + D, tmem, D), a.dev_status)) {
            ok = false;
            break;
          }
          const uint32_t vbase = aV + st * L::TILE_BYTES;
#pragma unroll
          for (int kk = 0; kk < kTileK / 16; ++kk) {
            // V is MN-major: LBO steps between the two 64-column halves, SBO
            // between the two 8-key groups of the 16-key step
            const uint64_t bdesc = il ? smem_desc_sw128(vbase + kk * 4096, 1024, 2048)
                                      : smem_desc_sw128(vbase + kk * 2048, kHalfBytes, 1024);
            // keys 0..63 (softmax group 0): P in columns 0..31, into O_0;
            // keys 64..127 (group 1): P in columns 64..95, into O_1
            const uint32_t pa = tS + (kk < 4 ? kk * 8 : 64 + (kk - 4) * 8);
            const uint32_t tO = tmem + 256 + (kk < 4 ? 0 : D);
            mma_bf16_ts(tO, pa, bdesc, IDESC_PV, (t == 0 && (kk & 3) == 0) ? 0u : 1u);
          }
          ++vt;
          mma_commit(o_done + sb);
        }
        if (!ok) break;
        ++qn;
        g += I.ntiles;
      }
      if (!ok) fail(abort, a.dev_status);
      mma_commit(mma_done);
      mbar_wait(mma_done, 0, no_abort, limit);
    }
    __syncwarp();
  } else if (warp < kWarpV) {
    // ------------------------------------------------------------- softmax
    SoftmaxShared sh{s_full, p_full, o_done, o_free, lbar, abort};
    // one copy of the softmax code serves both groups (J is a runtime value)
    softmax_role<D, UNIT, ENT, WIN>(a, sh, tmem, warp, lane, warp < 6 ? 0 : 1);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

__global__ void f32_to_bf16_kernel(const float4* __restrict__ src, uint2* __restrict__ dst,
                                   size_t n4) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float4 v = src[i];
    dst[i] = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
  }
}

template <int D, int KS, int VS, int UNIT, bool ENT = false, bool WIN = false>
cudaError_t launch_t(const AttnArgs& a, const CUtensorMap& tq, const CUtensorMap& tku,
                     const CUtensorMap& tvu, const CUtensorMap& tkf, const CUtensorMap& tvf,
                     const CUtensorMap& tki, const CUtensorMap& tvi, int num_sms,
                     cudaStream_t stream) {
  using L = Layout<D, KS, VS>;
  auto kern = attn_fwd_kernel<D, KS, VS, UNIT, ENT, WIN>;
  cudaError_t e = set_dyn_smem<attn_fwd_kernel<D, KS, VS, UNIT, ENT, WIN>>(L::ALLOC);
  if (e != cudaSuccess) return e;
  const int grid = a.n_items < num_sms ? a.n_items : num_sms;
  if (grid <= 0) return cudaSuccess;
  kern<<<grid, kThreads, L::ALLOC, stream>>>(a, tq, tku, tvu, tkf, tvf, tki, tvi);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(int d, const AttnArgs& a, const CUtensorMap& tq,
                             const CUtensorMap& tku, const CUtensorMap& tvu,
                             const CUtensorMap& tkf, const CUtensorMap& tvf,
                             const CUtensorMap& tki, const CUtensorMap& tvi, int num_sms,
                             cudaStream_t stream) {
  // dense attention with per-query entropy (the dense warm-up)
  if (a.entropy) {
    if (a.mode != kModeDense || a.unit != kTileK) return cudaErrorInvalidValue;
    if (d == 128)
      return launch_t<128, STA_KSTAGES, STA_VSTAGES, 128, true>(a, tq, tku, tvu, tkf, tvf, tki,
                                                                tvi, num_sms, stream);
    if (d == 64)
      return launch_t<64, STA_KSTAGES, STA_VSTAGES, 128, true>(a, tq, tku, tvu, tkf, tvf, tki,
                                                               tvi, num_sms, stream);
    return cudaErrorInvalidValue;
  }
  // routed lists (local windows) run their own instantiation, so that the
  // window code costs the other kernels nothing
  const bool routed = (a.mode == kModeRouted);
#define STA_ATTN_CASE(DD, UU)                                                                \
  if (d == DD && a.unit == UU)                                                               \
    return routed ? launch_t<DD, STA_KSTAGES, STA_VSTAGES, UU, false, true>(                 \
                        a, tq, tku, tvu, tkf, tvf, tki, tvi, num_sms, stream)                \
                  : launch_t<DD, STA_KSTAGES, STA_VSTAGES, UU, false, false>(                \
                        a, tq, tku, tvu, tkf, tvf, tki, tvi, num_sms, stream);
  STA_ATTN_CASE(128, 128)
  STA_ATTN_CASE(128, 64)
  STA_ATTN_CASE(128, 32)
  STA_ATTN_CASE(128, 16)
  STA_ATTN_CASE(64, 128)
  STA_ATTN_CASE(64, 64)
  STA_ATTN_CASE(64, 32)
  STA_ATTN_CASE(64, 16)
#undef STA_ATTN_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_f32_to_bf16(const float* src, __nv_bfloat16* dst, size_t n, cudaStream_t s) {
  if (n % 4 != 0) return cudaErrorInvalidValue;
  const size_t n4 = n / 4;
  const int block = 256;
  size_t grid = (n4 + block - 1) / block;
  if (grid > 148 * 16) grid = 148 * 16;
  if (grid == 0) return cudaSuccess;
  f32_to_bf16_kernel<<<static_cast<unsigned>(grid), block, 0, s>>>(
      reinterpret_cast<const float4*>(src), reinterpret_cast<uint2*>(dst), n4);
  return cudaGetLastError();
}

}  // namespace sta
