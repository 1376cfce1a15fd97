// sta_api.cu -- the C ABI (include/sta.h): argument checks, tensor-map
// construction and kernel dispatch.  Every entry point only enqueues work
// on the caller's stream; nothing here allocates device memory.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <stdint.h>

#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"

using namespace sta;

namespace {

constexpr int kVersion = 200;  // 0.2.0 (selector parameters gained the token layout)

// Last CUDA error a call of this thread ran into (sta_last_cuda_error).
thread_local cudaError_t g_last_cuda_error = cudaSuccess;

// An NVTX range named after the entry point, around each call that enqueues
// selector or attention work (recorded by profilers that trace NVTX, e.g.
// `ncu --nvtx --nvtx-include "sta_sparse_attn_fwd/"`; a no-op otherwise).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

bool failed(cudaError_t e) {
  if (e == cudaSuccess) return false;
  g_last_cuda_error = e;
  return true;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3D map over a [heads][N][d] bf16 tensor: dim0 = d (contiguous), dim1 = N,
// dim2 = heads; box = 64 columns (128 bytes, 128-byte swizzle) x rows x 1.
// Rows past N read as zero.
bool make_map(CUtensorMap* m, const void* base, int d, int N, int heads, int box_rows,
              CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(heads)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(N) * static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, dtype, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Five-dimensional view of a [heads][N][128] bf16 tensor for loading one
// key/value unit of `unit` rows (both 64-column halves) in a single TMA copy:
// dims (64 columns, 8 rows, 2 halves, N/8 row groups, heads) with byte
// strides (256, 128, 2048, N*256) and box (64, 8, 2, unit/8, 1).  The box
// lands in shared memory as [row group][half][8 rows][128 B], each 1 KB
// block one 128-byte-swizzle atom.  Only row groups below N/8 are in range,
// so a copy never reads past the head's last row.
bool interleaved_unit_map(CUtensorMap* m, const void* base, int N, int heads, int unit) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t groups = N >= 8 ? static_cast<cuuint64_t>(N / 8) : 1;
  cuuint64_t dims[5] = {64, 8, 2, groups, static_cast<cuuint64_t>(heads)};
  cuuint64_t strides[4] = {256, 128, 2048, static_cast<cuuint64_t>(N) * 256};
  cuuint32_t box[5] = {64, 8, 2, static_cast<cuuint32_t>(unit / 8), 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool pow2_unit(int u) { return u == 16 || u == 32 || u == 64 || u == 128; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

sta_status check_problem(const sta_problem* p) {
  if (!p) return STA_ERR_ARG;
  if (p->heads < 1 || p->F < 1 || p->H < 1 || p->W < 1) return STA_ERR_ARG;
  if (p->dtype != STA_BF16 && p->dtype != STA_F32) return STA_ERR_ARG;
  if (p->d != 64 && p->d != 128) return STA_ERR_UNSUPPORTED;
  const long long N = static_cast<long long>(p->F) * p->H * p->W;
  if (N > (1ll << 30)) return STA_ERR_UNSUPPORTED;
  if (N * p->heads > (1ll << 31) - 1) return STA_ERR_UNSUPPORTED;
  return STA_OK;
}

int num_sms_current() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

size_t staged_bytes(const sta_problem* p) {
  const size_t n = static_cast<size_t>(p->heads) * p->F * p->H * p->W * p->d;
  return round_up(n * 2, 256);
}

// bf16 views of q, k, v: the inputs themselves, or fp32 inputs rounded
// into the workspace.
sta_status stage_inputs(const sta_problem* p, const void* q, const void* k, const void* v,
                        void* ws, size_t ws_bytes, const __nv_bfloat16** qb,
                        const __nv_bfloat16** kb, const __nv_bfloat16** vb,
                        cudaStream_t stream) {
  if (p->dtype == STA_BF16) {
    *qb = static_cast<const __nv_bfloat16*>(q);
    *kb = static_cast<const __nv_bfloat16*>(k);
    *vb = static_cast<const __nv_bfloat16*>(v);
    return STA_OK;
  }
  const size_t one = staged_bytes(p);
  if (!ws || ws_bytes < 3 * one) return STA_ERR_WORKSPACE;
  const size_t n = static_cast<size_t>(p->heads) * p->F * p->H * p->W * p->d;
  __nv_bfloat16* base = static_cast<__nv_bfloat16*>(ws);
  __nv_bfloat16* dq = base;
  __nv_bfloat16* dk = reinterpret_cast<__nv_bfloat16*>(reinterpret_cast<uint8_t*>(ws) + one);
  __nv_bfloat16* dv = reinterpret_cast<__nv_bfloat16*>(reinterpret_cast<uint8_t*>(ws) + 2 * one);
  if (failed(launch_f32_to_bf16(static_cast<const float*>(q), dq, n, stream)) ||
      failed(launch_f32_to_bf16(static_cast<const float*>(k), dk, n, stream)) ||
      failed(launch_f32_to_bf16(static_cast<const float*>(v), dv, n, stream)))
    return STA_ERR_CUDA;
  *qb = dq;
  *kb = dk;
  *vb = dv;
  return STA_OK;
}

sta_status run_attention(const sta_problem* p, AttnArgs& a, const __nv_bfloat16* qb,
                         const __nv_bfloat16* kb, const __nv_bfloat16* vb, int unit,
                         cudaStream_t stream) {
  CUtensorMap tq, tku, tvu, tkf, tvf, tki, tvi;
  const int N = a.N;
  // d = 128 with 16-key units: one interleaved copy per unit,
  // 8-row boxes for a unit that reaches the last N % 8 rows
  const bool il = (p->d == 128 && unit < 32);
  const int unit_box = il ? 8 : unit;
  if (!make_map(&tq, qb, p->d, N, p->heads, kTileQ) ||
      !make_map(&tku, kb, p->d, N, p->heads, unit_box) ||
      !make_map(&tvu, vb, p->d, N, p->heads, unit_box) ||
      !make_map(&tkf, kb, p->d, N, p->heads, kTileK) ||
      !make_map(&tvf, vb, p->d, N, p->heads, kTileK) ||
      (il && (!interleaved_unit_map(&tki, kb, N, p->heads, unit) ||
              !interleaved_unit_map(&tvi, vb, N, p->heads, unit)))) {
    g_last_cuda_error = cudaErrorInvalidValue;
    return STA_ERR_CUDA;
  }
  if (!il) {
    tki = tkf;  // unused
    tvi = tvf;
  }
  const int sms = num_sms_current();
  if (sms <= 0) return STA_ERR_CUDA;
  a.unit = unit;
  a.q = qb;
  if (failed(launch_attention(p->d, a, tq, tku, tvu, tkf, tvf, tki, tvi, sms, stream)))
    return STA_ERR_CUDA;
  return STA_OK;
}

// Workspace carve-up of the content selectors (256-byte aligned segments).
struct SelWorkspace {
  size_t qbar = 0, kbar = 0, scores = 0, cent = 0, wts = 0, p = 0, prior_idx = 0, prior_cnt = 0;
  size_t kb_hi = 0, kb_lo = 0, c_hi = 0, c_lo = 0, total = 0;
};

SelWorkspace sel_workspace(const sta_problem* p, const sta_selector_params* sel) {
  SelWorkspace w;
  const size_t h = static_cast<size_t>(p->heads);
  const size_t N = static_cast<size_t>(p->F) * p->H * p->W;
  const size_t d = static_cast<size_t>(p->d);
  if (sel->block_q < 1 || sel->kv_unit < 1) return w;
  const size_t nqb = (N + sel->block_q - 1) / sel->block_q;
  const size_t nku = (N + sel->kv_unit - 1) / sel->kv_unit;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += round_up(bytes, 256);
    return at;
  };
  if (sel->kind == STA_SEL_DYNRAD) {
    w.qbar = take(h * nqb * d * 4);
    w.kbar = take(h * nku * d * 4);
    w.prior_idx = take(nqb * nku * 4);
    w.prior_cnt = take(nqb * 4);
  } else if (sel->kind == STA_SEL_ENTROPY) {
    w.qbar = take(h * nqb * d * 4);
    w.kbar = take(h * nku * d * 4);
    w.scores = take(h * nqb * nku * 4);
  } else if (sel->kind == STA_SEL_IBCS_SIP) {
    const size_t km = sel->km_k > 0 ? static_cast<size_t>(sel->km_k) : 1;
    w.kb_hi = take(h * nku * d * 2);
    w.kb_lo = take(h * nku * d * 2);
    w.c_hi = take(h * nqb * km * d * 2);
    w.c_lo = take(h * nqb * km * d * 2);
    w.wts = take(h * nqb * km * 4);
    w.p = take(h * nqb * ((nku + 3) & ~size_t(3)) * 4);  // rows padded to 16 bytes
  }
  w.total = off;
  return w;
}

// ceil(frac * n) with a relative slack of 1e-6 (so that a decimal fraction
// stored in binary does not add one), clamped to [lo, n].
int fraction_count(double frac, long long n, int lo) {
  long long m = static_cast<long long>(ceil(frac * static_cast<double>(n) * (1.0 - 1e-6)));
  if (m < lo) m = lo;
  if (m > n) m = n;
  return static_cast<int>(m);
}

}  // namespace

extern "C" {

int sta_version(void) { return kVersion; }

int sta_debug_build(void) { return STA_DEBUG ? 1 : 0; }

sta_status sta_selftest_index_check(int32_t* buf, int n, int index, int32_t* dev_status,
                                    sta_stream_t stream) {
  if (!buf || !dev_status || n < 1) return STA_ERR_ARG;
  // without the checks an out-of-range index would be stored as given
  if (!STA_DEBUG) return STA_ERR_UNSUPPORTED;
  if (failed(launch_index_check_selftest(buf, n, index, dev_status,
                                         reinterpret_cast<cudaStream_t>(stream))))
    return STA_ERR_CUDA;
  return STA_OK;
}

sta_status sta_selftest_bounded_wait(uint64_t limit_ns, int32_t* dev_status, int32_t* waited_ok,
                                     sta_stream_t stream) {
  if (!dev_status || !waited_ok) return STA_ERR_ARG;
  if (limit_ns == 0 || limit_ns > kWaitLimitNs) return STA_ERR_ARG;
  if (failed(launch_bounded_wait_selftest(limit_ns, dev_status, waited_ok,
                                          reinterpret_cast<cudaStream_t>(stream))))
    return STA_ERR_CUDA;
  return STA_OK;
}

const char* sta_last_cuda_error(void) {
  return g_last_cuda_error == cudaSuccess ? "no CUDA error" : cudaGetErrorString(g_last_cuda_error);
}

const char* sta_status_string(sta_status s) {
  switch (s) {
    case STA_OK: return "ok";
    case STA_ERR_ARG: return "invalid argument";
    case STA_ERR_UNSUPPORTED: return "unsupported shape or parameter";
    case STA_ERR_CAPACITY: return "list capacity exceeded";
    case STA_ERR_CUDA: return "CUDA error";
    case STA_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

const char* sta_dev_status_string(int32_t bits) {
  if (bits == 0) return "ok";
  if (bits & STA_DEV_DEBUG) return "debug build: an index check failed (access skipped)";
  if (bits & STA_DEV_TIMEOUT) return "timeout: a bounded wait ran out";
  if (bits & STA_DEV_BAD_INDEX) return "list entry out of range (skipped)";
  if (bits & STA_DEV_RANGE) return "importance operand beyond the fp16 range";
  if (bits & STA_DEV_CAPACITY) return "list row truncated at capacity";
  if (bits & STA_DEV_EMPTY_ROW) return "query row without kept keys (output 0)";
  return "unknown device status";
}

int sta_build_blocks_rows(const sta_problem* prob, const sta_selector_params* sel) {
  if (check_problem(prob) != STA_OK || !sel || sel->block_q < 1) return -1;
  const long long N = static_cast<long long>(prob->F) * prob->H * prob->W;
  const int nqb = static_cast<int>((N + sel->block_q - 1) / sel->block_q);
  switch (sel->kind) {
    case STA_SEL_RADIAL:
    case STA_SEL_ROUTED:
      return nqb;
    case STA_SEL_ENTROPY:
    case STA_SEL_IBCS_SIP:
    case STA_SEL_TRA_TOKEN:
    case STA_SEL_DYNRAD:
      return nqb * prob->heads;
  }
  return -1;
}

size_t sta_build_blocks_workspace(const sta_problem* prob, const sta_selector_params* sel) {
  if (check_problem(prob) != STA_OK || !sel) return 0;
  const SelWorkspace w = sel_workspace(prob, sel);
  return w.total;
}

sta_status sta_build_blocks(const sta_problem* prob, const sta_selector_params* sel,
                            const void* q, const void* k, sta_block_lists* out, void* workspace,
                            size_t workspace_bytes, int32_t* dev_status, sta_stream_t stream) {
  NvtxRange nvtx_range("sta_build_blocks");
  sta_status st = check_problem(prob);
  if (st != STA_OK) return st;
  if (!sel || !out || !out->idx || !out->cnt || out->cap < 1) return STA_ERR_ARG;
  if (!pow2_unit(sel->block_q) || !pow2_unit(sel->kv_unit)) return STA_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (sel->kind) {
    case STA_SEL_RADIAL: {
      if (sel->kv_unit != sel->block_q) return STA_ERR_UNSUPPORTED;
      const int S = prob->H * prob->W;
      if ((sel->block_q + S - 1) / S + 1 > 8) return STA_ERR_UNSUPPORTED;
      out->head_shared = 1;
      if (failed(launch_radial_lists(prob->F, prob->H, prob->W, sel->block_q, sel->radial_w0,
                              sel->radial_w_off, sel->radial_full_df, out->idx, out->cnt, out->cap,
                              out->required_cap, dev_status, s)))
        return STA_ERR_CUDA;
      return STA_OK;
    }
    case STA_SEL_ENTROPY: {
      if (prob->dtype != STA_BF16 || !q || !k) return q && k ? STA_ERR_UNSUPPORTED : STA_ERR_ARG;
      if (sel->kv_unit != sel->block_q) return STA_ERR_UNSUPPORTED;
      if (sel->ent_r_lo > sel->ent_r_hi || sel->ent_tile_h < 1 || sel->ent_tile_w < 1)
        return STA_ERR_ARG;
      const int N = prob->F * prob->H * prob->W;
      const int nb = (N + sel->block_q - 1) / sel->block_q;
      if (nb > entropy_max_blocks(prob->d)) return STA_ERR_UNSUPPORTED;
      // block cells are packed in 11 + 10 + 10 bits
      if (prob->F > 2047 || (prob->H - 1) / sel->ent_tile_h > 1023 ||
          (prob->W - 1) / sel->ent_tile_w > 1023)
        return STA_ERR_UNSUPPORTED;
      const SelWorkspace w = sel_workspace(prob, sel);
      if (!workspace || workspace_bytes < w.total ||
          (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return STA_ERR_WORKSPACE;
      uint8_t* ws = static_cast<uint8_t*>(workspace);
      float* qbar = reinterpret_cast<float*>(ws + w.qbar);
      float* kbar = reinterpret_cast<float*>(ws + w.kbar);
      out->head_shared = 0;
      const float scale = 1.0f / sqrtf(static_cast<float>(prob->d));
      if (failed(launch_block_means(static_cast<const __nv_bfloat16*>(q),
                             static_cast<const __nv_bfloat16*>(k), qbar, kbar, prob->heads, N,
                             prob->d, sel->block_q, s)))
        return STA_ERR_CUDA;
      if (failed(launch_entropy_lists(qbar, kbar, reinterpret_cast<float*>(ws + w.scores),
                                      prob->heads, prob->F, prob->H, prob->W, prob->d,
                                      sel->block_q, scale, sel->ent_alpha, sel->ent_beta,
                                      sel->ent_r_lo, sel->ent_r_hi, sel->ent_tile_h,
                                      sel->ent_tile_w, out->idx, out->cnt, out->cap,
                                      out->required_cap, out->entropy, out->radius, dev_status,
                                      s)))
        return STA_ERR_CUDA;
      return STA_OK;
    }
    case STA_SEL_DYNRAD: {
      if (prob->dtype != STA_BF16 || !q || !k) return q && k ? STA_ERR_UNSUPPORTED : STA_ERR_ARG;
      if (sel->dyn_mode != 0 && sel->dyn_mode != 1) return STA_ERR_ARG;
      if (sel->dyn_mode == 0 && !(sel->dyn_ratio > 0.f && sel->dyn_ratio <= 1.f))
        return STA_ERR_ARG;
      if (sel->dyn_mode == 1 && !(sel->dyn_threshold > 0.f && sel->dyn_threshold <= 1.f))
        return STA_ERR_ARG;
      if (sel->kv_unit != sel->block_q) return STA_ERR_UNSUPPORTED;
      const int S = prob->H * prob->W;
      if ((sel->block_q + S - 1) / S + 1 > 8) return STA_ERR_UNSUPPORTED;
      const int N = prob->F * prob->H * prob->W;
      const int nb = (N + sel->block_q - 1) / sel->block_q;
      if (nb > dynrad_max_candidates()) return STA_ERR_UNSUPPORTED;
      const SelWorkspace w = sel_workspace(prob, sel);
      if (!workspace || workspace_bytes < w.total ||
          (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return STA_ERR_WORKSPACE;
      uint8_t* ws = static_cast<uint8_t*>(workspace);
      float* qbar = reinterpret_cast<float*>(ws + w.qbar);
      float* kbar = reinterpret_cast<float*>(ws + w.kbar);
      int32_t* pidx = reinterpret_cast<int32_t*>(ws + w.prior_idx);
      int32_t* pcnt = reinterpret_cast<int32_t*>(ws + w.prior_cnt);
      out->head_shared = 0;
      const float scale = 1.0f / sqrtf(static_cast<float>(prob->d));
      // 1. block means, 2. the radial prior (shared by the heads), 3. selection
      if (failed(launch_block_means(static_cast<const __nv_bfloat16*>(q),
                                    static_cast<const __nv_bfloat16*>(k), qbar, kbar,
                                    prob->heads, N, prob->d, sel->block_q, s)) ||
          failed(launch_radial_lists(prob->F, prob->H, prob->W, sel->block_q, sel->radial_w0,
                                     sel->radial_w_off, sel->radial_full_df, pidx, pcnt, nb,
                                     nullptr, dev_status, s)) ||
          failed(launch_dynrad_lists(qbar, kbar, pidx, pcnt, nb, prob->heads, nb, prob->d, scale,
                                     sel->dyn_mode, sel->dyn_ratio, sel->dyn_threshold, out->idx,
                                     out->cnt, out->cap, out->required_cap, dev_status, s)))
        return STA_ERR_CUDA;
      return STA_OK;
    }
    case STA_SEL_TRA_TOKEN: {
      if (!sel->tra_entropy) return STA_ERR_ARG;
      if (!(sel->tra_tau > 0.f) || !(sel->tra_gamma >= 0.f) || sel->tra_vote < 1)
        return STA_ERR_ARG;
      if (sel->kv_unit != sel->block_q || sel->block_q > tra_max_block() ||
          prob->F > tra_max_frames())
        return STA_ERR_UNSUPPORTED;
      out->head_shared = 0;
      const int th = sel->layout_tile_h, tw = sel->layout_tile_w;
      if ((th == 0) != (tw == 0) || th < 0 || tw < 0 || th > prob->H || tw > prob->W)
        return STA_ERR_ARG;
      if (failed(launch_tra_token_lists(sel->tra_entropy, prob->heads, prob->F, prob->H, prob->W,
                                        sel->block_q, th == 0 ? 1 : th, th == 0 ? prob->W : tw,
                                        sel->tra_tau, sel->tra_gamma,
                                        sel->tra_vote, out->idx, out->cnt, out->cap,
                                        out->required_cap, dev_status, s)))
        return STA_ERR_CUDA;
      return STA_OK;
    }
    case STA_SEL_ROUTED: {
      if (!sel->difficulty || !out->routed_ids || !out->routed_flag) return STA_ERR_ARG;
      if (sel->win_f < 0 || sel->win_h < 1 || sel->win_w < 1) return STA_ERR_ARG;
      if (!(sel->dense_frac >= 0.f && sel->dense_frac <= 1.f)) return STA_ERR_ARG;
      const int N = prob->F * prob->H * prob->W;
      const int n_routed = fraction_count(sel->dense_frac, N, 0);
      out->head_shared = 1;
      out->n_routed = n_routed;
      if (failed(launch_routed_select(sel->difficulty, N, n_routed, out->routed_ids, out->routed_flag,
                               s)))
        return STA_ERR_CUDA;
      if (failed(launch_routed_local_lists(prob->F, prob->H, prob->W, sel->block_q, sel->kv_unit,
                                    sel->win_f, sel->win_h, sel->win_w, out->idx, out->cnt,
                                    out->cap, out->required_cap, dev_status, s)))
        return STA_ERR_CUDA;
      return STA_OK;
    }
    case STA_SEL_IBCS_SIP: {
      if (prob->dtype != STA_BF16 || !q || !k) return q && k ? STA_ERR_UNSUPPORTED : STA_ERR_ARG;
      if (sel->km_k != 1 && sel->km_k != 2 && sel->km_k != 4 && sel->km_k != 8)
        return STA_ERR_UNSUPPORTED;
      if (sel->km_iters < 1) return STA_ERR_ARG;
      if (prob->d != 128) return STA_ERR_UNSUPPORTED;  // tensor-core importance: d = 128
      if (!(sel->sample_frac > 0.f && sel->sample_frac <= 1.f)) return STA_ERR_ARG;
      const int N = prob->F * prob->H * prob->W;
      const int n_sub = (N + sel->kv_unit - 1) / sel->kv_unit;
      if (n_sub > ibcs_max_subblocks()) return STA_ERR_UNSUPPORTED;
      const SelWorkspace w = sel_workspace(prob, sel);
      if (!workspace || workspace_bytes < w.total ||
          (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return STA_ERR_WORKSPACE;
      uint8_t* ws = static_cast<uint8_t*>(workspace);
      float* wts = reinterpret_cast<float*>(ws + w.wts);
      float* pbuf = reinterpret_cast<float*>(ws + w.p);
      __half* kbh = reinterpret_cast<__half*>(ws + w.kb_hi);
      __half* kbl = reinterpret_cast<__half*>(ws + w.kb_lo);
      __half* ch = reinterpret_cast<__half*>(ws + w.c_hi);
      __half* cl = reinterpret_cast<__half*>(ws + w.c_lo);
      out->head_shared = 0;
      const int m = fraction_count(sel->sample_frac, n_sub, 1);
      const float scale = 1.0f / sqrtf(static_cast<float>(prob->d));
      const int nqb = (N + sel->block_q - 1) / sel->block_q;
      const int n_rows = nqb * sel->km_k;
      // 1. sub-block means, 2. k-means, both written as fp16 hi/lo pairs
      if (failed(launch_block_means_f16x2(static_cast<const __nv_bfloat16*>(k), kbh, kbl,
                                          prob->heads, N, prob->d, sel->kv_unit, dev_status,
                                          s)) ||
          failed(launch_kmeans(static_cast<const __nv_bfloat16*>(q), ch, cl, wts, prob->heads, N,
                               prob->d, sel->block_q, sel->km_k, sel->km_iters, dev_status, s)))
        return STA_ERR_CUDA;
      // 4. importance on the tensor cores, 5. water filling + Philox sampling
      CUtensorMap tch, tcl, tkh, tkl;
      if (!make_map(&tch, ch, prob->d, n_rows, prob->heads, 128, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) ||
          !make_map(&tcl, cl, prob->d, n_rows, prob->heads, 128, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) ||
          !make_map(&tkh, kbh, prob->d, n_sub, prob->heads, 128, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) ||
          !make_map(&tkl, kbl, prob->d, n_sub, prob->heads, 128, CU_TENSOR_MAP_DATA_TYPE_FLOAT16)) {
        g_last_cuda_error = cudaErrorInvalidValue;
        return STA_ERR_CUDA;
      }
      if (failed(launch_importance_tc(wts, pbuf, prob->heads, n_rows, nqb, sel->km_k, n_sub, N,
                                      sel->kv_unit,
                                      scale, tch, tcl, tkh, tkl, dev_status, s)) ||
          failed(launch_sip_sample(pbuf, prob->heads * nqb, n_sub, m, sel->seed, out->idx,
                                   out->logw, out->cnt, out->cap, out->required_cap, dev_status,
                                   s)))
        return STA_ERR_CUDA;
      return STA_OK;
    }
    default:
      return STA_ERR_UNSUPPORTED;
  }
}

size_t sta_attn_workspace(const sta_problem* prob) {
  if (check_problem(prob) != STA_OK) return 0;
  return prob->dtype == STA_F32 ? 3 * staged_bytes(prob) : 0;
}

}  // extern "C"

namespace {

// Argument checks shared by the sparse attention entry points (before any
// size or workspace check, so that both report the same codes).
sta_status check_sparse_args(const sta_problem* prob, const sta_attn_params* prm, const void* q,
                             const void* k, const void* v, const sta_block_lists* lists,
                             const void* o) {
  sta_status st = check_problem(prob);
  if (st != STA_OK) return st;
  if (!prm || !q || !k || !v || !lists || !o) return STA_ERR_ARG;
  if (!pow2_unit(prm->block_q) || !pow2_unit(prm->kv_unit)) return STA_ERR_UNSUPPORTED;
  if (!lists->idx || !lists->cnt || lists->cap < 1) return STA_ERR_ARG;
  return STA_OK;
}

}  // namespace

extern "C" {

sta_status sta_sparse_attn_fwd(const sta_problem* prob, const sta_attn_params* prm,
                               const void* q, const void* k, const void* v,
                               const sta_block_lists* lists, void* o, void* workspace,
                               size_t workspace_bytes, int32_t* dev_status, sta_stream_t stream) {
  NvtxRange nvtx_range("sta_sparse_attn_fwd");
  sta_status st = check_sparse_args(prob, prm, q, k, v, lists, o);
  if (st != STA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int N = prob->F * prob->H * prob->W;
  AttnArgs a = {};
  a.heads = prob->heads;
  a.N = N;
  a.F = prob->F;
  a.H = prob->H;
  a.W = prob->W;
  const float scale = prm->scale > 0.f ? prm->scale : 1.0f / sqrtf(static_cast<float>(prob->d));
  a.scale_log2 = scale * 1.4426950408889634f;
  a.block_q = prm->block_q;
  a.n_qb = (N + prm->block_q - 1) / prm->block_q;
  a.idx = lists->idx;
  a.cnt = lists->cnt;
  a.logw = lists->logw;
  a.cap = lists->cap;
  a.head_shared = lists->head_shared ? 1 : 0;
  a.o = o;
  a.out_f32 = prob->dtype == STA_F32;
  a.dev_status = dev_status;
  if (prm->mode == STA_ATTN_LISTS) {
    a.mode = kModeLists;
    a.n_items = prob->heads * a.n_qb;
  } else if (prm->mode == STA_ATTN_ROUTED) {
    if (!lists->routed_ids || !lists->routed_flag || lists->n_routed < 0 || lists->n_routed > N)
      return STA_ERR_ARG;
    if (!lists->head_shared) return STA_ERR_UNSUPPORTED;
    a.mode = kModeRouted;
    a.routed_ids = lists->routed_ids;
    a.routed_flag = lists->routed_flag;
    a.n_routed = lists->n_routed;
    a.n_dense_items = (lists->n_routed + kTileQ - 1) / kTileQ;
    a.win_f = prm->win_f;
    a.win_h = prm->win_h;
    a.win_w = prm->win_w;
    a.n_items = prob->heads * (a.n_dense_items + a.n_qb);
  } else {
    return STA_ERR_ARG;
  }
  const __nv_bfloat16 *qb, *kb, *vb;
  st = stage_inputs(prob, q, k, v, workspace, workspace_bytes, &qb, &kb, &vb, s);
  if (st != STA_OK) return st;
  return run_attention(prob, a, qb, kb, vb, prm->kv_unit, s);
}

namespace {

// Dense attention, with the per-query entropy written to `entropy` when it is
// not null (the dense warm-up of the token-level selector).
sta_status dense_attn(const sta_problem* prob, const void* q, const void* k, const void* v,
                      float scale, void* o, float* entropy, void* workspace,
                      size_t workspace_bytes, int32_t* dev_status, sta_stream_t stream) {
  sta_status st = check_problem(prob);
  if (st != STA_OK) return st;
  if (!q || !k || !v || !o) return STA_ERR_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int N = prob->F * prob->H * prob->W;
  AttnArgs a = {};
  a.heads = prob->heads;
  a.N = N;
  a.F = prob->F;
  a.H = prob->H;
  a.W = prob->W;
  const float sc = scale > 0.f ? scale : 1.0f / sqrtf(static_cast<float>(prob->d));
  a.scale_log2 = sc * 1.4426950408889634f;
  a.mode = kModeDense;
  a.block_q = kTileQ;
  a.unit = kTileK;
  a.n_qb = (N + kTileQ - 1) / kTileQ;
  a.n_items = prob->heads * a.n_qb;
  a.o = o;
  a.out_f32 = prob->dtype == STA_F32;
  a.dev_status = dev_status;
  a.entropy = entropy;
  const __nv_bfloat16 *qb, *kb, *vb;
  st = stage_inputs(prob, q, k, v, workspace, workspace_bytes, &qb, &kb, &vb, s);
  if (st != STA_OK) return st;
  return run_attention(prob, a, qb, kb, vb, kTileK, s);
}

}  // namespace

sta_status sta_dense_attn_fwd(const sta_problem* prob, const void* q, const void* k,
                              const void* v, float scale, void* o, void* workspace,
                              size_t workspace_bytes, int32_t* dev_status, sta_stream_t stream) {
  NvtxRange nvtx_range("sta_dense_attn_fwd");
  return dense_attn(prob, q, k, v, scale, o, nullptr, workspace, workspace_bytes, dev_status,
                    stream);
}

sta_status sta_dense_attn_entropy_fwd(const sta_problem* prob, const void* q, const void* k,
                                      const void* v, float scale, void* o, float* entropy,
                                      void* workspace, size_t workspace_bytes,
                                      int32_t* dev_status, sta_stream_t stream) {
  NvtxRange nvtx_range("sta_dense_attn_entropy_fwd");
  if (!entropy) return STA_ERR_ARG;
  return dense_attn(prob, q, k, v, scale, o, entropy, workspace, workspace_bytes, dev_status,
                    stream);
}

sta_status sta_permute_tokens(const sta_problem* prob, int tile_h, int tile_w, int inverse,
                              const void* in, void* out, sta_stream_t stream) {
  NvtxRange nvtx_range("sta_permute_tokens");
  sta_status st = check_problem(prob);
  if (st != STA_OK) return st;
  if (!in || !out || tile_h < 1 || tile_w < 1 || tile_h > prob->H || tile_w > prob->W)
    return STA_ERR_ARG;
  const int N = prob->F * prob->H * prob->W;
  const size_t elem = prob->dtype == STA_F32 ? 4 : 2;
  const size_t bytes = static_cast<size_t>(prob->heads) * N * prob->d * elem;
  const uintptr_t a = reinterpret_cast<uintptr_t>(in), b = reinterpret_cast<uintptr_t>(out);
  if (a < b + bytes && b < a + bytes) return STA_ERR_ARG;  // overlapping buffers
  if (a % 16 != 0 || b % 16 != 0) return STA_ERR_ARG;
  const TokLayout L{prob->H, prob->W, tile_h, tile_w};
  if (failed(launch_permute_rows(in, out, prob->heads, N, static_cast<int>(prob->d * elem), L,
                                 inverse ? 1 : 0, reinterpret_cast<cudaStream_t>(stream))))
    return STA_ERR_CUDA;
  return STA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// sta_sparse_attn_fwd_noalloc: sparse attention for callers that cannot
// allocate device memory.
//
// The only scratch the attention path needs is the bf16 copy of fp32 q, k, v
// that the tensor cores read.  sta_sparse_attn_fwd takes it from a caller
// workspace; this variant takes it from the fixed array below instead.  It
// is for callers that cannot allocate: a plugin that its host framework hands
// only the input and output buffers, with no access to the framework's
// allocator, or a latency-bound pipeline that bans allocation after start-up
// because cudaMalloc can synchronise the device and stall other streams.
//
// The array is part of the library's device image: each device the library
// is used on holds kStaticStageBytes until the process exits.  Host code
// cannot use the symbol's name as a device address (it names a host-side
// shadow), so its device address is looked up once per device with
// cudaGetSymbolAddress and cached.  A reset of the device's primary context
// (cudaDeviceReset) unloads the library's device image and makes the cached
// address stale: this entry point must not be used on a device after such a
// reset.
namespace {

constexpr size_t kStaticStageBytes = size_t(12) << 20;  // 12 MiB
constexpr int kMaxStaticDevices = 64;

static __device__ __align__(256) uint8_t g_static_stage[kStaticStageBytes];

std::mutex g_static_stage_mu;
void* g_static_stage_ptr[kMaxStaticDevices] = {};

// Device address of g_static_stage on the current device (set-up on the
// first call per device).
sta_status static_stage_address(void** out) {
  int dev = -1;
  if (failed(cudaGetDevice(&dev))) return STA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxStaticDevices) return STA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_static_stage_mu);
  if (!g_static_stage_ptr[dev]) {
    void* p = nullptr;
    if (failed(cudaGetSymbolAddress(&p, g_static_stage)) || !p) return STA_ERR_CUDA;
    g_static_stage_ptr[dev] = p;
  }
  *out = g_static_stage_ptr[dev];
  return STA_OK;
}

}  // namespace

extern "C" sta_status sta_sparse_attn_fwd_noalloc(const sta_problem* prob,
                                                  const sta_attn_params* prm, const void* q,
                                                  const void* k, const void* v,
                                                  const sta_block_lists* lists, void* o,
                                                  int32_t* dev_status, sta_stream_t stream) {
  sta_status st = check_sparse_args(prob, prm, q, k, v, lists, o);
  if (st != STA_OK) return st;
  if (prob->dtype != STA_F32) {
    // bf16 inputs feed the tensor cores directly: no scratch at all.
    return sta_sparse_attn_fwd(prob, prm, q, k, v, lists, o, nullptr, 0, dev_status, stream);
  }
  const size_t need = 3 * staged_bytes(prob);
  if (need > kStaticStageBytes) return STA_ERR_WORKSPACE;
  void* stage = nullptr;
  st = static_stage_address(&stage);
  if (st != STA_OK) return st;
  // Every byte the kernels read from the stage is written by this call's
  // conversion first, so nothing needs clearing.
  return sta_sparse_attn_fwd(prob, prm, q, k, v, lists, o, stage, kStaticStageBytes, dev_status,
                             stream);
}
