// api.cu — the C ABI of liblh.so: argument validation, size queries, buffer layouts and the launch sequences
// of the step-wise and fused entry points.  Semantics of every entry point are documented in include/lh.h.
#include <math.h>
#include <string.h>

#include <mutex>

#include "internal.h"

namespace lh {

// Per-device status word and wait limit (see LhDeviceState).
__device__ LhDeviceState g_lh_state = {0, 0, kWaitLimitNs};

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

// Fill the size table; returns LH_OK, LH_ERR_INVALID_ARG or LH_ERR_UNSUPPORTED.
int make_dims(const lh_params* P, LhDims* dm) {
  if (!P) return LH_ERR_INVALID_ARG;
  memset(dm, 0, sizeof(*dm));
  if (P->B < 1 || P->H < 1 || P->N < 1 || P->d < 1 || P->L < 1 || P->p < 2 || P->k < 1 || P->C < 1 ||
      (P->flags & ~LH_EXPAND_CHILDREN) != 0 || P->L > LH_MAX_LEVELS)
    return LH_ERR_INVALID_ARG;
  int64_t w = 1;
  for (int l = 1; l < P->L; ++l) {
    w *= P->p;
    if (w > P->N) return LH_ERR_INVALID_ARG;
  }
  if (P->N % w) return LH_ERR_INVALID_ARG;
  const bool expand = (P->flags & LH_EXPAND_CHILDREN) != 0;
  dm->B = P->B; dm->H = P->H; dm->N = P->N; dm->d = P->d; dm->L = P->L; dm->p = P->p; dm->k = P->k; dm->C = P->C;
  dm->expand = expand ? 1 : 0;
  const int64_t BH = (int64_t)P->B * P->H;
  int64_t S = 0, R = 0, Rs = 0, Rp = 0, Ksel = 0;
  int nPartial = 0;
  int64_t wl = 1;
  for (int l = 0; l < P->L; ++l) {
    const int64_t n = P->N / wl;
    dm->Nl[l] = (int)n;
    dm->wl[l] = (int)wl;
    dm->wlog[l] = 0;
    while ((int64_t(1) << dm->wlog[l]) < wl) ++dm->wlog[l];  // exact log2 when p is a power of two
    dm->off[l] = (int)R;
    if (l >= 1) dm->poff[l] = (int)Rp;
    // the level whose scores pick level l's entries: l itself, or its parent level with expand
    const int64_t n_rank = expand ? n / P->p : n;
    int64_t kl = n;
    if (l <= P->L - 2 && P->k < n_rank) {
      if (n_rank % P->C || P->k % P->C) return LH_ERR_INVALID_ARG;
      kl = expand ? (int64_t)P->k * P->p : P->k;
      if (l != nPartial) return LH_ERR_INVALID_ARG;  // unreachable: level sizes decrease
      dm->seloff[l] = (int)Ksel;
      Ksel += kl;
      ++nPartial;
    }
    dm->kl[l] = (int)kl;
    S += kl;
    R += n;
    const bool scored = expand ? l >= 1 : l <= P->L - 2;
    if (scored) {
      dm->score_mask |= 1u << l;
      dm->soff[l] = (int)Rs;
      Rs += n;
    }
    if (l >= 1) Rp += n;
    wl *= P->p;
  }
  dm->BH = (int)BH;
  dm->S = (int)S;
  dm->R = (int)R;
  dm->Rs = (int)Rs;
  dm->Rp = (int)Rp;
  dm->nPartial = nPartial;
  dm->Ksel = (int)Ksel;
  // what the kernels are built for
  if (P->d != 64 && P->d != 128) return LH_ERR_UNSUPPORTED;
  if (P->p != 2 && P->p != 4 && P->p != 8) return LH_ERR_UNSUPPORTED;
  if (P->L > kMaxL || w > 512) return LH_ERR_UNSUPPORTED;
  if (nPartial > 0 && P->k / P->C > 512) return LH_ERR_UNSUPPORTED;
  if (BH > 65535 || R > INT32_MAX / 2 || S > INT32_MAX / 2) return LH_ERR_UNSUPPORTED;
  return LH_OK;
}

struct CtxLayout {
  size_t qg, kg, vg, og, lse, idx_g, slot, total;
};
CtxLayout ctx_layout(const LhDims& dm) {
  CtxLayout c;
  const size_t rows = (size_t)dm.BH * dm.S;
  size_t o = 0;
  c.qg = o; o = align_up(o + rows * dm.d * 2);
  c.kg = o; o = align_up(o + rows * dm.d * 2);
  c.vg = o; o = align_up(o + rows * dm.d * 2);
  c.og = o; o = align_up(o + rows * dm.d * 4);
  c.lse = o; o = align_up(o + rows * 4);
  c.idx_g = o; o = align_up(o + rows * 4);
  c.slot = o; o = align_up(o + (size_t)dm.BH * dm.R * 4);
  c.total = o;
  return c;
}

struct WsLayout {
  // forward / selection
  size_t scores, coarse[3], sel, fwd_total;
  // backward
  size_t dog, dog16, stats, amax, dinv, dqacc, dkg, dvg, bwd_total;
  size_t total;
};
WsLayout ws_layout(const LhDims& dm) {
  WsLayout w;
  size_t o = 0;
  w.scores = o; o = align_up(o + (size_t)dm.BH * dm.Rs * 4);
  const size_t coarse = (size_t)dm.BH * dm.Nl[dm.L - 1] * dm.d * 2;
  for (int i = 0; i < 3; ++i) { w.coarse[i] = o; o = align_up(o + coarse); }
  w.sel = o; o = align_up(o + (size_t)dm.BH * dm.Ksel * 4);
  w.fwd_total = o;
  const size_t rows = (size_t)dm.BH * dm.S;
  o = 0;
  w.dog = o; o = align_up(o + rows * dm.d * 4);    // fp32 window sums
  w.dog16 = o; o = align_up(o + rows * dm.d * 2);  // fp16, scaled per head
  w.stats = o; o = align_up(o + (size_t)dm.BH * stats_stride(dm) * 2 * 4);  // -LSE log2 e, -D / sqrt(d)
  w.amax = o; o = align_up(o + (size_t)dm.BH * 4);
  w.dinv = o; o = align_up(o + (size_t)dm.BH * 4);
  w.dqacc = o; o = align_up(o + rows * dm.d * 4);
  w.dkg = o; o = align_up(o + rows * dm.d * 4);
  w.dvg = o; o = align_up(o + rows * dm.d * 4);
  w.bwd_total = o;
  w.total = w.fwd_total > w.bwd_total ? w.fwd_total : w.bwd_total;
  if (w.total == 0) w.total = kAlign;
  return w;
}

inline bool aligned16(const void* p) { return p && ((uintptr_t)p & 15u) == 0; }

// Device status word of the current device.
int status_ptr(int** out) {
  static std::mutex mu;
  static int* cache[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return LH_ERR_CUDA;
  std::lock_guard<std::mutex> g(mu);
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_lh_state) != cudaSuccess) return LH_ERR_CUDA;
    cache[dev] = &static_cast<LhDeviceState*>(p)->status;
  }
  *out = cache[dev];
  return LH_OK;
}

int prepare(const lh_params* P, LhDims* dm) {
  int rc = make_dims(P, dm);
  if (rc) return rc;
  return status_ptr(&dm->status);
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace

int make_tmap_f32_3d(CUtensorMap* map, const void* base, int d, int rows, int bh, int box_cols, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return LH_ERR_CUDA;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)bh};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 4, (cuuint64_t)rows * d * 4};
  const cuuint32_t box[3] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? LH_OK : LH_ERR_CUDA;
}

int make_tmap_f16_3d(CUtensorMap* map, const void* base, int d, int rows, int bh, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return LH_ERR_CUDA;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)bh};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)rows * d * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? LH_OK : LH_ERR_CUDA;
}

int make_tmap_stats(CUtensorMap* map, const float* stats, int S, int bh, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return LH_ERR_CUDA;
  const uint64_t stride = (uint64_t)((S + 3) & ~3) * 4;
  const cuuint64_t dims[3] = {(cuuint64_t)S, (cuuint64_t)bh, 2};
  const cuuint64_t strides[2] = {(cuuint64_t)stride, (cuuint64_t)(stride * bh)};
  const cuuint32_t box[3] = {(cuuint32_t)box_rows, 1, 2};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(stats), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? LH_OK : LH_ERR_CUDA;
}

int make_tmap_f16_4d(CUtensorMap* map, const void* base, int d, int rows, int bh, int blocks, uint64_t block_stride,
                     int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return LH_ERR_CUDA;
  const uint64_t plain = (uint64_t)rows * d * 2 * bh;
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)bh, (cuuint64_t)blocks};
  const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)rows * d * 2,
                                 (cuuint64_t)(blocks > 1 ? block_stride : ((plain + 15) & ~uint64_t(15)))};
  const cuuint32_t box[4] = {64, (cuuint32_t)box_rows, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? LH_OK : LH_ERR_CUDA;
}

}  // namespace lh

using namespace lh;

#define LH_TRY(expr)        \
  do {                      \
    const int rc_ = (expr); \
    if (rc_) return rc_;    \
  } while (0)

extern "C" {

const char* lh_error_string(int status) {
  switch (status) {
    case LH_OK: return "ok";
    case LH_ERR_INVALID_ARG: return "invalid argument";
    case LH_ERR_UNSUPPORTED: return "unsupported shape";
    case LH_ERR_CUDA: return "CUDA error";
    case LH_ERR_TIMEOUT: return "device wait timed out";
    case LH_ERR_WORKSPACE: return "workspace too small";
    case LH_ERR_RANGE: return "value outside the fp16 operand range";
    default: return "unknown status";
  }
}

int lh_validate(const lh_params* P) {
  LhDims dm;
  return make_dims(P, &dm);
}

int64_t lh_S(const lh_params* P) {
  LhDims dm;
  const int rc = make_dims(P, &dm);
  return (rc == LH_OK || rc == LH_ERR_UNSUPPORTED) ? dm.S : -1;
}

int64_t lh_level_size(const lh_params* P, int level) {
  LhDims dm;
  const int rc = make_dims(P, &dm);
  if ((rc != LH_OK && rc != LH_ERR_UNSUPPORTED) || level < 0 || level >= dm.L) return -1;
  return dm.Nl[level];
}

int64_t lh_level_offset(const lh_params* P, int level) {
  LhDims dm;
  const int rc = make_dims(P, &dm);
  if ((rc != LH_OK && rc != LH_ERR_UNSUPPORTED) || level < 0 || level >= dm.L) return -1;
  return dm.off[level];
}

int64_t lh_pyramid_rows(const lh_params* P) {
  LhDims dm;
  const int rc = make_dims(P, &dm);
  return (rc == LH_OK || rc == LH_ERR_UNSUPPORTED) ? dm.Rp : -1;
}

int64_t lh_score_rows(const lh_params* P) {
  LhDims dm;
  const int rc = make_dims(P, &dm);
  return (rc == LH_OK || rc == LH_ERR_UNSUPPORTED) ? dm.Rs : -1;
}

int64_t lh_slot_rows(const lh_params* P) {
  LhDims dm;
  const int rc = make_dims(P, &dm);
  return (rc == LH_OK || rc == LH_ERR_UNSUPPORTED) ? dm.R : -1;
}

size_t lh_ctx_bytes(const lh_params* P) {
  LhDims dm;
  if (make_dims(P, &dm) != LH_OK) return 0;
  return ctx_layout(dm).total;
}

int lh_ctx_layout(const lh_params* P, lh_ctx_layout_t* out) {
  LhDims dm;
  LH_TRY(make_dims(P, &dm));
  if (!out) return LH_ERR_INVALID_ARG;
  const CtxLayout c = ctx_layout(dm);
  out->qg = c.qg; out->kg = c.kg; out->vg = c.vg; out->og = c.og;
  out->lse = c.lse; out->idx_g = c.idx_g; out->slot = c.slot; out->total = c.total;
  return LH_OK;
}

size_t lh_workspace_bytes(const lh_params* P) {
  LhDims dm;
  if (make_dims(P, &dm) != LH_OK) return 0;
  return ws_layout(dm).total;
}

int lh_pool(const lh_params* P, const void* x, void* pyr, void* stream) {
  LhDims dm;
  LH_TRY(prepare(P, &dm));
  if (dm.L == 1) return LH_OK;
  if (!aligned16(x) || !aligned16(pyr)) return LH_ERR_INVALID_ARG;
  PoolJobs jobs;
  memset(&jobs, 0, sizeof(jobs));
  PoolJob& j = jobs.job[0];
  j.x = x;
  j.pyr = pyr;
  j.pyr_rows = dm.Rp;
  for (int l = 1; l < dm.L; ++l) {
    j.write_mask |= 1u << l;
    j.row_off[l] = dm.poff[l];
  }
  return launch_pool_score(jobs, 1, dm, (cudaStream_t)stream);
}

int lh_score_topk(const lh_params* P, const void* k, const float* scores_in, float* scores_out, int32_t* idx_g,
                  int32_t* slot, void* ws, size_t ws_bytes, void* stream) {
  LhDims dm;
  LH_TRY(prepare(P, &dm));
  cudaStream_t st = (cudaStream_t)stream;
  if (!aligned16(idx_g) || !aligned16(slot)) return LH_ERR_INVALID_ARG;
  const WsLayout w = ws_layout(dm);
  if (!aligned16(ws) || ws_bytes < w.total) return ws ? LH_ERR_WORKSPACE : LH_ERR_INVALID_ARG;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  const float* scores = scores_in;
  if (dm.L >= 2 && !scores_in) {
    if (!aligned16(k) || (scores_out && !aligned16(scores_out))) return LH_ERR_INVALID_ARG;
    float* dst = scores_out ? scores_out : reinterpret_cast<float*>(wsb + w.scores);
    PoolJobs jobs;
    memset(&jobs, 0, sizeof(jobs));
    jobs.job[0].x = k;
    jobs.job[0].scores = dst;
    LH_TRY(launch_pool_score(jobs, 1, dm, st));
    scores = dst;
  } else if (dm.L >= 2 && !aligned16(scores_in)) {
    return LH_ERR_INVALID_ARG;
  }
  int32_t* sel = reinterpret_cast<int32_t*>(wsb + w.sel);
  LH_TRY(launch_topk(scores, sel, slot, dm, st));
  return launch_order(sel, idx_g, slot, dm, st);
}

int lh_gather(const lh_params* P, const void* q, const void* k, const void* v, const void* q_pyr, const void* k_pyr,
              const void* v_pyr, const int32_t* idx_g, void* qg, void* kg, void* vg, void* stream) {
  LhDims dm;
  LH_TRY(prepare(P, &dm));
  const void* xs[3] = {q, k, v};
  const void* ps[3] = {q_pyr, k_pyr, v_pyr};
  void* outs[3] = {qg, kg, vg};
  GatherJobs jobs;
  memset(&jobs, 0, sizeof(jobs));
  if (!aligned16(idx_g)) return LH_ERR_INVALID_ARG;
  for (int i = 0; i < 3; ++i) {
    if (!aligned16(xs[i]) || !aligned16(outs[i])) return LH_ERR_INVALID_ARG;
    if (dm.L > 1 && !aligned16(ps[i])) return LH_ERR_INVALID_ARG;
    GatherJob& j = jobs.job[i];
    j.x = xs[i];
    j.pyr = ps[i];
    j.pyr_rows = dm.Rp;
    for (int l = 1; l < dm.L; ++l) {
      j.pyr_mask |= 1u << l;
      j.row_off[l] = dm.poff[l];
    }
    j.out = outs[i];
  }
  return launch_gather(jobs, 3, idx_g, dm, (cudaStream_t)stream);
}

int lh_attend(const lh_params* P, const void* qg, const void* kg, const void* vg, float* og, float* lse,
              void* stream) {
  LhDims dm;
  LH_TRY(prepare(P, &dm));
  if (!aligned16(qg) || !aligned16(kg) || !aligned16(vg) || !aligned16(og) || !aligned16(lse))
    return LH_ERR_INVALID_ARG;
  return launch_attn_fwd(qg, kv_plain(kg, vg), og, lse, dm, (cudaStream_t)stream);
}

int lh_scatter(const lh_params* P, const float* og, const int32_t* slot, void* o, void* stream) {
  LhDims dm;
  LH_TRY(prepare(P, &dm));
  if (!aligned16(og) || !aligned16(slot) || !aligned16(o)) return LH_ERR_INVALID_ARG;
  return launch_scatter(og, slot, o, dm, (cudaStream_t)stream);
}

}  // extern "C"

namespace {

// Steps 1-4a of the forward (pool, score, top-K, order, gather) into the context.
int forward_select(const LhDims& dm, const void* q, const void* k, const void* v, uint8_t* cb, const CtxLayout& c,
                   uint8_t* wsb, const WsLayout& w, cudaStream_t st) {
  const void* xs[3] = {q, k, v};
  const int top = dm.L - 1;
  // 1-2: pool Q, K, V in one launch; only the coarsest level is stored, plus the key scores
  if (dm.L >= 2) {
    PoolJobs pj;
    memset(&pj, 0, sizeof(pj));
    for (int i = 0; i < 3; ++i) {
      pj.job[i].x = xs[i];
      pj.job[i].pyr = wsb + w.coarse[i];
      pj.job[i].pyr_rows = dm.Nl[top];
      pj.job[i].write_mask = 1u << top;
      pj.job[i].row_off[top] = 0;
    }
    pj.job[1].scores = reinterpret_cast<float*>(wsb + w.scores);
    LH_TRY(launch_pool_score(pj, 3, dm, st));
  }
  // 3: top-K and the gathered order
  int32_t* idx_g = reinterpret_cast<int32_t*>(cb + c.idx_g);
  int32_t* slot = reinterpret_cast<int32_t*>(cb + c.slot);
  int32_t* sel = reinterpret_cast<int32_t*>(wsb + w.sel);
  LH_TRY(launch_topk(reinterpret_cast<float*>(wsb + w.scores), sel, slot, dm, st));
  LH_TRY(launch_order(sel, idx_g, slot, dm, st));
  // 4a: gather (levels 1..L-2 recomputed from the raw rows with the same summation tree)
  GatherJobs gj;
  memset(&gj, 0, sizeof(gj));
  const size_t outs[3] = {c.qg, c.kg, c.vg};
  for (int i = 0; i < 3; ++i) {
    gj.job[i].x = xs[i];
    gj.job[i].pyr = wsb + w.coarse[i];
    gj.job[i].pyr_rows = dm.Nl[top];
    gj.job[i].pyr_mask = dm.L >= 2 ? (1u << top) : 0u;
    gj.job[i].row_off[top] = 0;
    gj.job[i].out = cb + outs[i];
  }
  return launch_gather(gj, 3, idx_g, dm, st);
}

// The backward's steps before the attention: dO_g window sums (plus, under context parallelism, the next rank's
// part of the last windows), the per-head scale, fp16 dO_g, D, and the zeroed dQ accumulator.
int backward_prep(const LhDims& dm, const void* dout, const uint8_t* cb, const CtxLayout& c, uint8_t* wsb,
                  const WsLayout& w, const float* halo_next, cudaStream_t st) {
  const int32_t* idx_g = reinterpret_cast<const int32_t*>(cb + c.idx_g);
  float* dog = reinterpret_cast<float*>(wsb + w.dog);
  unsigned int* amax = reinterpret_cast<unsigned int*>(wsb + w.amax);
  if (cudaMemsetAsync(amax, 0, (size_t)dm.BH * 4, st) != cudaSuccess) return LH_ERR_CUDA;
  LH_TRY(launch_scatter_bwd(dout, idx_g, dog, amax, dm, st));
  if (halo_next)
    LH_TRY(launch_dog_halo(dog, reinterpret_cast<const int32_t*>(cb + c.slot), halo_next, amax, dm, st));
  return launch_bwd_prep(dog, reinterpret_cast<const float*>(cb + c.og), reinterpret_cast<const float*>(cb + c.lse),
                         amax, wsb + w.dog16, reinterpret_cast<float*>(wsb + w.stats),
                         reinterpret_cast<float*>(wsb + w.dinv), reinterpret_cast<float*>(wsb + w.dqacc), dm, st);
}

}  // namespace

extern "C" {

int lh_forward(const lh_params* P, const void* q, const void* k, const void* v, void* o, void* ctx, void* ws,
               size_t ws_bytes, void* stream) {
  LhDims dm;
  LH_TRY(prepare(P, &dm));
  cudaStream_t st = (cudaStream_t)stream;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(ctx))
    return LH_ERR_INVALID_ARG;
  const WsLayout w = ws_layout(dm);
  if (!aligned16(ws) || ws_bytes < w.total) return ws ? LH_ERR_WORKSPACE : LH_ERR_INVALID_ARG;
  const CtxLayout c = ctx_layout(dm);
  uint8_t* cb = static_cast<uint8_t*>(ctx);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  LH_TRY(forward_select(dm, q, k, v, cb, c, wsb, w, st));
  // 4b: attention over the gathered sequence
  float* og = reinterpret_cast<float*>(cb + c.og);
  LH_TRY(launch_attn_fwd(cb + c.qg, kv_plain(cb + c.kg, cb + c.vg), og, reinterpret_cast<float*>(cb + c.lse), dm, st));
  // 5: scatter back
  return launch_scatter(og, reinterpret_cast<const int32_t*>(cb + c.slot), o, dm, st);
}

int lh_backward(const lh_params* P, const void* dout, const void* ctx, void* dq, void* dk, void* dv, void* ws,
                size_t ws_bytes, void* stream) {
  LhDims dm;
  LH_TRY(prepare(P, &dm));
  cudaStream_t st = (cudaStream_t)stream;
  if (!aligned16(dout) || !aligned16(ctx) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return LH_ERR_INVALID_ARG;
  const WsLayout w = ws_layout(dm);
  if (!aligned16(ws) || ws_bytes < w.total) return ws ? LH_ERR_WORKSPACE : LH_ERR_INVALID_ARG;
  const CtxLayout c = ctx_layout(dm);
  const uint8_t* cb = static_cast<const uint8_t*>(ctx);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  LH_TRY(backward_prep(dm, dout, cb, c, wsb, w, nullptr, st));
  float* dqacc = reinterpret_cast<float*>(wsb + w.dqacc);
  float* dkg = reinterpret_cast<float*>(wsb + w.dkg);
  float* dvg = reinterpret_cast<float*>(wsb + w.dvg);
  LH_TRY(launch_attn_bwd(cb + c.qg, kv_plain(cb + c.kg, cb + c.vg), wsb + w.dog16,
                         reinterpret_cast<const float*>(wsb + w.stats), reinterpret_cast<const float*>(wsb + w.dinv),
                         dqacc, dkg, dvg, 0, dm, st));
  return launch_unpool_bwd(dqacc, dkg, dvg, reinterpret_cast<const int32_t*>(cb + c.slot), dq, dk, dv, dm, st);
}

int lh_scatter_bwd(const lh_params* P, const void* dout, const int32_t* idx_g, float* dog, void* stream) {
  LhDims dm;
  LH_TRY(prepare(P, &dm));
  if (!aligned16(dout) || !aligned16(idx_g) || !aligned16(dog)) return LH_ERR_INVALID_ARG;
  return launch_scatter_bwd(dout, idx_g, dog, nullptr, dm, (cudaStream_t)stream);
}

int lh_attend_bwd(const lh_params* P, const void* qg, const void* kg, const void* vg, const float* og,
                  const float* lse, const float* dog, float* dqg, float* dkg, float* dvg, void* ws, size_t ws_bytes,
                  void* stream) {
  LhDims dm;
  LH_TRY(prepare(P, &dm));
  cudaStream_t st = (cudaStream_t)stream;
  if (!aligned16(qg) || !aligned16(kg) || !aligned16(vg) || !aligned16(og) || !aligned16(lse) || !aligned16(dog) ||
      !aligned16(dqg) || !aligned16(dkg) || !aligned16(dvg))
    return LH_ERR_INVALID_ARG;
  const WsLayout w = ws_layout(dm);
  if (!aligned16(ws) || ws_bytes < w.total) return ws ? LH_ERR_WORKSPACE : LH_ERR_INVALID_ARG;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  float* stats = reinterpret_cast<float*>(wsb + w.stats);
  float* dinv = reinterpret_cast<float*>(wsb + w.dinv);
  unsigned int* amax = reinterpret_cast<unsigned int*>(wsb + w.amax);
  if (cudaMemsetAsync(amax, 0, (size_t)dm.BH * 4, st) != cudaSuccess) return LH_ERR_CUDA;
  LH_TRY(launch_absmax(dog, amax, dm, st));
  LH_TRY(launch_bwd_prep(dog, og, lse, amax, wsb + w.dog16, stats, dinv, dqg, dm, st));
  return launch_attn_bwd(qg, kv_plain(kg, vg), wsb + w.dog16, stats, dinv, dqg, dkg, dvg, 0, dm, st);
}

int lh_set_wait_limit_ns(uint64_t ns) {
  int* p = nullptr;
  if (status_ptr(&p)) return LH_ERR_CUDA;
  const unsigned long long v = ns ? (unsigned long long)ns : (unsigned long long)kWaitLimitNs;
  if (cudaDeviceSynchronize() != cudaSuccess) return LH_ERR_CUDA;
  if (cudaMemcpy(&reinterpret_cast<LhDeviceState*>(p)->wait_limit_ns, &v, sizeof(v), cudaMemcpyHostToDevice) !=
      cudaSuccess)
    return LH_ERR_CUDA;
  return LH_OK;
}

int lh_get_status(void* stream) {
  int* p = nullptr;
  if (status_ptr(&p)) return LH_ERR_CUDA;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return LH_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return LH_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return LH_ERR_CUDA;
  return v;
}

}  // extern "C"

// ------------------------------------------------------------------------------------------------------------
// Selection without caller-provided scratch (lh_score_topk_static).
//
// Some callers cannot allocate device memory at the point where they need the selection: a runtime that plans
// all of its device memory once at start-up and forbids allocation on its step path, or a hook inside another
// framework that is handed only the tensors it reads and writes.  For them this entry point keeps its scratch
// (the per-level selection lists and, when the caller passes no score buffer, the scores) in one fixed device
// array owned by the library.
// ------------------------------------------------------------------------------------------------------------

namespace lh {
namespace {

// Loaded with the library on every device that uses it and held until the process exits.
static __device__ __align__(256) unsigned char g_static_scratch[LH_STATIC_SCRATCH_BYTES];

// Device address of g_static_scratch on the current device, looked up once per device.  The symbol's name is a
// host-side stand-in in host code, so kernels must be given this address instead.
int static_scratch_ptr(unsigned char** out) {
  static std::mutex mu;
  static unsigned char* cache[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return LH_ERR_CUDA;
  std::lock_guard<std::mutex> g(mu);
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess) return LH_ERR_CUDA;
    cache[dev] = static_cast<unsigned char*>(p);
  }
  *out = cache[dev];
  return LH_OK;
}

}  // namespace
}  // namespace lh

extern "C" int lh_score_topk_static(const lh_params* P, const void* k, const float* scores_in, float* scores_out,
                                    int32_t* idx_g, int32_t* slot, void* stream) {
  LhDims dm;
  LH_TRY(prepare(P, &dm));
  cudaStream_t st = (cudaStream_t)stream;
  if (!aligned16(idx_g) || !aligned16(slot)) return LH_ERR_INVALID_ARG;
  const bool own_scores = dm.L >= 2 && !scores_in && !scores_out;
  if (dm.L >= 2 && !scores_in && !aligned16(k)) return LH_ERR_INVALID_ARG;
  if (dm.L >= 2 && scores_in && !aligned16(scores_in)) return LH_ERR_INVALID_ARG;
  if (scores_out && !aligned16(scores_out)) return LH_ERR_INVALID_ARG;
  // scratch: the selection lists, then (only when the caller gives no score buffer) the scores
  const size_t sel_bytes = align_up((size_t)dm.BH * dm.Ksel * 4);
  const size_t need = sel_bytes + (own_scores ? align_up((size_t)dm.BH * dm.Rs * 4) : 0);
  if (need > (size_t)LH_STATIC_SCRATCH_BYTES) return LH_ERR_WORKSPACE;
  unsigned char* scratch = nullptr;
  LH_TRY(static_scratch_ptr(&scratch));
  int32_t* sel = reinterpret_cast<int32_t*>(scratch);
  const float* scores = scores_in;
  if (dm.L >= 2 && !scores_in) {
    float* dst = scores_out ? scores_out : reinterpret_cast<float*>(scratch + sel_bytes);
    PoolJobs jobs;
    memset(&jobs, 0, sizeof(jobs));
    jobs.job[0].x = k;
    jobs.job[0].scores = dst;
    LH_TRY(launch_pool_score(jobs, 1, dm, st));
    scores = dst;
  }
  LH_TRY(launch_topk(scores, sel, slot, dm, st));
  return launch_order(sel, idx_g, slot, dm, st);
}

// ------------------------------------------------------------------------------------------------------------
// Context parallelism: the sequence split into G equal shards at chunk boundaries, one per rank.
// ------------------------------------------------------------------------------------------------------------

namespace lh {
namespace {

// The shard's parameters and the checks that make the split exact: G | C and G | k keep every chunk, and therefore
// every pick, inside one shard (each rank selects exactly the global selection's entries of its tokens, S/G of
// them); the gathered rows per rank must fill whole 128-row attention tiles when G > 1.
int cp_local(const lh_params* P, int G, int rank, LhDims* glob, LhDims* loc, lh_params* Ploc) {
  if (!P || G < 1 || rank < 0 || rank >= G) return LH_ERR_INVALID_ARG;
  LH_TRY(make_dims(P, glob));
  if (P->C % G || P->k % G || P->N % G) return LH_ERR_INVALID_ARG;
  *Ploc = *P;
  Ploc->N = P->N / G;
  Ploc->k = P->k / G;
  Ploc->C = P->C / G;
  LH_TRY(make_dims(Ploc, loc));
  if ((int64_t)loc->S * G != glob->S) return LH_ERR_INVALID_ARG;  // unreachable when the checks above hold
  if (G > 1 && loc->S % 128 != 0) return LH_ERR_UNSUPPORTED;
  return LH_OK;
}

// cp_local plus the device status word (device entry points only).
int cp_prepare(const lh_params* P, int G, int rank, LhDims* glob, LhDims* loc, lh_params* Ploc) {
  LH_TRY(cp_local(P, G, rank, glob, loc, Ploc));
  return status_ptr(&loc->status);
}

struct CpSizes {
  size_t kv_offset, kv_bytes, v_offset, halo_bytes, dkv_bytes;
};
CpSizes cp_sizes(const LhDims& loc) {
  const CtxLayout c = ctx_layout(loc);
  const size_t rows = (size_t)loc.BH * loc.S * loc.d;
  CpSizes z;
  z.kv_offset = c.kg;
  z.v_offset = c.vg - c.kg;
  z.kv_bytes = align_up(z.v_offset + rows * 2);
  z.halo_bytes = (size_t)loc.BH * loc.L * loc.d * 4;
  z.dkv_bytes = 2 * rows * 4;
  return z;
}

}  // namespace
}  // namespace lh

extern "C" {

int lh_cp_layout(const lh_params* P, int G, lh_cp_layout_t* out) {
  LhDims glob, loc;
  lh_params Ploc;
  if (!out) return LH_ERR_INVALID_ARG;
  LH_TRY(cp_local(P, G, 0, &glob, &loc, &Ploc));
  const CpSizes z = cp_sizes(loc);
  out->local = Ploc;
  out->S_local = loc.S;
  out->kv_offset = z.kv_offset;
  out->kv_bytes = z.kv_bytes;
  out->v_offset = z.v_offset;
  out->halo_bytes = z.halo_bytes;
  out->dkv_bytes = z.dkv_bytes;
  return LH_OK;
}

int lh_cp_forward_select(const lh_params* P, int G, int rank, const void* q, const void* k, const void* v, void* ctx,
                         void* ws, size_t ws_bytes, void* stream) {
  LhDims glob, dm;
  lh_params Ploc;
  LH_TRY(cp_prepare(P, G, rank, &glob, &dm, &Ploc));
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(ctx)) return LH_ERR_INVALID_ARG;
  const WsLayout w = ws_layout(dm);
  if (!aligned16(ws) || ws_bytes < w.total) return ws ? LH_ERR_WORKSPACE : LH_ERR_INVALID_ARG;
  return forward_select(dm, q, k, v, static_cast<uint8_t*>(ctx), ctx_layout(dm), static_cast<uint8_t*>(ws), w,
                        (cudaStream_t)stream);
}

int lh_cp_forward_attend(const lh_params* P, int G, int rank, void* ctx, const void* kv_all, float* halo_out,
                         void* stream) {
  LhDims glob, dm;
  lh_params Ploc;
  LH_TRY(cp_prepare(P, G, rank, &glob, &dm, &Ploc));
  if (!aligned16(ctx) || !aligned16(kv_all) || !aligned16(halo_out)) return LH_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  const CtxLayout c = ctx_layout(dm);
  const CpSizes z = cp_sizes(dm);
  uint8_t* cb = static_cast<uint8_t*>(ctx);
  const uint8_t* kv = static_cast<const uint8_t*>(kv_all);
  const KvSource src{kv, kv + z.v_offset, G, (uint64_t)z.kv_bytes, rank * dm.S};
  float* og = reinterpret_cast<float*>(cb + c.og);
  LH_TRY(launch_attn_fwd(cb + c.qg, src, og, reinterpret_cast<float*>(cb + c.lse), dm, st));
  return launch_halo_fwd(og, reinterpret_cast<const int32_t*>(cb + c.slot), halo_out, dm, st);
}

int lh_cp_forward_scatter(const lh_params* P, int G, int rank, const void* ctx, const float* halo_prev, void* o,
                          void* stream) {
  LhDims glob, dm;
  lh_params Ploc;
  LH_TRY(cp_prepare(P, G, rank, &glob, &dm, &Ploc));
  if (!aligned16(ctx) || !aligned16(o) || (rank > 0 && !aligned16(halo_prev))) return LH_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  const CtxLayout c = ctx_layout(dm);
  const uint8_t* cb = static_cast<const uint8_t*>(ctx);
  const float* og = reinterpret_cast<const float*>(cb + c.og);
  const int32_t* slot = reinterpret_cast<const int32_t*>(cb + c.slot);
  LH_TRY(launch_scatter(og, slot, o, dm, st));
  return rank > 0 ? launch_scatter_halo(og, slot, halo_prev, o, dm, st) : LH_OK;
}

int lh_cp_backward_halo(const lh_params* P, int G, int rank, const void* dout, float* halo_out, void* stream) {
  LhDims glob, dm;
  lh_params Ploc;
  LH_TRY(cp_prepare(P, G, rank, &glob, &dm, &Ploc));
  if (!aligned16(dout) || !aligned16(halo_out)) return LH_ERR_INVALID_ARG;
  return launch_halo_bwd(dout, halo_out, dm, (cudaStream_t)stream);
}

int lh_cp_backward_attend(const lh_params* P, int G, int rank, const void* dout, const void* ctx, const void* kv_all,
                          const float* halo_next, float* dkv_part, void* ws, size_t ws_bytes, void* stream) {
  LhDims glob, dm;
  lh_params Ploc;
  LH_TRY(cp_prepare(P, G, rank, &glob, &dm, &Ploc));
  if (!aligned16(dout) || !aligned16(ctx) || !aligned16(kv_all) || !aligned16(dkv_part) ||
      (rank < G - 1 && !aligned16(halo_next)))
    return LH_ERR_INVALID_ARG;
  const WsLayout w = ws_layout(dm);
  if (!aligned16(ws) || ws_bytes < w.total) return ws ? LH_ERR_WORKSPACE : LH_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  const CtxLayout c = ctx_layout(dm);
  const CpSizes z = cp_sizes(dm);
  const uint8_t* cb = static_cast<const uint8_t*>(ctx);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  LH_TRY(backward_prep(dm, dout, cb, c, wsb, w, rank < G - 1 ? halo_next : nullptr, st));
  // blocks of ranks after this one see none of its queries: their share of the exchange is zero
  const size_t block_floats = z.dkv_bytes / 4;
  if (rank < G - 1 &&
      cudaMemsetAsync(dkv_part + (rank + 1) * block_floats, 0, (G - 1 - rank) * z.dkv_bytes, st) != cudaSuccess)
    return LH_ERR_CUDA;
  const uint8_t* kv = static_cast<const uint8_t*>(kv_all);
  const KvSource src{kv, kv + z.v_offset, G, (uint64_t)z.kv_bytes, rank * dm.S};
  const size_t rows = (size_t)dm.BH * dm.S * dm.d;
  return launch_attn_bwd(cb + c.qg, src, wsb + w.dog16, reinterpret_cast<const float*>(wsb + w.stats),
                         reinterpret_cast<const float*>(wsb + w.dinv), reinterpret_cast<float*>(wsb + w.dqacc),
                         dkv_part, dkv_part + rows, block_floats, dm, st);
}

int lh_cp_backward_unpool(const lh_params* P, int G, int rank, const void* ctx, const float* dkv, void* dq, void* dk,
                          void* dv, void* ws, size_t ws_bytes, void* stream) {
  LhDims glob, dm;
  lh_params Ploc;
  LH_TRY(cp_prepare(P, G, rank, &glob, &dm, &Ploc));
  if (!aligned16(ctx) || !aligned16(dkv) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return LH_ERR_INVALID_ARG;
  const WsLayout w = ws_layout(dm);
  if (!aligned16(ws) || ws_bytes < w.total) return ws ? LH_ERR_WORKSPACE : LH_ERR_INVALID_ARG;
  const CtxLayout c = ctx_layout(dm);
  const uint8_t* cb = static_cast<const uint8_t*>(ctx);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  const size_t rows = (size_t)dm.BH * dm.S * dm.d;
  return launch_unpool_bwd(reinterpret_cast<const float*>(wsb + w.dqacc), dkv, dkv + rows,
                           reinterpret_cast<const int32_t*>(cb + c.slot), dq, dk, dv, dm, (cudaStream_t)stream);
}

}  // extern "C"
