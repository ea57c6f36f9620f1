// scatter.cu — step 5 (offset scatter-back) and the streaming steps of the backward.
//
// Scatter follows [W]'s figure caption (scatter-back to the original positions) and [E] "Как four-stage
// pipeline…" (outputs redistributed with a causality-preserving offset): entry (l, j), ending at token
// E = (j+1) p^l - 1, contributes to tokens E .. E + p^l - 1, levels summed.  Token t therefore reads, per level,
// the entry j = floor((t+1)/p^l) - 1 when it is selected.
//
// The backward has no gradient through the selection ([E] "Как four-stage pipeline…"; [W] 深度洞察):
//   scatter backward: dO_g[s] = sum of dO over the window E_s .. min(E_s + w - 1, N - 1)   (fp32);
//   unpool backward:  dX[t] = sum_l dX_g[slot(l, floor(t/p^l))] / p^l over selected entries.
// Between them, the attention backward takes dO_g as fp16 operands.  dO_g is a sum of up to p^(L-1) rows, so
// it is scaled per head by a power of two (largest magnitude brought into [2^9, 2^10)) before rounding to
// fp16; D = rowsum(dO_g o O_g) is formed from the same rounded, scaled values, and the attention backward
// multiplies its results by the inverse scale.
//
// Layout: a group of d/8 lanes per row, each lane 8 features; fp32 accumulation, one rounding at the end.
#include "internal.h"

namespace lh {

namespace {

__device__ __forceinline__ int level_of(int gid, const LhDims& dm) {
  int lev = 0;
#pragma unroll
  for (int l = 1; l < LH_MAX_LEVELS; ++l)
    if (l < dm.L && gid >= dm.off[l]) lev = l;
  return lev;
}

__device__ __forceinline__ uint4 pack8_rn(const float (&a)[8]) {
  return make_uint4(pack_bf16x2_rn(a[0], a[1]), pack_bf16x2_rn(a[2], a[3]), pack_bf16x2_rn(a[4], a[5]),
                    pack_bf16x2_rn(a[6], a[7]));
}

// 8 consecutive fp32 values (32 bytes).
__device__ __forceinline__ void load8f(const float* p, float (&f)[8]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
__device__ __forceinline__ void store8f(float* p, const float (&f)[8]) {
  reinterpret_cast<float4*>(p)[0] = make_float4(f[0], f[1], f[2], f[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(f[4], f[5], f[6], f[7]);
}

// Fold a per-row maximum magnitude m (held by the G lanes of a row group) into amax[bh] with few atomics: rows of
// a warp are consecutive, so the warp spans one head (one atomic) or two (one atomic per row group).  Clamped
// idle groups repeat the last row and are harmless for a maximum.
template <int G>
__device__ __forceinline__ void head_max_atomic(float m, int bh, bool active, int lane, unsigned int* amax) {
#pragma unroll
  for (int off = 1; off < G; off <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  const int bh0 = __shfl_sync(0xffffffffu, bh, 0);
  if (__all_sync(0xffffffffu, bh == bh0)) {
#pragma unroll
    for (int off = G; off < 32; off <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if ((threadIdx.x & 31) == 0 && active) atomicMax(amax + bh, __float_as_uint(m));
  } else if (lane == 0 && active) {
    atomicMax(amax + bh, __float_as_uint(m));
  }
}

// Power-of-two scale bringing the largest magnitude `amax` into [2^9, 2^10); 1 for an all-zero head.
__device__ __forceinline__ float head_scale(float amax) {
  if (!(amax > 0.f) || !isfinite(amax)) return 1.f;
  int e;
  frexpf(amax, &e);  // amax = m 2^e, m in [0.5, 1)
  return ldexpf(1.f, 10 - e);
}

// Tokens per row group in the token-major kernels: every slot lookup of the group is issued before any row load,
// so a thread keeps up to kMaxL * kTok independent loads in flight instead of a chain of dependent ones.
constexpr int kTok = 4;
constexpr int kMaxL = 5;

// Row group g covers the kTok tokens whose "key" is g*kTok .. g*kTok + kTok - 1, where key = t + 1 for the offset
// scatter (entry j = key/w - 1) and key = t for the unpool (j = key/w).  Windows are powers of two, so for every
// level with w >= kTok the whole group reads ONE entry (one slot lookup, one row load, added to all kTok tokens);
// only narrower levels need per-token lookups.  Rows are summed in fp32 with per-level weights.
template <int D, bool kOffset>
__device__ __forceinline__ void token_sum(const float* __restrict__ src, const int32_t* __restrict__ sl, int bh,
                                          int key0, int lane, const LhDims& dm, float (&acc)[kTok][8]) {
  int s[kMaxL][kTok];
#pragma unroll
  for (int lev = 0; lev < kMaxL; ++lev) {
#pragma unroll
    for (int u = 0; u < kTok; ++u) s[lev][u] = -1;
    if (lev >= dm.L) continue;
    const int sh = dm.wlog[lev];
    if ((1 << sh) >= kTok) {
      const int j = (key0 >> sh) - (kOffset ? 1 : 0);
      if (j >= 0 && j < dm.Nl[lev]) s[lev][0] = sl[dm.off[lev] + j];
    } else {
#pragma unroll
      for (int u = 0; u < kTok; ++u) {
        const int j = ((key0 + u) >> sh) - (kOffset ? 1 : 0);
        if (j >= 0 && j < dm.Nl[lev]) s[lev][u] = sl[dm.off[lev] + j];
      }
    }
  }
#pragma unroll
  for (int u = 0; u < kTok; ++u)
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[u][i] = 0.f;
#pragma unroll
  for (int lev = 0; lev < kMaxL; ++lev) {
    if (lev >= dm.L) continue;
    const int sh = dm.wlog[lev];
    const float wgt = kOffset ? 1.0f : __uint_as_float((127u - (uint32_t)sh) << 23);  // 2^-sh, exact
    if ((1 << sh) >= kTok) {
      if (s[lev][0] >= 0) {
        float f[8];
        load8f(src + ((int64_t)bh * dm.S + s[lev][0]) * D + lane * 8, f);
#pragma unroll
        for (int u = 0; u < kTok; ++u)
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[u][i] = fmaf(f[i], wgt, acc[u][i]);
      }
    } else {
#pragma unroll
      for (int u = 0; u < kTok; ++u) {
        if (s[lev][u] >= 0) {
          float f[8];
          load8f(src + ((int64_t)bh * dm.S + s[lev][u]) * D + lane * 8, f);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[u][i] = fmaf(f[i], wgt, acc[u][i]);
        }
      }
    }
  }
}

template <int D>
__global__ void __launch_bounds__(256) scatter_kernel(const float* __restrict__ og, const int32_t* __restrict__ slot,
                                                      __nv_bfloat16* __restrict__ o, LhDims dm) {
  constexpr int G = D / 8;
  const int lane = threadIdx.x % G;
  const int gph = (dm.N + kTok) / kTok;  // row groups per head: keys t + 1 = 1 .. N
  const int64_t ngrp = (int64_t)dm.BH * gph;
  // grid-stride over row groups: a few resident blocks per SM instead of one short-lived block per 64 tokens
  for (int64_t grp = (int64_t)blockIdx.x * (256 / G) + threadIdx.x / G; grp < ngrp;
       grp += (int64_t)gridDim.x * (256 / G)) {
    const int bh = (int)(grp / gph);
    const int key0 = (int)(grp % gph) * kTok;
    float acc[kTok][8];
    token_sum<D, true>(og, slot + (int64_t)bh * dm.R, bh, key0, lane, dm, acc);
#pragma unroll
    for (int u = 0; u < kTok; ++u) {
      const int t = key0 + u - 1;
      if (t >= 0 && t < dm.N) st_stream16(o + ((int64_t)bh * dm.N + t) * D + lane * 8, pack8_rn(acc[u]));
    }
  }
}

// One group per gathered row: dog[s] = fp32 window sum of dout.  With amax non-null, also the running per-head
// maximum magnitude (non-negative fp32 bit patterns order like their values).
template <int D>
__global__ void __launch_bounds__(256) scatter_bwd_kernel(const __nv_bfloat16* __restrict__ dout,
                                                          const int32_t* __restrict__ idx_g, float* __restrict__ dog,
                                                          unsigned int* __restrict__ amax, LhDims dm) {
  constexpr int G = D / 8;
  const int lane = threadIdx.x % G;
  const int64_t total = (int64_t)dm.BH * dm.S;
  const int64_t row0 = (int64_t)blockIdx.x * (256 / G) + threadIdx.x / G;
  const bool active = row0 < total;
  const int64_t row = active ? row0 : total - 1;
  const int bh = (int)(row / dm.S);
  const int gid = idx_g[row];
  const int lev = level_of(gid, dm);
  const int j = gid - dm.off[lev];
  const int w = dm.wl[lev];
  const int t0 = (j + 1) * w - 1;
  const int t1 = min(t0 + w - 1, dm.N - 1);
  const __nv_bfloat16* src = dout + ((int64_t)bh * dm.N) * D + lane * 8;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  int t = t0;
  for (; t + 3 <= t1; t += 4) {  // four rows in flight
    uint4 r[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) r[u] = ld_stream16(src + (int64_t)(t + u) * D);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float f[8];
      unpack8(r[u], f);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += f[i];
    }
  }
  for (; t <= t1; ++t) {
    float f[8];
    unpack8(ld_stream16(src + (int64_t)t * D), f);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] += f[i];
  }
  if (active) store8f(dog + row * D + lane * 8, acc);
  if (amax) {
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(acc[i]));
    head_max_atomic<G>(m, bh, active, lane, amax);
  }
}

// Per-head maximum magnitude of an fp32 [BH, S, d] tensor (for the stand-alone attention backward).
template <int D>
__global__ void __launch_bounds__(256) absmax_kernel(const float* __restrict__ x, unsigned int* __restrict__ amax,
                                                     LhDims dm) {
  constexpr int G = D / 8;
  const int lane = threadIdx.x % G;
  const int64_t total = (int64_t)dm.BH * dm.S;
  const int64_t row0 = (int64_t)blockIdx.x * (256 / G) + threadIdx.x / G;
  const bool active = row0 < total;
  const int64_t row = active ? row0 : total - 1;
  float f[8];
  load8f(x + row * D + lane * 8, f);
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(f[i]));
  head_max_atomic<G>(m, (int)(row / dm.S), active, lane, amax);
}

// dog16[s] = fp16_RN(dog[s] * scale_bh), D[s] = <dog16[s], og[s]> (scaled domain), dqacc[s] = 0, and the inverse
// scale of each head.
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const float* __restrict__ dog, const float* __restrict__ og,
                                                       const unsigned int* __restrict__ amax, __half* __restrict__ dog16,
                                                       float* __restrict__ dvec, float* __restrict__ dinv,
                                                       float* __restrict__ dqacc, LhDims dm) {
  constexpr int G = D / 8;
  const int lane = threadIdx.x % G;
  const int64_t total = (int64_t)dm.BH * dm.S;
  const int64_t row0 = (int64_t)blockIdx.x * (256 / G) + threadIdx.x / G;
  const bool active = row0 < total;
  const int64_t row = active ? row0 : total - 1;
  const int bh = (int)(row / dm.S);
  const float sc = head_scale(__uint_as_float(amax[bh]));
  float a[8], b[8];
  load8f(dog + row * D + lane * 8, a);
  load8f(og + row * D + lane * 8, b);
  uint32_t h[4];
  float dot = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __half2 v = __floats2half2_rn(a[2 * i] * sc, a[2 * i + 1] * sc);
    h[i] = *reinterpret_cast<uint32_t*>(&v);
    const float2 r = __half22float2(v);
    dot = fmaf(r.x, b[2 * i], dot);
    dot = fmaf(r.y, b[2 * i + 1], dot);
  }
#pragma unroll
  for (int off = 1; off < G; off <<= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
  if (active) {
    st16(dog16 + row * D + lane * 8, make_uint4(h[0], h[1], h[2], h[3]));
    if (lane == 0) dvec[row] = dot;
    if (lane == 0 && row % dm.S == 0) dinv[bh] = 1.f / sc;
    const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    store8f(dqacc + row * D + lane * 8, z);
  }
}

// blockIdx.y selects the tensor: 0 = dQ, 1 = dK, 2 = dV (fp32 gathered gradients).
template <int D>
__global__ void __launch_bounds__(256) unpool_bwd_kernel(const float* __restrict__ dqg, const float* __restrict__ dkg,
                                                         const float* __restrict__ dvg, const int32_t* __restrict__ slot,
                                                         __nv_bfloat16* dq, __nv_bfloat16* dk, __nv_bfloat16* dv,
                                                         LhDims dm) {
  constexpr int G = D / 8;
  const int which = blockIdx.y;
  const int lane = threadIdx.x % G;
  const int gph = (dm.N + kTok - 1) / kTok;
  const int64_t ngrp = (int64_t)dm.BH * gph;
  const float* src = which == 0 ? dqg : (which == 1 ? dkg : dvg);
  __nv_bfloat16* out = which == 0 ? dq : (which == 1 ? dk : dv);
  for (int64_t grp = (int64_t)blockIdx.x * (256 / G) + threadIdx.x / G; grp < ngrp;
       grp += (int64_t)gridDim.x * (256 / G)) {
    const int bh = (int)(grp / gph);
    const int t0 = (int)(grp % gph) * kTok;  // key = t
    float acc[kTok][8];
    token_sum<D, false>(src, slot + (int64_t)bh * dm.R, bh, t0, lane, dm, acc);
#pragma unroll
    for (int u = 0; u < kTok; ++u)
      if (t0 + u < dm.N) st_stream16(out + ((int64_t)bh * dm.N + t0 + u) * D + lane * 8, pack8_rn(acc[u]));
  }
}

template <int D>
int blocks_for(int64_t rows) {
  return (int)((rows + 256 / (D / 8) - 1) / (256 / (D / 8)));
}

// Blocks for a grid-stride kernel: enough for every row group, capped at what the device keeps resident at once
// (blocks per SM from the occupancy calculator times the SM count), so the loop has no ragged last wave.
template <typename Kernel>
int resident_blocks(Kernel kernel, int64_t need) {
  int dev = 0, sms = 148, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, 256, 0);
  const int64_t cap = (int64_t)sms * (per_sm > 0 ? per_sm : 1);
  return (int)(need < cap ? need : cap);
}

// `slices` launches share the device (gridDim.y), so each gets 1/slices of the resident blocks.
template <int D, typename Kernel>
int token_blocks(Kernel kernel, const LhDims& dm, int slices) {
  const int b = resident_blocks(kernel, blocks_for<D>((int64_t)dm.BH * ((dm.N + kTok - 1) / kTok))) / slices;
  return b > 0 ? b : 1;
}

}  // namespace

int launch_scatter(const float* og, const int32_t* slot, void* o, const LhDims& dm, cudaStream_t st) {
  KernelTimer timer("scatter", st);
  if (dm.d == 64)
    scatter_kernel<64><<<token_blocks<64>(scatter_kernel<64>, dm, 1), 256, 0, st>>>(og, slot, (__nv_bfloat16*)o, dm);
  else
    scatter_kernel<128><<<token_blocks<128>(scatter_kernel<128>, dm, 1), 256, 0, st>>>(og, slot, (__nv_bfloat16*)o, dm);
  return check_launch();
}

int launch_scatter_bwd(const void* dout, const int32_t* idx_g, float* dog, unsigned int* amax, const LhDims& dm,
                       cudaStream_t st) {
  const int64_t rows = (int64_t)dm.BH * dm.S;
  KernelTimer timer("scatter_bwd", st);
  if (dm.d == 64)
    scatter_bwd_kernel<64><<<blocks_for<64>(rows), 256, 0, st>>>((const __nv_bfloat16*)dout, idx_g, dog, amax, dm);
  else
    scatter_bwd_kernel<128><<<blocks_for<128>(rows), 256, 0, st>>>((const __nv_bfloat16*)dout, idx_g, dog, amax, dm);
  return check_launch();
}

int launch_absmax(const float* x, unsigned int* amax, const LhDims& dm, cudaStream_t st) {
  const int64_t rows = (int64_t)dm.BH * dm.S;
  KernelTimer timer("absmax", st);
  if (dm.d == 64)
    absmax_kernel<64><<<blocks_for<64>(rows), 256, 0, st>>>(x, amax, dm);
  else
    absmax_kernel<128><<<blocks_for<128>(rows), 256, 0, st>>>(x, amax, dm);
  return check_launch();
}

int launch_bwd_prep(const float* dog, const float* og, const unsigned int* amax, void* dog16, float* dvec, float* dinv,
                    float* dqacc, const LhDims& dm, cudaStream_t st) {
  const int64_t rows = (int64_t)dm.BH * dm.S;
  KernelTimer timer("bwd_prep", st);
  if (dm.d == 64)
    bwd_prep_kernel<64><<<blocks_for<64>(rows), 256, 0, st>>>(dog, og, amax, (__half*)dog16, dvec, dinv, dqacc, dm);
  else
    bwd_prep_kernel<128><<<blocks_for<128>(rows), 256, 0, st>>>(dog, og, amax, (__half*)dog16, dvec, dinv, dqacc, dm);
  return check_launch();
}

int launch_unpool_bwd(const float* dqg, const float* dkg, const float* dvg, const int32_t* slot, void* dq, void* dk,
                      void* dv, const LhDims& dm, cudaStream_t st) {
  KernelTimer timer("unpool_bwd", st);
  if (dm.d == 64)
    unpool_bwd_kernel<64><<<dim3(token_blocks<64>(unpool_bwd_kernel<64>, dm, 3), 3), 256, 0, st>>>(
        dqg, dkg, dvg, slot, (__nv_bfloat16*)dq, (__nv_bfloat16*)dk, (__nv_bfloat16*)dv, dm);
  else
    unpool_bwd_kernel<128><<<dim3(token_blocks<128>(unpool_bwd_kernel<128>, dm, 3), 3), 256, 0, st>>>(
        dqg, dkg, dvg, slot, (__nv_bfloat16*)dq, (__nv_bfloat16*)dk, (__nv_bfloat16*)dv, dm);
  return check_launch();
}

}  // namespace lh
