// scatter.cu — step 5 (offset scatter-back) and the streaming steps of the backward.
//
// Scatter follows [W]'s figure caption (scatter-back to the original positions) and [E] "Как four-stage
// pipeline…" (outputs redistributed with a causality-preserving offset): entry (l, j), ending at token
// E = (j+1) p^l - 1, contributes to tokens E .. E + p^l - 1, levels summed.  Token t therefore reads, per level,
// the entry j = floor((t+1)/p^l) - 1 when it is selected.
//
// The backward has no gradient through the selection ([E] "Как four-stage pipeline…"; [W] 深度洞察):
//   scatter backward: dO_g[s] = sum of dO over the window E_s .. min(E_s + w - 1, N - 1);
//   unpool backward:  dX[t] = sum_l dX_g[slot(l, floor(t/p^l))] / p^l over selected entries.
//
// Layout: a group of d/8 lanes per row, each lane 8 features (16 bytes); fp32 accumulation, one bf16 rounding.
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

template <int D>
__global__ void __launch_bounds__(256) scatter_kernel(const __nv_bfloat16* __restrict__ og,
                                                      const int32_t* __restrict__ slot, __nv_bfloat16* __restrict__ o,
                                                      LhDims dm) {
  constexpr int G = D / 8;
  const int lane = threadIdx.x % G;
  const int64_t row = (int64_t)blockIdx.x * (256 / G) + threadIdx.x / G;
  if (row >= (int64_t)dm.BH * dm.N) return;
  const int bh = (int)(row / dm.N);
  const int t = (int)(row % dm.N);
  const int32_t* sl = slot + (int64_t)bh * dm.R;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int lev = 0; lev < dm.L; ++lev) {
    const int j = (t + 1) / dm.wl[lev] - 1;
    if (j < 0) continue;
    const int s = sl[dm.off[lev] + j];
    if (s < 0) continue;
    float f[8];
    unpack8(ld16(og + ((int64_t)bh * dm.S + s) * D + lane * 8), f);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] += f[i];
  }
  st_stream16(o + row * D + lane * 8, pack8_rn(acc));
}

// One group per gathered row.  Optionally also D[s] = <dO_g[s], O_g[s]> (with the rounded dO_g) for the
// attention backward, and zeroes the fp32 dQ_g accumulator row.
template <int D>
__global__ void __launch_bounds__(256) scatter_bwd_kernel(const __nv_bfloat16* __restrict__ dout,
                                                          const int32_t* __restrict__ idx_g,
                                                          __nv_bfloat16* __restrict__ dog,
                                                          const __nv_bfloat16* __restrict__ og, float* __restrict__ dvec,
                                                          float* __restrict__ dqacc, LhDims dm) {
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
  const uint4 packed = pack8_rn(acc);
  if (active) st16(dog + row * D + lane * 8, packed);
  if (dvec) {
    float rd[8], of[8];
    unpack8(packed, rd);
    unpack8(ld16(og + row * D + lane * 8), of);
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) dot = fmaf(rd[i], of[i], dot);
#pragma unroll
    for (int off = 1; off < G; off <<= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
    if (active && lane == 0) dvec[row] = dot;
  }
  if (dqacc && active) {
    float4* z = reinterpret_cast<float4*>(dqacc + row * D + lane * 8);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// D[s] = <dO_g[s], O_g[s]> and a zeroed fp32 dQ_g accumulator, for the stand-alone attention backward.
template <int D>
__global__ void __launch_bounds__(256) attn_prep_kernel(const __nv_bfloat16* __restrict__ og,
                                                        const __nv_bfloat16* __restrict__ dog,
                                                        float* __restrict__ dvec, float* __restrict__ dqacc,
                                                        LhDims dm) {
  constexpr int G = D / 8;
  const int lane = threadIdx.x % G;
  const int64_t total = (int64_t)dm.BH * dm.S;
  const int64_t row0 = (int64_t)blockIdx.x * (256 / G) + threadIdx.x / G;
  const bool active = row0 < total;
  const int64_t row = active ? row0 : total - 1;
  float a[8], b[8];
  unpack8(ld16(dog + row * D + lane * 8), a);
  unpack8(ld16(og + row * D + lane * 8), b);
  float dot = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) dot = fmaf(a[i], b[i], dot);
#pragma unroll
  for (int off = 1; off < G; off <<= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
  if (active) {
    if (lane == 0) dvec[row] = dot;
    float4* z = reinterpret_cast<float4*>(dqacc + row * D + lane * 8);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// blockIdx.y = 0: dQ from the fp32 accumulator; 1: dK; 2: dV (bf16 gathered gradients).
template <int D>
__global__ void __launch_bounds__(256) unpool_bwd_kernel(const float* __restrict__ dqg,
                                                         const __nv_bfloat16* __restrict__ dkg,
                                                         const __nv_bfloat16* __restrict__ dvg,
                                                         const int32_t* __restrict__ slot, __nv_bfloat16* dq,
                                                         __nv_bfloat16* dk, __nv_bfloat16* dv, LhDims dm) {
  constexpr int G = D / 8;
  const int which = blockIdx.y;
  const int lane = threadIdx.x % G;
  const int64_t row = (int64_t)blockIdx.x * (256 / G) + threadIdx.x / G;
  if (row >= (int64_t)dm.BH * dm.N) return;
  const int bh = (int)(row / dm.N);
  const int t = (int)(row % dm.N);
  const int32_t* sl = slot + (int64_t)bh * dm.R;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int lev = 0; lev < dm.L; ++lev) {
    const int s = sl[dm.off[lev] + t / dm.wl[lev]];
    if (s < 0) continue;
    const float inv_w = 1.0f / (float)dm.wl[lev];  // exact: power-of-two window
    const int64_t srow = (int64_t)bh * dm.S + s;
    float f[8];
    if (which == 0) {
      const float4* p = reinterpret_cast<const float4*>(dqg + srow * D + lane * 8);
      const float4 a = p[0], b = p[1];
      f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    } else {
      unpack8(ld16((which == 1 ? dkg : dvg) + srow * D + lane * 8), f);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = fmaf(f[i], inv_w, acc[i]);
  }
  __nv_bfloat16* out = which == 0 ? dq : (which == 1 ? dk : dv);
  st_stream16(out + row * D + lane * 8, pack8_rn(acc));
}

template <int D>
int blocks_for(int64_t rows) {
  return (int)((rows + 256 / (D / 8) - 1) / (256 / (D / 8)));
}

}  // namespace

int launch_scatter(const void* og, const int32_t* slot, void* o, const LhDims& dm, cudaStream_t st) {
  const int64_t rows = (int64_t)dm.BH * dm.N;
  KernelTimer timer("scatter", st);
  if (dm.d == 64)
    scatter_kernel<64><<<blocks_for<64>(rows), 256, 0, st>>>((const __nv_bfloat16*)og, slot, (__nv_bfloat16*)o, dm);
  else
    scatter_kernel<128><<<blocks_for<128>(rows), 256, 0, st>>>((const __nv_bfloat16*)og, slot, (__nv_bfloat16*)o,
                                                                dm);
  return check_launch();
}

int launch_scatter_bwd(const void* dout, const int32_t* idx_g, void* dog, const void* og, float* dvec, float* dqacc,
                       const LhDims& dm, cudaStream_t st) {
  const int64_t rows = (int64_t)dm.BH * dm.S;
  KernelTimer timer("scatter_bwd", st);
  if (dm.d == 64)
    scatter_bwd_kernel<64><<<blocks_for<64>(rows), 256, 0, st>>>((const __nv_bfloat16*)dout, idx_g,
                                                                  (__nv_bfloat16*)dog, (const __nv_bfloat16*)og,
                                                                  dvec, dqacc, dm);
  else
    scatter_bwd_kernel<128><<<blocks_for<128>(rows), 256, 0, st>>>((const __nv_bfloat16*)dout, idx_g,
                                                                    (__nv_bfloat16*)dog, (const __nv_bfloat16*)og,
                                                                    dvec, dqacc, dm);
  return check_launch();
}

int launch_attn_prep(const void* og, const void* dog, float* dvec, float* dqacc, const LhDims& dm, cudaStream_t st) {
  const int64_t rows = (int64_t)dm.BH * dm.S;
  KernelTimer timer("attn_prep", st);
  if (dm.d == 64)
    attn_prep_kernel<64><<<blocks_for<64>(rows), 256, 0, st>>>((const __nv_bfloat16*)og, (const __nv_bfloat16*)dog,
                                                                dvec, dqacc, dm);
  else
    attn_prep_kernel<128><<<blocks_for<128>(rows), 256, 0, st>>>((const __nv_bfloat16*)og,
                                                                  (const __nv_bfloat16*)dog, dvec, dqacc, dm);
  return check_launch();
}

int launch_unpool_bwd(const float* dqg, const void* dkg, const void* dvg, const int32_t* slot, void* dq, void* dk,
                      void* dv, const LhDims& dm, cudaStream_t st) {
  const int64_t rows = (int64_t)dm.BH * dm.N;
  KernelTimer timer("unpool_bwd", st);
  if (dm.d == 64)
    unpool_bwd_kernel<64><<<dim3(blocks_for<64>(rows), 3), 256, 0, st>>>(
        dqg, (const __nv_bfloat16*)dkg, (const __nv_bfloat16*)dvg, slot, (__nv_bfloat16*)dq, (__nv_bfloat16*)dk,
        (__nv_bfloat16*)dv, dm);
  else
    unpool_bwd_kernel<128><<<dim3(blocks_for<128>(rows), 3), 256, 0, st>>>(
        dqg, (const __nv_bfloat16*)dkg, (const __nv_bfloat16*)dvg, slot, (__nv_bfloat16*)dq, (__nv_bfloat16*)dk,
        (__nv_bfloat16*)dv, dm);
  return check_launch();
}

}  // namespace lh
