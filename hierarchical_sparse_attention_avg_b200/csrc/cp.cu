// cp.cu — the small exchange-side kernels of context parallelism (the sequence split across ranks).
//
// [E] "Може ли този подход да скалира отвъд един GPU…": beyond ~100K tokens the layer runs context-parallel; pooling,
// scoring and top-K stay local to each shard and the gathered subsequence, being dense, takes part in ordinary
// ring attention.  Here the N tokens are split into G equal shards at chunk boundaries (G | C), so every pyramid
// entry lies inside one shard and each rank's selection is the global selection restricted to its shard.  Two
// steps of the layer reach across a shard edge, and only by less than one coarsest window:
//   forward  — token t < w_l - 1 of rank r receives, at level l, the output of rank r-1's last level-l entry;
//   backward — the window sum dO_g of rank r's last level-l entry runs into the first w_l - 1 tokens of rank r+1.
// Each rank therefore hands its neighbour one row per (head, level): the kernels below build those "halo" rows
// and fold the received ones in.  A halo block is fp32 [BH][L][d].
#include "internal.h"

namespace lh {

namespace {

// One warp per (head, level): the output row of the shard's last level-l entry, or zeros when it is not selected.
template <int D>
__global__ void __launch_bounds__(256) halo_fwd_kernel(const float* __restrict__ og, const int32_t* __restrict__ slot,
                                                       float* __restrict__ halo, LhDims dm) {
  constexpr int V = D / 32;  // features per lane
  const int w = blockIdx.x * 8 + threadIdx.x / 32, lane = threadIdx.x % 32;
  if (w >= dm.BH * dm.L) return;
  const int bh = w / dm.L, lev = w % dm.L;
  const int s = slot[(int64_t)bh * dm.R + dm.off[lev] + dm.Nl[lev] - 1];
  float* dst = halo + (int64_t)w * D + lane * V;
#pragma unroll
  for (int i = 0; i < V; ++i) dst[i] = s >= 0 ? og[((int64_t)bh * dm.S + s) * D + lane * V + i] : 0.f;
}

// One warp per token t < w_{L-1} - 1 of a head: O[t] recomputed with the previous rank's halo rows for the levels
// whose candidate entry lies in the previous shard (j = -1), summed with the shard's own entries in level order
// and rounded once.  Runs after the ordinary scatter, which gave these tokens only their local contributions.
template <int D>
__global__ void __launch_bounds__(256) scatter_halo_kernel(const float* __restrict__ og,
                                                           const int32_t* __restrict__ slot,
                                                           const float* __restrict__ halo, __nv_bfloat16* __restrict__ o,
                                                           LhDims dm) {
  constexpr int V = D / 32;
  const int t = blockIdx.x * 8 + threadIdx.x / 32, lane = threadIdx.x % 32;
  const int bh = blockIdx.y;
  if (t >= dm.wl[dm.L - 1] - 1) return;
  float acc[V];
#pragma unroll
  for (int i = 0; i < V; ++i) acc[i] = 0.f;
  for (int lev = 0; lev < dm.L; ++lev) {
    const int j = (t + 1) / dm.wl[lev] - 1;
    const float* src = nullptr;
    if (j < 0) {
      src = halo + ((int64_t)bh * dm.L + lev) * D;
    } else {
      const int s = slot[(int64_t)bh * dm.R + dm.off[lev] + j];
      if (s >= 0) src = og + ((int64_t)bh * dm.S + s) * D;
    }
    if (src) {
#pragma unroll
      for (int i = 0; i < V; ++i) acc[i] += src[lane * V + i];
    }
  }
  __nv_bfloat16* dst = o + ((int64_t)bh * dm.N + t) * D + lane * V;
#pragma unroll
  for (int i = 0; i < V; i += 2) *reinterpret_cast<uint32_t*>(dst + i) = pack_bf16x2_rn(acc[i], acc[i + 1]);
}

// One warp per (head, level): the sum of the shard's first w_l - 1 upstream-gradient rows (fp32), the part of the
// previous rank's last level-l window that lies in this shard.
template <int D>
__global__ void __launch_bounds__(256) halo_bwd_kernel(const __nv_bfloat16* __restrict__ dout, float* __restrict__ halo,
                                                       LhDims dm) {
  constexpr int V = D / 32;
  const int w = blockIdx.x * 8 + threadIdx.x / 32, lane = threadIdx.x % 32;
  if (w >= dm.BH * dm.L) return;
  const int bh = w / dm.L, lev = w % dm.L;
  float acc[V];
#pragma unroll
  for (int i = 0; i < V; ++i) acc[i] = 0.f;
  for (int t = 0; t < dm.wl[lev] - 1; ++t) {
    const __nv_bfloat16* src = dout + ((int64_t)bh * dm.N + t) * D + lane * V;
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] += __bfloat162float(src[i]);
  }
  float* dst = halo + (int64_t)w * D + lane * V;
#pragma unroll
  for (int i = 0; i < V; ++i) dst[i] = acc[i];
}

// One warp per (head, level): the next rank's partial window sum added to dO_g of the shard's last level-l entry
// (when selected), and the head's largest magnitude raised to cover the new row.  Runs after the scatter backward
// and before the per-head scaling of dO_g.
template <int D>
__global__ void __launch_bounds__(256) dog_halo_kernel(float* __restrict__ dog, const int32_t* __restrict__ slot,
                                                       const float* __restrict__ halo, unsigned int* __restrict__ amax,
                                                       LhDims dm) {
  constexpr int V = D / 32;
  const int w = blockIdx.x * 8 + threadIdx.x / 32, lane = threadIdx.x % 32;
  if (w >= dm.BH * dm.L) return;
  const int bh = w / dm.L, lev = w % dm.L;
  const int s = slot[(int64_t)bh * dm.R + dm.off[lev] + dm.Nl[lev] - 1];
  if (s < 0) return;  // warp-uniform
  float* row = dog + ((int64_t)bh * dm.S + s) * D + lane * V;
  const float* add = halo + (int64_t)w * D + lane * V;
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < V; ++i) {
    row[i] += add[i];
    m = fmaxf(m, fabsf(row[i]));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  if (lane == 0) atomicMax(amax + bh, __float_as_uint(m));
}

inline unsigned warp_blocks(int warps) { return (unsigned)((warps + 7) / 8); }

}  // namespace

int launch_halo_fwd(const float* og, const int32_t* slot, float* halo, const LhDims& dm, cudaStream_t st) {
  KernelTimer timer("cp_halo", st);
  const unsigned nb = warp_blocks(dm.BH * dm.L);
  if (dm.d == 64) halo_fwd_kernel<64><<<nb, 256, 0, st>>>(og, slot, halo, dm);
  else halo_fwd_kernel<128><<<nb, 256, 0, st>>>(og, slot, halo, dm);
  return check_launch();
}

int launch_scatter_halo(const float* og, const int32_t* slot, const float* halo, void* o, const LhDims& dm,
                        cudaStream_t st) {
  const int ntok = dm.wl[dm.L - 1] - 1;
  if (ntok <= 0) return LH_OK;
  KernelTimer timer("cp_halo", st);
  dim3 grid(warp_blocks(ntok), dm.BH);
  auto* out = reinterpret_cast<__nv_bfloat16*>(o);
  if (dm.d == 64) scatter_halo_kernel<64><<<grid, 256, 0, st>>>(og, slot, halo, out, dm);
  else scatter_halo_kernel<128><<<grid, 256, 0, st>>>(og, slot, halo, out, dm);
  return check_launch();
}

int launch_halo_bwd(const void* dout, float* halo, const LhDims& dm, cudaStream_t st) {
  KernelTimer timer("cp_halo", st);
  const unsigned nb = warp_blocks(dm.BH * dm.L);
  auto* src = reinterpret_cast<const __nv_bfloat16*>(dout);
  if (dm.d == 64) halo_bwd_kernel<64><<<nb, 256, 0, st>>>(src, halo, dm);
  else halo_bwd_kernel<128><<<nb, 256, 0, st>>>(src, halo, dm);
  return check_launch();
}

int launch_dog_halo(float* dog, const int32_t* slot, const float* halo, unsigned int* amax, const LhDims& dm,
                    cudaStream_t st) {
  KernelTimer timer("cp_halo", st);
  const unsigned nb = warp_blocks(dm.BH * dm.L);
  if (dm.d == 64) dog_halo_kernel<64><<<nb, 256, 0, st>>>(dog, slot, halo, amax, dm);
  else dog_halo_kernel<128><<<nb, 256, 0, st>>>(dog, slot, halo, amax, dm);
  return check_launch();
}

}  // namespace lh
