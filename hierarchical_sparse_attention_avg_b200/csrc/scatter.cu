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

// Power-of-two scale bringing the largest magnitude `amax` into [2^9, 2^10); 1 for an all-zero or non-finite head.
// The exponent is read from the bits and the scale is capped at 2^126, so that both the scale and its inverse stay
// finite normal fp32 numbers: a head whose largest magnitude is below 2^-116 (subnormal values included) is scaled
// by 2^126 and keeps its values below 2^10.
__device__ __forceinline__ float head_scale(float amax) {
  if (!(amax > 0.f) || !isfinite(amax)) return 1.f;
  const int biased = (int)((__float_as_uint(amax) >> 23) & 0xFFu);  // 0 for a subnormal amax
  const int e = (biased == 0 ? -126 : biased - 127) + 1;               // amax < 2^e
  const int s = 10 - e < 126 ? 10 - e : 126;
  return __uint_as_float((uint32_t)(s + 127) << 23);
}

// Window sums for the scatter-back (offset, one tensor) and the unpool backward (three tensors).
//
// A tile is T consecutive "keys" of one head, key0 a multiple of T; key = t + 1 for the scatter (entry
// j = key/w - 1) and key = t for the unpool (j = key/w).  Windows are powers of two, so a level with w <= T has
// T/w entries in the tile and a wider level exactly one.  Per tile:
//   1. every thread holds at most kH slots of the tile's entry list (loaded one tile ahead); a block-wide
//      ballot scan numbers the selected entries (compact index) and lists their source rows;
//   2. each warp copies the selected rows of its own entries, every tensor, to shared memory with cp.async (the
//      first M rows of the tile; rows beyond M, which only very dense selections reach, are read from global
//      memory where they are used), and marks the keys that a selected "fine" entry covers in a bitmap;
//   3. a row group (d/8 lanes) owns PP consecutive keys.  Levels with w >= PP ("uniform") have one entry for the
//      whole group: their rows are summed once into a base row, rounded, packed and stored to every key.  Levels
//      with w < PP ("fine") differ per key: each key marked in the bitmap is then recomputed as base + its fine
//      rows (fp32, one rounding) and stored again over the base value.  Weights are 1 (scatter) and
//      2^-level-shift (unpool, exact).
// The loop is software-pipelined over the block's tiles: while tile i is summed and stored, the rows of tile
// i+1 are in flight to the other shared-memory stage and the slots of tile i+2 to registers, so no tile waits
// for a full memory round trip.
constexpr int kWinThreads = 256;
constexpr int kWinWarps = kWinThreads / 32;
constexpr int kWinStageBytes = 24 * 1024;  // staged rows per stage, all tensors

template <int D, int P, int NT>
struct WinCfg {
  static constexpr int G = D / 8;                  // lanes per row
  static constexpr int RG = kWinThreads / G;       // row groups
  static constexpr int PP = (NT == 1 && D == 128) ? 16 : 8;  // keys per row group
  static constexpr int T = RG * PP;                // keys per tile
  static constexpr int M = kWinStageBytes / (NT * D * 4);
  static constexpr int LP = P == 2 ? 1 : (P == 4 ? 2 : 3);  // log2 p
  // entries of level l in a tile, and the first entry of level l in the tile's list
  __host__ __device__ static constexpr int n_ent(int l) { return (1 << (l * LP)) <= T ? T >> (l * LP) : 1; }
  __host__ __device__ static constexpr int ent_base(int l) { return l == 0 ? 0 : ent_base(l - 1) + n_ent(l - 1); }
  static constexpr int kMaxEnt = ent_base(kMaxL);
  static constexpr int kH = (kMaxEnt + kWinThreads - 1) / kWinThreads;  // entries per thread
  static constexpr int kWords = T / 32;                                  // fine-key bitmap words
  __host__ __device__ static constexpr bool uniform(int l) { return (1 << (l * LP)) >= PP; }
  __host__ __device__ static constexpr float weight(int l, bool offset) {
    return offset ? 1.0f : 1.0f / (float)(1 << (l * LP));  // exact: a power of two
  }
  static_assert(T % 32 == 0 && PP <= 32 && 32 % PP == 0, "row groups tile the bitmap words");
};

// The tile-independent part of one of a thread's entries: level (-1 beyond the last level), shift, offset in
// the level's run within the tile, entry offset including the scatter's -1, level size, slot-row offset, and
// whether the level is fine.
struct WinEntry {
  int lev, sh, r, e, nl, off;
  bool fine;
};

template <int D, int P, int NT, bool kOffset>
__device__ __forceinline__ WinEntry win_entry(int i, const LhDims& dm) {
  using C = WinCfg<D, P, NT>;
  WinEntry w{-1, 0, 0, 0, 0, 0, false};
#pragma unroll
  for (int l = 0; l < kMaxL; ++l) {
    if (l < dm.L && i >= C::ent_base(l) && i < C::ent_base(l) + C::n_ent(l)) {
      w.lev = l;
      w.sh = l * C::LP;
      w.r = i - C::ent_base(l);
      w.e = w.r - (kOffset ? 1 : 0);
      w.nl = dm.Nl[l];
      w.off = dm.off[l];
      w.fine = !C::uniform(l);
    }
  }
  return w;
}

// Slot of entry `w` in the tile of head bh starting at key0 (-1: not selected, or outside the level).
__device__ __forceinline__ int win_slot(const WinEntry& w, int bh, int key0, const int32_t* __restrict__ slot,
                                        const LhDims& dm) {
  const int j = (key0 >> w.sh) + w.e;
  return (w.lev >= 0 && j >= 0 && j < w.nl) ? slot[(int64_t)bh * dm.R + w.off + j] : -1;
}

// Numbers the selected entries of a tile (compact index into s_cidx, source row into s_src), starts the copy of
// the first M selected rows of every tensor into stage buffer `buf`, clears the stage's fine-key bitmap and
// returns in (fw, fm) the bitmap word and bits of each selected fine entry of this thread (fm = 0: none), to be
// set once the clearing is visible to every thread.
template <int D, int P, int NT>
__device__ __forceinline__ void win_stage(const int (&s)[WinCfg<D, P, NT>::kH],
                                          const WinEntry (&we)[WinCfg<D, P, NT>::kH], int bh,
                                          const float* const (&src)[3], const LhDims& dm, int* s_cidx, int* s_src,
                                          int* s_wcount, unsigned* s_fine, float* buf,
                                          int (&fw)[WinCfg<D, P, NT>::kH], unsigned (&fm)[WinCfg<D, P, NT>::kH]) {
  using C = WinCfg<D, P, NT>;
  constexpr int kH = C::kH;
  const int tid = threadIdx.x, wid = tid >> 5, wl = tid & 31;
  unsigned m[kH];
#pragma unroll
  for (int h = 0; h < kH; ++h) {
    m[h] = __ballot_sync(0xffffffffu, s[h] >= 0);
    if (wl == 0) s_wcount[h * kWinWarps + wid] = __popc(m[h]);
    // a fine entry at run offset r covers tile keys r*w .. r*w + w - 1 (w < PP <= 32: one bitmap word)
    const int k0 = we[h].r << we[h].sh;
    fw[h] = k0 >> 5;
    fm[h] = (s[h] >= 0 && we[h].fine) ? ((2u << ((1 << we[h].sh) - 1)) - 1u) << (k0 & 31) : 0u;
  }
  __syncthreads();
  if (tid < C::kWords) s_fine[tid] = 0u;
  int c[kH];
  int run = 0;  // selected entries of the earlier groups
#pragma unroll
  for (int h = 0; h < kH; ++h) {
    const int4 lo = *reinterpret_cast<const int4*>(s_wcount + h * kWinWarps);
    const int4 hi = *reinterpret_cast<const int4*>(s_wcount + h * kWinWarps + 4);
    const int w8[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
    int pre = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < kWinWarps; ++w) {
      pre += w < wid ? w8[w] : 0;
      tot += w8[w];
    }
    c[h] = s[h] >= 0 ? run + pre + __popc(m[h] & ((1u << wl) - 1u)) : -1;
    run += tot;
    const int i = tid + h * kWinThreads;
    if (i < C::kMaxEnt) s_cidx[i] = c[h];
    if (c[h] >= 0) s_src[c[h]] = s[h];
  }
  // the warp copies the rows of its own selected entries: lane x moves 16-byte chunks x, x + 32, ...
  constexpr int kChunks = D / 4;  // 16-byte chunks per fp32 row
#pragma unroll
  for (int h = 0; h < kH; ++h) {
    unsigned mm = m[h];
    while (mm) {
      const int src_lane = __ffs(mm) - 1;
      mm &= mm - 1;
      const int cc = __shfl_sync(0xffffffffu, c[h], src_lane);
      const int row = __shfl_sync(0xffffffffu, s[h], src_lane);
      if (cc < C::M) {
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const float* g = src[t] + ((int64_t)bh * dm.S + row) * D;
          float* sb = buf + (t * C::M + cc) * D;
#pragma unroll
          for (int x = wl; x < kChunks; x += 32) cp_async16(smem_u32(sb + x * 4), g + x * 4);
        }
      }
    }
  }
}

template <int kH>
__device__ __forceinline__ void win_mark(const int (&fw)[kH], const unsigned (&fm)[kH], unsigned* s_fine) {
#pragma unroll
  for (int h = 0; h < kH; ++h)
    if (fm[h]) atomicOr(s_fine + fw[h], fm[h]);
}

template <int D, int P, bool kOffset, int NT>
__global__ void __launch_bounds__(kWinThreads, 4) window_sum_kernel(const float* __restrict__ src0,
                                                                   const float* __restrict__ src1,
                                                                   const float* __restrict__ src2,
                                                                   const int32_t* __restrict__ slot,
                                                                   __nv_bfloat16* dst0, __nv_bfloat16* dst1,
                                                                   __nv_bfloat16* dst2, LhDims dm) {
  using C = WinCfg<D, P, NT>;
  constexpr int G = C::G, PP = C::PP, T = C::T, M = C::M, LP = C::LP, kH = C::kH;
  extern __shared__ __align__(16) float s_buf[];  // [2 stages][NT][M][D]
  __shared__ int s_cidx[2][C::kMaxEnt];
  __shared__ int s_src[2][C::kMaxEnt];
  __shared__ __align__(16) int s_wcount[2][kH * kWinWarps];
  __shared__ unsigned s_fine[2][C::kWords];
  const float* const src[3] = {src0, src1, src2};
  __nv_bfloat16* const dst[3] = {dst0, dst1, dst2};
  const int tid = threadIdx.x, lane = tid % G, x0 = (tid / G) * PP;
  // Tiles are numbered head-major (tile = bh * tph + kt) and visited with stride gridDim.x; (bh, kt) is advanced
  // incrementally.  Three tiles are live: the one summed (0), the one staged (1) and the one whose slots load (2).
  const int tph = (dm.N + (kOffset ? 1 : 0) + T - 1) / T;  // tiles per head
  const int sq = (int)(gridDim.x / (unsigned)tph), sr = (int)(gridDim.x % (unsigned)tph);
  int bh0 = (int)(blockIdx.x / (unsigned)tph), kt0 = (int)(blockIdx.x % (unsigned)tph);
  if (bh0 >= dm.BH) return;
  int bh1 = bh0 + sq, kt1 = kt0 + sr;
  if (kt1 >= tph) { kt1 -= tph; ++bh1; }
  int bh2 = bh1 + sq, kt2 = kt1 + sr;
  if (kt2 >= tph) { kt2 -= tph; ++bh2; }
  WinEntry we[kH];
#pragma unroll
  for (int h = 0; h < kH; ++h) we[h] = win_entry<D, P, NT, kOffset>(tid + h * kWinThreads, dm);
  int sl[kH], fw[kH];
  unsigned fm[kH];
#pragma unroll
  for (int h = 0; h < kH; ++h) sl[h] = win_slot(we[h], bh0, kt0 * T, slot, dm);
  win_stage<D, P, NT>(sl, we, bh0, src, dm, s_cidx[0], s_src[0], s_wcount[0], s_fine[0], s_buf, fw, fm);
  cp_async_commit();
  if (bh1 < dm.BH)
#pragma unroll
    for (int h = 0; h < kH; ++h) sl[h] = win_slot(we[h], bh1, kt1 * T, slot, dm);
  __syncthreads();
  win_mark<kH>(fw, fm, s_fine[0]);
  for (int it = 0; bh0 < dm.BH; ++it) {
    const int b = it & 1;
    const bool has1 = bh1 < dm.BH;  // block-uniform
    if (has1)
      win_stage<D, P, NT>(sl, we, bh1, src, dm, s_cidx[b ^ 1], s_src[b ^ 1], s_wcount[b ^ 1], s_fine[b ^ 1],
                          s_buf + (b ^ 1) * NT * M * D, fw, fm);
    cp_async_commit();
    if (bh2 < dm.BH)
#pragma unroll
      for (int h = 0; h < kH; ++h) sl[h] = win_slot(we[h], bh2, kt2 * T, slot, dm);
    cp_async_wait<1>();  // this thread's copies for the summed tile are done ...
    __syncthreads();     // ... and everyone's are visible, as is the cleared bitmap of the staged tile
    if (has1) win_mark<kH>(fw, fm, s_fine[b ^ 1]);
    const int bh = bh0, key0 = kt0 * T;
    const int* ci = s_cidx[b];
    const int* cs = s_src[b];
    const float* sb = s_buf + b * NT * M * D;
    const int64_t gbase = (int64_t)bh * dm.S * D + lane * 8;  // row 0 of this head in the sources
    // the source row of compact index c (staged copy when c < M), at this thread's 8 features
    auto row_ptr = [&](int t, int c) -> const float* {
      return c < M ? sb + (t * M + c) * D + lane * 8 : src[t] + gbase + (int64_t)cs[c] * D;
    };
    const unsigned fine = (s_fine[b][x0 >> 5] >> (x0 & 31)) & (PP == 32 ? ~0u : (1u << PP) - 1u);
    const int tok0 = key0 + x0 - (kOffset ? 1 : 0);  // token of this row group's first key
    const int64_t obase = ((int64_t)bh * dm.N + tok0) * D + lane * 8;
    const bool whole = tok0 >= 0 && tok0 + PP <= dm.N;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      float base[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int l = 0; l < kMaxL; ++l) {
        if (C::uniform(l) && l < dm.L) {
          const int c = ci[C::ent_base(l) + ((1 << (l * LP)) <= T ? x0 >> (l * LP) : 0)];
          if (c >= 0) {
            float f[8];
            load8f(row_ptr(t, c), f);
#pragma unroll
            for (int e8 = 0; e8 < 8; ++e8) base[e8] = fmaf(f[e8], C::weight(l, kOffset), base[e8]);
          }
        }
      }
      const uint4 packed = pack8_rn(base);
      __nv_bfloat16* out = dst[t] + obase;
      if (whole) {
#pragma unroll
        for (int q = 0; q < PP; ++q) st_stream16(out + q * D, packed);
      } else {
#pragma unroll
        for (int q = 0; q < PP; ++q)
          if (tok0 + q >= 0 && tok0 + q < dm.N) st_stream16(out + q * D, packed);
      }
      // keys with a selected fine entry: base + fine rows, stored over the base value (same thread, same address)
      unsigned f = fine;
      while (f) {
        const int q = __ffs(f) - 1;
        f &= f - 1u;
        if (tok0 + q < 0 || tok0 + q >= dm.N) continue;
        float acc[8];
#pragma unroll
        for (int e8 = 0; e8 < 8; ++e8) acc[e8] = base[e8];
#pragma unroll
        for (int l = 0; l < kMaxL; ++l) {
          if (!C::uniform(l) && l < dm.L) {
            const int c = ci[C::ent_base(l) + ((x0 + q) >> (l * LP))];
            if (c >= 0) {
              float fr[8];
              load8f(row_ptr(t, c), fr);
#pragma unroll
              for (int e8 = 0; e8 < 8; ++e8) acc[e8] = fmaf(fr[e8], C::weight(l, kOffset), acc[e8]);
            }
          }
        }
        st_stream16(out + q * D, pack8_rn(acc));
      }
    }
    bh0 = bh1; kt0 = kt1;
    bh1 = bh2; kt1 = kt2;
    bh2 += sq; kt2 += sr;
    if (kt2 >= tph) { kt2 -= tph; ++bh2; }
  }
  cp_async_wait<0>();
}

// Scatter backward.  A gathered row sums a window of 1 to p^(L-1) upstream rows, so a row group that summed its
// own row's whole window would keep its block alive for the longest window (eight round trips for a 64-row
// window) while most rows need one.  Instead the windows of the block's rows (one row per row group) are cut into
// chunks of up to kSbChunk consecutive upstream rows, numbered row by row; in each round every row group loads and
// sums one chunk (all its rows in flight at once) into a shared slot, and after the round's barrier each row group
// adds the slots of its own row in chunk order.  The order of every addition is fixed by the row's window, so the
// result does not depend on the schedule.
constexpr int kSbThreads = 256;
constexpr int kSbChunk = 8;

template <int D>
__global__ void __launch_bounds__(kSbThreads) scatter_bwd_kernel(const __nv_bfloat16* __restrict__ dout,
                                                                 const int32_t* __restrict__ idx_g,
                                                                 float* __restrict__ dog,
                                                                 unsigned int* __restrict__ amax, LhDims dm) {
  constexpr int G = D / 8;             // lanes per row
  constexpr int NG = kSbThreads / G;   // row groups = rows per block (16 or 32)
  __shared__ int64_t s_src[NG];        // element offset of the row's first upstream row
  __shared__ int s_len[NG];            // upstream rows in the row's window (0: no row)
  __shared__ int s_base[NG + 1];       // first chunk of each row; s_base[NG] = chunks of the block
  __shared__ __align__(16) float s_part[2][NG][D];
  const int lane = threadIdx.x % G, g = threadIdx.x / G;
  const int64_t total = (int64_t)dm.BH * dm.S;
  const int64_t row0 = (int64_t)blockIdx.x * NG + g;
  const bool active = row0 < total;
  const int64_t row = active ? row0 : total - 1;
  const int bh = (int)(row / dm.S);
  if (lane == 0) {
    int len = 0;
    int64_t src = 0;
    if (active) {
      const int gid = idx_g[row];
      const int lev = level_of(gid, dm);
      const int j = gid - dm.off[lev];
      const int w = dm.wl[lev];
      const int t0 = (j + 1) * w - 1;
      const int t1 = min(t0 + w - 1, dm.N - 1);
      len = t1 - t0 + 1;
      src = ((int64_t)bh * dm.N + t0) * D;
    }
    s_len[g] = len;
    s_src[g] = src;
  }
  __syncthreads();
  if (threadIdx.x < 32) {  // chunk counts, inclusive scan over the row groups
    const int r = threadIdx.x;
    int c = r < NG ? (s_len[r] + kSbChunk - 1) / kSbChunk : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, c, off);
      if (r >= off) c += y;
    }
    if (r < NG) s_base[r + 1] = c;
    if (r == 0) s_base[0] = 0;
  }
  __syncthreads();
  const int T = s_base[NG], first = s_base[g], last = s_base[g + 1];
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int w0 = 0, b = 0; w0 < T; w0 += NG, b ^= 1) {
    const int tau = w0 + g;  // this row group's chunk in the round
    if (tau < T) {
      int r = 0;  // the row of chunk tau: the last r with s_base[r] <= tau
#pragma unroll
      for (int step = NG / 2; step > 0; step >>= 1)
        if (s_base[r + step] <= tau) r += step;
      const int c = tau - s_base[r];
      const int n = min(kSbChunk, s_len[r] - c * kSbChunk);
      const __nv_bfloat16* src = dout + s_src[r] + (int64_t)c * kSbChunk * D + lane * 8;
      uint4 v[kSbChunk];
#pragma unroll
      for (int u = 0; u < kSbChunk; ++u)
        if (u < n) v[u] = ld_stream16(src + (int64_t)u * D);
      float part[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int u = 0; u < kSbChunk; ++u) {
        if (u < n) {
          float f[8];
          unpack8(v[u], f);
#pragma unroll
          for (int i = 0; i < 8; ++i) part[i] += f[i];
        }
      }
      store8f(&s_part[b][g][lane * 8], part);
    }
    __syncthreads();  // the round's slots are written (and the slots of two rounds back were read by their owners)
    for (int t = max(first, w0); t < min(last, w0 + NG); ++t) {
      float f[8];
      load8f(&s_part[b][t - w0][lane * 8], f);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += f[i];
    }
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
                                                       const float* __restrict__ lse,
                                                       const unsigned int* __restrict__ amax, __half* __restrict__ dog16,
                                                       float* __restrict__ stats, float* __restrict__ dinv,
                                                       float* __restrict__ dqacc, LhDims dm) {
  constexpr int G = D / 8;
  constexpr float kLog2e = 1.4426950408889634f;
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
    if (lane == 0) {
      const int64_t srow = (int64_t)bh * stats_stride(dm) + row % dm.S;
      stats[srow] = -lse[row] * kLog2e;
      stats[(int64_t)dm.BH * stats_stride(dm) + srow] = -dot * rsqrtf((float)D);
    }
    if (lane == 0 && row % dm.S == 0) dinv[bh] = 1.f / sc;
    const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    store8f(dqacc + row * D + lane * 8, z);
  }
}


template <int D>
int blocks_for(int64_t rows) {
  return (int)((rows + 256 / (D / 8) - 1) / (256 / (D / 8)));
}

// Launch a window_sum_kernel with a grid of at most the blocks the device keeps resident at once (occupancy
// times the SM count): each block pipelines over many tiles.
template <int D, int P, bool kOffset, int NT>
int launch_window_sum(const float* s0, const float* s1, const float* s2, const int32_t* slot, __nv_bfloat16* d0,
                      __nv_bfloat16* d1, __nv_bfloat16* d2, const LhDims& dm, cudaStream_t st) {
  using C = WinCfg<D, P, NT>;
  auto kernel = window_sum_kernel<D, P, kOffset, NT>;
  const int smem = 2 * NT * C::M * D * (int)sizeof(float);
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return LH_ERR_CUDA;
  const int64_t tiles = (int64_t)dm.BH * ((dm.N + (kOffset ? 1 : 0) + C::T - 1) / C::T);
  if (tiles >= (int64_t)1 << 31) return LH_ERR_UNSUPPORTED;
  int dev = 0, sms = 148, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kWinThreads, smem);
  const int64_t cap = (int64_t)sms * (per_sm > 0 ? per_sm : 1);
  const int grid = (int)(tiles < cap ? tiles : cap);
  kernel<<<grid, kWinThreads, smem, st>>>(s0, s1, s2, slot, d0, d1, d2, dm);
  return check_launch();
}

template <bool kOffset, int NT>
int window_sum(const float* s0, const float* s1, const float* s2, const int32_t* slot, void* d0, void* d1, void* d2,
               const LhDims& dm, cudaStream_t st) {
  __nv_bfloat16 *o0 = (__nv_bfloat16*)d0, *o1 = (__nv_bfloat16*)d1, *o2 = (__nv_bfloat16*)d2;
#define LH_WIN(DD, PPV) \
  if (dm.d == DD && dm.p == PPV) return launch_window_sum<DD, PPV, kOffset, NT>(s0, s1, s2, slot, o0, o1, o2, dm, st);
  LH_WIN(64, 2) LH_WIN(64, 4) LH_WIN(64, 8) LH_WIN(128, 2) LH_WIN(128, 4) LH_WIN(128, 8)
#undef LH_WIN
  return LH_ERR_UNSUPPORTED;
}

}  // namespace

int launch_scatter(const float* og, const int32_t* slot, void* o, const LhDims& dm, cudaStream_t st) {
  KernelTimer timer("scatter", st);
  return window_sum<true, 1>(og, og, og, slot, o, o, o, dm, st);
}

int launch_scatter_bwd(const void* dout, const int32_t* idx_g, float* dog, unsigned int* amax, const LhDims& dm,
                       cudaStream_t st) {
  const int64_t rows = (int64_t)dm.BH * dm.S;
  KernelTimer timer("scatter_bwd", st);
  if (dm.d == 64)
    scatter_bwd_kernel<64><<<(unsigned)((rows + kSbThreads / 8 - 1) / (kSbThreads / 8)), kSbThreads, 0, st>>>(
        (const __nv_bfloat16*)dout, idx_g, dog, amax, dm);
  else
    scatter_bwd_kernel<128><<<(unsigned)((rows + kSbThreads / 16 - 1) / (kSbThreads / 16)), kSbThreads, 0, st>>>(
        (const __nv_bfloat16*)dout, idx_g, dog, amax, dm);
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

int launch_bwd_prep(const float* dog, const float* og, const float* lse, const unsigned int* amax, void* dog16,
                    float* stats, float* dinv, float* dqacc, const LhDims& dm, cudaStream_t st) {
  const int64_t rows = (int64_t)dm.BH * dm.S;
  KernelTimer timer("bwd_prep", st);
  if (dm.d == 64)
    bwd_prep_kernel<64><<<blocks_for<64>(rows), 256, 0, st>>>(dog, og, lse, amax, (__half*)dog16, stats, dinv, dqacc,
                                                              dm);
  else
    bwd_prep_kernel<128><<<blocks_for<128>(rows), 256, 0, st>>>(dog, og, lse, amax, (__half*)dog16, stats, dinv,
                                                                dqacc, dm);
  return check_launch();
}

int launch_unpool_bwd(const float* dqg, const float* dkg, const float* dvg, const int32_t* slot, void* dq, void* dk,
                      void* dv, const LhDims& dm, cudaStream_t st) {
  KernelTimer timer("unpool_bwd", st);
  return window_sum<false, 3>(dqg, dkg, dvg, slot, dq, dk, dv, dm, st);
}

}  // namespace lh
