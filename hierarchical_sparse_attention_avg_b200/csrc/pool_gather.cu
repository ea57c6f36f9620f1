// pool_gather.cu — step 1 (symmetric average-pool pyramid), step 2 (per-head l2-norm score) and the row
// gather of step 4.
//
// Pooling follows [W] 核心方法 §1 对称金字塔池化 (Q, K and V average-pooled alike into a multi-level
// pyramid); scoring follows [W] 核心方法 §2 and [E] "Как four-stage pipeline…" (parameter-free per-head l2
// norm).  The arithmetic is the one the layer's definition fixes so that results are bit-exact everywhere:
//   level sums in fp64, each level summing its p children left to right from the first child;
//   pooled value = bf16_RN(sum / p^l);
//   score = fp32_RN(sum of squares: 8 left to right per 8-feature group, then a pairwise tree over groups).
//
// Thread layout: a "group" of d/8 lanes owns one row, each lane 8 features (one 16-byte vector).  The pairwise
// tree over the groups of a row is an xor-butterfly over those lanes (float addition is commutative, so every
// lane ends with the same bits).
#include "internal.h"

namespace lh {

namespace {

constexpr int kPoolThreads = 256;
constexpr int kPoolStages = 3;  // batches of raw rows in flight per thread (cp.async into private shared slots)

__host__ __device__ constexpr int pool_batch(int W) { return W < 8 ? W : 8; }

__host__ __device__ constexpr int ipow(int b, int e) { return e == 0 ? 1 : b * ipow(b, e - 1); }

__device__ __forceinline__ void load_row8(const uint4& raw, double (&x)[8]) {
  float f[8];
  unpack8(raw, f);
#pragma unroll
  for (int i = 0; i < 8; ++i) x[i] = f64_of(f[i]);
}

// Score of one row: squared l2 norm of the (bf16) values x, summed in the fixed order, rounded to fp32.
template <int G>
__device__ __forceinline__ float row_score(const double (&x)[8]) {
  double s = x[0] * x[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) s = fma(x[i], x[i], s);  // x*x is exact in fp64: fma == add of the square
#pragma unroll
  for (int off = 1; off < G; off <<= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  return f32_rn_of(s);
}

// This lane's share of a row's score: the squares of its 8 values summed left to right in fp64.
__device__ __forceinline__ double lane_sq8(const float (&xf)[8]) {
  double s = f64_of(xf[0]) * f64_of(xf[0]);
#pragma unroll
  for (int i = 1; i < 8; ++i) s = fma(f64_of(xf[i]), f64_of(xf[i]), s);
  return s;
}

// Scores of 4 rows at once from each lane's shares part[u] (row u of the group of 4).  The pairwise tree over a
// row's G lanes is the xor butterfly of row_score (partners L^1, then L^2, ...); its first two rounds are done
// transposed: in round m each lane keeps half of its remaining rows (the upper half when bit m of the lane is set)
// and adds its partner's shares of those rows, which the partner sends; the later rounds (L^4, L^8) pair lanes that
// hold the same row.  Every addition has the same two operands as in the per-row butterfly, so the sums are
// bit-identical, and lane L ends with the score of row 2 (L & 1) + ((L >> 1) & 1).  Returns that row.
template <int G>
__device__ __forceinline__ int rows4_score(const double (&part)[4], int lane, float& score) {
  const bool b0 = lane & 1, b1 = (lane >> 1) & 1;
  double r2[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const double got = __shfl_xor_sync(0xffffffffu, b0 ? part[i] : part[i + 2], 1);
    r2[i] = (b0 ? part[i + 2] : part[i]) + got;
  }
  double r = (b1 ? r2[1] : r2[0]) + __shfl_xor_sync(0xffffffffu, b1 ? r2[0] : r2[1], 2);
#pragma unroll
  for (int off = 4; off < G; off <<= 1) r += __shfl_xor_sync(0xffffffffu, r, off);
  score = f32_rn_of(r);
  return 2 * b0 + b1;
}

// Round 8 fp64 sums / w to bf16 (single rounding), returning packed bits and the bf16 values as fp64.
__device__ __forceinline__ uint4 round_pooled(const double (&sum)[8], double inv_w, double (&val)[8]) {
  uint32_t b[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    b[i] = f64_to_bf16_bits_rne(sum[i] * inv_w);  // inv_w = 1/p^l is exact for power-of-two p
    val[i] = f64_of(__uint_as_float(b[i] << 16));
  }
  return make_uint4(b[0] | (b[1] << 16), b[2] | (b[3] << 16), b[4] | (b[5] << 16), b[6] | (b[7] << 16));
}

// Level-1 sums in fp32.  A level-1 entry sums p bf16 values; the sum is carried twice in fp32, rounded toward
// +inf and toward -inf (IEEE directed rounding, subnormals kept).  The two chains bracket the exact value and stay
// apart once any step rounded, so they are equal exactly when every step was exact -- the common case for p bf16
// values -- and an exact fp32 sum is also what the fp64 order of the definition produces.  Then the pooled value
// bf16_RN(sum / p) is the bf16 rounding of the fp32 value sum * 2^-log2(p) (exact while that is a normal number)
// and the fp64 sum for the levels above is one widening per entry instead of one per element.  A lane whose
// chains differ recomputes the entry in fp64 from the raw values.
__device__ __forceinline__ float add_up(float a, float b) {
  float r;
  asm("add.rp.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float add_dn(float a, float b) {
  float r;
  asm("add.rm.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float mul_rn(float a, float b) {  // no flush of subnormal results
  float r;
  asm("mul.rn.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}
// Upper and lower chain agree: same bits, or both zero (an exact zero sum is +0 upward and -0 downward).
__device__ __forceinline__ bool same_sum(float up, float dn) {
  const uint32_t a = __float_as_uint(up), b = __float_as_uint(dn);
  return a == b || ((a | b) & 0x7FFFFFFFu) == 0u;
}
// Zero or a normal, finite number (tested on the bits, independent of flush-to-zero).
__device__ __forceinline__ bool zero_or_normal(float x) {
  const uint32_t e = (__float_as_uint(x) >> 23) & 0xFFu;
  return (__float_as_uint(x) & 0x7FFFFFFFu) == 0u || (e != 0u && e != 0xFFu);
}

// One group builds every level of the pyramid over one block of W = P^(L-1) consecutive tokens of one head (one
// coarsest entry): level 1 as above, levels >= 2 in fp64 registers, in the order the definition fixes.  The raw
// rows stream through kPoolStages batches of TB rows per thread, copied with cp.async into shared-memory slots
// private to the thread (so no block barrier is needed) while earlier batches are summed.
// kScore: 0 = no scores; 1 = score levels 0..L-2; 2 = score levels 1..L-1 (children-expansion variant).  Scored
// level l is written at row dm.soff[l] of the head's score array.
template <int D, int P, int L, int kScore>
__device__ __forceinline__ void pool_score_body(const PoolJob& job, unsigned block, const LhDims& dm) {
  constexpr int G = D / 8;
  constexpr int GPB = kPoolThreads / G;
  constexpr int W = ipow(P, L - 1);
  constexpr int TB = pool_batch(W);  // tokens per batch (a multiple of P)
  constexpr int NB = W / TB;          // batches per block
  static_assert(TB % P == 0, "batch must hold whole level-1 entries");
  extern __shared__ uint4 s_raw[];    // [kPoolStages][TB][kPoolThreads]

  const int lane = threadIdx.x % G;
  const int64_t group = (int64_t)block * GPB + threadIdx.x / G;
  const int nblk = dm.N / W;
  const int64_t total = (int64_t)dm.BH * nblk;
  const bool active = group < total;
  const int64_t gi = active ? group : total - 1;  // idle groups shadow a valid one (shuffles need the warp)
  const int bh = (int)(gi / nblk);
  const int blk = (int)(gi % nblk);

  const __nv_bfloat16* xrow =
      reinterpret_cast<const __nv_bfloat16*>(job.x) + ((int64_t)bh * dm.N + (int64_t)blk * W) * D + lane * 8;
  float* scores = kScore ? job.scores + (int64_t)bh * dm.Rs : nullptr;  // jobs with scores run as kScore
  __nv_bfloat16* pyr = reinterpret_cast<__nv_bfloat16*>(job.pyr);

  double acc[L][8];  // acc[l]: running fp64 sum of the current level-l entry (l >= 1)

  uint4* my = s_raw + threadIdx.x;  // this thread's slot u of stage st: my[(st * TB + u) * kPoolThreads]
  auto issue = [&](int bi) {
    const int st = bi % kPoolStages;
#pragma unroll
    for (int u = 0; u < TB; ++u)
      cp_async16(smem_u32(my + (st * TB + u) * kPoolThreads), xrow + (int64_t)(bi * TB + u) * D);
  };
#pragma unroll
  for (int bi = 0; bi < kPoolStages - 1; ++bi) {
    if (bi < NB) issue(bi);
    cp_async_commit();
  }
#pragma unroll 1
  for (int bi = 0; bi < NB; ++bi) {
    if (bi + kPoolStages - 1 < NB) issue(bi + kPoolStages - 1);
    cp_async_commit();
    cp_async_wait<kPoolStages - 1>();  // batch bi has landed in this thread's slots
    const int t0 = bi * TB;
    const uint4* raw_s = my + (bi % kPoolStages) * TB * kPoolThreads;  // row u at raw_s[u * kPoolThreads]

    // level 0 is scored whenever L >= 2 (not in the children-expansion variant): the 4 rows of a level-1 entry
    // together when p = 4 (rows4_score), else row by row
    constexpr bool kRows4 = kScore == 1 && P == 4;
#pragma unroll
    for (int g1 = 0; g1 < TB / P; ++g1) {
      float up[8], dn[8];
      double part[4];
#pragma unroll
      for (int c = 0; c < P; ++c) {
        float xf[8];
        unpack8(raw_s[(g1 * P + c) * kPoolThreads], xf);
        if (kRows4) {
          part[c & 3] = lane_sq8(xf);
        } else if (kScore == 1) {
          double x[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) x[i] = f64_of(xf[i]);
          float s = row_score<G>(x);
          if (active && lane == 0) scores[dm.soff[0] + (int64_t)blk * W + t0 + g1 * P + c] = s;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          up[i] = (c == 0) ? xf[i] : add_up(up[i], xf[i]);
          dn[i] = (c == 0) ? xf[i] : add_dn(dn[i], xf[i]);
        }
      }
      if constexpr (kRows4) {  // the entry's 4 level-0 scores: lanes 0..3 of a row group hold one row each
        float sc;
        const int row = rows4_score<G>(part, lane, sc);
        if (active && lane < 4) scores[dm.soff[0] + (int64_t)blk * W + t0 + g1 * P + row] = sc;
      }
      bool exact = true;
#pragma unroll
      for (int i = 0; i < 8; ++i) exact &= same_sum(up[i], dn[i]);
      const int j1 = blk * (W / P) + t0 / P + g1;  // global level-1 index
      const bool write1 = (job.write_mask >> 1) & 1u;
      const bool score1 = (kScore == 1 && 1 <= L - 2) || kScore == 2;
      // the fp64 level-1 sum: needed above level 1, and for the rounding when the fp32 one is not exact
      if (!exact) {
#pragma unroll
        for (int c = 0; c < P; ++c) {
          double x[8];
          load_row8(raw_s[(g1 * P + c) * kPoolThreads], x);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[1][i] = (c == 0) ? x[i] : acc[1][i] + x[i];
        }
      } else if (L > 2) {
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[1][i] = f64_of(up[i]);
      }
      if (write1 || score1) {
        uint4 packed;
        bool fast = exact;
        float pv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          pv[i] = mul_rn(up[i], 1.0f / (float)P);  // exact scaling by a power of two while the result is normal
          fast &= zero_or_normal(pv[i]);
        }
        if (fast) {
          packed = make_uint4(pack_bf16x2_rn(pv[0], pv[1]), pack_bf16x2_rn(pv[2], pv[3]),
                              pack_bf16x2_rn(pv[4], pv[5]), pack_bf16x2_rn(pv[6], pv[7]));
        } else {
          if (exact && L <= 2) {
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[1][i] = f64_of(up[i]);
          }
          double unused[8];
          packed = round_pooled(acc[1], 1.0 / (double)P, unused);
        }
        if (write1 && active) st16(pyr + ((int64_t)bh * job.pyr_rows + job.row_off[1] + j1) * D + lane * 8, packed);
        if (score1) {
          float vf[8];
          unpack8(packed, vf);
          double v[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) v[i] = f64_of(vf[i]);
          const float sc = row_score<G>(v);
          if (active && lane == 0) scores[dm.soff[1] + j1] = sc;
        }
      }
      // levels >= 2: walk up while parents complete
      int jloc = t0 / P + g1;  // index of the completed level-1 entry inside this block
#pragma unroll
      for (int lev = 2; lev < L; ++lev) {
        const int c = jloc % P;  // child index of the completed level-(lev-1) entry
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[lev][i] = (c == 0) ? acc[lev - 1][i] : acc[lev][i] + acc[lev - 1][i];
        if (c != P - 1) break;
        jloc /= P;
        const int64_t j = (int64_t)blk * (W / ipow(P, lev)) + jloc;  // global index at level lev
        const bool write = (job.write_mask >> lev) & 1u;
        const bool score = (kScore == 1 && lev <= L - 2) || kScore == 2;
        if (write || score) {
          double val[8];
          const uint4 packed = round_pooled(acc[lev], 1.0 / (double)ipow(P, lev), val);
          if (write && active)
            st16(pyr + ((int64_t)bh * job.pyr_rows + job.row_off[lev] + j) * D + lane * 8, packed);
          if (score) {
            float s = row_score<G>(val);
            if (active && lane == 0) scores[dm.soff[lev] + j] = s;
          }
        }
      }
    }
  }
}

// One launch for every job; the job is the grid's fastest index, so each SM holds blocks of every job at once: the
// scored job's blocks are bound by instruction issue, the others by memory, and they overlap.  kScore is the scored
// job's mode (jobs without a score array run the unscored body).
template <int D, int P, int L, int kScore>
__global__ void __launch_bounds__(kPoolThreads, 2) pool_score_kernel(PoolJobs jobs, int njobs, LhDims dm) {
  const int ji = (int)(blockIdx.x % (unsigned)njobs);
  const unsigned block = blockIdx.x / (unsigned)njobs;
  if (kScore != 0 && jobs.job[ji].scores != nullptr)
    pool_score_body<D, P, L, kScore>(jobs.job[ji], block, dm);
  else
    pool_score_body<D, P, L, 0>(jobs.job[ji], block, dm);
}

// ---- Gather (step 4).  One warp per gathered row: lane i holds features [2*NW*i, 2*NW*i + 2*NW) (NW 32-bit
// words: d=128 -> 8 bytes, d=64 -> 4 bytes), so a row's level decides the warp's path as a whole.

// One lane's share of one row: 2*NW bf16 values.
template <int NW>
struct RowW {
  uint32_t w[NW];
};

template <int NW>
__device__ __forceinline__ RowW<NW> ld_roww(const __nv_bfloat16* p) {
  RowW<NW> r;
  if constexpr (NW == 2) {
    uint2 v;
    asm volatile("ld.global.nc.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    r.w[0] = v.x;
    r.w[1] = v.y;
  } else {
    asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(r.w[0]) : "l"(p));
  }
  return r;
}

// Packed pair of fp32 values (low word first), the operand of the sm_100a f32x2 instructions.
__device__ __forceinline__ uint64_t f32x2_of_bf16x2(uint32_t w) {
  return ((uint64_t)(w & 0xFFFF0000u) << 32) | (uint64_t)(w << 16);
}
__device__ __forceinline__ uint64_t add2_up(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rp.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t add2_dn(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rm.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ float sub_rn(float a, float b) {  // no flush of subnormal results
  float r;
  asm("sub.rn.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

// Interval sums.  The sum of a level-LEV entry is carried twice in fp32, every addition rounded up in one copy and
// down in the other, in the definition's tree order (p children left to right at every level, each child being
// the sum of its own children).  Rounding is monotone, so the upper copy never falls below the exact sum and the
// lower never rises above it, and a copy that rounded once stays strictly apart from it.  Equal copies therefore
// mean that every partial sum of the tree is exact in fp32 -- hence also in fp64, where the definition takes them
// -- and that the common value is the sum the definition fixes.
template <int NW, int P, int LEV>
__device__ __forceinline__ void iv_regs(const RowW<NW>* raw, uint64_t (&up)[NW], uint64_t (&dn)[NW]) {
#pragma unroll
  for (int c = 0; c < P; ++c) {
    uint64_t cu[NW], cd[NW];
    if constexpr (LEV == 1) {
#pragma unroll
      for (int i = 0; i < NW; ++i) cu[i] = cd[i] = f32x2_of_bf16x2(raw[c].w[i]);
    } else {
      iv_regs<NW, P, LEV - 1>(raw + c * ipow(P, LEV - 1), cu, cd);
    }
#pragma unroll
    for (int i = 0; i < NW; ++i) {
      up[i] = c == 0 ? cu[i] : add2_up(up[i], cu[i]);
      dn[i] = c == 0 ? cd[i] : add2_dn(dn[i], cd[i]);
    }
  }
}

// The interval of the level-LEV entry whose first raw row is at p (rows d = 64*NW apart): all raw loads in flight
// at once while the entry covers at most 16 rows, else child by child.
template <int NW, int P, int LEV>
__device__ __forceinline__ void iv_mem(const __nv_bfloat16* p, uint64_t (&up)[NW], uint64_t (&dn)[NW]) {
  constexpr int D = 64 * NW;
  constexpr int R = ipow(P, LEV);
  if constexpr (R <= 16) {
    RowW<NW> raw[R];
#pragma unroll
    for (int u = 0; u < R; ++u) raw[u] = ld_roww<NW>(p + (int64_t)u * D);
    iv_regs<NW, P, LEV>(raw, up, dn);
  } else {
    constexpr int CW = ipow(P, LEV - 1);
#pragma unroll 1
    for (int c = 0; c < P; ++c) {
      uint64_t cu[NW], cd[NW];
      iv_mem<NW, P, LEV - 1>(p + (int64_t)c * CW * D, cu, cd);
#pragma unroll
      for (int i = 0; i < NW; ++i) {
        up[i] = c == 0 ? cu[i] : add2_up(up[i], cu[i]);
        dn[i] = c == 0 ? cd[i] : add2_dn(dn[i], cd[i]);
      }
    }
  }
}

// The pooled bf16 values from an interval: true when both copies agree on every value and sum * 2^-(LEV log2 p)
// is zero or a normal number (then that fp32 product is exact and its bf16 rounding is the definition's).
template <int NW>
__device__ __forceinline__ bool iv_finish(const uint64_t (&up)[NW], const uint64_t (&dn)[NW], float scale,
                                          RowW<NW>& out) {
  uint32_t diff = 0u;
  bool normal = true;
#pragma unroll
  for (int i = 0; i < NW; ++i) {
    const float u0 = __uint_as_float((uint32_t)up[i]), u1 = __uint_as_float((uint32_t)(up[i] >> 32));
    const float d0 = __uint_as_float((uint32_t)dn[i]), d1 = __uint_as_float((uint32_t)(dn[i] >> 32));
    // x - y is zero exactly when x == y (gradual underflow); inf - inf and NaN give NaN, never zero
    diff |= __float_as_uint(sub_rn(u0, d0)) | __float_as_uint(sub_rn(u1, d1));
    const float v0 = mul_rn(u0, scale), v1 = mul_rn(u1, scale);
    normal &= zero_or_normal(v0) & zero_or_normal(v1);
    out.w[i] = pack_bf16x2_rn(v0, v1);
  }
  return normal && (diff & 0x7FFFFFFFu) == 0u;
}

// The definition's tree in fp64, for lanes whose interval did not close: the raw rows one at a time, level-1
// sums from the raw values, and every completed entry added into its parent (children left to right from the
// first).  A real call with the level as an argument: the path is rare, and inlined it would set the register
// budget of the whole kernel.
template <int NW, int P>
__device__ __noinline__ RowW<NW> pooled_f64(const __nv_bfloat16* p, int lev) {
  constexpr int D = 64 * NW;
  double acc[LH_MAX_LEVELS][2 * NW];  // acc[l]: running sum of the current level-l entry (l >= 1)
  int rows = 1;
  for (int l = 0; l < lev; ++l) rows *= P;
#pragma unroll 1
  for (int u = 0; u < rows; ++u) {
    const RowW<NW> r = ld_roww<NW>(p + (int64_t)u * D);
    double x[2 * NW];
#pragma unroll
    for (int i = 0; i < NW; ++i) {
      x[2 * i] = f64_of(__uint_as_float(r.w[i] << 16));
      x[2 * i + 1] = f64_of(__uint_as_float(r.w[i] & 0xFFFF0000u));
    }
    int j = u;  // index of the entry just completed one level down
#pragma unroll 1
    for (int l = 1; l <= lev; ++l) {
      const int c = j % P;
#pragma unroll
      for (int e = 0; e < 2 * NW; ++e) {
        const double ch = l == 1 ? x[e] : acc[l - 1][e];
        acc[l][e] = c == 0 ? ch : acc[l][e] + ch;
      }
      if (c != P - 1) break;
      j /= P;
    }
  }
  double inv_w = 1.0;
  for (int l = 0; l < lev; ++l) inv_w *= 1.0 / (double)P;  // exact: p is a power of two
  RowW<NW> out;
#pragma unroll
  for (int i = 0; i < NW; ++i)
    out.w[i] = f64_to_bf16_bits_rne(acc[lev][2 * i] * inv_w) | (f64_to_bf16_bits_rne(acc[lev][2 * i + 1] * inv_w) << 16);
  return out;
}

template <int NW, int P, int LEV>
__device__ __forceinline__ RowW<NW> pooled_lev(const __nv_bfloat16* p) {
  uint64_t up[NW], dn[NW];
  iv_mem<NW, P, LEV>(p, up, dn);
  RowW<NW> out;
  if (!iv_finish<NW>(up, dn, 1.0f / (float)ipow(P, LEV), out)) out = pooled_f64<NW, P>(p, LEV);
  return out;
}

// Pooled (bf16) value of a level-lev entry recomputed from its raw rows, bit-identical to the pool kernel's.
// Levels above 3 are never recomputed by the layer (it keeps at most five levels and stores the coarsest);
// they take the fp64 path.
template <int NW, int P>
__device__ __forceinline__ RowW<NW> pooled_row(const __nv_bfloat16* p, int lev) {
  switch (lev) {
    case 1: return pooled_lev<NW, P, 1>(p);
    case 2: return pooled_lev<NW, P, 2>(p);
    case 3: return pooled_lev<NW, P, 3>(p);
    default: return pooled_f64<NW, P>(p, lev);
  }
}

// bf16 -> fp16 (the attention kernels' operand format) and store.  Exact for every bf16 value of magnitude in
// [2^-14, 65504]; smaller ones round to fp16 subnormals, larger ones set *overflow.
template <int NW>
__device__ __forceinline__ void st_f16(__half* p, const RowW<NW>& v, bool& overflow) {
  uint32_t o[NW];
#pragma unroll
  for (int i = 0; i < NW; ++i) {
    const float lo = __uint_as_float(v.w[i] << 16), hi = __uint_as_float(v.w[i] & 0xFFFF0000u);
    __half2 h = __floats2half2_rn(lo, hi);
    o[i] = *reinterpret_cast<uint32_t*>(&h);
    overflow |= fabsf(lo) > 65504.f || fabsf(hi) > 65504.f;
  }
  if constexpr (NW == 2)
    *reinterpret_cast<uint2*>(p) = make_uint2(o[0], o[1]);
  else
    *reinterpret_cast<uint32_t*>(p) = o[0];
}

__device__ __forceinline__ int64_t shfl64(int64_t v, int src) {
  const int lo = __shfl_sync(0xffffffffu, (int)(uint32_t)v, src);
  const int hi = __shfl_sync(0xffffffffu, (int)(uint32_t)((uint64_t)v >> 32), src);
  return (int64_t)(((uint64_t)(uint32_t)hi << 32) | (uint32_t)lo);
}

// Each warp takes a run of kGatherRun consecutive gathered rows of one job: lane i reads the index of row i (one
// coalesced load) and works out its source; then, kGatherBatch rows at a time, the warp issues the loads of all
// copied rows (level 0 from x, stored levels from the pyramid) together, recomputes the pooled rows one by one
// while those are in flight, and stores everything as fp16.
constexpr int kGatherWarps = 4;
constexpr int kGatherRun = 32;
constexpr int kGatherBatch = 8;
constexpr int kSrcCopy = 0x100;  // code bit: the row is copied (bit 0: from the pyramid); else code = its level

template <int D, int P>
__global__ void __launch_bounds__(kGatherWarps * 32) gather_kernel(GatherJobs jobs, const int32_t* __restrict__ idx_g,
                                                                   LhDims dm) {
  constexpr int NW = D / 64;
  const GatherJob& job = jobs.job[blockIdx.y];
  const int lane = threadIdx.x & 31;
  const int64_t rows = (int64_t)dm.BH * dm.S;
  const int64_t row0 = ((int64_t)blockIdx.x * kGatherWarps + threadIdx.x / 32) * kGatherRun;
  if (row0 >= rows) return;  // whole warps only
  const __nv_bfloat16* x = reinterpret_cast<const __nv_bfloat16*>(job.x);
  const __nv_bfloat16* pyr = reinterpret_cast<const __nv_bfloat16*>(job.pyr);
  __half* out = reinterpret_cast<__half*>(job.out);

  int code = -1;  // -1: past the last row
  int64_t src = 0;  // element offset of the row's first source row
  if (row0 + lane < rows) {
    const int64_t row = row0 + lane;
    const int bh = (int)(row / dm.S);
    const int gid = idx_g[row];
    int lev = 0;
#pragma unroll
    for (int l = 1; l < LH_MAX_LEVELS; ++l)
      if (l < dm.L && gid >= dm.off[l]) lev = l;
    const int j = gid - dm.off[lev];
    if (lev == 0) {
      code = kSrcCopy;
      src = ((int64_t)bh * dm.N + j) * D;
    } else if ((job.pyr_mask >> lev) & 1u) {
      code = kSrcCopy | 1;
      src = ((int64_t)bh * job.pyr_rows + job.row_off[lev] + j) * D;
    } else {
      code = lev;
      src = ((int64_t)bh * dm.N + (int64_t)j * dm.wl[lev]) * D;
    }
  }
  const int col = lane * 2 * NW;
  bool overflow = false;
#pragma unroll 1
  for (int b0 = 0; b0 < kGatherRun && row0 + b0 < rows; b0 += kGatherBatch) {
    RowW<NW> v[kGatherBatch];
    int cr[kGatherBatch];
#pragma unroll
    for (int r = 0; r < kGatherBatch; ++r) {
      cr[r] = __shfl_sync(0xffffffffu, code, b0 + r);
      const int64_t sr = shfl64(src, b0 + r);
      if (cr[r] >= kSrcCopy) v[r] = ld_roww<NW>(((cr[r] & 1) ? pyr : x) + sr + col);
    }
#pragma unroll 1
    for (int r = 0; r < kGatherBatch; ++r) {
      const int c = __shfl_sync(0xffffffffu, code, b0 + r);
      const int64_t sr = shfl64(src, b0 + r);
      if (c >= 1 && c < kSrcCopy) st_f16<NW>(out + (row0 + b0 + r) * D + col, pooled_row<NW, P>(x + sr + col, c), overflow);
    }
#pragma unroll
    for (int r = 0; r < kGatherBatch; ++r)
      if (cr[r] >= kSrcCopy) st_f16<NW>(out + (row0 + b0 + r) * D + col, v[r], overflow);
  }
  if (overflow) set_status(dm.status, LH_ERR_RANGE);
}

template <int D, int P, int L, int kScore>
int launch_pool_kind(const PoolJobs& jobs, int njobs, const LhDims& dm, cudaStream_t st) {
  constexpr int G = D / 8;
  constexpr int W = ipow(P, L - 1);
  const int64_t groups = (int64_t)dm.BH * (dm.N / W);
  const int64_t blocks = (groups + kPoolThreads / G - 1) / (kPoolThreads / G);
  if (blocks * njobs > 0x7fffffff) return LH_ERR_UNSUPPORTED;
  const int smem = kPoolStages * pool_batch(W) * kPoolThreads * (int)sizeof(uint4);
  auto kernel = pool_score_kernel<D, P, L, kScore>;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return LH_ERR_CUDA;
  kernel<<<(unsigned)(blocks * njobs), kPoolThreads, smem, st>>>(jobs, njobs, dm);
  return check_launch();
}

template <int D, int P, int L>
int launch_pool_t(const PoolJobs& jobs, int njobs, const LhDims& dm, cudaStream_t st) {
  if (njobs <= 0) return LH_OK;
  bool scored = false;
  for (int i = 0; i < njobs; ++i) scored |= jobs.job[i].scores != nullptr;
  if (!scored) return launch_pool_kind<D, P, L, 0>(jobs, njobs, dm, st);
  return dm.expand ? launch_pool_kind<D, P, L, 2>(jobs, njobs, dm, st) : launch_pool_kind<D, P, L, 1>(jobs, njobs, dm, st);
}

template <int D, int P>
int launch_pool_dp(const PoolJobs& jobs, int njobs, const LhDims& dm, cudaStream_t st) {
  switch (dm.L) {
    case 2: return launch_pool_t<D, P, 2>(jobs, njobs, dm, st);
    case 3: return launch_pool_t<D, P, 3>(jobs, njobs, dm, st);
    case 4: return launch_pool_t<D, P, 4>(jobs, njobs, dm, st);
    case 5:
      if constexpr (P <= 4) return launch_pool_t<D, P, 5>(jobs, njobs, dm, st);
      return LH_ERR_UNSUPPORTED;
    default: return LH_ERR_UNSUPPORTED;
  }
}

template <int D>
int launch_pool_d(const PoolJobs& jobs, int njobs, const LhDims& dm, cudaStream_t st) {
  switch (dm.p) {
    case 2: return launch_pool_dp<D, 2>(jobs, njobs, dm, st);
    case 4: return launch_pool_dp<D, 4>(jobs, njobs, dm, st);
    case 8: return launch_pool_dp<D, 8>(jobs, njobs, dm, st);
    default: return LH_ERR_UNSUPPORTED;
  }
}

template <int D>
int launch_gather_d(const GatherJobs& jobs, int njobs, const int32_t* idx_g, const LhDims& dm, cudaStream_t st) {
  const int64_t rows = (int64_t)dm.BH * dm.S;
  const int64_t warps = (rows + kGatherRun - 1) / kGatherRun;
  const int64_t blocks = (warps + kGatherWarps - 1) / kGatherWarps;
  if (blocks == 0) return LH_OK;
  if (blocks > 0x7fffffff) return LH_ERR_UNSUPPORTED;
  dim3 grid((unsigned)blocks, njobs);
  switch (dm.p) {
    case 2: gather_kernel<D, 2><<<grid, kGatherWarps * 32, 0, st>>>(jobs, idx_g, dm); break;
    case 4: gather_kernel<D, 4><<<grid, kGatherWarps * 32, 0, st>>>(jobs, idx_g, dm); break;
    case 8: gather_kernel<D, 8><<<grid, kGatherWarps * 32, 0, st>>>(jobs, idx_g, dm); break;
    default: return LH_ERR_UNSUPPORTED;
  }
  return check_launch();
}

}  // namespace

int launch_pool_score(const PoolJobs& jobs, int njobs, const LhDims& dm, cudaStream_t st) {
  if (dm.L < 2) return LH_OK;  // a single level has nothing to pool and nothing to score
  KernelTimer timer("pool_score", st);
  return dm.d == 64 ? launch_pool_d<64>(jobs, njobs, dm, st) : launch_pool_d<128>(jobs, njobs, dm, st);
}

int launch_gather(const GatherJobs& jobs, int njobs, const int32_t* idx_g, const LhDims& dm, cudaStream_t st) {
  KernelTimer timer("gather", st);
  return dm.d == 64 ? launch_gather_d<64>(jobs, njobs, idx_g, dm, st)
                    : launch_gather_d<128>(jobs, njobs, idx_g, dm, st);
}

}  // namespace lh
