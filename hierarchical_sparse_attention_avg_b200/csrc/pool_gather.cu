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
  for (int i = 0; i < 8; ++i) x[i] = (double)f[i];
}

// Score of one row: squared l2 norm of the (bf16) values x, summed in the fixed order, rounded to fp32.
template <int G>
__device__ __forceinline__ float row_score(const double (&x)[8]) {
  double s = x[0] * x[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) s = fma(x[i], x[i], s);  // x*x is exact in fp64: fma == add of the square
#pragma unroll
  for (int off = 1; off < G; off <<= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  return __double2float_rn(s);
}

// Round 8 fp64 sums / w to bf16 (single rounding), returning packed bits and the bf16 values as fp64.
__device__ __forceinline__ uint4 round_pooled(const double (&sum)[8], double inv_w, double (&val)[8]) {
  uint32_t b[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    b[i] = f64_to_bf16_bits_rne(sum[i] * inv_w);  // inv_w = 1/p^l is exact for power-of-two p
    val[i] = (double)__uint_as_float(b[i] << 16);
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
template <int D, int P, int L, bool kScore>
__global__ void __launch_bounds__(kPoolThreads) pool_score_kernel(PoolJobs jobs, LhDims dm) {
  constexpr int G = D / 8;
  constexpr int GPB = kPoolThreads / G;
  constexpr int W = ipow(P, L - 1);
  constexpr int TB = pool_batch(W);  // tokens per batch (a multiple of P)
  constexpr int NB = W / TB;          // batches per block
  static_assert(TB % P == 0, "batch must hold whole level-1 entries");
  extern __shared__ uint4 s_raw[];    // [kPoolStages][TB][kPoolThreads]

  const PoolJob& job = jobs.job[blockIdx.y];
  const int lane = threadIdx.x % G;
  const int64_t group = (int64_t)blockIdx.x * GPB + threadIdx.x / G;
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

#pragma unroll
    for (int g1 = 0; g1 < TB / P; ++g1) {
      float up[8], dn[8];
#pragma unroll
      for (int c = 0; c < P; ++c) {
        float xf[8];
        unpack8(raw_s[(g1 * P + c) * kPoolThreads], xf);
        if (kScore) {  // level 0 is scored whenever L >= 2
          double x[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) x[i] = (double)xf[i];
          float s = row_score<G>(x);
          if (active && lane == 0) scores[dm.off[0] + (int64_t)blk * W + t0 + g1 * P + c] = s;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          up[i] = (c == 0) ? xf[i] : add_up(up[i], xf[i]);
          dn[i] = (c == 0) ? xf[i] : add_dn(dn[i], xf[i]);
        }
      }
      bool exact = true;
#pragma unroll
      for (int i = 0; i < 8; ++i) exact &= same_sum(up[i], dn[i]);
      const int j1 = blk * (W / P) + t0 / P + g1;  // global level-1 index
      const bool write1 = (job.write_mask >> 1) & 1u;
      const bool score1 = kScore && 1 <= L - 2;
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
        for (int i = 0; i < 8; ++i) acc[1][i] = (double)up[i];
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
            for (int i = 0; i < 8; ++i) acc[1][i] = (double)up[i];
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
          for (int i = 0; i < 8; ++i) v[i] = (double)vf[i];
          const float sc = row_score<G>(v);
          if (active && lane == 0) scores[dm.off[1] + j1] = sc;
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
        const bool score = kScore && lev <= L - 2;
        if (write || score) {
          double val[8];
          const uint4 packed = round_pooled(acc[lev], 1.0 / (double)ipow(P, lev), val);
          if (write && active)
            st16(pyr + ((int64_t)bh * job.pyr_rows + job.row_off[lev] + j) * D + lane * 8, packed);
          if (score) {
            float s = row_score<G>(val);
            if (active && lane == 0) scores[dm.off[lev] + j] = s;
          }
        }
      }
    }
  }
}

// Level-1 entry of P raw rows (already loaded) summed with the exact fp32 chains described above; the result
// tells whether the chains agree (then `up` is the sum the definition fixes).
template <int P>
__device__ __forceinline__ bool level1_f32(const uint4* raw, float (&up)[8]) {
  float dn[8];
#pragma unroll
  for (int c = 0; c < P; ++c) {
    float x[8];
    unpack8(raw[c], x);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      up[i] = (c == 0) ? x[i] : add_up(up[i], x[i]);
      dn[i] = (c == 0) ? x[i] : add_dn(dn[i], x[i]);
    }
  }
  bool exact = true;
#pragma unroll
  for (int i = 0; i < 8; ++i) exact &= same_sum(up[i], dn[i]);
  return exact;
}

// fp64 sum of the level-LEV entry at p in the definition's tree order: level-1 sums from the fp32 chains when
// exact (one widening per entry), else in fp64 from the raw values.
template <int P>
__device__ __forceinline__ void level1_f64(const uint4* raw, double (&out)[8]) {
  float up[8];
  if (level1_f32<P>(raw, up)) {
#pragma unroll
    for (int i = 0; i < 8; ++i) out[i] = (double)up[i];
  } else {
#pragma unroll
    for (int c = 0; c < P; ++c) {
      double x[8];
      load_row8(raw[c], x);
#pragma unroll
      for (int i = 0; i < 8; ++i) out[i] = (c == 0) ? x[i] : out[i] + x[i];
    }
  }
}

// The tree over raw rows already in registers (P^LEV of them).
template <int P, int LEV>
__device__ __forceinline__ void tree_from_raw(const uint4* raw, double (&out)[8]) {
  if constexpr (LEV == 1) {
    level1_f64<P>(raw, out);
  } else {
#pragma unroll
    for (int c = 0; c < P; ++c) {
      double ch[8];
      tree_from_raw<P, LEV - 1>(raw + c * ipow(P, LEV - 1), ch);
#pragma unroll
      for (int i = 0; i < 8; ++i) out[i] = (c == 0) ? ch[i] : out[i] + ch[i];
    }
  }
}

template <int D, int P, int LEV>
__device__ __forceinline__ void tree_sum(const __nv_bfloat16* p, double (&out)[8]) {
  if constexpr (ipow(P, LEV) <= 16) {
    // few enough rows to keep all of their loads in flight at once; the sums keep the tree order
    constexpr int R = ipow(P, LEV);
    uint4 raw[R];
#pragma unroll
    for (int u = 0; u < R; ++u) raw[u] = ld16(p + (int64_t)u * D);
    tree_from_raw<P, LEV>(raw, out);
  } else if constexpr (LEV == 1) {
    uint4 raw[P];
#pragma unroll
    for (int u = 0; u < P; ++u) raw[u] = ld16(p + (int64_t)u * D);
    level1_f64<P>(raw, out);
  } else {
    constexpr int CW = ipow(P, LEV - 1);
#pragma unroll 1
    for (int c = 0; c < P; ++c) {
      double ch[8];
      tree_sum<D, P, LEV - 1>(p + (int64_t)c * CW * D, ch);
#pragma unroll
      for (int i = 0; i < 8; ++i) out[i] = (c == 0) ? ch[i] : out[i] + ch[i];
    }
  }
}

// Pooled (bf16) value of entry (lev, j) recomputed from the raw rows with the same summation tree as the pool
// kernel: a level-1 entry whose fp32 chains agree is rounded straight from fp32.
template <int D, int P>
__device__ __forceinline__ uint4 pooled_row(const __nv_bfloat16* x0, int lev) {
  double s[8], val[8];
  if (lev == 1) {
    uint4 raw[P];
#pragma unroll
    for (int u = 0; u < P; ++u) raw[u] = ld16(x0 + (int64_t)u * D);
    float up[8], pv[8];
    bool fast = level1_f32<P>(raw, up);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      pv[i] = mul_rn(up[i], 1.0f / (float)P);
      fast &= zero_or_normal(pv[i]);
    }
    if (fast)
      return make_uint4(pack_bf16x2_rn(pv[0], pv[1]), pack_bf16x2_rn(pv[2], pv[3]), pack_bf16x2_rn(pv[4], pv[5]),
                        pack_bf16x2_rn(pv[6], pv[7]));
    tree_sum<D, P, 1>(x0, s);
  } else if (lev == 2) {
    tree_sum<D, P, 2>(x0, s);
  } else if (lev == 3) {
    tree_sum<D, P, 3>(x0, s);
  } else {
    tree_sum<D, P, 4>(x0, s);
  }
  return round_pooled(s, 1.0 / (double)ipow(P, lev), val);
}

// One group per gathered row (b, h, s): copy (level 0), read (pyramid) or recompute (pooled) the row, and store
// it as fp16, the operand format of the attention kernels (every bf16 value of magnitude in [2^-14, 65504] is
// exact in fp16; a larger one records LH_ERR_RANGE).
// Small blocks (kGatherThreads), many per SM: rows cost from one to p^(L-2) raw rows, and a block retires only
// with its slowest row.
constexpr int kGatherThreads = 32;

template <int D, int P>
__global__ void __launch_bounds__(kGatherThreads, 16) gather_kernel(GatherJobs jobs, const int32_t* __restrict__ idx_g,
                                                                 LhDims dm) {
  constexpr int G = D / 8;
  const GatherJob& job = jobs.job[blockIdx.y];
  const int lane = threadIdx.x % G;
  const int64_t row = (int64_t)blockIdx.x * (kGatherThreads / G) + threadIdx.x / G;
  if (row >= (int64_t)dm.BH * dm.S) return;
  const int bh = (int)(row / dm.S);
  const int gid = idx_g[row];
  int lev = 0;
#pragma unroll
  for (int l = 1; l < LH_MAX_LEVELS; ++l)
    if (l < dm.L && gid >= dm.off[l]) lev = l;
  const int j = gid - dm.off[lev];
  const __nv_bfloat16* x = reinterpret_cast<const __nv_bfloat16*>(job.x);
  uint4 v;
  if (lev == 0) {
    v = ld16(x + ((int64_t)bh * dm.N + j) * D + lane * 8);
  } else if ((job.pyr_mask >> lev) & 1u) {
    v = ld16(reinterpret_cast<const __nv_bfloat16*>(job.pyr) +
             ((int64_t)bh * job.pyr_rows + job.row_off[lev] + j) * D + lane * 8);
  } else {
    v = pooled_row<D, P>(x + ((int64_t)bh * dm.N + (int64_t)j * dm.wl[lev]) * D + lane * 8, lev);
  }
  bool overflow = false;
  const uint4 h = bf16x8_to_f16x8(v, overflow);
  if (overflow) set_status(dm.status, LH_ERR_RANGE);
  st16(reinterpret_cast<__half*>(job.out) + row * D + lane * 8, h);
}

// Jobs with scores and jobs without run as two launches of the two specialisations (the one without carries no
// scoring code and fewer registers).
template <int D, int P, int L, bool kScore>
int launch_pool_kind(const PoolJobs& all, int njobs, const LhDims& dm, cudaStream_t st) {
  PoolJobs jobs;
  int n = 0;
  for (int i = 0; i < njobs; ++i)
    if ((all.job[i].scores != nullptr) == kScore) jobs.job[n++] = all.job[i];
  if (n == 0) return LH_OK;
  constexpr int G = D / 8;
  constexpr int W = ipow(P, L - 1);
  const int64_t groups = (int64_t)dm.BH * (dm.N / W);
  const int64_t blocks = (groups + kPoolThreads / G - 1) / (kPoolThreads / G);
  if (blocks > 0x7fffffff) return LH_ERR_UNSUPPORTED;
  const int smem = kPoolStages * pool_batch(W) * kPoolThreads * (int)sizeof(uint4);
  auto kernel = pool_score_kernel<D, P, L, kScore>;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return LH_ERR_CUDA;
  kernel<<<dim3((unsigned)blocks, n), kPoolThreads, smem, st>>>(jobs, dm);
  return check_launch();
}

template <int D, int P, int L>
int launch_pool_t(const PoolJobs& jobs, int njobs, const LhDims& dm, cudaStream_t st) {
  const int rc = launch_pool_kind<D, P, L, false>(jobs, njobs, dm, st);
  return rc != LH_OK ? rc : launch_pool_kind<D, P, L, true>(jobs, njobs, dm, st);
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
  constexpr int G = D / 8;
  const int64_t rows = (int64_t)dm.BH * dm.S;
  const int64_t blocks = (rows + kGatherThreads / G - 1) / (kGatherThreads / G);
  dim3 grid((unsigned)blocks, njobs);
  switch (dm.p) {
    case 2: gather_kernel<D, 2><<<grid, kGatherThreads, 0, st>>>(jobs, idx_g, dm); break;
    case 4: gather_kernel<D, 4><<<grid, kGatherThreads, 0, st>>>(jobs, idx_g, dm); break;
    case 8: gather_kernel<D, 8><<<grid, kGatherThreads, 0, st>>>(jobs, idx_g, dm); break;
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
