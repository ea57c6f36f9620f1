// attn_fwd.cu — causal attention over the gathered sequence (step 4), forward, on the tcgen05 tensor cores.
//
// O_g = softmax(Q_g K_g^T / sqrt(d) + M) V_g with M = -inf above the diagonal, plus the natural-log row LSE: the
// standard scaled-dot-product attention the pages run on the gathered rows ([W] 核心方法 §3 标准 FlashAttention
// 调用; [H] "How Lighthouse Attention Works").  The pages call a library kernel here; this is a kernel of its own.
//
// One CTA (128 threads) per (head, 128-row query tile), heaviest tiles first.  For each 128-row key tile:
//   TMA (128-byte swizzle) brings K_j and V_j into a two-stage ring while the previous tile computes;
//   one thread issues S = Q K_j^T (tcgen05.mma, M = N = 128, fp32 accumulator in tensor memory);
//   every thread owns one query row = one TMEM lane: it reads its 128 scores, applies the causal mask on the
//   diagonal tile, updates the running max (O in tensor memory is rescaled when any row of the warp grows),
//   exponentiates in base 2 and writes P (bf16) into a swizzled shared-memory tile.  Keeping the reference at
//   the running max makes the dominant key's P exactly 1, so O = P V stays consistent with the fp32 P the
//   backward recomputes (D = rowsum(dO o O) then matches sum_b P dP);
//   one thread issues O += P V_j (A = P K-major, B = V_j MN-major, fp32 accumulator in tensor memory).
// O_g is written in fp32: the backward's D and the scatter-back read it at full accumulator precision.
// Every wait is bounded; a timeout records LH_ERR_TIMEOUT and the block leaves after draining its own copies
// and MMAs.
#include "internal.h"

namespace lh {

namespace {

constexpr int kThreads = 128;
constexpr int kTile = 128;                 // query rows and key rows per tile
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <int D>
struct FwdLayout {
  static constexpr uint32_t TILE = kTile * D * 2;  // bytes of one [128][D] bf16 tile (D/64 swizzled blocks)
  static constexpr uint32_t Q = 0;
  static constexpr uint32_t K = TILE;              // two stages
  static constexpr uint32_t V = 3 * TILE;          // two stages
  static constexpr uint32_t P = 5 * TILE;          // [128][128] bf16, two 64-column swizzled blocks
  static constexpr uint32_t BAR = P + kTile * kTile * 2;
  static constexpr uint32_t BYTES = BAR + 128;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, float* __restrict__ og,
                    float* __restrict__ lse, int S, int ntiles, float scale_log2, int* status) {
  using Lay = FwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t bar_q = sb + Lay::BAR, bar_kv0 = bar_q + 8, bar_s = bar_q + 24, bar_o = bar_q + 32;
  const uint32_t bar_drain = bar_q + 40;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int qt = ntiles - 1 - (int)blockIdx.x;  // heaviest query tiles first
  const int bh = blockIdx.y;
  const int nkv = qt + 1;

  if (threadIdx.x == 0) {
    s_abort = 0;
    mbar_init(bar_q, 1);
    mbar_init(bar_kv0, 1);
    mbar_init(bar_kv0 + 8, 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    mbar_init(bar_drain, 1);
    fence_mbar_init();
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 0) tmem_alloc(smem_u32(&s_tmem), 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const uint32_t tS = tmem;        // columns [0, 128): scores
  const uint32_t tO = tmem + 128;  // columns [128, 128 + D): output accumulator
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;

  constexpr uint32_t idesc_qk = idesc_f32acc(kFmtF16, 128, 128, 0, 0);
  constexpr uint32_t idesc_pv = idesc_f32acc(kFmtF16, 128, D, 0, 1);

  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bar_q, Lay::TILE);
    for (int db = 0; db < D / 64; ++db) tma_load_3d(sb + Lay::Q + db * 16384, &tmQ, bar_q, db * 64, qt * kTile, bh);
    mbar_arrive_expect_tx(bar_kv0, 2 * Lay::TILE);
    for (int db = 0; db < D / 64; ++db) {
      tma_load_3d(sb + Lay::K + db * 16384, &tmK, bar_kv0, db * 64, 0, bh);
      tma_load_3d(sb + Lay::V + db * 16384, &tmV, bar_kv0, db * 64, 0, bh);
    }
  }

  const int row = warp * 32 + lane;  // query row inside the tile = TMEM lane
  float m_run = -INFINITY, l_run = 0.f;
  int issued_kv = 1;                 // K/V tiles whose loads were issued
  bool ok = true;

  for (int j = 0; j < nkv && ok; ++j) {
    const int st = j & 1;
    const uint32_t sK = sb + Lay::K + st * Lay::TILE, sV = sb + Lay::V + st * Lay::TILE;
    if (threadIdx.x == 0) {
      bool got = (j > 0 || mbar_wait(bar_q, 0, &s_abort, status)) &&
                 mbar_wait(bar_kv0 + 8 * st, (j >> 1) & 1, &s_abort, status);
      if (got) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_ss(tS, sdesc_sw128(sb + Lay::Q + koff, 16, 1024), sdesc_sw128(sK + koff, 16, 1024), idesc_qk,
                       kk > 0);
        }
        umma_commit(bar_s);
        if (j + 1 < nkv) {  // the other stage was released by the PV product of tile j-1 (waited below)
          const uint32_t bar = bar_kv0 + 8 * (st ^ 1);
          const uint32_t sK2 = sb + Lay::K + (st ^ 1) * Lay::TILE, sV2 = sb + Lay::V + (st ^ 1) * Lay::TILE;
          mbar_arrive_expect_tx(bar, 2 * Lay::TILE);
          for (int db = 0; db < D / 64; ++db) {
            tma_load_3d(sK2 + db * 16384, &tmK, bar, db * 64, (j + 1) * kTile, bh);
            tma_load_3d(sV2 + db * 16384, &tmV, bar, db * 64, (j + 1) * kTile, bh);
          }
          issued_kv = j + 2;
        }
      } else {
        s_abort = 1;
      }
    }
    ok = mbar_wait(bar_s, j & 1, &s_abort, status);
    if (!__syncthreads_and(ok)) {
      ok = false;
      break;
    }
    tc_fence_after();

    float s[4][32];
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_ld32(tS + lane_base + c * 32, s[c]);
    tmem_ld_wait();

    const bool diag = (j == qt);
    float mx = -INFINITY;
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        float x = s[c][i] * scale_log2;
        if (diag && (c * 32 + i) > row) x = -INFINITY;
        s[c][i] = x;
        mx = fmaxf(mx, x);
      }
    const bool grow = mx > m_run;
    const float m_new = grow ? mx : m_run;
    const float alpha = ex2(m_run - m_new);  // 1 without growth; 0 on the first tile
    if (j > 0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        tmem_ld32(tO + lane_base + c * 32, o);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] *= alpha;
        tmem_st32(tO + lane_base + c * 32, o);
      }
      tmem_st_wait();
    }
    m_run = m_new;
    float rs = 0.f;
    uint8_t* sP = smem + Lay::P;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
#pragma unroll
      for (int q8 = 0; q8 < 4; ++q8) {
        float p[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          p[i] = ex2(s[c][q8 * 8 + i] - m_run);
          rs += p[i];
        }
        const int col = c * 32 + q8 * 8;  // first key column of this 16-byte chunk
        const uint4 v = make_uint4(pack_half2_rn(p[0], p[1]), pack_half2_rn(p[2], p[3]),
                                   pack_half2_rn(p[4], p[5]), pack_half2_rn(p[6], p[7]));
        *reinterpret_cast<uint4*>(sP + (col >> 6) * 16384 + sw128_offset(row, (col & 63) >> 3)) = v;
      }
    }
    l_run = l_run * alpha + rs;
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < kTile / 16; ++kk) {
        const uint64_t a = sdesc_sw128(sb + Lay::P + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
        const uint64_t b = sdesc_sw128(sV + kk * 2048, 16384, 1024);
        umma_ss(tO, a, b, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
      }
      umma_commit(bar_o);
    }
    ok = mbar_wait(bar_o, j & 1, &s_abort, status);
    if (!__syncthreads_and(ok)) {
      ok = false;
      break;
    }
    tc_fence_after();
  }

  if (ok) {
    const int grow_idx = qt * kTile + row;
    const float inv_l = 1.0f / l_run;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      float o[32];
      tmem_ld32(tO + lane_base + c * 32, o);
      tmem_ld_wait();
      if (grow_idx < S) {
        float4* dst = reinterpret_cast<float4*>(og + ((int64_t)bh * S + grow_idx) * D + c * 32);
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4)
          dst[q4] = make_float4(o[q4 * 4 + 0] * inv_l, o[q4 * 4 + 1] * inv_l, o[q4 * 4 + 2] * inv_l,
                                o[q4 * 4 + 3] * inv_l);
      }
    }
    if (grow_idx < S) lse[(int64_t)bh * S + grow_idx] = (m_run + __log2f(l_run)) * kLn2;
  } else if (threadIdx.x == 0) {
    // drain: outstanding TMA copies and MMAs must finish before shared and tensor memory are released
    umma_commit(bar_drain);
    mbar_wait_teardown(bar_drain, 0);
    mbar_wait_teardown(bar_q, 0);
    // only the last two K/V tiles can still be in flight, one per stage (older phases were consumed)
    for (int t = issued_kv >= 2 ? issued_kv - 2 : 0; t < issued_kv; ++t)
      mbar_wait_teardown(bar_kv0 + 8 * (t & 1), (t >> 1) & 1);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <int D>
int launch_fwd_t(const void* qg, const void* kg, const void* vg, float* og, float* lse, const LhDims& dm,
                 cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  if (make_tmap_f16_3d(&mq, qg, D, dm.S, dm.BH) || make_tmap_f16_3d(&mk, kg, D, dm.S, dm.BH) ||
      make_tmap_f16_3d(&mv, vg, D, dm.S, dm.BH))
    return LH_ERR_CUDA;
  const int smem = FwdLayout<D>::BYTES + 1024;
  if (cudaFuncSetAttribute(attn_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return LH_ERR_CUDA;
  const int nt = (dm.S + kTile - 1) / kTile;
  const float scale_log2 = kLog2e / sqrtf((float)D);
  KernelTimer timer("attn_fwd", st);
  attn_fwd_kernel<D><<<dim3(nt, dm.BH), kThreads, smem, st>>>(mq, mk, mv, og, lse, dm.S, nt,
                                                               scale_log2, dm.status);
  return check_launch();
}

}  // namespace

int launch_attn_fwd(const void* qg, const void* kg, const void* vg, float* og, float* lse, const LhDims& dm,
                    cudaStream_t st) {
  return dm.d == 64 ? launch_fwd_t<64>(qg, kg, vg, og, lse, dm, st) : launch_fwd_t<128>(qg, kg, vg, og, lse, dm, st);
}

}  // namespace lh
