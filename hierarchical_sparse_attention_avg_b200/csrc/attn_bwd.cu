// attn_bwd.cu — causal attention backward over the gathered sequence, on the tcgen05 tensor cores.
//
// Textbook softmax backward of O_g = softmax(Q_g K_g^T / sqrt(d) + M) V_g: with P = exp(S / sqrt(d) - LSE),
// dV = P^T dO, dP = dO V^T, dS = P o (dP - D) / sqrt(d) with D = rowsum(dO o O), dQ = dS K, dK = dS^T Q.  The pages
// leave this to the attention library's autograd ([W] 深度洞察; [E] "Как four-stage pipeline…"); this is a kernel
// of its own.
//
// One CTA (128 threads) per (head, 128-row key tile); K_j, V_j stay in shared memory while the query tiles
// i >= j stream through (TMA, 128-byte swizzle).  Per query tile:
//   S^T = K_j Q_i^T and dP^T = V_j dO_i^T (tensor memory, M = 128 key rows, N = 128 query rows);
//   each thread owns one key row (one TMEM lane): P^T and dS^T rows go to swizzled shared-memory tiles (bf16);
//   dV_j += P^T dO_i and dK_j += dS^T Q_i accumulate in tensor memory for the whole loop;
//   dQ_i^T = K_j^T dS^T (M = 128 over the head dimension, N = 128 query rows) lands in the S^T columns, and each
//   thread (one feature) adds its 128 values to the fp32 dQ accumulator in global memory: a warp's 32 lanes
//   touch 32 consecutive floats of one row, so every atomic instruction is one coalesced 128-byte reduction.
// For d = 64 the dQ^T product still uses M = 128; lanes 64..127 are ignored.
// Operands are fp16 (gathered Q, K, V exactly; P in [0, 1]; dO_g and dS scaled per head by a power of two so
// that their largest magnitudes sit near 2^10): the layer's window-summed dO_g makes the dS and dV sums cancel
// strongly, and bf16 operands (8-bit significands) were measured to exceed the 2e-2 + 2e-2|ref| tolerance where
// fp16 (11-bit) stays within it at the same tensor-core rate.  Results are multiplied by the inverse scale; a
// dS beyond the fp16 range records LH_ERR_RANGE.
#include "internal.h"

namespace lh {

namespace {

constexpr int kThreads = 128;
constexpr int kTile = 128;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct BwdLayout {
  static constexpr uint32_t TILE = kTile * D * 2;
  static constexpr uint32_t K = 0;
  static constexpr uint32_t V = TILE;
  static constexpr uint32_t Q = 2 * TILE;
  static constexpr uint32_t DO = 3 * TILE;
  static constexpr uint32_t P = 4 * TILE;              // [128 key][128 query] bf16, two swizzled blocks
  static constexpr uint32_t DS = P + kTile * kTile * 2;
  static constexpr uint32_t LSE = DS + kTile * kTile * 2;  // 128 fp32: LSE * log2(e) of the query tile
  static constexpr uint32_t DV = LSE + 512;                // 128 fp32: D of the query tile
  static constexpr uint32_t BAR = DV + 512;
  static constexpr uint32_t BYTES = BAR + 128;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const float* __restrict__ lse, const float* __restrict__ dvec, const float* __restrict__ dinv,
                    float* __restrict__ dqacc, float* __restrict__ dkg, float* __restrict__ dvg, int S, int ntiles,
                    float scale, int* status) {
  using Lay = BwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t bar_kv = sb + Lay::BAR, bar_qd = bar_kv + 8, bar_mm1 = bar_kv + 16, bar_mm2 = bar_kv + 24;
  const uint32_t bar_drain = bar_kv + 32;
  float* s_lse = reinterpret_cast<float*>(smem + Lay::LSE);
  float* s_d = reinterpret_cast<float*>(smem + Lay::DV);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int kt = blockIdx.x;  // key tile: tile 0 meets the most query tiles and is scheduled first
  const int bh = blockIdx.y;
  const float scale_log2 = scale * kLog2e;

  if (threadIdx.x == 0) {
    s_abort = 0;
    mbar_init(bar_kv, 1);
    mbar_init(bar_qd, 1);
    mbar_init(bar_mm1, 1);
    mbar_init(bar_mm2, 1);
    mbar_init(bar_drain, 1);
    fence_mbar_init();
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmDO);
  }
  if (warp == 0) tmem_alloc(smem_u32(&s_tmem), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const uint32_t tS = tmem;            // S^T, later dQ^T
  const uint32_t tDP = tmem + 128;     // dP^T
  const uint32_t tDV = tmem + 256;     // dV accumulator (D columns)
  const uint32_t tDK = tmem + 256 + D; // dK accumulator (D columns)
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;

  constexpr uint32_t idesc_kk = idesc_f32acc(kFmtF16, 128, 128, 0, 0);  // both operands K-major
  constexpr uint32_t idesc_acc = idesc_f32acc(kFmtF16, 128, D, 0, 1);   // A K-major, B MN-major
  constexpr uint32_t idesc_dq = idesc_f32acc(kFmtF16, 128, 128, 1, 1);  // both operands MN-major
  const float inv_scale = dinv[bh];                                     // undoes the per-head dO_g scale

  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bar_kv, 2 * Lay::TILE);
    for (int db = 0; db < D / 64; ++db) {
      tma_load_3d(sb + Lay::K + db * 16384, &tmK, bar_kv, db * 64, kt * kTile, bh);
      tma_load_3d(sb + Lay::V + db * 16384, &tmV, bar_kv, db * 64, kt * kTile, bh);
    }
    mbar_arrive_expect_tx(bar_qd, 2 * Lay::TILE);
    for (int db = 0; db < D / 64; ++db) {
      tma_load_3d(sb + Lay::Q + db * 16384, &tmQ, bar_qd, db * 64, kt * kTile, bh);
      tma_load_3d(sb + Lay::DO + db * 16384, &tmDO, bar_qd, db * 64, kt * kTile, bh);
    }
  }

  const int r = warp * 32 + lane;  // TMEM lane: key row of S^T/dP^T/dV/dK, feature of dQ^T
  bool ok = true;
  int issued_qd = 1;

  for (int i = kt; i < ntiles && ok; ++i) {
    const int it = i - kt;
    {  // query-tile statistics into shared memory (rows beyond S contribute nothing)
      const int q = i * kTile + r;
      s_lse[r] = q < S ? lse[(int64_t)bh * S + q] * kLog2e : INFINITY;
      s_d[r] = q < S ? dvec[(int64_t)bh * S + q] : 0.f;
    }
    if (threadIdx.x == 0) {
      const bool got = (it > 0 || mbar_wait(bar_kv, 0, &s_abort, status)) &&
                       mbar_wait(bar_qd, it & 1, &s_abort, status);
      if (got) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_ss(tS, sdesc_sw128(sb + Lay::K + koff, 16, 1024), sdesc_sw128(sb + Lay::Q + koff, 16, 1024),
                       idesc_kk, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_ss(tDP, sdesc_sw128(sb + Lay::V + koff, 16, 1024), sdesc_sw128(sb + Lay::DO + koff, 16, 1024),
                       idesc_kk, kk > 0);
        }
        umma_commit(bar_mm1);
      } else {
        s_abort = 1;
      }
    }
    ok = mbar_wait(bar_mm1, it & 1, &s_abort, status);
    if (!__syncthreads_and(ok)) {
      ok = false;
      break;
    }
    tc_fence_after();

    // P^T and dS^T rows of key r
    const bool diag = (i == kt);
    uint8_t* sP = smem + Lay::P;
    uint8_t* sDS = smem + Lay::DS;
    float ds_max = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float sv[32], dp[32];
      tmem_ld32(tS + lane_base + c * 32, sv);
      tmem_ld32(tDP + lane_base + c * 32, dp);
      tmem_ld_wait();
#pragma unroll
      for (int q8 = 0; q8 < 4; ++q8) {
        float p[8], ds[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int qc = c * 32 + q8 * 8 + e;  // query column inside the tile
          float pv = ex2(sv[q8 * 8 + e] * scale_log2 - s_lse[qc]);
          if (diag && qc < r) pv = 0.f;        // query qc does not see key r
          p[e] = pv;
          ds[e] = pv * (dp[q8 * 8 + e] - s_d[qc]) * scale;  // scaled by the head's dO_g scale
          ds_max = fmaxf(ds_max, fabsf(ds[e]));
        }
        const int col = c * 32 + q8 * 8;
        const uint32_t off = (col >> 6) * 16384 + sw128_offset(r, (col & 63) >> 3);
        *reinterpret_cast<uint4*>(sP + off) =
            make_uint4(pack_half2_rn(p[0], p[1]), pack_half2_rn(p[2], p[3]), pack_half2_rn(p[4], p[5]),
                       pack_half2_rn(p[6], p[7]));
        *reinterpret_cast<uint4*>(sDS + off) =
            make_uint4(pack_half2_rn(ds[0], ds[1]), pack_half2_rn(ds[2], ds[3]), pack_half2_rn(ds[4], ds[5]),
                       pack_half2_rn(ds[6], ds[7]));
      }
    }
    if (__any_sync(0xffffffffu, !(ds_max <= 65504.f)) && lane == 0) set_status(status, LH_ERR_RANGE);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < kTile / 16; ++kk) {  // reduction over the 128 query rows
        const uint32_t aoff = (kk >> 2) * 16384 + (kk & 3) * 32;
        umma_ss(tDV, sdesc_sw128(sb + Lay::P + aoff, 16, 1024), sdesc_sw128(sb + Lay::DO + kk * 2048, 16384, 1024),
                     idesc_acc, (it > 0 || kk > 0) ? 1u : 0u);
        umma_ss(tDK, sdesc_sw128(sb + Lay::DS + aoff, 16, 1024), sdesc_sw128(sb + Lay::Q + kk * 2048, 16384, 1024),
                     idesc_acc, (it > 0 || kk > 0) ? 1u : 0u);
      }
#pragma unroll
      for (int kk = 0; kk < kTile / 16; ++kk) {  // reduction over the 128 key rows
        umma_ss(tS, sdesc_sw128(sb + Lay::K + kk * 2048, 16384, 1024),
                     sdesc_sw128(sb + Lay::DS + kk * 2048, 16384, 1024), idesc_dq, kk > 0);
      }
      umma_commit(bar_mm2);
    }
    ok = mbar_wait(bar_mm2, it & 1, &s_abort, status);
    if (!__syncthreads_and(ok)) {
      ok = false;
      break;
    }
    tc_fence_after();
    if (threadIdx.x == 0 && i + 1 < ntiles) {  // Q_i and dO_i are no longer read
      mbar_arrive_expect_tx(bar_qd, 2 * Lay::TILE);
      for (int db = 0; db < D / 64; ++db) {
        tma_load_3d(sb + Lay::Q + db * 16384, &tmQ, bar_qd, db * 64, (i + 1) * kTile, bh);
        tma_load_3d(sb + Lay::DO + db * 16384, &tmDO, bar_qd, db * 64, (i + 1) * kTile, bh);
      }
      issued_qd = it + 2;
    }
    // dQ^T: lane r = feature r, columns = the 128 query rows of tile i
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float v[32];
      tmem_ld32(tS + lane_base + c * 32, v);
      tmem_ld_wait();
      if (r < D) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int q = i * kTile + c * 32 + e;
          if (q < S) atomicAdd(dqacc + ((int64_t)bh * S + q) * D + r, v[e] * inv_scale);
        }
      }
    }
    tc_fence_before();
    __syncthreads();  // S^T columns, P and dS tiles and the statistics are reused by the next query tile
    tc_fence_after();
  }

  if (ok) {
    const int krow = kt * kTile + r;
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      const uint32_t tacc = which == 0 ? tDV : tDK;
      float* dst_base = which == 0 ? dvg : dkg;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float v[32];
        tmem_ld32(tacc + lane_base + c * 32, v);
        tmem_ld_wait();
        if (krow < S) {
          float4* dst = reinterpret_cast<float4*>(dst_base + ((int64_t)bh * S + krow) * D + c * 32);
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)
            dst[q4] = make_float4(v[q4 * 4 + 0] * inv_scale, v[q4 * 4 + 1] * inv_scale, v[q4 * 4 + 2] * inv_scale,
                                  v[q4 * 4 + 3] * inv_scale);
        }
      }
    }
  } else if (threadIdx.x == 0) {
    umma_commit(bar_drain);
    mbar_wait_teardown(bar_drain, 0);
    mbar_wait_teardown(bar_kv, 0);
    mbar_wait_teardown(bar_qd, (issued_qd - 1) & 1);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D>
int launch_bwd_t(const void* qg, const void* kg, const void* vg, const void* dog16, const float* lse, const float* dvec,
                 const float* dinv, float* dqacc, float* dkg, float* dvg, const LhDims& dm, cudaStream_t st) {
  CUtensorMap mq, mk, mv, mdo;
  if (make_tmap_f16_3d(&mq, qg, D, dm.S, dm.BH) || make_tmap_f16_3d(&mk, kg, D, dm.S, dm.BH) ||
      make_tmap_f16_3d(&mv, vg, D, dm.S, dm.BH) || make_tmap_f16_3d(&mdo, dog16, D, dm.S, dm.BH))
    return LH_ERR_CUDA;
  const int smem = BwdLayout<D>::BYTES + 1024;
  if (cudaFuncSetAttribute(attn_bwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return LH_ERR_CUDA;
  const int nt = (dm.S + kTile - 1) / kTile;
  KernelTimer timer("attn_bwd", st);
  attn_bwd_kernel<D><<<dim3(nt, dm.BH), kThreads, smem, st>>>(mq, mk, mv, mdo, lse, dvec, dinv, dqacc, dkg, dvg,
                                                               dm.S, nt, 1.0f / sqrtf((float)D), dm.status);
  return check_launch();
}

}  // namespace

int launch_attn_bwd(const void* qg, const void* kg, const void* vg, const void* dog16, const float* lse,
                    const float* dvec, const float* dinv, float* dqacc, float* dkg, float* dvg, const LhDims& dm,
                    cudaStream_t st) {
  return dm.d == 64 ? launch_bwd_t<64>(qg, kg, vg, dog16, lse, dvec, dinv, dqacc, dkg, dvg, dm, st)
                    : launch_bwd_t<128>(qg, kg, vg, dog16, lse, dvec, dinv, dqacc, dkg, dvg, dm, st);
}

}  // namespace lh
