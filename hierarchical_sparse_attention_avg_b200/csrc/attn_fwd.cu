// attn_fwd.cu — causal attention over the gathered sequence (step 4), forward, on the tcgen05 tensor cores.
//
// O_g = softmax(Q_g K_g^T / sqrt(d) + M) V_g with M = -inf above the diagonal, plus the natural-log row LSE: the
// standard scaled-dot-product attention the pages run on the gathered rows ([W] 核心方法 §3 标准 FlashAttention
// 调用; [H] "How Lighthouse Attention Works").  The pages call a library kernel here; this is a kernel of its own.
//
// One CTA per (head, 128-row query tile), heaviest tiles first, with warp roles:
//   warp 0     TMA producer: Q once; K_j and V_j into two-stage rings with their own full/empty barriers;
//   warp 1     MMA issuer (one thread): S_j = Q K_j^T into one of two TMEM score buffers, then O_b += P_j V_j;
//   warps 2-5  softmax, one query row (= one TMEM lane) per thread.
// The MMA thread issues S_{j+1} before O += P_j V_j, so the tensor core computes the next scores while the
// softmax works on the current ones.  There are two O accumulators in tensor memory: tile j accumulates into O_b,
// b = j mod 2, so before the softmax rescales O_b to its new running max and overwrites P buffer b it only waits
// for the product of tile j-2 (long finished in steady state).  At the end the two accumulators are brought to
// the final max and added.  The reference max is always the running max itself, so the dominant key's P is
// exactly 1 and O = P V stays consistent with the fp32 P the backward recomputes; O_g is stored in fp32.
// Operands are fp16 (Q, K, V exact from their bf16 values; P in [0, 1]); accumulators fp32.
// Every wait is bounded; a timeout records LH_ERR_TIMEOUT and every role leaves after draining its own work.
#include "internal.h"

namespace lh {

namespace {

constexpr int kThreads = 192;
constexpr int kTile = 128;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct FwdLayout {
  static constexpr uint32_t TILE = kTile * D * 2;  // one [128][D] fp16 tile (D/64 swizzled 16 KB blocks)
  static constexpr uint32_t PT = kTile * kTile * 2;  // one [128][128] fp16 P tile
  static constexpr uint32_t Q = 0;
  static constexpr uint32_t K = TILE;              // 2 stages
  static constexpr uint32_t V = 3 * TILE;          // 2 stages
  static constexpr uint32_t P = 5 * TILE;          // 2 buffers
  static constexpr uint32_t BAR = P + 2 * PT;
  // barriers (8 bytes each)
  static constexpr uint32_t B_Q = 0, B_KF = 1, B_KE = 3, B_VF = 5, B_VE = 7, B_SF = 9, B_SE = 11, B_PF = 13,
                            B_OD = 15, B_DRAIN = 17, NBAR = 18;
  static constexpr uint32_t BYTES = BAR + NBAR * 8;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, float* __restrict__ og, float* __restrict__ lse, int S,
                    int ntiles, float scale_log2, int* status) {
  using Lay = FwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](uint32_t i) { return sb + Lay::BAR + 8u * i; };

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int qt = ntiles - 1 - (int)blockIdx.x;  // heaviest query tiles first
  const int bh = blockIdx.y;
  const int nkv = qt + 1;

  if (threadIdx.x == 0) {
    s_abort = 0;
    mbar_init(bar(Lay::B_Q), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(Lay::B_KF + b), 1);
      mbar_init(bar(Lay::B_KE + b), 1);
      mbar_init(bar(Lay::B_VF + b), 1);
      mbar_init(bar(Lay::B_VE + b), 1);
      mbar_init(bar(Lay::B_SF + b), 1);
      mbar_init(bar(Lay::B_SE + b), kTile);
      mbar_init(bar(Lay::B_PF + b), kTile);
      mbar_init(bar(Lay::B_OD + b), 1);
    }
    mbar_init(bar(Lay::B_DRAIN), 1);
    fence_mbar_init();
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 1) tmem_alloc(smem_u32(&s_tmem), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;  // columns: S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [384,384+D)

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int kv_issued = 0;
      bool ok = true;
      mbar_arrive_expect_tx(bar(Lay::B_Q), Lay::TILE);
      for (int db = 0; db < D / 64; ++db)
        tma_load_3d(sb + Lay::Q + db * 16384, &tmQ, bar(Lay::B_Q), db * 64, qt * kTile, bh);
      for (int j = 0; j < nkv && ok; ++j) {
        const int b = j & 1;
        const uint32_t ph = ((j >> 1) - 1) & 1;  // phase of the previous use of this stage
        if (j >= 2) ok = mbar_wait(bar(Lay::B_KE + b), ph, &s_abort, status);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(Lay::B_KF + b), Lay::TILE);
        for (int db = 0; db < D / 64; ++db)
          tma_load_3d(sb + Lay::K + b * Lay::TILE + db * 16384, &tmK, bar(Lay::B_KF + b), db * 64, j * kTile, bh);
        if (j >= 2) ok = mbar_wait(bar(Lay::B_VE + b), ph, &s_abort, status);
        if (!ok) {
          kv_issued = j;  // K_j in flight without its V
          mbar_wait_teardown(bar(Lay::B_KF + b), (j >> 1) & 1);
          break;
        }
        mbar_arrive_expect_tx(bar(Lay::B_VF + b), Lay::TILE);
        for (int db = 0; db < D / 64; ++db)
          tma_load_3d(sb + Lay::V + b * Lay::TILE + db * 16384, &tmV, bar(Lay::B_VF + b), db * 64, j * kTile, bh);
        kv_issued = j + 1;
      }
      if (!ok) {  // drain the copies this thread issued before leaving
        mbar_wait_teardown(bar(Lay::B_Q), 0);
        for (int j = kv_issued >= 2 ? kv_issued - 2 : 0; j < kv_issued; ++j) {
          mbar_wait_teardown(bar(Lay::B_KF + (j & 1)), (j >> 1) & 1);
          mbar_wait_teardown(bar(Lay::B_VF + (j & 1)), (j >> 1) & 1);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_f32acc(kFmtF16, 128, 128, 0, 0);
      constexpr uint32_t idesc_pv = idesc_f32acc(kFmtF16, 128, D, 0, 1);
      bool ok = mbar_wait(bar(Lay::B_Q), 0, &s_abort, status);
      auto issue_pv = [&](int jp) {
        const int bp = jp & 1;
        const uint32_t php = (jp >> 1) & 1;
        if (!mbar_wait(bar(Lay::B_VF + bp), php, &s_abort, status)) return false;
        if (!mbar_wait(bar(Lay::B_PF + bp), php, &s_abort, status)) return false;
        tc_fence_after();
        const uint32_t tO = tmem + 256 + 128 * bp;
        const uint32_t sP = sb + Lay::P + bp * Lay::PT, sV = sb + Lay::V + bp * Lay::TILE;
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          umma_ss(tO, sdesc_sw128(sP + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                  sdesc_sw128(sV + kk * 2048, 16384, 1024), idesc_pv, (jp >= 2 || kk > 0) ? 1u : 0u);
        umma_commit(bar(Lay::B_OD + bp));
        umma_commit(bar(Lay::B_VE + bp));
        return true;
      };
      for (int j = 0; j < nkv && ok; ++j) {
        const int b = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        ok = mbar_wait(bar(Lay::B_KF + b), ph, &s_abort, status);
        if (ok && j >= 2) ok = mbar_wait(bar(Lay::B_SE + b), ph ^ 1, &s_abort, status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t tS = tmem + 128 * b;
        const uint32_t sK = sb + Lay::K + b * Lay::TILE;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_ss(tS, sdesc_sw128(sb + Lay::Q + koff, 16, 1024), sdesc_sw128(sK + koff, 16, 1024), idesc_qk,
                  kk > 0 ? 1u : 0u);
        }
        umma_commit(bar(Lay::B_SF + b));
        umma_commit(bar(Lay::B_KE + b));
        if (j >= 1) ok = issue_pv(j - 1);
      }
      if (ok) issue_pv(nkv - 1);
      // drain: every product issued above completes before the block releases its memory
      umma_commit(bar(Lay::B_DRAIN));
      mbar_wait_teardown(bar(Lay::B_DRAIN), 0);
    }
  } else {
    // ---------------------------------------------------------------- softmax (warps 2..5)
    const int quarter = warp & 3;  // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    float m_run = -INFINITY, l_run = 0.f;
    float m_ref[2] = {-INFINITY, -INFINITY};
    bool ok = true;
    for (int j = 0; j < nkv && ok; ++j) {
      const int b = j & 1;
      const uint32_t ph = (j >> 1) & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(Lay::B_SF + b), ph, &s_abort, status));  // warp-uniform
      if (!ok) break;
      tc_fence_after();
      float s[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tmem + 128 * b + lane_base + c * 32, s[c]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(bar(Lay::B_SE + b));  // score buffer b may be overwritten by S_{j+2}

      // row max of the raw scores (the scale is positive), as 8 independent chains; keys above the diagonal of
      // the last tile are masked first
      if (j == qt) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c * 32 + i > row) s[c][i] = -INFINITY;
      }
      float mx8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx8[k] = fmaxf(s[0][k], s[0][k + 8]);
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (c > 0 || i >= 16) mx8[i & 7] = fmaxf(mx8[i & 7], s[c][i]);
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) * scale_log2;
      const float m_new = fmaxf(m_run, mx);
      l_run *= ex2(m_run - m_new);  // 1 without growth; 0 on the first tile
      m_run = m_new;
      // P of this tile (fp16, in [0, 1]) = 2^(s * scale - m) and its row sum (8 independent chains)
      uint32_t pk[64];
      float rs8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float p0 = ex2(fmaf(s[c][i], scale_log2, -m_run)), p1 = ex2(fmaf(s[c][i + 1], scale_log2, -m_run));
          rs8[(i >> 1) & 7] += p0 + p1;
          pk[c * 16 + i / 2] = pack_half2_rn(p0, p1);
        }
      const float rs = ((rs8[0] + rs8[1]) + (rs8[2] + rs8[3])) + ((rs8[4] + rs8[5]) + (rs8[6] + rs8[7]));
      l_run += rs;
      // O_b and P buffer b are free once the product of tile j-2 has completed
      if (j >= 2) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(Lay::B_OD + b), ph ^ 1, &s_abort, status));
        if (!ok) break;
        tc_fence_after();
        const float alpha = ex2(m_ref[b] - m_run);
        if (__any_sync(0xffffffffu, alpha != 1.0f)) {
          const uint32_t tO = tmem + 256 + 128 * b + lane_base;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            float o[32];
            tmem_ld32(tO + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(tO + c * 32, o);
          }
          tmem_st_wait();
        }
      }
      m_ref[b] = m_run;
      uint8_t* sP = smem + Lay::P + b * Lay::PT;
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {  // 16-byte chunk ch holds keys 8*ch .. 8*ch+7
        const uint4 v = make_uint4(pk[ch * 4 + 0], pk[ch * 4 + 1], pk[ch * 4 + 2], pk[ch * 4 + 3]);
        *reinterpret_cast<uint4*>(sP + (ch >> 3) * 16384 + sw128_offset(row, ch & 7)) = v;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(Lay::B_PF + b));
    }
    // epilogue: wait for the last products, bring both accumulators to the final max, normalise, store
    if (ok) {
      const int jl = nkv - 1;
      ok = mbar_wait(bar(Lay::B_OD + (jl & 1)), (jl >> 1) & 1, &s_abort, status);
      if (ok && nkv >= 2) ok = mbar_wait(bar(Lay::B_OD + ((jl - 1) & 1)), ((jl - 1) >> 1) & 1, &s_abort, status);
    }
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.0f / l_run;
      const float a0 = ex2(m_ref[0] - m_run) * inv_l;
      const float a1 = nkv >= 2 ? ex2(m_ref[1] - m_run) * inv_l : 0.f;
      const int grow_idx = qt * kTile + row;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float o0[32], o1[32];
        tmem_ld32(tmem + 256 + lane_base + c * 32, o0);
        tmem_ld32(tmem + 384 + lane_base + c * 32, o1);
        tmem_ld_wait();
        if (grow_idx < S) {
          float4* dst = reinterpret_cast<float4*>(og + ((int64_t)bh * S + grow_idx) * D + c * 32);
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            float r[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i = q4 * 4 + e;
              r[e] = nkv >= 2 ? fmaf(o0[i], a0, o1[i] * a1) : o0[i] * a0;
            }
            dst[q4] = make_float4(r[0], r[1], r[2], r[3]);
          }
        }
      }
      if (grow_idx < S) lse[(int64_t)bh * S + grow_idx] = (m_run + __log2f(l_run)) * kLn2;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
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
  attn_fwd_kernel<D><<<dim3(nt, dm.BH), kThreads, smem, st>>>(mq, mk, mv, og, lse, dm.S, nt, scale_log2, dm.status);
  return check_launch();
}

}  // namespace

int launch_attn_fwd(const void* qg, const void* kg, const void* vg, float* og, float* lse, const LhDims& dm,
                    cudaStream_t st) {
  return dm.d == 64 ? launch_fwd_t<64>(qg, kg, vg, og, lse, dm, st) : launch_fwd_t<128>(qg, kg, vg, og, lse, dm, st);
}

}  // namespace lh
