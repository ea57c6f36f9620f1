// attn_fwd.cu — causal attention over the gathered sequence (step 4), forward, on the tcgen05 tensor cores.
//
// O_g = softmax(Q_g K_g^T / sqrt(d) + M) V_g with M = -inf above the diagonal, plus the natural-log row LSE: the
// standard scaled-dot-product attention the pages run on the gathered rows ([W] 核心方法 §3 标准 FlashAttention
// 调用; [H] "How Lighthouse Attention Works").  The pages call a library kernel here; this is a kernel of its own.
//
// One CTA per (head, pair of 128-row query tiles), heaviest pairs first, with warp roles:
//   warp 0     TMA producer: both query tiles once; K_j and V_j into two-stage rings (full/empty barriers);
//   warp 1     MMA issuer (one thread);
//   warps 2-5  softmax of query tile 0, warps 6-9 softmax of query tile 1: one query row (= TMEM lane) per thread.
// Tensor memory per query tile q: S_q (128 fp32 columns; P_q, fp16, is written over its first 64 columns once the
// scores are read) and the accumulator O_q (d columns).  The MMA thread alternates the tiles:
//   ... O_0 += P_0,j V_j | S_0,j+1 = Q_0 K_j+1^T | O_1 += P_1,j V_j | S_1,j+1 = Q_1 K_j+1^T ...
// so the tensor core works on one tile while the other tile's softmax runs.  Tensor-core operations complete in
// issue order, so the commit that publishes S_q,j+1 also means O_q += P_q,j V_j is done: the softmax may rescale
// O_q to a new reference max right after reading the scores, with no further wait, and the next S may overwrite
// P_q.  The reference max of a row moves only when the row max exceeds it by more than 2^kSlack, so P lies in
// [0, 2^kSlack] (fp16 keeps its relative precision there) and O is rarely rescaled; the row sum uses the same P,
// and O_g is stored in fp32.  Operands fp16 (Q, K, V exact from their bf16 values), accumulators fp32.
// Every wait is bounded; a timeout records LH_ERR_TIMEOUT and every role leaves after draining its own work.
#include "internal.h"

namespace lh {

namespace {

constexpr int kThreads = 320;
constexpr int kTile = 128;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kSlack = 8.0f;  // largest log2 of P
// Below this many CTAs (query-tile pairs) per head the grid runs head-fastest, so every head's longest CTAs start
// in the first waves instead of trailing the grid (512K, S = 20K: 1.67 -> 1.56 ms); above it the pairs of one head
// run together and share its keys and values in L2, which dominates at very long S (dense 512K: 1024 ms against
// 1267 head-fastest).
constexpr int kHeadFastBelow = 512;

template <int D>
struct FwdLayout {
  static constexpr uint32_t TILE = kTile * D * 2;  // one [128][D] fp16 tile (D/64 swizzled 16 KB blocks)
  static constexpr uint32_t Q = 0;                 // 2 query tiles
  static constexpr uint32_t K = 2 * TILE;          // 2 stages
  static constexpr uint32_t V = 4 * TILE;          // 2 stages
  static constexpr uint32_t BAR = 6 * TILE;
  // barriers (8 bytes each); per-stage pairs at +0/+1, per-query-tile pairs at +0/+1
  static constexpr uint32_t B_Q = 0, B_KF = 1, B_KE = 3, B_VF = 5, B_VE = 7, B_SF = 9, B_PF = 11, B_OD = 13,
                            B_DRAIN = 15, NBAR = 16;
  static constexpr uint32_t BYTES = BAR + NBAR * 8;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, float* __restrict__ og, float* __restrict__ lse, int S,
                    int npair, int q_tile0, int kv_tpb, int head_fast, float scale_log2, int* status) {
  using Lay = FwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ WaitCtl s_wait;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](uint32_t i) { return sb + Lay::BAR + 8u * i; };

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // heaviest pairs first; with head_fast the head is the grid's fastest index
  const int pt = npair - 1 - (int)(head_fast ? blockIdx.y : blockIdx.x);
  const int bh = head_fast ? blockIdx.x : blockIdx.y;
  const int ntile = (S + kTile - 1) / kTile;
  const bool v1 = 2 * pt + 1 < ntile;    // the pair's second query tile exists
  // key tiles are numbered globally: the local query tile t is global tile q_tile0 + t (context parallelism puts
  // the local queries after q_tile0 tiles of earlier ranks' keys); key tile j is tile j % kv_tpb of block j / kv_tpb
  const int nkv0 = q_tile0 + 2 * pt + 1;  // key tiles of query tile 0 (its diagonal is the last one)
  const int nkv = v1 ? nkv0 + 1 : nkv0;  // key tiles loaded (= those of query tile 1 when it exists)

  if (threadIdx.x == 0) {
    wait_ctl_init(&s_wait, status);
    mbar_init(bar(Lay::B_Q), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(Lay::B_KF + b), 1);
      mbar_init(bar(Lay::B_KE + b), 1);
      mbar_init(bar(Lay::B_VF + b), 1);
      mbar_init(bar(Lay::B_VE + b), 1);
      mbar_init(bar(Lay::B_SF + b), 1);
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
  const uint32_t tmem = s_tmem;  // columns: S/P of tile q at 128 q, O of tile q at 256 + 128 q

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int kv_issued = 0;
      bool ok = true;
      mbar_arrive_expect_tx(bar(Lay::B_Q), (v1 ? 2 : 1) * Lay::TILE);
      for (int q = 0; q < (v1 ? 2 : 1); ++q)
        for (int db = 0; db < D / 64; ++db)
          tma_load_3d(sb + Lay::Q + q * Lay::TILE + db * 16384, &tmQ, bar(Lay::B_Q), db * 64,
                      (2 * pt + q) * kTile, bh);
      for (int j = 0; j < nkv && ok; ++j) {
        const int b = j & 1;
        const uint32_t ph = ((j >> 1) - 1) & 1;  // phase of the previous use of this stage
        if (j >= 2) ok = mbar_wait(bar(Lay::B_KE + b), ph, &s_wait, status);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(Lay::B_KF + b), Lay::TILE);
        for (int db = 0; db < D / 64; ++db)
          tma_load_4d(sb + Lay::K + b * Lay::TILE + db * 16384, &tmK, bar(Lay::B_KF + b), db * 64,
                      (j % kv_tpb) * kTile, bh, j / kv_tpb);
        if (j >= 2) ok = mbar_wait(bar(Lay::B_VE + b), ph, &s_wait, status);
        if (!ok) {
          kv_issued = j;  // K_j in flight without its V
          mbar_wait_teardown(bar(Lay::B_KF + b), (j >> 1) & 1);
          break;
        }
        mbar_arrive_expect_tx(bar(Lay::B_VF + b), Lay::TILE);
        for (int db = 0; db < D / 64; ++db)
          tma_load_4d(sb + Lay::V + b * Lay::TILE + db * 16384, &tmV, bar(Lay::B_VF + b), db * 64,
                      (j % kv_tpb) * kTile, bh, j / kv_tpb);
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
      auto mma_s = [&](int q, int j) {  // S_q,j = Q_q K_j^T
        const uint32_t tS = tmem + 128 * q;
        const uint32_t sQ = sb + Lay::Q + q * Lay::TILE, sK = sb + Lay::K + (j & 1) * Lay::TILE;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_ss(tS, sdesc_sw128(sQ + koff, 16, 1024), sdesc_sw128(sK + koff, 16, 1024), idesc_qk,
                  kk > 0 ? 1u : 0u);
        }
        umma_commit(bar(Lay::B_SF + q));
      };
      auto mma_pv = [&](int q, int j) {  // O_q (+)= P_q,j V_j, P from tensor memory
        const uint32_t tO = tmem + 256 + 128 * q, tP = tmem + 128 * q;
        const uint32_t sV = sb + Lay::V + (j & 1) * Lay::TILE;
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          umma_ts(tO, tP + kk * 8, sdesc_sw128(sV + kk * 2048, 16384, 1024), idesc_pv,
                  (j > 0 || kk > 0) ? 1u : 0u);
      };
      bool ok = mbar_wait(bar(Lay::B_Q), 0, &s_wait, status);
      if (ok) ok = mbar_wait(bar(Lay::B_KF), 0, &s_wait, status);
      if (ok) {
        tc_fence_after();
        mma_s(0, 0);
        if (v1) mma_s(1, 0);
        umma_commit(bar(Lay::B_KE));
      }
      for (int j = 0; j < nkv && ok; ++j) {
        const int b = j & 1;
        const int nx = j + 1;
        ok = mbar_wait(bar(Lay::B_VF + b), (j >> 1) & 1, &s_wait, status);
        if (ok && j < nkv0) {
          ok = mbar_wait(bar(Lay::B_PF + 0), j & 1, &s_wait, status);
          if (ok) {
            tc_fence_after();
            mma_pv(0, j);
          }
        }
        if (ok && nx < nkv) {
          ok = mbar_wait(bar(Lay::B_KF + (nx & 1)), (nx >> 1) & 1, &s_wait, status);
          if (ok && nx < nkv0) {
            tc_fence_after();
            mma_s(0, nx);
          }
        }
        if (ok && v1) {
          ok = mbar_wait(bar(Lay::B_PF + 1), j & 1, &s_wait, status);
          if (ok) {
            tc_fence_after();
            mma_pv(1, j);
          }
        }
        if (!ok) break;
        umma_commit(bar(Lay::B_VE + b));
        if (nx < nkv) {
          if (v1) mma_s(1, nx);
          umma_commit(bar(Lay::B_KE + (nx & 1)));
        }
      }
      umma_commit(bar(Lay::B_OD + 0));
      umma_commit(bar(Lay::B_OD + 1));
      // drain: every product issued above completes before the block releases its memory
      umma_commit(bar(Lay::B_DRAIN));
      mbar_wait_teardown(bar(Lay::B_DRAIN), 0);
    }
  } else {
    // ---------------------------------------------------------------- softmax (warps 2..5: tile 0, 6..9: tile 1)
    const int q = (warp - 2) >> 2;
    if (q == 0 || v1) {
      const int quarter = warp & 3;  // TMEM lane quarter this warp may access
      const int row = quarter * 32 + lane;
      const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
      const uint32_t tS = tmem + 128 * q + lane_base, tO = tmem + 256 + 128 * q + lane_base;
      const int nkv_q = nkv0 + q;
      const int diag = q_tile0 + 2 * pt + q;  // global key tile on the diagonal
      float m_run = -INFINITY, l_run = 0.f;
      bool ok = true;
      for (int j = 0; j < nkv_q && ok; ++j) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(Lay::B_SF + q), j & 1, &s_wait, status));  // warp-uniform
        if (!ok) break;
        tc_fence_after();
        float s[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, s[c]);
        tmem_ld_wait();
        if (j == diag) {  // keys above the diagonal
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (c * 32 + i > row) s[c][i] = -INFINITY;
        }
        // row max of the raw scores (the scale is positive), as 8 independent chains: chain k takes columns
        // k, k + 8, ..., k + 120, two new ones per three-input max
        auto col = [&](int x) { return s[x >> 5][x & 31]; };
        float mx8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          float m = fmax3(col(k), col(k + 8), col(k + 16));
#pragma unroll
          for (int t = 3; t + 1 < 16; t += 2) m = fmax3(m, col(k + 8 * t), col(k + 8 * t + 8));
          mx8[k] = fmaxf(m, col(k + 120));
        }
        const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])) *
                         scale_log2;
        // The reference max moves only when some row of the warp exceeds it by more than kSlack (log2 units):
        // P = 2^(s scale - m_ref) then stays in [0, 2^kSlack], well inside fp16, and O is rescaled rarely.
        float alpha = 1.0f;
        const bool move = __any_sync(0xffffffffu, mx > m_run + kSlack);  // always on the first tile
        if (move) {
          const float m_new = fmaxf(m_run, mx);
          alpha = ex2(m_run - m_new);  // 0 on the first tile
          l_run *= alpha;
          m_run = m_new;
        }
        // P = 2^(s * scale - m) in fp16 over the first 64 columns of S (each half stored as soon as it
        // is packed, so the scores it came from are dead), and its row sum; arguments and sums as fp32 pairs
        uint64_t rs2[4] = {0ull, 0ull, 0ull, 0ull};
        const uint64_t scl2 = f2pack(scale_log2, scale_log2), nm2 = f2pack(-m_run, -m_run), one2 = f2pack(1.f, 1.f);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float pk[32];
#pragma unroll
          for (int c = 2 * h; c < 2 * h + 2; ++c)
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              const uint64_t arg = fma_f32x2(f2pack(s[c][i], s[c][i + 1]), scl2, nm2);
              const float p0 = ex2(f2lo(arg)), p1 = ex2(f2hi(arg));
              const uint64_t p2 = f2pack(p0, p1);
              rs2[(i >> 1) & 3] = fma_f32x2(p2, one2, rs2[(i >> 1) & 3]);
              pk[(c & 1) * 16 + i / 2] = __uint_as_float(pack_half2_rn(p0, p1));
            }
          tmem_st32(tS + 32 * h, pk);
        }
        float rs8[8] = {f2lo(rs2[0]), f2hi(rs2[0]), f2lo(rs2[1]), f2hi(rs2[1]),
                        f2lo(rs2[2]), f2hi(rs2[2]), f2lo(rs2[3]), f2hi(rs2[3])};
        // O_q += P_q,j-1 V_j-1 has completed (it was issued before S_q,j): bring O_q to the new max
        if (j > 0 && move) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            float o[32];
            tmem_ld32(tO + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(tO + c * 32, o);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar(Lay::B_PF + q));
        l_run += ((rs8[0] + rs8[1]) + (rs8[2] + rs8[3])) + ((rs8[4] + rs8[5]) + (rs8[6] + rs8[7]));
      }
      // epilogue: wait for the last product, normalise, store
      if (ok) ok = mbar_wait(bar(Lay::B_OD + q), 0, &s_wait, status);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
        const float inv_l = 1.0f / l_run;
        const int grow_idx = (2 * pt + q) * kTile + row;  // local query row
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_ld_wait();
          if (grow_idx < S) {
            float4* dst = reinterpret_cast<float4*>(og + ((int64_t)bh * S + grow_idx) * D + c * 32);
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              dst[q4] = make_float4(o[q4 * 4] * inv_l, o[q4 * 4 + 1] * inv_l, o[q4 * 4 + 2] * inv_l,
                                    o[q4 * 4 + 3] * inv_l);
          }
        }
        if (grow_idx < S) lse[(int64_t)bh * S + grow_idx] = (m_run + __log2f(l_run)) * kLn2;
      }
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
int launch_fwd_t(const void* qg, const KvSource& kv, float* og, float* lse, const LhDims& dm, cudaStream_t st) {
  if (kv.q_off % kTile != 0 || (kv.blocks > 1 && dm.S % kTile != 0)) return LH_ERR_UNSUPPORTED;
  CUtensorMap mq, mk, mv;
  if (make_tmap_f16_3d(&mq, qg, D, dm.S, dm.BH) ||
      make_tmap_f16_4d(&mk, kv.k, D, dm.S, dm.BH, kv.blocks, kv.block_stride) ||
      make_tmap_f16_4d(&mv, kv.v, D, dm.S, dm.BH, kv.blocks, kv.block_stride))
    return LH_ERR_CUDA;
  // at least 120 KB, so that one CTA (and its 512 tensor-memory columns) occupies an SM
  int smem = FwdLayout<D>::BYTES + 1024;
  if (smem < 120 * 1024) smem = 120 * 1024;
  if (cudaFuncSetAttribute(attn_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return LH_ERR_CUDA;
  const int nt = (dm.S + kTile - 1) / kTile;
  const int npair = (nt + 1) / 2;
  const float scale_log2 = kLog2e / sqrtf((float)D);
  KernelTimer timer("attn_fwd", st);
  const int head_fast = npair < kHeadFastBelow;
  const dim3 grid = head_fast ? dim3(dm.BH, npair) : dim3(npair, dm.BH);
  attn_fwd_kernel<D><<<grid, kThreads, smem, st>>>(mq, mk, mv, og, lse, dm.S, npair, kv.q_off / kTile, nt, head_fast,
                                                   scale_log2, dm.status);
  return check_launch();
}

}  // namespace

int launch_attn_fwd(const void* qg, const KvSource& kv, float* og, float* lse, const LhDims& dm, cudaStream_t st) {
  return dm.d == 64 ? launch_fwd_t<64>(qg, kv, og, lse, dm, st) : launch_fwd_t<128>(qg, kv, og, lse, dm, st);
}

}  // namespace lh
