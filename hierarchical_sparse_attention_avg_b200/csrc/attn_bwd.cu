// attn_bwd.cu — causal attention backward over the gathered sequence, on the tcgen05 tensor cores.
//
// Textbook softmax backward of O_g = softmax(Q_g K_g^T / sqrt(d) + M) V_g: with P = exp(S / sqrt(d) - LSE),
// dV = P^T dO, dP = dO V^T, dS = P o (dP - D) / sqrt(d) with D = rowsum(dO o O), dQ = dS K, dK = dS^T Q.  The pages
// leave this to the attention library's autograd ([W] 深度洞察; [E] "Как four-stage pipeline…"); this is a kernel
// of its own.
//
// One CTA per (head, 128-row key tile); K_j and V_j stay in shared memory while the 64-row query sub-tiles i that
// can see them stream through.  Warp roles:
//   warp 0      TMA producer: K_j, V_j once; Q_i, dO_i and the sub-tile's statistics into a three-stage ring;
//   warp 1      MMA issuer (one thread): S^T = K_j Q_i^T and dP^T = V_j dO_i^T into one of two TMEM buffer pairs,
//               then, for the previous sub-tile, dV += P^T dO, dK += dS^T Q (accumulated in TMEM for the whole
//               loop) and dQ^T = K_j^T dS^T (into the consumed S^T columns);
//   warps 2-9   compute, two warps per TMEM lane quarter (one key row per thread), each on 32 of the sub-tile's 64
//               query columns: the P^T and dS^T values (fp16) go to tensor memory over the S^T and dP^T columns
//               they came from (there they are the A operands of dV += P^T dO and dK += dS^T Q), and dS^T also to
//               shared memory (the B operand of dQ^T);
//   warps 10-13 drain: one feature (TMEM lane) per thread moves dQ^T out of TMEM into a shared-memory tile that
//               one thread adds to the fp32 dQ accumulator with TMA bulk tensor reduce-add.
// The MMA thread issues S^T/dP^T of sub-tile i+1 before the products of sub-tile i, so the tensor core works while
// the compute warps do.  64-row sub-tiles keep the double-buffered S^T/dP^T (4 x 64 columns) and the dV/dK
// accumulators (2 x d columns) inside the 512 tensor-memory columns.  Per sub-tile the shared memory carries about
// 290 KB (operands of the three products with both operands there, TMA writes, dS^T, the dQ staging), which bounds
// the tensor side at 128 B/clk.
#include "internal.h"

namespace lh {

namespace {

constexpr int kThreads = 448;
constexpr int kKTile = 128;  // key rows per CTA
constexpr int kQTile = 64;   // query rows per sub-tile
constexpr int kStages = 3;   // Q/dO ring depth
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kBarCompute = 1, kBarDrain = 2;  // named barrier ids (0 is __syncthreads)
// Below this many key tiles per head the grid runs head-fastest (one head's CTAs do not fill the 148 SMs).
constexpr int kHeadFastBelow = 148;

template <int D>
struct BwdLayout {
  static constexpr uint32_t KT = kKTile * D * 2;       // K or V tile
  static constexpr uint32_t QT = kQTile * D * 2;       // Q or dO sub-tile (d-blocks of 8 KB)
  static constexpr uint32_t PT = kKTile * kQTile * 2;  // P^T or dS^T tile: 128 rows x 128 bytes (16 KB)
  static constexpr uint32_t K = 0;
  static constexpr uint32_t V = KT;
  static constexpr uint32_t Q = 2 * KT;                      // kStages
  static constexpr uint32_t DO = Q + kStages * QT;           // kStages
  static constexpr uint32_t DS = DO + kStages * QT;          // 2 buffers (dS^T, the B operand of dQ^T)
  static constexpr uint32_t DQ = DS + 2 * PT;                // staging: [d/32][64 q][32 f] fp32
  static constexpr uint32_t ST = 2 * kQTile * 4;             // one stage's statistics: [2][64] fp32
  static constexpr uint32_t STAT = DQ + kQTile * D * 4;      // kStages x {-LSE log2 e, -D/sqrt(d)} of the sub-tile
  static constexpr uint32_t BAR = STAT + kStages * ST;
  static constexpr uint32_t B_KV = 0, B_QF = 1, B_QE = 1 + kStages, B_SF = 1 + 2 * kStages, B_DSF = B_SF + 2,
                            B_MM = B_DSF + 2, B_DQF = B_MM + 2, B_FIN = B_DQF + 2, B_DRAIN = B_FIN + 1,
                            NBAR = B_DRAIN + 1;
  static constexpr uint32_t BYTES = BAR + NBAR * 8;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const __grid_constant__ CUtensorMap tmDQ, const __grid_constant__ CUtensorMap tmST,
                    const float* __restrict__ dinv, float* __restrict__ dkg,
                    float* __restrict__ dvg, uint64_t dkv_block_stride, int S, int q_off, int kv_tpb, int head_fast,
                    float scale, int* status) {
  using Lay = BwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ WaitCtl s_wait;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](uint32_t i) { return sb + Lay::BAR + 8u * i; };

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // key tiles are numbered globally (tile kt is tile kt % kv_tpb of block kt / kv_tpb); the S local query rows are
  // global rows q_off .. q_off + S - 1 (q_off = 0 without context parallelism, else a multiple of 128)
  // key tile: tile 0 meets the most query sub-tiles and is scheduled first; with head_fast the head is the grid's
  // fastest index (short sequences: every head's heavy tiles start in the first wave)
  const int kt = head_fast ? blockIdx.y : blockIdx.x;
  const int bh = head_fast ? blockIdx.x : blockIdx.y;
  const int kblk = kt / kv_tpb, krow0 = (kt % kv_tpb) * kKTile;  // block of the key tile and its first row there
  const int nq = (S + kQTile - 1) / kQTile;
  const int i0 = max(0, 2 * kt - q_off / kQTile);  // first local sub-tile with a query at or after the tile's first key
  const int nit = nq - i0;
  const float scale_log2 = scale * kLog2e;
  const float inv_scale = dinv[bh];

  if (threadIdx.x == 0) {
    wait_ctl_init(&s_wait, status);
    mbar_init(bar(Lay::B_KV), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(Lay::B_QF + s), 1);
      mbar_init(bar(Lay::B_QE + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(Lay::B_SF + b), 1);
      mbar_init(bar(Lay::B_DSF + b), 256);
      mbar_init(bar(Lay::B_MM + b), 1);
      mbar_init(bar(Lay::B_DQF + b), 128);
    }
    mbar_init(bar(Lay::B_FIN), 1);
    mbar_init(bar(Lay::B_DRAIN), 1);
    fence_mbar_init();
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmDO);
    prefetch_tmap(&tmDQ);
    prefetch_tmap(&tmST);
  }
  if (warp == 1) tmem_alloc(smem_u32(&s_tmem), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  // columns: S^T buffer b at 128 b, dP^T buffer b at 128 b + 64; dV at 256; dK at 256 + D
  const uint32_t tDV = tmem + 256, tDK = tmem + 256 + D;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      bool ok = true;
      int issued = 0;
      mbar_arrive_expect_tx(bar(Lay::B_KV), 2 * Lay::KT);
      for (int db = 0; db < D / 64; ++db) {
        tma_load_4d(sb + Lay::K + db * 16384, &tmK, bar(Lay::B_KV), db * 64, krow0, bh, kblk);
        tma_load_4d(sb + Lay::V + db * 16384, &tmV, bar(Lay::B_KV), db * 64, krow0, bh, kblk);
      }
      for (int it = 0; it < nit && ok; ++it) {
        const int s = it % kStages;
        if (it >= kStages) ok = mbar_wait(bar(Lay::B_QE + s), ((it / kStages) - 1) & 1, &s_wait, status);
        if (!ok) break;
        const int row = (i0 + it) * kQTile;
        mbar_arrive_expect_tx(bar(Lay::B_QF + s), 2 * Lay::QT + Lay::ST);
        for (int db = 0; db < D / 64; ++db) {
          tma_load_3d(sb + Lay::Q + s * Lay::QT + db * 8192, &tmQ, bar(Lay::B_QF + s), db * 64, row, bh);
          tma_load_3d(sb + Lay::DO + s * Lay::QT + db * 8192, &tmDO, bar(Lay::B_QF + s), db * 64, row, bh);
        }
        tma_load_3d(sb + Lay::STAT + s * Lay::ST, &tmST, bar(Lay::B_QF + s), row, bh, 0);  // both planes
        issued = it + 1;
      }
      if (!ok) {
        mbar_wait_teardown(bar(Lay::B_KV), 0);
        for (int it = issued >= kStages ? issued - kStages : 0; it < issued; ++it)
          mbar_wait_teardown(bar(Lay::B_QF + it % kStages), (it / kStages) & 1);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_f32acc(kFmtF16, 128, kQTile, 0, 0);   // K-major x K-major
      constexpr uint32_t idesc_acc = idesc_f32acc(kFmtF16, 128, D, 0, 1);      // K-major x MN-major
      constexpr uint32_t idesc_dq = idesc_f32acc(kFmtF16, 128, kQTile, 1, 1);  // MN-major x MN-major
      bool ok = mbar_wait(bar(Lay::B_KV), 0, &s_wait, status);
      auto products = [&](int jt) {  // dV, dK, dQ^T of sub-tile jt
        const int b = jt & 1, s = jt % kStages;
        if (!mbar_wait(bar(Lay::B_DSF + b), (jt >> 1) & 1, &s_wait, status)) return false;
        tc_fence_after();
        const uint32_t sDS = sb + Lay::DS + b * Lay::PT;
        const uint32_t sQ = sb + Lay::Q + s * Lay::QT, sDO = sb + Lay::DO + s * Lay::QT;
        // P^T and dS^T (fp16 pairs) sit over the first 32 columns of the S^T and dP^T buffers
        const uint32_t tP = tmem + 128 * b, tDS = tmem + 128 * b + 64;
#pragma unroll
        for (int kk = 0; kk < kQTile / 16; ++kk) {  // reduction over the 64 queries
          const uint32_t acc = (jt > 0 || kk > 0) ? 1u : 0u;
          const uint32_t pc = (kk >> 1) * 32 + (kk & 1) * 8;  // column half h = kk/2 packed at 32 h
          umma_ts(tDV, tP + pc, sdesc_sw128(sDO + kk * 2048, 8192, 1024), idesc_acc, acc);
          umma_ts(tDK, tDS + pc, sdesc_sw128(sQ + kk * 2048, 8192, 1024), idesc_acc, acc);
        }
#pragma unroll
        for (int kk = 0; kk < kKTile / 16; ++kk)  // reduction over the 128 keys
          umma_ss(tmem + 128 * b, sdesc_sw128(sb + Lay::K + kk * 2048, 16384, 1024),
                  sdesc_sw128(sDS + kk * 2048, 8192, 1024), idesc_dq, kk > 0 ? 1u : 0u);
        umma_commit(bar(Lay::B_MM + b));
        umma_commit(bar(Lay::B_QE + s));
        return true;
      };
      for (int it = 0; it < nit && ok; ++it) {
        const int b = it & 1, s = it % kStages;
        ok = mbar_wait(bar(Lay::B_QF + s), (it / kStages) & 1, &s_wait, status);
        // buffer pair b: its dQ^T of sub-tile it-2 has been read out of tensor memory
        if (ok && it >= 2) ok = mbar_wait(bar(Lay::B_DQF + b), ((it >> 1) - 1) & 1, &s_wait, status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t sQ = sb + Lay::Q + s * Lay::QT, sDO = sb + Lay::DO + s * Lay::QT;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ko = (kk >> 2) * 16384 + (kk & 3) * 32, qo = (kk >> 2) * 8192 + (kk & 3) * 32;
          umma_ss(tmem + 128 * b, sdesc_sw128(sb + Lay::K + ko, 16, 1024), sdesc_sw128(sQ + qo, 16, 1024), idesc_s,
                  kk > 0 ? 1u : 0u);
          umma_ss(tmem + 128 * b + 64, sdesc_sw128(sb + Lay::V + ko, 16, 1024), sdesc_sw128(sDO + qo, 16, 1024),
                  idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar(Lay::B_SF + b));
        if (it >= 1) ok = products(it - 1);
      }
      if (ok && nit >= 1) ok = products(nit - 1);
      umma_commit(bar(Lay::B_FIN));  // dV, dK final once every product above has completed
      umma_commit(bar(Lay::B_DRAIN));
      mbar_wait_teardown(bar(Lay::B_DRAIN), 0);
    }
  } else if (warp < 10) {
    // ---------------------------------------------------------------- compute: P^T and dS^T, one key row per
    // thread, 32 query columns (half hc of the sub-tile) per warp
    const int quarter = warp & 3;
    const int hc = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;  // key row inside the tile = TMEM lane
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int key = kt * kKTile + r;  // global key row
    bool ok = true;
    const uint64_t scl2 = f2pack(scale_log2, scale_log2), sc2 = f2pack(scale, scale);
    for (int it = 0; it < nit && ok; ++it) {
      const int b = it & 1, s = it % kStages, i = i0 + it;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(Lay::B_SF + b), (it >> 1) & 1, &s_wait, status));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(Lay::B_QF + s), (it / kStages) & 1, &s_wait, status));
      if (!ok) break;
      float sv[32], dp[32];
      tc_fence_after();
      tmem_ld32(tmem + 128 * b + lane_base + 32 * hc, sv);
      tmem_ld32(tmem + 128 * b + 64 + lane_base + 32 * hc, dp);
      tmem_ld_wait();
      uint32_t pk[16], dk[16];
      {
        const int qg0 = q_off + i * kQTile + 32 * hc;  // global row of this half's first query
        const bool diag = qg0 < key;
        __half2 hm[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) hm[k] = __float2half2_rn(0.f);
        const ulonglong2* nl4 = reinterpret_cast<const ulonglong2*>(smem + Lay::STAT + s * Lay::ST) + 8 * hc;
        const ulonglong2* nd4 = reinterpret_cast<const ulonglong2*>(smem + Lay::STAT + s * Lay::ST + kQTile * 4) + 8 * hc;
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          const ulonglong2 nl = nl4[c >> 2], nd = nd4[c >> 2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int cc = c + 2 * h;
            const uint64_t arg = fma_f32x2(f2pack(sv[cc], sv[cc + 1]), scl2, h ? nl.y : nl.x);
            float p0 = ex2(f2lo(arg)), p1 = ex2(f2hi(arg));
            if (diag) {
              if (qg0 + cc < key) p0 = 0.f;
              if (qg0 + cc + 1 < key) p1 = 0.f;
            }
            const uint64_t p2 = f2pack(p0, p1);
            const uint64_t d2 = mul_f32x2(p2, fma_f32x2(f2pack(dp[cc], dp[cc + 1]), sc2, h ? nd.y : nd.x));
            pk[cc / 2] = pack_half2_rn(p0, p1);
            dk[cc / 2] = pack_half2_rn(f2lo(d2), f2hi(d2));
            const __half2 hv = *reinterpret_cast<const __half2*>(&dk[cc / 2]);
            hm[(cc / 2) & 3] = __hmax2_nan(hm[(cc / 2) & 3], __habs2(hv));
          }
        }
        const __half2 h01 = __hmax2_nan(hm[0], hm[1]), h23 = __hmax2_nan(hm[2], hm[3]);
        const float2 mf = __half22float2(__hmax2_nan(h01, h23));
        if (__any_sync(0xffffffffu, !(mf.x <= 65504.f && mf.y <= 65504.f)) && lane == 0)
          set_status(status, LH_ERR_RANGE);
        if (it >= 2) ok = __all_sync(0xffffffffu, mbar_wait(bar(Lay::B_MM + b), ((it >> 1) - 1) & 1, &s_wait,
                                                            status));
      }
      if (ok) {
        tmem_st16(tmem + 128 * b + lane_base + 32 * hc, pk);
        tmem_st16(tmem + 128 * b + 64 + lane_base + 32 * hc, dk);
        uint8_t* sDS = smem + Lay::DS + b * Lay::PT;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {  // 16-byte chunk 4 hc + ch holds queries 8 (4 hc + ch) .. + 7
          const uint32_t off = sw128_offset(r, 4 * hc + ch);
          *reinterpret_cast<uint4*>(sDS + off) = make_uint4(dk[4 * ch], dk[4 * ch + 1], dk[4 * ch + 2], dk[4 * ch + 3]);
        }
        fence_proxy_async_smem();
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar(Lay::B_DSF + b));
      }
    }
    // epilogue: dV (column half 0's warps) or dK (half 1's) rows of this key tile, final after B_FIN
    ok = named_barrier_and(kBarCompute, 256, ok);
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(Lay::B_FIN), 0, &s_wait, status));
    if (ok) {
      tc_fence_after();
      const uint32_t tacc = hc == 0 ? tDV : tDK;
      float* dst_base = hc == 0 ? dvg : dkg;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float v[32];
        tmem_ld32(tacc + lane_base + c * 32, v);
        tmem_ld_wait();
        if (krow0 + r < S) {
          float4* dst = reinterpret_cast<float4*>(dst_base + kblk * dkv_block_stride +
                                                  ((int64_t)bh * S + krow0 + r) * D + c * 32);
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)
            dst[q4] = make_float4(v[q4 * 4 + 0] * inv_scale, v[q4 * 4 + 1] * inv_scale, v[q4 * 4 + 2] * inv_scale,
                                  v[q4 * 4 + 3] * inv_scale);
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- drain: dQ^T -> shared tile -> TMA reduce-add
    const int quarter = warp & 3;
    const int f = quarter * 32 + lane;  // feature = TMEM lane of dQ^T
    const int dt = threadIdx.x - 320;   // 0..127 inside the drain group
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    float* stage = reinterpret_cast<float*>(smem + Lay::DQ);
    bool ok = true;
    for (int it = 0; it < nit; ++it) {
      const int b = it & 1, i = i0 + it;
      ok = __all_sync(0xffffffffu, ok && mbar_wait(bar(Lay::B_MM + b), (it >> 1) & 1, &s_wait, status));
      float v[64];
      if (ok) {
        tc_fence_after();
        tmem_ld32(tmem + 128 * b + lane_base, *reinterpret_cast<float(*)[32]>(&v[0]));
        tmem_ld32(tmem + 128 * b + lane_base + 32, *reinterpret_cast<float(*)[32]>(&v[32]));
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(bar(Lay::B_DQF + b));  // TMEM pair b may take the next S^T
      }
      // the previous reduce must have finished reading the staging tile before it is overwritten
      if (dt == 0) bulk_wait_group_read0();
      ok = named_barrier_and(kBarDrain, 128, ok);
      if (!ok) break;
      if (f < D) {
        float* col = stage + (f >> 5) * (kQTile * 32) + (f & 31);  // box (f/32): [64 q][32 f]
#pragma unroll
        for (int c = 0; c < kQTile; ++c) col[c * 32] = v[c] * inv_scale;
      }
      fence_proxy_async_smem();
      named_barrier_and(kBarDrain, 128, true);
      if (dt == 0) {
        for (int fb = 0; fb < D / 32; ++fb)
          tma_reduce_add_3d(&tmDQ, smem_u32(stage + fb * kQTile * 32), fb * 32, i * kQTile, bh);
        bulk_commit_group();
      }
    }
    if (dt == 0) bulk_wait_group0();  // every reduction has landed before the block exits
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D>
int launch_bwd_t(const void* qg, const KvSource& kv, const void* dog16, const float* stats, const float* dinv,
                 float* dqacc, float* dkg, float* dvg, uint64_t dkv_block_stride, const LhDims& dm, cudaStream_t st) {
  if (kv.q_off % kKTile != 0 || (kv.blocks > 1 && dm.S % kKTile != 0)) return LH_ERR_UNSUPPORTED;
  CUtensorMap mq, mk, mv, mdo, mdq, mst;
  if (make_tmap_f16_3d(&mq, qg, D, dm.S, dm.BH, kQTile) ||
      make_tmap_f16_4d(&mk, kv.k, D, dm.S, dm.BH, kv.blocks, kv.block_stride, kKTile) ||
      make_tmap_f16_4d(&mv, kv.v, D, dm.S, dm.BH, kv.blocks, kv.block_stride, kKTile) ||
      make_tmap_f16_3d(&mdo, dog16, D, dm.S, dm.BH, kQTile) ||
      make_tmap_f32_3d(&mdq, dqacc, D, dm.S, dm.BH, 32, kQTile) || make_tmap_stats(&mst, stats, dm.S, dm.BH, kQTile))
    return LH_ERR_CUDA;
  const int smem = BwdLayout<D>::BYTES + 1024;
  if (cudaFuncSetAttribute(attn_bwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return LH_ERR_CUDA;
  const int tpb = (dm.S + kKTile - 1) / kKTile;            // key tiles per block
  const int nt = (kv.q_off + dm.S + kKTile - 1) / kKTile;  // key tiles the local queries see
  KernelTimer timer("attn_bwd", st);
  const int head_fast = nt < kHeadFastBelow;
  const dim3 grid = head_fast ? dim3(dm.BH, nt) : dim3(nt, dm.BH);
  attn_bwd_kernel<D><<<grid, kThreads, smem, st>>>(mq, mk, mv, mdo, mdq, mst, dinv, dkg, dvg, dkv_block_stride, dm.S,
                                                   kv.q_off, tpb, head_fast, 1.0f / sqrtf((float)D), dm.status);
  return check_launch();
}

}  // namespace

int launch_attn_bwd(const void* qg, const KvSource& kv, const void* dog16, const float* stats, const float* dinv,
                    float* dqacc, float* dkg, float* dvg, uint64_t dkv_block_stride, const LhDims& dm, cudaStream_t st) {
  return dm.d == 64 ? launch_bwd_t<64>(qg, kv, dog16, stats, dinv, dqacc, dkg, dvg, dkv_block_stride, dm, st)
                    : launch_bwd_t<128>(qg, kv, dog16, stats, dinv, dqacc, dkg, dvg, dkv_block_stride, dm, st);
}

}  // namespace lh
