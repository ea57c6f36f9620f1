// lh_common.cuh — device-side helpers shared by the Lighthouse kernels (sm_100a only).
//
// Contents: the per-call size table (LhDims), bf16/fp64 conversions with the rounding the layer fixes,
// the device status word and bounded waits, and thin inline-PTX wrappers for mbarriers, TMA, and the
// fifth-generation tensor core (tcgen05 + tensor memory).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/lh.h"

namespace lh {

// Largest level count the kernels are built for (the entry points reject more); loops over levels unroll to it.
constexpr int kMaxL = 5;

// ------------------------------------------------------------------------------------------------------------
// Sizes of one call, computed on the host and passed by value.
// ------------------------------------------------------------------------------------------------------------
struct LhDims {
  int B, H, N, d, L, p, k, C;
  int BH;
  int S;
  int R;       // slot rows per head: sum_l N_l
  int Rs;      // score rows per head: sum of N_l over the scored levels
  int Rp;      // pyramid rows per head: sum_{l>=1} N_l
  int Ksel;    // selection-list rows per head: sum over partially selected levels of kl
  int nPartial;  // levels 0..nPartial-1 are partially selected; the rest are kept whole
  int expand;    // children-expansion variant (LH_EXPAND_CHILDREN): level l keeps the children of level l+1's picks
  unsigned score_mask;  // bit l set: level l is scored (0..L-2, or 1..L-1 with expand)
  int Nl[LH_MAX_LEVELS];     // entries of level l
  int wl[LH_MAX_LEVELS];     // tokens per entry of level l
  int wlog[LH_MAX_LEVELS];   // log2(wl[l]) (windows are powers of two for every supported p)
  int off[LH_MAX_LEVELS];    // global pyramid id (= slot row) of entry (l, 0)
  int poff[LH_MAX_LEVELS];   // row of level l (>= 1) inside the per-head pyramid of lh_pool
  int kl[LH_MAX_LEVELS];     // selected entries of level l
  int soff[LH_MAX_LEVELS];   // row of scored level l inside the per-head score array
  int seloff[LH_MAX_LEVELS]; // row of level l inside the per-head selection list (partial levels only)
  int* status;               // device status word of the current device (first error wins)
};

// ------------------------------------------------------------------------------------------------------------
// Device status word (first error wins) and the bound on every device-side wait.
// ------------------------------------------------------------------------------------------------------------
__device__ __forceinline__ void set_status(int* status, int code) { atomicCAS(status, 0, code); }

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bound of the waits taken while tearing down after an abort (they wait for the block's own copies and products,
// which always complete).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// The device status word is the first member of this per-device record; the kernels receive a pointer to it.  The
// record also holds the bound on every ordinary device-side wait (lh_set_wait_limit_ns; 2 s by default).
struct LhDeviceState {
  int status;
  int pad;
  unsigned long long wait_limit_ns;
};
__device__ __forceinline__ uint64_t wait_limit_ns(const int* status) {
  return reinterpret_cast<const volatile LhDeviceState*>(status)->wait_limit_ns;
}

// ------------------------------------------------------------------------------------------------------------
// Number formats.
// ------------------------------------------------------------------------------------------------------------
__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b16) { return __uint_as_float(b16 << 16); }

// Unpack 8 bf16 values held in a 16-byte vector to fp32 (exact).
__device__ __forceinline__ void unpack8(const uint4& r, float (&f)[8]) {
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// 8 bf16 values -> 8 fp16 values.  Exact for every bf16 value of magnitude in [2^-14, 65504]; smaller ones are
// rounded to fp16 subnormals, larger ones become infinities and set *overflow.
__device__ __forceinline__ uint4 bf16x8_to_f16x8(const uint4& r, bool& overflow) {
  float f[8];
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __half2 h = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
    o[i] = *reinterpret_cast<uint32_t*>(&h);
    overflow |= fabsf(f[2 * i]) > 65504.f || fabsf(f[2 * i + 1]) > 65504.f;
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// fp32 <-> fp64 conversions that keep subnormal values whatever the compiler's flush-to-zero setting (the library
// is built with fast math, which would otherwise flush them in C++ conversions).
__device__ __forceinline__ double f64_of(float x) {
  double r;
  asm("cvt.f64.f32 %0, %1;" : "=d"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float f32_rn_of(double x) {
  float r;
  asm("cvt.rn.f32.f64 %0, %1;" : "=f"(r) : "d"(x));
  return r;
}
__device__ __forceinline__ float f32_rz_of(double x) {
  float r;
  asm("cvt.rz.f32.f64 %0, %1;" : "=f"(r) : "d"(x));
  return r;
}

// fp64 -> bf16 with a single round-to-nearest-even.  Method: round to fp32 toward zero, then make the result
// "round to odd" by forcing its last bit when the conversion was inexact, then round that fp32 value to bf16
// to nearest-even.  fp32 carries more than two extra bits over bf16, so the two steps equal one direct
// rounding (Boldo & Melquiond, "Emulation of FMA and correctly rounded sums: proved algorithms using rounding
// to odd", IEEE Trans. Computers 2008).  The last step is done on the bits (the bf16 conversion instruction
// is not relied on for fp32 subnormals).
__device__ __forceinline__ uint32_t f64_to_bf16_bits_rne(double x) {
  uint32_t b = __float_as_uint(f32_rz_of(x));
  if (f64_of(__uint_as_float(b)) != x) b |= 1u;
  if ((b & 0x7F800000u) == 0x7F800000u) return (b >> 16) | ((b & 0xFFFFu) ? 0x40u : 0u);  // inf stays, NaN quiet
  return (b + 0x7FFFu + ((b >> 16) & 1u)) >> 16;  // round to nearest, ties to even, on the bits
}

// ------------------------------------------------------------------------------------------------------------
// Vector memory access.
// ------------------------------------------------------------------------------------------------------------
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}
__device__ __forceinline__ uint4 ld16(const void* p) { return *reinterpret_cast<const uint4*>(p); }
__device__ __forceinline__ void st16(void* p, const uint4& v) { *reinterpret_cast<uint4*>(p) = v; }
__device__ __forceinline__ void st_stream16(void* p, const uint4& v) {
  asm volatile("st.global.L1::no_allocate.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

// ------------------------------------------------------------------------------------------------------------
// Shared memory, mbarriers and TMA.
// ------------------------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte asynchronous global -> shared copy (L2 only); copies are grouped per thread by commit, and a wait
// returns once at most N of this thread's most recent groups are still pending.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of the completion of phase `parity`.
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Per-block wait control in shared memory: the abort flag (set by the first wait that gives up, so that every
// other wait of the block returns at once) and the wait limit, read once from the device record at block start.
struct WaitCtl {
  int abort;
  int pad;
  unsigned long long limit_ns;
};
__device__ __forceinline__ void wait_ctl_init(WaitCtl* w, const int* status) {
  w->abort = 0;
  w->limit_ns = wait_limit_ns(status);
}

// Wait for phase `parity` of an mbarrier.  Returns false (and records LH_ERR_TIMEOUT) once the wait has lasted
// longer than the block's wait limit, or immediately once the block's abort flag is set.  The elapsed time is checked
// before each blocking try, so a limit of 1 ns makes every wait that finds its phase incomplete give up at once.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile WaitCtl* w, int* status) {
  if (mbar_test_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (w->abort) return false;
    const uint64_t limit = w->limit_ns;
    if (limit <= 1 || globaltimer_ns() - t0 > limit) {
      set_status(status, LH_ERR_TIMEOUT);
      w->abort = 1;
      return false;
    }
    if (mbar_try_wait(bar, parity)) return true;
  }
}

// Bounded wait used while tearing down after an abort: ignores the abort flag.
__device__ __forceinline__ bool mbar_wait_teardown(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 3-D tiled TMA load (no multicast) into shared memory, completion counted on `bar`.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
      "[%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// 4-D tiled TMA load (no multicast) into shared memory, completion counted on `bar`.
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1,
                                            int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], "
      "[%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// 3-D tiled TMA reduce-add (fp32) of a shared-memory box into global memory; completion tracked by bulk groups.
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* map, uint32_t src, int c0, int c1, int c2) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until the shared-memory sources of all committed bulk groups have been read.
__device__ __forceinline__ void bulk_wait_group_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until all committed bulk groups have completed.
__device__ __forceinline__ void bulk_wait_group0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Named barrier over `count` threads (a multiple of 32) that also returns the AND of `pred` over them.
__device__ __forceinline__ bool named_barrier_and(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------------------------------------------------------------
// tcgen05: tensor memory and the fifth-generation MMA (cta_group::1 throughout).
// ------------------------------------------------------------------------------------------------------------

// Allocate `ncols` TMEM columns (power of two >= 32); the base address is written to shared memory at `dst`.
// Must be executed by one whole warp.
__device__ __forceinline__ void tmem_alloc(uint32_t dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, 16-bit inputs (fp16 or bf16, per the instruction descriptor), fp32
// accumulation; issued by one thread.
__device__ __forceinline__ void umma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]: the M x K A operand (16-bit) is read from tensor memory, lane i holding row i
// with its K elements packed two per 32-bit column (lower half first); B comes from a shared-memory descriptor.
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when all tcgen05.mma previously issued by this thread have completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// Instruction descriptor for kind::f16 with fp32 D (bit layout of the sm_100 UMMA instruction descriptor: D format
// [4,6), A format [7,10), B format [10,13), A major bit 15, B major bit 16, N>>3 at [17,23), M>>4 at [24,29)).
// fmt: 0 = fp16, 1 = bf16 (A and B always share it).  major: 0 = K-major, 1 = MN-major.
__host__ __device__ constexpr uint32_t idesc_f32acc(int fmt, int M, int N, int a_mn, int b_mn) {
  return (1u << 4) | ((uint32_t)fmt << 7) | ((uint32_t)fmt << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
constexpr int kFmtF16 = 0;
constexpr int kFmtBF16 = 1;

__device__ __forceinline__ uint32_t pack_half2_rn(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 layout: start address >> 4 at [0,14), leading
// byte offset >> 4 at [16,30), stride byte offset >> 4 at [32,46), version 1 at [46,48), layout type
// SWIZZLE_128B = 2 at [61,64)).  All swizzle atoms (8 rows x 128 bytes) must be 1024-byte aligned.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}

// 32 lanes x 32 columns of 32-bit TMEM words: thread i of the warp receives lane (base lane + i), columns
// [col, col + 32).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,"
      "%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}
// 32 lanes x 16 columns store (thread i of the warp writes lane base + i, columns [col, col + 16)).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Packed pairs of fp32 values (low word = first value), the operands of the sm_100a f32x2 instructions.
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
  return ((uint64_t)__float_as_uint(hi) << 32) | (uint64_t)__float_as_uint(lo);
}
__device__ __forceinline__ float f2lo(uint64_t v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float f2hi(uint64_t v) { return __uint_as_float((uint32_t)(v >> 32)); }
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
// Largest of three values (the three-input max.f32 of sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Hardware base-2 exponential (MUFU), flush-to-zero.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` inside a 128-byte-swizzled tile whose rows are
// 128 bytes long (8-row, 1024-byte swizzle atoms): chunk index XOR (row mod 8).
__device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t chunk) {
  return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

}  // namespace lh
