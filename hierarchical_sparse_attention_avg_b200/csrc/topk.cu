// topk.cu — step 3 (chunked, stratified top-K per level) and the gathered order of step 4.
//
// Selection follows [W] 核心方法 §2 ("Chunked Bitonic Top-K" kernel) and [C] "Four-Stage Pipeline Wraps Standard
// FlashAttention" (per-level stratified top-K, coarsest level always kept whole): every level l <= L-2 with fewer
// picks than entries is cut into C equal contiguous chunks, and each chunk keeps its k/C entries of largest
// score, ties to the lower index.  In the children-expansion variant (the reading that reproduces the size example
// of [E] "Какво точно промени Nous Research в attention пътя?") the chunks and scores are those of level l+1, and
// level l keeps the p children of every pick.
//
// Keys: the score's fp32 bit pattern is mapped to an unsigned integer that orders like the value (negative numbers:
// all bits flipped; others: sign bit set; -0 is first made +0, so that the two zeros tie); key = (ordered score
// << 32) | (0xFFFFFFFF - index) is unique, and a larger key means a higher score or, on equal scores, a lower
// index.  Sentinel key 0 is below every real key (the index part of a real key is never 0).
//
// One CTA (8 warps) per (head, level, chunk).  Each warp keeps a running top-M (M = picks rounded up to a power
// of two) of its share of the chunk in registers, M/32 keys per lane, sorted descending.  Keys of the warp's
// blocks that exceed the running M-th largest key are compacted (ballot) into a per-warp shared-memory buffer;
// a key at or below it can never enter the warp's top M, since M larger-or-equal keys are already held and keys
// are unique.  When the next block's candidates would overflow the buffer, and at the end, the buffer is
// bitonic-sorted ascending (register compare-exchange for partners in the same lane, warp shuffles otherwise);
// the element-wise maximum of the descending running list and the ascending buffer is a bitonic sequence that
// holds the top M of both, which one bitonic merge sorts descending again.  The eight warp lists are merged the
// same way through shared memory.
#include "internal.h"

namespace lh {

namespace {

__device__ __forceinline__ uint64_t make_key(float score, uint32_t index) {
  uint32_t u = __float_as_uint(score);
  if (u == 0x80000000u) u = 0u;  // -0 ties with +0
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((uint64_t)u << 32) | (uint64_t)(0xFFFFFFFFu - index);
}
__device__ __forceinline__ uint32_t key_index(uint64_t key) { return 0xFFFFFFFFu - (uint32_t)key; }

__device__ __forceinline__ uint64_t shfl_xor64(uint64_t v, int mask) {
  uint32_t lo = (uint32_t)v, hi = (uint32_t)(v >> 32);
  lo = __shfl_xor_sync(0xffffffffu, lo, mask);
  hi = __shfl_xor_sync(0xffffffffu, hi, mask);
  return ((uint64_t)hi << 32) | lo;
}

__device__ __forceinline__ uint64_t shfl_idx64(uint64_t v, int src) {
  uint32_t lo = (uint32_t)v, hi = (uint32_t)(v >> 32);
  lo = __shfl_sync(0xffffffffu, lo, src);
  hi = __shfl_sync(0xffffffffu, hi, src);
  return ((uint64_t)hi << 32) | lo;
}

// Compare-exchange stage of a bitonic network over M = 32*R keys, element e = lane*R + r.  Pair (e, e^J), e the
// lower element; when `up` the lower element receives the minimum.
template <int R, int J>
__device__ __forceinline__ void cx_stage(uint64_t (&key)[R], int lane, int K /* 0 = all descending */) {
  if constexpr (J >= R) {
    constexpr int LJ = J / R;
    const bool lower = (lane & LJ) == 0;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int e = lane * R + r;
      const bool up = K ? ((e & K) == 0) : false;
      const uint64_t other = shfl_xor64(key[r], LJ);
      const bool take_min = (lower == up);
      const uint64_t mn = key[r] < other ? key[r] : other;
      const uint64_t mx = key[r] < other ? other : key[r];
      key[r] = take_min ? mn : mx;
    }
  } else {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if ((r & J) == 0) {
        const int e = lane * R + r;
        const bool up = K ? ((e & K) == 0) : false;
        const uint64_t a = key[r], b = key[r | J];
        const uint64_t mn = a < b ? a : b, mx = a < b ? b : a;
        key[r] = up ? mn : mx;
        key[r | J] = up ? mx : mn;
      }
    }
  }
}

template <int R, int K, int J>
__device__ __forceinline__ void sort_stages(uint64_t (&key)[R], int lane) {
  cx_stage<R, J>(key, lane, K);
  if constexpr (J > 1) sort_stages<R, K, J / 2>(key, lane);
}

// Bitonic sort ascending of the warp's M = 32*R keys.
template <int R, int K>
__device__ __forceinline__ void bitonic_sort_asc(uint64_t (&key)[R], int lane) {
  sort_stages<R, K, K / 2>(key, lane);
  if constexpr (K < 32 * R) bitonic_sort_asc<R, K * 2>(key, lane);
}

template <int R, int J>
__device__ __forceinline__ void merge_desc(uint64_t (&key)[R], int lane) {
  cx_stage<R, J>(key, lane, 0);
  if constexpr (J > 1) merge_desc<R, J / 2>(key, lane);
}

template <int M>
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ scores, int32_t* __restrict__ sel,
                                                   int32_t* __restrict__ slot, LhDims dm) {
  constexpr int R = M / 32;
  __shared__ uint64_t s_top[8][M];
  __shared__ uint32_t s_idx[M];

  // lev: the level whose selection list this block writes; rlev: the level whose entries it ranks (lev itself, or
  // its parent level in the children-expansion variant, where each pick brings its p children at level lev)
  const int c = blockIdx.x, lev = blockIdx.y, bh = blockIdx.z;
  const int rlev = lev + dm.expand;
  const int nc = dm.Nl[rlev] / dm.C;
  const int m = dm.k / dm.C;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const float* sc = scores + (int64_t)bh * dm.Rs + dm.soff[rlev] + (int64_t)c * nc;
  const int nslot = dm.Nl[lev] / dm.C;  // entries of level lev in this chunk
  int32_t* sl = slot + (int64_t)bh * dm.R + dm.off[lev] + (int64_t)c * nslot;

  for (int i = threadIdx.x; i < nslot; i += 256) sl[i] = -1;  // positions of the picks are written later

  uint64_t top[R];
#pragma unroll
  for (int r = 0; r < R; ++r) top[r] = 0;
  uint64_t thr = 0;  // the running M-th largest key (0: fewer than M keys so far)
  uint64_t* buf = s_top[warp];  // candidate buffer (the warp's merge slot is free until the end)
  int cnt = 0;                  // keys in the buffer (warp-uniform)
  auto flush = [&]() {          // fold the buffer into the running list
    __syncwarp();
    uint64_t key[R];
#pragma unroll
    for (int r = 0; r < R; ++r) key[r] = lane * R + r < cnt ? buf[lane * R + r] : 0ull;
    __syncwarp();
    bitonic_sort_asc<R, 2>(key, lane);
#pragma unroll
    for (int r = 0; r < R; ++r) key[r] = top[r] > key[r] ? top[r] : key[r];
    merge_desc<R, M / 2>(key, lane);
#pragma unroll
    for (int r = 0; r < R; ++r) top[r] = key[r];
    thr = shfl_idx64(top[R - 1], 31);
    cnt = 0;
  };
  const unsigned lt = (1u << lane) - 1u;  // lanes below this one
  const int nblocks = (nc + M - 1) / M;
  for (int b = warp; b < nblocks; b += 8) {
    uint64_t key[R];
    int nb = 0;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int e = b * M + r * 32 + lane;  // coalesced: element r*32 + lane of the block
      key[r] = e < nc ? make_key(sc[e], (uint32_t)(c * nc + e)) : 0ull;
      nb += __popc(__ballot_sync(0xffffffffu, key[r] > thr));
    }
    if (cnt + nb > M) flush();
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const bool keep = key[r] > thr;
      const unsigned vote = __ballot_sync(0xffffffffu, keep);
      if (keep) buf[cnt + __popc(vote & lt)] = key[r];
      cnt += __popc(vote);
    }
  }
  if (cnt > 0) flush();
  __syncwarp();
#pragma unroll
  for (int r = 0; r < R; ++r) s_top[warp][lane * R + r] = top[r];
  __syncthreads();
  if (warp == 0) {
    for (int w = 1; w < 8; ++w) {
      uint64_t key[R];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const uint64_t other = s_top[w][M - 1 - (lane * R + r)];  // reversed: ascending
        key[r] = top[r] > other ? top[r] : other;
      }
      merge_desc<R, M / 2>(key, lane);
#pragma unroll
      for (int r = 0; r < R; ++r) top[r] = key[r];
    }
#pragma unroll
    for (int r = 0; r < R; ++r) s_idx[lane * R + r] = key_index(top[r]);
  }
  __syncthreads();
  // the first m keys are the picks; emit their indices in ascending order (rank = number of smaller indices), or,
  // in the children-expansion variant, the p children of each pick (consecutive, so the list stays ascending)
  const int fan = dm.expand ? dm.p : 1;
  for (int i = threadIdx.x; i < m; i += 256) {
    const uint32_t me = s_idx[i];
    int rank = 0;
    for (int q = 0; q < m; ++q) rank += s_idx[q] < me;
    int32_t* dst = sel + (int64_t)bh * dm.Ksel + dm.seloff[lev] + ((int64_t)c * m + rank) * fan;
    for (int e = 0; e < fan; ++e) dst[e] = (int32_t)me * fan + e;
  }
}

// Number of entries of `list` (ascending, length n) that are <= x.
__device__ __forceinline__ int count_le(const int32_t* list, int n, int x) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (list[mid] <= x) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

// One thread per selected entry: its position in the gathered order = its rank in its own level plus, for every
// other level, the number of selected entries ordered before it (end E' < E for finer levels, E' <= E for
// coarser levels: equal ends go coarser first).
__global__ void __launch_bounds__(256) order_kernel(const int32_t* __restrict__ sel, int32_t* __restrict__ idx_g,
                                                    int32_t* __restrict__ slot, LhDims dm) {
  const int bh = blockIdx.y;
  const int u = blockIdx.x * 256 + threadIdx.x;
  if (u >= dm.S) return;
  int lev = 0, base = 0;
  while (u >= base + dm.kl[lev]) {
    base += dm.kl[lev];
    ++lev;
  }
  const int r = u - base;
  const int32_t* sel_bh = sel + (int64_t)bh * dm.Ksel;
  const int j = lev < dm.nPartial ? sel_bh[dm.seloff[lev] + r] : r;
  const int64_t E = (int64_t)(j + 1) * dm.wl[lev] - 1;
  int64_t pos = r;
  for (int l2 = 0; l2 < dm.L; ++l2) {
    if (l2 == lev) continue;
    const int coarser = l2 > lev ? 1 : 0;
    const int64_t J = (E + coarser) / dm.wl[l2] - 1;  // largest index j' of level l2 ordered before (lev, j)
    if (l2 >= dm.nPartial) pos += J + 1;
    else pos += count_le(sel_bh + dm.seloff[l2], dm.kl[l2], (int)J);
  }
  const int gid = dm.off[lev] + j;
  idx_g[(int64_t)bh * dm.S + pos] = gid;
  slot[(int64_t)bh * dm.R + gid] = (int32_t)pos;
}

}  // namespace

int launch_topk(const float* scores, int32_t* sel, int32_t* slot, const LhDims& dm, cudaStream_t st) {
  if (dm.nPartial == 0) return LH_OK;
  const int m = dm.k / dm.C;
  int M = 32;
  while (M < m) M <<= 1;
  dim3 grid(dm.C, dm.nPartial, dm.BH);
  KernelTimer timer("topk", st);
  switch (M) {
    case 32: topk_kernel<32><<<grid, 256, 0, st>>>(scores, sel, slot, dm); break;
    case 64: topk_kernel<64><<<grid, 256, 0, st>>>(scores, sel, slot, dm); break;
    case 128: topk_kernel<128><<<grid, 256, 0, st>>>(scores, sel, slot, dm); break;
    case 256: topk_kernel<256><<<grid, 256, 0, st>>>(scores, sel, slot, dm); break;
    case 512: topk_kernel<512><<<grid, 256, 0, st>>>(scores, sel, slot, dm); break;
    default: return LH_ERR_UNSUPPORTED;
  }
  return check_launch();
}

int launch_order(const int32_t* sel, int32_t* idx_g, int32_t* slot, const LhDims& dm, cudaStream_t st) {
  dim3 grid((dm.S + 255) / 256, dm.BH);
  KernelTimer timer("order", st);
  order_kernel<<<grid, 256, 0, st>>>(sel, idx_g, slot, dm);
  return check_launch();
}

}  // namespace lh
