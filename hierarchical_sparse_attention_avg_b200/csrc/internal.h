// internal.h — host-side declarations shared by the library's translation units (not part of the ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lh_common.cuh"

namespace lh {

// One pooling job: one input tensor, optional pyramid output (levels chosen by write_mask, level l written at
// row row_off[l] of a per-head block of pyr_rows rows), optional score output (levels 0..L-2).
struct PoolJob {
  const void* x;
  void* pyr;
  int pyr_rows;
  uint32_t write_mask;  // bit l set: write level l (1 <= l <= L-1)
  int row_off[LH_MAX_LEVELS];
  float* scores;        // [BH, Rs] or nullptr
};
struct PoolJobs {
  PoolJob job[3];
};

// One gather job: rows of one tensor.  Source of level l >= 1: pyr (per-head rows pyr_rows, level l at
// row_off[l]) when non-null for that level, else recomputed from x.
struct GatherJob {
  const void* x;
  const void* pyr;
  int pyr_rows;
  uint32_t pyr_mask;  // bit l set: level l is read from pyr
  int row_off[LH_MAX_LEVELS];
  void* out;          // [BH, S, d]
};
struct GatherJobs {
  GatherJob job[3];
};

int launch_pool_score(const PoolJobs& jobs, int njobs, const LhDims& dm, cudaStream_t st);
int launch_gather(const GatherJobs& jobs, int njobs, const int32_t* idx_g, const LhDims& dm, cudaStream_t st);
int launch_topk(const float* scores, int32_t* sel, int32_t* slot, const LhDims& dm, cudaStream_t st);
int launch_order(const int32_t* sel, int32_t* idx_g, int32_t* slot, const LhDims& dm, cudaStream_t st);
// og (fp32 [BH, S, d]) is the attention output at accumulator precision.
int launch_scatter(const float* og, const int32_t* slot, void* o, const LhDims& dm, cudaStream_t st);
// dog[s] = fp32 window sum of dout; with amax non-null also the per-head maximum magnitude (atomicMax on the bit
// pattern; amax must start at 0).
int launch_scatter_bwd(const void* dout, const int32_t* idx_g, float* dog, unsigned int* amax, const LhDims& dm,
                       cudaStream_t st);
// Per-head maximum magnitude of an fp32 [BH, S, d] tensor (amax must start at 0).
int launch_absmax(const float* x, unsigned int* amax, const LhDims& dm, cudaStream_t st);
// Rows per head of the attention backward's statistics planes (S rounded up to a multiple of 4, so that each row of
// the planes starts on a 16-byte boundary for the tensor map).
__host__ __device__ inline int stats_stride(const LhDims& dm) { return (dm.S + 3) & ~3; }
// dog16 = fp16(dog * scale_bh), dinv[bh] = 1/scale_bh, dqacc = 0, and the statistics the attention backward reads,
// stats fp32 [2][BH][stats_stride]: plane 0 = -LSE log2(e) (lse: natural-log LSE of the forward), plane 1 =
// -<dog16, og> / sqrt(d).
int launch_bwd_prep(const float* dog, const float* og, const float* lse, const unsigned int* amax, void* dog16,
                    float* stats, float* dinv, float* dqacc, const LhDims& dm, cudaStream_t st);
int launch_unpool_bwd(const float* dqg, const float* dkg, const float* dvg, const int32_t* slot, void* dq, void* dk,
                      void* dv, const LhDims& dm, cudaStream_t st);
// Keys and values of the attention: `blocks` blocks of dm.S rows each (one per rank of a context-parallel group;
// a single block otherwise), block g of K at k + g * block_stride bytes (V likewise), each fp16 [BH, S, d].  The
// queries (dm.S local rows) have global rows q_off .. q_off + S - 1 (q_off a multiple of 128; 0 without context
// parallelism) and see every key of global row <= their own, i.e. the first q_off + S keys.
struct KvSource {
  const void* k;
  const void* v;
  int blocks;
  uint64_t block_stride;
  int q_off;
};
inline KvSource kv_plain(const void* k, const void* v) { return KvSource{k, v, 1, 0, 0}; }

int launch_attn_fwd(const void* qg, const KvSource& kv, float* og, float* lse, const LhDims& dm, cudaStream_t st);
// qg, dog16: fp16 [BH, S, d] (dog16 scaled per head); stats from launch_bwd_prep; dinv: inverse scales.  dqacc
// (fp32, zeroed) accumulates dQ_g of the local queries; dK_g and dV_g (fp32) of the key rows of block g are written
// to dkg / dvg + g * dkv_block_stride floats, [BH, S, d] each.
int launch_attn_bwd(const void* qg, const KvSource& kv, const void* dog16, const float* stats, const float* dinv,
                    float* dqacc, float* dkg, float* dvg, uint64_t dkv_block_stride, const LhDims& dm,
                    cudaStream_t st);

// Context parallelism: halo rows exchanged between neighbouring ranks (fp32 [BH][L][d], see cp.cu).
int launch_halo_fwd(const float* og, const int32_t* slot, float* halo, const LhDims& dm, cudaStream_t st);
int launch_scatter_halo(const float* og, const int32_t* slot, const float* halo, void* o, const LhDims& dm,
                        cudaStream_t st);
int launch_halo_bwd(const void* dout, float* halo, const LhDims& dm, cudaStream_t st);
int launch_dog_halo(float* dog, const int32_t* slot, const float* halo, unsigned int* amax, const LhDims& dm,
                    cudaStream_t st);

// Encode a 3-D fp16 tensor map over [BH][rows][d] with a {64, box_rows, 1} box and 128-byte swizzle.
int make_tmap_f16_3d(CUtensorMap* map, const void* base, int d, int rows, int bh, int box_rows = 128);
// Encode a 4-D fp16 tensor map over [blocks][BH][rows][d] (block stride in bytes) with a {64, box_rows, 1, 1} box
// and 128-byte swizzle.
int make_tmap_f16_4d(CUtensorMap* map, const void* base, int d, int rows, int bh, int blocks, uint64_t block_stride,
                     int box_rows = 128);
// Encode the tensor map of the statistics planes of launch_bwd_prep: [2][BH][S] fp32 (row stride stats_stride), box
// {box_rows, 1, 2} (one sub-tile's rows of both planes), no swizzle; rows beyond S read as zero.
int make_tmap_stats(CUtensorMap* map, const float* stats, int S, int bh, int box_rows);
// Encode a 3-D fp32 tensor map over [BH][rows][d] with a {box_cols, box_rows, 1} box, no swizzle.
int make_tmap_f32_3d(CUtensorMap* map, const void* base, int d, int rows, int bh, int box_cols, int box_rows);

inline int check_launch() { return cudaGetLastError() == cudaSuccess ? LH_OK : LH_ERR_CUDA; }

// Brackets the kernel launches of its scope with CUDA events on `st` while tracing is enabled
// (lh_profile_enable); a no-op otherwise.
class KernelTimer {
 public:
  KernelTimer(const char* name, cudaStream_t st);
  ~KernelTimer();

 private:
  int slot_ = -1;
  cudaStream_t st_;
};

}  // namespace lh
