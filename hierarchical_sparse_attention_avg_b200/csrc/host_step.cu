// host_step.cu — one forward + backward of the layer on host-resident tensors, with the PCIe copies overlapped.
//
// The pages describe the layer on device tensors only; this entry point is plumbing for callers whose Q, K, V and
// dO live in host memory.  Heads are independent through every step of the layer (pool, score, selection, gather,
// attention and scatter all work within one head), so the step runs in chunks of consecutive heads of one batch
// row: chunk g's host-to-device copies (on the caller's h2d stream), its lh_forward + lh_backward (on the compute
// stream) and its device-to-host copies (on the d2h stream) overlap with the neighbouring chunks', and the two copy
// directions share the full-duplex link.  Three chunks' tensors are resident at a time (slots 0..2 of the caller's
// device buffer): chunk g's inputs are copied in while chunk g-1 is computed and chunk g-2 is copied out, so
// neither copy direction waits for a computation; one context and one workspace serve every chunk, in order, on
// the compute stream.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "lh.h"

namespace {

constexpr int kSlots = 3;
constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct StepLayout {
  size_t tensor;       // bytes of one bf16 chunk tensor [hc, N, d]
  size_t tensor_al;    // the same, aligned
  size_t slot;         // 8 tensors: q, k, v, dout, o, dq, dk, dv
  size_t ctx, ctx_off;
  size_t ws, ws_off;
  size_t total;
};

// Parameters of one chunk (one batch row, hc heads); false when P or hc cannot be chunked.
bool chunk_params(const lh_params* P, int hc, lh_params* Pc) {
  if (!P || hc <= 0 || P->H <= 0 || P->H % hc != 0) return false;
  *Pc = *P;
  Pc->B = 1;
  Pc->H = hc;
  return true;
}

bool step_layout(const lh_params* P, int hc, StepLayout* L) {
  lh_params Pc;
  if (!chunk_params(P, hc, &Pc) || P->B <= 0 || lh_S(&Pc) < 0) return false;
  L->ctx = lh_ctx_bytes(&Pc);
  L->ws = lh_workspace_bytes(&Pc);
  if (L->ctx == 0 || L->ws == 0) return false;
  L->tensor = (size_t)hc * (size_t)P->N * (size_t)P->d * 2;
  L->tensor_al = align_up(L->tensor);
  L->slot = 8 * L->tensor_al;
  L->ctx_off = kSlots * L->slot;
  L->ws_off = L->ctx_off + align_up(L->ctx);
  L->total = L->ws_off + align_up(L->ws);
  return true;
}

// Events of the pipeline, created on first use per device and kept for the life of the process.
struct StepEvents {
  bool ready = false;
  cudaEvent_t start, h2d[kSlots], comp[kSlots], d2h[kSlots];
};
constexpr int kMaxDevices = 64;
StepEvents g_events[kMaxDevices];

int events_for_current_device(StepEvents** out) {
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LH_ERR_CUDA;
  std::lock_guard<std::mutex> g(mu);
  StepEvents& e = g_events[dev];
  if (!e.ready) {
    // create all events or none: on a failure the ones already created are destroyed
    constexpr int kPer = 3;  // events per slot
    cudaEvent_t* all[1 + kPer * kSlots] = {&e.start};
    for (int s = 0; s < kSlots; ++s) {
      all[1 + kPer * s] = &e.h2d[s];
      all[2 + kPer * s] = &e.comp[s];
      all[3 + kPer * s] = &e.d2h[s];
    }
    for (int i = 0; i < 1 + kPer * kSlots; ++i) {
      if (cudaEventCreateWithFlags(all[i], cudaEventDisableTiming) != cudaSuccess) {
        for (int j = 0; j < i; ++j) cudaEventDestroy(*all[j]);
        return LH_ERR_CUDA;
      }
    }
    e.ready = true;
  }
  *out = &e;
  return LH_OK;
}

#define STEP_CUDA(x)                              \
  do {                                            \
    if ((x) != cudaSuccess) return LH_ERR_CUDA;   \
  } while (0)

}  // namespace

extern "C" size_t lh_step_host_bytes(const lh_params* P, int heads_per_chunk) {
  StepLayout L;
  return step_layout(P, heads_per_chunk, &L) ? L.total : 0;
}

extern "C" int lh_step_host(const lh_params* P, const void* q, const void* k, const void* v, const void* dout,
                            void* o, void* dq, void* dk, void* dv, int heads_per_chunk, void* dev, size_t dev_bytes,
                            void* stream, void* h2d_stream, void* d2h_stream) {
  StepLayout L;
  lh_params Pc;
  if (!P || !chunk_params(P, heads_per_chunk, &Pc) || !step_layout(P, heads_per_chunk, &L)) return LH_ERR_INVALID_ARG;
  const void* in[4] = {q, k, v, dout};
  void* outp[4] = {o, dq, dk, dv};
  for (int i = 0; i < 4; ++i)
    if (!in[i] || !outp[i]) return LH_ERR_INVALID_ARG;
  if (!dev || (reinterpret_cast<uintptr_t>(dev) % kAlign) != 0) return LH_ERR_INVALID_ARG;
  if (dev_bytes < L.total) return LH_ERR_WORKSPACE;

  StepEvents* ev = nullptr;
  const int erc = events_for_current_device(&ev);
  if (erc != LH_OK) return erc;
  cudaStream_t cs = (cudaStream_t)stream, hs = (cudaStream_t)h2d_stream, ds = (cudaStream_t)d2h_stream;
  char* base = static_cast<char*>(dev);
  void* ctx = base + L.ctx_off;
  void* ws = base + L.ws_off;

  // the copies start after whatever the caller enqueued on the compute stream before this call
  STEP_CUDA(cudaEventRecord(ev->start, cs));
  STEP_CUDA(cudaStreamWaitEvent(hs, ev->start, 0));

  const int per_row = P->H / heads_per_chunk;
  const int nchunks = P->B * per_row;
  for (int g = 0; g < nchunks; ++g) {
    const int s = g % kSlots;
    const int b = g / per_row, h0 = (g % per_row) * heads_per_chunk;
    const size_t off = ((size_t)b * P->H + h0) * (size_t)P->N * (size_t)P->d * 2;  // byte offset of the chunk
    char* slot = base + s * L.slot;
    auto t = [&](int i) { return static_cast<void*>(slot + i * L.tensor_al); };
    // slot s is free once the chunk that used it before (g - kSlots) has been copied out (after its compute)
    if (g >= kSlots) STEP_CUDA(cudaStreamWaitEvent(hs, ev->d2h[s], 0));
    for (int i = 0; i < 4; ++i)
      STEP_CUDA(cudaMemcpyAsync(t(i), static_cast<const char*>(in[i]) + off, L.tensor, cudaMemcpyHostToDevice, hs));
    STEP_CUDA(cudaEventRecord(ev->h2d[s], hs));
    STEP_CUDA(cudaStreamWaitEvent(cs, ev->h2d[s], 0));
    int rc = lh_forward(&Pc, t(0), t(1), t(2), t(4), ctx, ws, L.ws, cs);
    if (rc == LH_OK) rc = lh_backward(&Pc, t(3), ctx, t(5), t(6), t(7), ws, L.ws, cs);
    if (rc != LH_OK) return rc;
    STEP_CUDA(cudaEventRecord(ev->comp[s], cs));
    STEP_CUDA(cudaStreamWaitEvent(ds, ev->comp[s], 0));
    for (int i = 0; i < 4; ++i)
      STEP_CUDA(cudaMemcpyAsync(static_cast<char*>(outp[i]) + off, t(4 + i), L.tensor, cudaMemcpyDeviceToHost, ds));
    STEP_CUDA(cudaEventRecord(ev->d2h[s], ds));
  }
  // the compute stream is ordered after the last device-to-host copies
  for (int s = 0; s < kSlots && s < nchunks; ++s) STEP_CUDA(cudaStreamWaitEvent(cs, ev->d2h[s], 0));
  return LH_OK;
}
