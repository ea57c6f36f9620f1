// trace.cu — optional per-kernel device timing (lh_profile_enable / lh_profile_read).
#include <string.h>

#include <mutex>
#include <string>
#include <vector>

#include "internal.h"

namespace lh {

namespace {

struct Record {
  std::string name;
  cudaEvent_t start, stop;
  bool done;
};

std::mutex g_mu;
bool g_on = false;
std::vector<Record> g_records;
std::vector<cudaEvent_t> g_pool;

cudaEvent_t take_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

}  // namespace

KernelTimer::KernelTimer(const char* name, cudaStream_t st) : st_(st) {
  std::lock_guard<std::mutex> g(g_mu);
  if (!g_on) return;
  cudaEvent_t a = take_event(), b = take_event();
  if (!a || !b) return;
  cudaEventRecord(a, st);
  g_records.push_back(Record{name, a, b, false});
  slot_ = (int)g_records.size() - 1;
}

KernelTimer::~KernelTimer() {
  if (slot_ < 0) return;
  std::lock_guard<std::mutex> g(g_mu);
  if (slot_ >= (int)g_records.size()) return;
  cudaEventRecord(g_records[slot_].stop, st_);
  g_records[slot_].done = true;
}

}  // namespace lh

extern "C" {

int lh_profile_enable(int on) {
  std::lock_guard<std::mutex> g(lh::g_mu);
  lh::g_on = on != 0;
  return LH_OK;
}

int lh_profile_read(lh_kernel_time_t* out, int max_entries) {
  std::lock_guard<std::mutex> g(lh::g_mu);
  std::vector<lh_kernel_time_t> acc;
  int rc = 0;
  for (auto& r : lh::g_records) {
    if (r.done) {
      float ms = 0.f;
      if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess) {
        rc = -LH_ERR_CUDA;
      } else {
        size_t i = 0;
        while (i < acc.size() && strncmp(acc[i].name, r.name.c_str(), sizeof(acc[i].name)) != 0) ++i;
        if (i == acc.size()) {
          lh_kernel_time_t t;
          memset(&t, 0, sizeof(t));
          strncpy(t.name, r.name.c_str(), sizeof(t.name) - 1);
          acc.push_back(t);
        }
        acc[i].launches += 1;
        acc[i].ms += ms;
      }
    }
    lh::g_pool.push_back(r.start);
    lh::g_pool.push_back(r.stop);
  }
  lh::g_records.clear();
  if (rc) return rc;
  const int n = (int)acc.size() < max_entries ? (int)acc.size() : max_entries;
  for (int i = 0; i < n && out; ++i) out[i] = acc[i];
  return n;
}

}  // extern "C"
