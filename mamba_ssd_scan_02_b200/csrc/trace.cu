// trace.cu -- optional CUDA-event tracing of the library's kernel launches (host code).
#include <atomic>
#include <mutex>
#include <string.h>
#include <vector>

#include "plan.h"

namespace ssd {
namespace {

struct Rec {
  cudaEvent_t start, stop;
  char name[48];
  bool used;
};

std::mutex g_mu;
std::atomic<bool> g_on{false};  // read without the lock on every launch
std::vector<Rec> g_recs;  // events are created once and reused after each read
size_t g_next = 0;

}  // namespace

bool trace_enabled() { return g_on.load(); }

int trace_begin(cudaStream_t s) {
  if (!g_on.load()) return -1;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_next == g_recs.size()) {
    Rec r{};
    if (cudaEventCreate(&r.start) != cudaSuccess || cudaEventCreate(&r.stop) != cudaSuccess) return -1;
    g_recs.push_back(r);
  }
  const int slot = (int)g_next++;
  g_recs[slot].used = false;
  cudaEventRecord(g_recs[slot].start, s);
  return slot;
}

void trace_end(int slot, const char *name, cudaStream_t s) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (slot < 0 || (size_t)slot >= g_recs.size()) return;
  cudaEventRecord(g_recs[slot].stop, s);
  strncpy(g_recs[slot].name, name, sizeof(g_recs[slot].name) - 1);
  g_recs[slot].used = true;
}

}  // namespace ssd

extern "C" {

int ssd_trace_enable(int on) {
  std::lock_guard<std::mutex> lk(ssd::g_mu);
  const int prev = ssd::g_on.exchange(on != 0) ? 1 : 0;
  return prev;
}

int ssd_trace_read(ssd_trace_record_t *out, int max_records) {
  std::lock_guard<std::mutex> lk(ssd::g_mu);
  int n = 0;
  int rc = 0;
  for (size_t i = 0; i < ssd::g_next; ++i) {
    ssd::Rec &r = ssd::g_recs[i];
    if (!r.used) continue;
    if (cudaEventSynchronize(r.stop) != cudaSuccess) rc = -1;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess) rc = -1;
    if (out && n < max_records) {
      memcpy(out[n].name, r.name, sizeof(out[n].name));
      out[n].ms = ms;
      ++n;
    }
  }
  ssd::g_next = 0;
  return rc < 0 ? -1 : n;
}

}  // extern "C"
