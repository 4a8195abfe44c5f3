// noalloc.cu -- ssd_prefill_noalloc: the prefill with its scratch in a fixed device array.
//
// Who needs it: code that is not allowed to create device allocations of its own -- for
// example a host program whose device memory is owned by a framework's caching allocator or a
// fixed memory pool, or one that must not call cudaMalloc/cudaFree because those calls can
// synchronise the device and stall unrelated work.  Such a caller still owns every input and
// output buffer; only the library's scratch moves into memory the library reserves itself.
//
// The scratch is one file-scope __device__ array of SSD_NOALLOC_WORKSPACE_BYTES per device.
// It is created when the library's device code is loaded on a device and lives until the
// process exits, so every GPU that loads this library holds it.  Host code cannot take the
// array's address directly (the host-side name is only a stand-in for the symbol); the first
// call on each device looks the address up with cudaGetSymbolAddress while that device is
// current, and later calls on that device reuse it.  That lookup is the only set-up work, so
// the first call on a device should happen before the caller starts any stream capture.
//
// All calls share the array and it keeps whatever the previous call left in it.  No call reads
// scratch that an earlier step of the same call has not written (every region is produced in
// full before it is consumed), so nothing has to be cleared between calls.  Two calls whose
// kernels can overlap on the GPU -- issued on different streams without ordering, or from
// different host threads -- would use the same scratch at the same time and race; callers must
// order them (for example by issuing them on one stream).
#include <mutex>

#include "common.cuh"
#include "plan.h"

namespace ssd {
namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[SSD_NOALLOC_WORKSPACE_BYTES];

constexpr int kMaxDev = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDev] = {};

// Device address of the scratch array on the current device (looked up once per device).
cudaError_t scratch_address(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace ssd

extern "C" ssd_status_t ssd_prefill_noalloc(const ssd_config_t *cfg, const ssd_prefill_args_t *args,
                                            void *stream) {
  if (!cfg || !args) return SSD_ERR_INVALID_ARG;
  // An invalid config reports 0 bytes here; ssd_prefill then returns the precise error.
  if (ssd_workspace_size(cfg) > SSD_NOALLOC_WORKSPACE_BYTES) return SSD_ERR_WORKSPACE;
  void *scratch = nullptr;
  if (ssd::scratch_address(&scratch) != cudaSuccess) return SSD_ERR_CUDA;
  ssd_prefill_args_t a = *args;
  a.workspace = scratch;
  a.workspace_bytes = SSD_NOALLOC_WORKSPACE_BYTES;
  return ssd_prefill(cfg, &a, stream);
}
