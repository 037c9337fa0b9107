// noalloc.cu -- moe_reader_forward_noalloc: the sparse step with its scratch
// in a fixed device array, for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc or an allocating library: serving
// loops that forbid any allocation after start-up so that their memory
// footprint stays fixed, and hosts whose device memory belongs to another
// runtime's allocator, which this library cannot call.  For them this entry
// point keeps the step's workspace in a file-scope __device__ array of a
// fixed size, which every GPU that loads the library holds until the
// process exits.  Its device error word (offset 0, set by a bounded wait
// that ran out) is read and cleared by moe_reader_check_error(NULL, stream).
#include <cstdio>
#include <mutex>

#include "../../include/moe_reader.h"
#include "common.cuh"
#include "kernels.h"

namespace {

constexpr size_t kScratchBytes = 8u << 20;  // 8 MiB per device

// Zero-initialised when the module loads on a device.  In host code this name
// is only a stand-in for the device array: its device address comes from
// cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

}  // namespace

// Device address of the scratch array on the current device (set up on the
// first call on each device).  Returns nullptr and fills *err on failure.
void* moe::noalloc_scratch(cudaError_t* err) {
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    *err = cudaGetSymbolAddress(&p, g_scratch);
    if (*err != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

extern "C" moe_status moe_reader_forward_noalloc(const moe_reader_layer* layer, int B, int k, int c,
                                                 const uint16_t* x, const uint16_t* residual, uint16_t* y,
                                                 void* stream) {
  cudaError_t err = cudaSuccess;
  void* scratch = moe::noalloc_scratch(&err);
  if (!scratch) return moe::set_last_error(MOE_ECUDA, "scratch set-up (cudaGetSymbolAddress) failed");
  // The combine counters in the scratch must be zero when a step begins.  The
  // kernels leave them zero, but the array keeps whatever an earlier
  // (possibly interrupted) call left, so the forward clears them once the
  // arguments have been validated, before its first launch.  Shapes whose
  // workspace exceeds the array are rejected by the same validation
  // ("workspace has N bytes, needs M") with nothing enqueued.
  return moe::forward_scratch(layer, B, k, c, x, residual, y, scratch, kScratchBytes, stream);
}
