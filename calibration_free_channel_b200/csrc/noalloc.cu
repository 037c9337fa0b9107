// noalloc.cu -- moe_reader_forward_noalloc: the sparse step with its scratch
// in a fixed device array, for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc or an allocating library: code that
// runs while a stream is being captured into a CUDA graph (allocation is not
// a capturable operation), serving loops that forbid any allocation after
// start-up so their memory footprint stays fixed, and hosts whose device
// allocator belongs to another runtime.  For them this entry point keeps the
// step's workspace in a file-scope __device__ array of a fixed size, which
// every GPU that loads the library holds until the process exits.
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

// Device address of the scratch array on the current device (set up on the
// first call on each device).  Returns nullptr and fills *err on failure.
void* scratch_address(cudaError_t* err) {
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

}  // namespace

extern "C" moe_status moe_reader_forward_noalloc(const moe_reader_layer* layer, int B, int k, int c,
                                                 const uint16_t* x, const uint16_t* residual, uint16_t* y,
                                                 void* stream) {
  if (!layer) return moe::set_last_error(MOE_EINVAL, "layer is NULL");
  // Shapes whose workspace exceeds the fixed array are rejected by the
  // forward's own validation below ("workspace has N bytes, needs M"),
  // before anything is enqueued.
  const size_t need = moe_reader_workspace_bytes(B, layer->E, layer->top_e, layer->I, layer->d, k, c, layer->r);
  cudaError_t err = cudaSuccess;
  void* scratch = scratch_address(&err);
  if (!scratch) return moe::set_last_error(MOE_ECUDA, "scratch set-up (cudaGetSymbolAddress) failed");
  if (need > 0 && need <= kScratchBytes) {
    // The combine counters at the start of the workspace must be zero when a
    // step begins.  The kernels leave them zero, but the array keeps whatever
    // an earlier (possibly interrupted) call left, so clear them here.
    moe::Workspace ws;
    moe::workspace_layout(1, 1, 1, 16, 0, 0, scratch, &ws);
    err = cudaMemsetAsync(ws.counters, 0, sizeof(unsigned) * moe::kMaxTokens * moe::kMaxCluster,
                          static_cast<cudaStream_t>(stream));
    if (err != cudaSuccess) return moe::set_last_error(MOE_ECUDA, "clearing the scratch counters failed");
  }
  return moe_reader_forward(layer, B, k, c, x, residual, y, nullptr, scratch, kScratchBytes, stream);
}
