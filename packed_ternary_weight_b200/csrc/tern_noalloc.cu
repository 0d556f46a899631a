// tern_gemv_noalloc: the single-token GEMV of tern_gemv for callers that cannot
// allocate device memory themselves -- for example code that runs where
// cudaMalloc is not allowed (inside a custom allocator or memory-pool
// callback, in a plugin whose host framework owns every device allocation, or
// between steps of a pre-planned memory budget) and so cannot provide the
// workspace that tern_gemv uses to combine partial sums when it splits K
// across thread blocks.
//
// Its workspace is instead a fixed array in device memory that belongs to the
// library: every GPU that loads the library holds kNoAllocScratchBytes of it
// until the process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "tern_internal.h"

namespace {

// Fixed device scratch shared by every tern_gemv_noalloc call on a device.
constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;  // 1 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device. In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device (with that device current) and cached.
tern_status scratch_on_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TERN_ECUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return TERN_ECUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return TERN_OK;
}

}  // namespace

extern "C" tern_status tern_gemv_noalloc(const tern_desc* desc, const void* d_packed, tern_act act, const void* d_x,
                                         const float* d_xscale, tern_out out, void* d_y, void* stream) {
  size_t need = 0;
  tern_status st = tern_workspace_size(desc, 1, &need);
  if (st != TERN_OK) return st;
  if (need > kNoAllocScratchBytes) return TERN_ENOSPACE;  // layer too large for the fixed scratch
  void* scratch = nullptr;
  st = scratch_on_current_device(&scratch);
  if (st != TERN_OK) return st;
  // The scratch keeps whatever the previous call left; the arrival counters at
  // its start must be zero, so clear the part this call may use.
  if (need > 0 &&
      cudaMemsetAsync(scratch, 0, need, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return TERN_ECUDA;
  return tern_gemv(desc, d_packed, act, d_x, d_xscale, out, d_y, need > 0 ? scratch : nullptr, need, stream);
}
