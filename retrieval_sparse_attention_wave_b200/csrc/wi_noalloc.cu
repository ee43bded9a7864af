// Decode without any allocation: the workspace of wi_decode_noalloc lives in
// a fixed device array of this library instead of caller memory.
//
// Some callers cannot allocate device memory at the point where they decode:
// code running inside a CUDA stream capture (cudaMalloc is not a capturable
// operation and fails or invalidates the capture), serving loops whose device
// memory is owned up front by a fixed arena that hands out no further blocks,
// and C callers embedded in runtimes that expose no device allocator at all.
// For them this entry point takes only inputs and outputs.
#include <mutex>

#include "wi.h"
#include "wi_common.cuh"
#include "wi_plan.h"

namespace {

constexpr size_t kScratchBytes = (size_t)WI_NOALLOC_SCRATCH_MIB << 20;

// Scratch shared by every wi_decode_noalloc call on a device.  Every GPU that
// loads the library holds it until the process exits.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_ptr[kMaxDevices];  // device address of g_scratch, per device

// The device address of g_scratch on the current device.  Host code only sees
// a host-side stand-in under the name g_scratch, so the address is looked up
// once per device with that device current.
wi_status scratch_ptr(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) return WI_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess || !p) return WI_ERR_CUDA;
    g_ptr[dev] = p;
  }
  *out = g_ptr[dev];
  return WI_OK;
}

}  // namespace

extern "C" wi_status wi_decode_noalloc(const void* q, const wi_index* idx,
                                       const wi_decode_params* p, float* out, float* lse,
                                       wi_stream_t stream) {
  size_t total = 0, zero_prefix = 0;
  wi_status st = wi::decode_workspace_extent(idx, p, &total, &zero_prefix);
  if (st != WI_OK) return st;
  if (total > kScratchBytes) return WI_ERR_WORKSPACE;  // larger than the fixed scratch
  void* ws = nullptr;
  if ((st = scratch_ptr(&ws)) != WI_OK) return st;
  // the scratch keeps the previous call's contents: clear what must start at zero
  const cudaError_t e =
      cudaMemsetAsync(ws, 0, zero_prefix, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return WI_ERR_CUDA;
  return wi_decode(q, idx, p, out, lse, ws, total, stream);
}
