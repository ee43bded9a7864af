// Decode without any allocation: the workspace of wi_decode_noalloc lives in
// a fixed device array of this library instead of caller memory.
//
// Some callers cannot allocate device memory at the point where they decode:
// code running inside a CUDA stream capture (cudaMalloc is not a capturable
// operation and fails or invalidates the capture), serving loops whose device
// memory is owned up front by a fixed arena that hands out no further blocks,
// and C callers embedded in runtimes that expose no device allocator at all.
// For them this entry point takes only inputs and outputs.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <mutex>

#include "wi.h"
#include "wi_common.cuh"
#include "wi_plan.h"

namespace {

constexpr size_t kScratchBytes = (size_t)WI_NOALLOC_SCRATCH_MIB << 20;

// Scratch shared by every wi_decode_noalloc call on a device.  Every GPU that
// loads the library holds it until the process exits.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

// Device address of g_scratch per CUDA context.  In host code the name
// g_scratch is only a host-side stand-in, so the address is looked up once
// per context with that context current.  Keying by the context's unique id
// (not the device number, nor the context handle, which a context created
// after a device reset may reuse) makes such a context look the address up
// again instead of reusing a stale one.
constexpr int kMaxContexts = 64;
std::mutex g_mu;
unsigned long long g_ctx[kMaxContexts];
void* g_ptr[kMaxContexts];
int g_n = 0;

// The current context's unique id, or 0 when it cannot be read.
unsigned long long current_ctx_id() {
  static std::once_flag once;
  static PFN_cuCtxGetCurrent_v4000 get_ctx = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_ctx = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_ctx || !get_id || get_ctx(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

wi_status scratch_ptr(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return WI_ERR_CUDA;
  // make the device's primary context current (a no-op when it already is)
  if (cudaFree(nullptr) != cudaSuccess) return WI_ERR_CUDA;
  const unsigned long long ctx = current_ctx_id();
  if (ctx == 0) return WI_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  for (int i = 0; i < g_n; ++i)
    if (g_ctx[i] == ctx) { *out = g_ptr[i]; return WI_OK; }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return WI_ERR_CUDA;
  if (g_n < kMaxContexts) { g_ctx[g_n] = ctx; g_ptr[g_n] = p; ++g_n; }
  *out = p;
  return WI_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" wi_status wi_decode_noalloc(const void* q, const wi_index* idx,
                                       const wi_decode_params* p, float* out, float* lse,
                                       wi_stream_t stream) {
  // every argument error is returned before the first CUDA call
  if (!q || !out || !aligned(q, 16) || !aligned(out, 4) || (lse && !aligned(lse, 4)))
    return WI_ERR_INVALID_ARG;
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
