// Decode launches of the wave index: the steady kernel, then the scan and
// gather kernels of the call's key type, head size and group size (compiled
// one key type and head size per file, wi_decode_<type>_d<size>.cu).  See wi_decode_kernels.cuh for
// what each kernel computes.
#include <algorithm>
#include <cstring>

#include "wi_decode_kernels.cuh"

namespace wi {

const char* const kDecodeStageNames[kDecodeStages] = {"steady", "scan", "gather"};

// compiled one key type and head size per file
WI_DECODE_EXTERN(__nv_bfloat16, 128)
WI_DECODE_EXTERN(__nv_bfloat16, 64)
WI_DECODE_EXTERN(float, 128)
WI_DECODE_EXTERN(float, 64)

namespace {

template <typename F>
cudaError_t with_types(int dtype, int D, int G, F&& f) {
  auto byG = [&]<typename T, int DD>() -> cudaError_t {
    switch (G) {
      case 1: return f.template operator()<T, DD, 1>();
      case 2: return f.template operator()<T, DD, 2>();
      case 4: return f.template operator()<T, DD, 4>();
      case 8: return f.template operator()<T, DD, 8>();
    }
    return cudaErrorInvalidValue;
  };
  if (dtype == WI_BF16) {
    if (D == 128) return byG.template operator()<__nv_bfloat16, 128>();
    if (D == 64) return byG.template operator()<__nv_bfloat16, 64>();
  } else {
    if (D == 128) return byG.template operator()<float, 128>();
    if (D == 64) return byG.template operator()<float, 64>();
  }
  return cudaErrorInvalidValue;
}

}  // namespace

size_t decode_scan_smem(int dtype, int D, int G, int slots, int exact_only) {
  size_t r = 0;
  with_types(dtype, D, G, [&]<typename T, int DD, int GG>() -> cudaError_t {
    r = ScanSmem<T, DD, GG>::total(slots, exact_only);
    return cudaSuccess;
  });
  return r;
}

size_t decode_scan_slot_bytes(int dtype, int D, int G, int exact_only) {
  size_t r = 0;
  with_types(dtype, D, G, [&]<typename T, int DD, int GG>() -> cudaError_t {
    r = ScanSmem<T, DD, GG>::tile_bytes(exact_only) + ScanSmem<T, DD, GG>::kSide;
    return cudaSuccess;
  });
  return r;
}

size_t decode_gather_smem(int dtype, int D, int G) {
  size_t r = 0;
  with_types(dtype, D, G, [&]<typename T, int DD, int GG>() -> cudaError_t {
    r = GatherSmem<T, DD, GG>::kTotal;
    return cudaSuccess;
  });
  return r;
}

size_t decode_steady_smem(int cap) { return (size_t)8 * pow2_at_least(std::max(cap, 1)); }

cudaError_t launch_decode(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
  unsigned char* ws = a.ws;
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + p.off_status);
  cudaEvent_t* ev = a.stage_events;
  if (ev) cudaEventRecord(ev[0], s);
  const ChunkMap cm = chunk_map(p);
  // K0: steady zone (a normal launch: everything before it in the stream is done)
  SteadyArgs sa{a.invperm, a.labels, a.offsets, p.n_sink, p.window, p.cap,
                reinterpret_cast<int32_t*>(ws + p.off_info),
                reinterpret_cast<int32_t*>(ws + p.off_st_slot),
                reinterpret_cast<int2*>(ws + p.off_pc), reinterpret_cast<int2*>(ws + p.off_nonc),
                reinterpret_cast<int32_t*>(ws + p.off_hist), reinterpret_cast<int32_t*>(ws + p.off_cnt1),
                reinterpret_cast<int32_t*>(ws + p.off_cnt2)};
  const size_t st_smem = decode_steady_smem(p.cap);
  set_smem(wave_steady_kernel, st_smem);
  const cudaError_t e = launch_ex(wave_steady_kernel, dim3(p.U), dim3(256), st_smem, s, false,
                                  p.geo, sa, status);
  if (e != cudaSuccess) return e;
  return with_types(p.dtype, p.D, p.G, [&]<typename T, int D, int G>() -> cudaError_t {
    return launch_decode_typed<T, D, G>(p, a, cm, s);
  });
}

}  // namespace wi
