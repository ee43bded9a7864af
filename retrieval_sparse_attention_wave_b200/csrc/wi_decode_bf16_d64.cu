// Scan and gather kernels for bf16 keys, head size 64.
#include "wi_decode_kernels.cuh"

namespace wi {
WI_DECODE_INSTANTIATE(__nv_bfloat16, 64)
}  // namespace wi
