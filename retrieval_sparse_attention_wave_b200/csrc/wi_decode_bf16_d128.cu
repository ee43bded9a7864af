// Scan and gather kernels for bf16 keys, head size 128.
#include "wi_decode_kernels.cuh"

namespace wi {
WI_DECODE_INSTANTIATE(__nv_bfloat16, 128)
}  // namespace wi
