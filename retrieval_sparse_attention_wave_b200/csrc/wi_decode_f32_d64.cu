// Scan and gather kernels for f32 keys, head size 64.
#include "wi_decode_kernels.cuh"

namespace wi {
WI_DECODE_INSTANTIATE(float, 64)
}  // namespace wi
