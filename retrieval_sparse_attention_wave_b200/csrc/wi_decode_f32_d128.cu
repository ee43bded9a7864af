// Scan and gather kernels for f32 keys, head size 128.
#include "wi_decode_kernels.cuh"

namespace wi {
WI_DECODE_INSTANTIATE(float, 128)
}  // namespace wi
