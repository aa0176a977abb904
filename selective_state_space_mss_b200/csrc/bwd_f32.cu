// bwd_f32.cu -- backward-pass launchers for fp32 io, every N.
#include "backward.cuh"

namespace mss_host {
MSS_INSTANTIATE_BACKWARD(float, 1)
MSS_INSTANTIATE_BACKWARD(float, 2)
MSS_INSTANTIATE_BACKWARD(float, 4)
MSS_INSTANTIATE_BACKWARD(float, 8)
MSS_INSTANTIATE_BACKWARD(float, 16)
}  // namespace mss_host
