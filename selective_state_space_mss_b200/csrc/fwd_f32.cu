// fwd_f32.cu -- forward-pass launchers for fp32 io, every N.
#include "forward.cuh"

namespace mss_host {
MSS_INSTANTIATE_FORWARD(float, 1)
MSS_INSTANTIATE_FORWARD(float, 2)
MSS_INSTANTIATE_FORWARD(float, 4)
MSS_INSTANTIATE_FORWARD(float, 8)
MSS_INSTANTIATE_FORWARD(float, 16)
}  // namespace mss_host
