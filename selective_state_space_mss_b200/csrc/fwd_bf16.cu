// fwd_bf16.cu -- forward-pass launchers for bf16 io with N = 1, 2, 4, 8.
#include "forward.cuh"

namespace mss_host {
MSS_INSTANTIATE_FORWARD(mss::bf16_t, 1)
MSS_INSTANTIATE_FORWARD(mss::bf16_t, 2)
MSS_INSTANTIATE_FORWARD(mss::bf16_t, 4)
MSS_INSTANTIATE_FORWARD(mss::bf16_t, 8)
}  // namespace mss_host
