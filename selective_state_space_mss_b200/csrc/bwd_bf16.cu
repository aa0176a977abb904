// bwd_bf16.cu -- backward-pass launchers for bf16 io, every N.
#include "backward.cuh"

namespace mss_host {
MSS_INSTANTIATE_BACKWARD(mss::bf16_t, 1)
MSS_INSTANTIATE_BACKWARD(mss::bf16_t, 2)
MSS_INSTANTIATE_BACKWARD(mss::bf16_t, 4)
MSS_INSTANTIATE_BACKWARD(mss::bf16_t, 8)
MSS_INSTANTIATE_BACKWARD(mss::bf16_t, 16)
}  // namespace mss_host
