// fwd_bf16_n16.cu -- forward-pass launchers for bf16 io with N = 16 (the
// largest set of kernel variants; those with the causal convolution in front
// are compiled in fwd_bf16_n16_conv.cu).
#include "forward.cuh"

namespace mss_host {
MSS_EXTERN_SEQ_CONV(mss::bf16_t, 16)
MSS_INSTANTIATE_FORWARD(mss::bf16_t, 16)
}  // namespace mss_host
