// fwd_bf16_n16_conv.cu -- the throughput-kernel launches for bf16 io, N = 16,
// with the causal convolution in front of the scan.
#include "forward.cuh"

namespace mss_host {
MSS_INSTANTIATE_SEQ_CONV(mss::bf16_t, 16)
}  // namespace mss_host
