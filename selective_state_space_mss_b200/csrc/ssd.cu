// ssd.cu -- host-side launch of the structured-state-space-duality forward
// pass (ssd_mma.cuh).
#include <cuda_runtime.h>

#include "host_common.h"
#include "launch.h"
#include "ssd_mma.cuh"

namespace mss_host {

template <int NS, bool kGate, bool kSoftplus>
int launch_ssd_variant(const mss::SsdParams& p, cudaStream_t s) {
    using Ly = mss::SsdLayout<NS>;
    auto kern = mss::ssd_fwd_kernel<NS, kGate, kSoftplus>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Ly::kSmemBytes) != cudaSuccess)
        return MSS_ERR_CUDA;
    const int64_t blocks = p.batch * p.nheads;
    if (blocks > 0x7fffffffLL) return MSS_ERR_SHAPE;
    kern<<<dim3(unsigned(blocks)), Ly::kThreads, Ly::kSmemBytes, s>>>(p);
    return launch_status();
}

template <int NS>
int launch_ssd_n(const mss::SsdParams& p, cudaStream_t s) {
    if (p.z)
        return p.softplus ? launch_ssd_variant<NS, true, true>(p, s) : launch_ssd_variant<NS, true, false>(p, s);
    return p.softplus ? launch_ssd_variant<NS, false, true>(p, s) : launch_ssd_variant<NS, false, false>(p, s);
}

int launch_ssd(const mss::SsdParams& p, int dstate, cudaStream_t s) {
    return dstate == 64 ? launch_ssd_n<64>(p, s) : launch_ssd_n<128>(p, s);
}

}  // namespace mss_host
