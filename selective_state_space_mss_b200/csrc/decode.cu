// decode.cu -- host-side launch of the single-token decode update: the
// bulk-staged kernel (state_update_tma.cuh) where the shape and alignment
// allow it, the per-thread kernel (state_update.cuh) otherwise.
#include <algorithm>
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "host_common.h"
#include "launch.h"
#include "state_update.cuh"
#include "state_update_tma.cuh"

namespace mss_host {

// Resident blocks of the bulk-staged decode kernel on the current device.
template <typename T, int N>
int decode_tma_slots() {
    static std::mutex mu;
    static int cache[kMaxDevices] = {};
    return per_device(cache, mu, [](int dev) {
        return resident_blocks(mss::state_update_tma_kernel<T, N>, mss::DecodeTile<T, N>::kThreads,
                               mss::DecodeTile<T, N>::kSmemBytes, dev);
    });
}

template <typename T, int N>
int launch_decode(mss::StepParams p, cudaStream_t s) {
    const int64_t rows = p.batch * p.dim;
    const bool vec = aligned(p.state, 16) && aligned(p.A, 16);
    if constexpr (N == 4 || N == 8 || N == 16) {
        // bulk-staged kernel when every streamed tensor is 16-byte aligned and
        // dim is a whole number of tiles
        using Ly = mss::DecodeTile<T, N>;
        const bool bulk_ok = vec && aligned(p.u, 16) && aligned(p.delta, 16) && aligned(p.y, 16) &&
                             (!p.z || aligned(p.z, 16)) && (p.conv_width < 2 || aligned(p.conv_state, 16)) &&
                             p.dim % Ly::kRows == 0 && p.batch <= 0x7fffffffLL;
        if (bulk_ok) {
            const int64_t n_cblocks = p.dim / Ly::kRows;
            const int slots = decode_tma_slots<T, N>();
            if (slots <= 0) return MSS_ERR_CUDA;
            // batch rows of a channel block served by separate CTAs
            const int64_t bsplit = std::max<int64_t>(1, std::min<int64_t>(p.batch, slots / n_cblocks));
            const int64_t grid = n_cblocks * bsplit;
            if (grid <= 0x7fffffffLL) {
                mss::state_update_tma_kernel<T, N><<<dim3(unsigned(grid)), Ly::kThreads, Ly::kSmemBytes, s>>>(
                    p, int(n_cblocks), int(bsplit));
                return launch_status();
            }
        }
    }
    constexpr int TPC = N < 4 ? 1 : N / 4;
    const int threads = 256;
    const int64_t blocks = ((rows - p.row0) * TPC + threads - 1) / threads;
    if (blocks > 0x7fffffffLL) return MSS_ERR_SHAPE;
    if (vec)
        mss::state_update_kernel<T, N, true><<<dim3(unsigned(blocks)), threads, 0, s>>>(p);
    else
        mss::state_update_kernel<T, N, false><<<dim3(unsigned(blocks)), threads, 0, s>>>(p);
    return launch_status();
}

#define MSS_INSTANTIATE_DECODE(T, N) template int launch_decode<T, N>(mss::StepParams, cudaStream_t);
MSS_INSTANTIATE_DECODE(mss::bf16_t, 1)
MSS_INSTANTIATE_DECODE(mss::bf16_t, 2)
MSS_INSTANTIATE_DECODE(mss::bf16_t, 4)
MSS_INSTANTIATE_DECODE(mss::bf16_t, 8)
MSS_INSTANTIATE_DECODE(mss::bf16_t, 16)
MSS_INSTANTIATE_DECODE(float, 1)
MSS_INSTANTIATE_DECODE(float, 2)
MSS_INSTANTIATE_DECODE(float, 4)
MSS_INSTANTIATE_DECODE(float, 8)
MSS_INSTANTIATE_DECODE(float, 16)
#undef MSS_INSTANTIATE_DECODE

}  // namespace mss_host
