// host_common.h -- host-side helpers shared by the library's translation
// units: argument arithmetic, alignment and overlap tests, dispatch on N,
// launch status, and a per-device cache for device queries.
#pragma once

#include <cstdint>
#include <mutex>
#include <type_traits>

#include <cuda_runtime.h>

#include "../../include/mss.h"
#include "mss_params.h"

namespace mss_host {

inline bool mul_ok(int64_t a, int64_t b, int64_t* out) { return !__builtin_mul_overflow(a, b, out); }

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline bool valid_n(int64_t n) { return n == 1 || n == 2 || n == 4 || n == 8 || n == 16; }

// [p, p + bytes) and [q, q + qbytes) overlap (null or empty ranges never do)
inline bool overlaps(const void* p, int64_t bytes, const void* q, int64_t qbytes) {
    if (!p || !q || bytes <= 0 || qbytes <= 0) return false;
    const uintptr_t a = reinterpret_cast<uintptr_t>(p), b = reinterpret_cast<uintptr_t>(q);
    return a < b + uint64_t(qbytes) && b < a + uint64_t(bytes);
}

// Dispatch on N: calls f(std::integral_constant<int, N>).
template <typename F>
auto with_n(int64_t n, F&& f) -> decltype(f(std::integral_constant<int, 1>{})) {
    switch (n) {
        case 1: return f(std::integral_constant<int, 1>{});
        case 2: return f(std::integral_constant<int, 2>{});
        case 4: return f(std::integral_constant<int, 4>{});
        case 8: return f(std::integral_constant<int, 8>{});
        case 16: return f(std::integral_constant<int, 16>{});
        default: return MSS_ERR_UNSUPPORTED_N;
    }
}

// The sizes the tiled kernels take (grid limits, 32-bit tensor-map row
// coordinates); the backward pass's workspace size follows the same test.
inline bool seq_shape_ok(int64_t batch, int64_t dim, int64_t seqlen, int64_t N, int esz, unsigned flags) {
    if (flags & MSS_FLAG_SIMPLE) return false;
    if (N != 4 && N != 8 && N != 16) return false;
    if ((seqlen * esz) % 16 != 0) return false;
    if (batch * dim >= (int64_t(1) << 31) || seqlen >= (int64_t(1) << 31)) return false;
    if ((dim + 15) / 16 > 0x7fffffffLL || batch > 65535) return false;
    return true;
}

// The throughput kernel's requirements; otherwise the scalar kernel runs.
inline bool seq_eligible(const mss::ScanParams& p, int64_t N, int esz, unsigned flags) {
    if (!seq_shape_ok(p.batch, p.dim, p.seqlen, N, esz, flags)) return false;
    const void* v[] = {p.u, p.delta, p.z, p.B, p.C, p.y};
    for (const void* q : v)
        if (q && !aligned(q, 16)) return false;
    return true;
}

inline int launch_status() { return cudaGetLastError() == cudaSuccess ? MSS_OK : MSS_ERR_CUDA; }

constexpr int kMaxDevices = 64;

// A positive value computed by `query()` once per device and kept; 0 when
// there is no current device or the query fails (it is then retried).
template <typename Query>
int per_device(int (&cache)[kMaxDevices], std::mutex& mu, Query&& query) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    std::lock_guard<std::mutex> lock(mu);
    if (cache[dev] <= 0) cache[dev] = query(dev);
    return cache[dev] > 0 ? cache[dev] : 0;
}

// Streaming multiprocessors x resident blocks of `kern` with `threads`
// threads and `smem` bytes of dynamic shared memory, on device `dev`.
template <typename Kernel>
int resident_blocks(Kernel kern, int threads, int smem, int dev) {
    int sms = 0, occ = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    if (smem > 48 * 1024 && cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, threads, smem) != cudaSuccess || occ < 1) return 0;
    return sms * occ;
}

}  // namespace mss_host
