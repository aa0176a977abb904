// pipe_probe.cu -- throughput loops for the pipes the scan kernels are bound
// by (a measurement aid behind mss_probe_pipe_rates; no scan runs here).
//
// Every SM runs 8 CTAs of 256 threads (all 64 warp slots of an SM), each
// thread 8 independent dependency chains of one instruction kind:
//   0  fp32 fma            (FFMA, one lane operation per result)
//   1  packed fp32 fma     (f32x2, two lane operations per instruction)
//   2  ex2.approx          (the multi-function unit)
//   3  shfl.sync.bfly      (warp shuffle)
// Each CTA records its SM (%smid) and the SM cycle counter after a CTA
// barrier at the start and at the end; the host takes, per SM, the span from
// the first start to the last end of the CTAs it ran, so that staggered CTA
// starts count against the rate rather than inflating it.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <vector>

#include "../../include/mss.h"
#include "mss_device.cuh"

namespace mss {

constexpr int kProbeThreads = 256;
constexpr int kProbeCtasPerSm = 8;
constexpr int kProbeChains = 8;
constexpr int kProbeMaxCtas = 4096;

__device__ long long g_probe_t0[kProbeMaxCtas];
__device__ long long g_probe_t1[kProbeMaxCtas];
__device__ int g_probe_sm[kProbeMaxCtas];
__device__ float g_probe_sink[kProbeMaxCtas];

__device__ __forceinline__ int smid() {
    int r;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(r));
    return r;
}

template <int kKind>
__global__ void __launch_bounds__(kProbeThreads) pipe_probe_kernel(int iters, float a, float b) {
    float x[kProbeChains];
    float2 x2[kProbeChains];
#pragma unroll
    for (int i = 0; i < kProbeChains; ++i) {
        x[i] = 1e-3f * float(threadIdx.x) + 0.125f * float(i);
        x2[i] = make_float2(x[i], x[i] + 0.5f);
    }
    const float2 a2 = make_float2(a, a), b2 = make_float2(b, b);
    __syncthreads();
    const long long start = clock64();
#pragma unroll 8
    for (int k = 0; k < iters; ++k) {
#pragma unroll
        for (int i = 0; i < kProbeChains; ++i) {
            if constexpr (kKind == 0) x[i] = fmaf(x[i], a, b);
            if constexpr (kKind == 1) x2[i] = __ffma2_rn(x2[i], a2, b2);
            if constexpr (kKind == 2) x[i] = ex2_approx(-x[i]);
            if constexpr (kKind == 3) x[i] = __shfl_xor_sync(0xffffffffu, x[i], 1 << (i & 3));
        }
    }
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < kProbeChains; ++i) s += (kKind == 1) ? x2[i].x + x2[i].y : x[i];
    __syncthreads();
    const long long end = clock64();
    // the chains' results stay live through one store per CTA
    s = __shfl_xor_sync(0xffffffffu, s, 16) + s;
    if (threadIdx.x == 0) {
        g_probe_t0[blockIdx.x] = start;
        g_probe_t1[blockIdx.x] = end;
        g_probe_sm[blockIdx.x] = smid();
        g_probe_sink[blockIdx.x] = s;
    }
}

}  // namespace mss

namespace {

template <int kKind>
int run_probe(int n_ctas, int iters, cudaStream_t st) {
    mss::pipe_probe_kernel<kKind><<<n_ctas, mss::kProbeThreads, 0, st>>>(iters, 0.999f, 1e-3f);
    return cudaGetLastError() == cudaSuccess ? MSS_OK : MSS_ERR_CUDA;
}

// operations of one kind per thread, per chain and iteration (lane operations
// for the fma kinds, results for the others)
constexpr double kOpsPerStep[4] = {1.0, 2.0, 1.0, 1.0};

}  // namespace

extern "C" MSS_API int mss_probe_pipe_rates(double* rates, int n_rates, void* stream) {
    if (!rates) return MSS_ERR_NULL;
    if (n_rates < 0) return MSS_ERR_SHAPE;
    int dev = 0, n_sm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return MSS_ERR_CUDA;
    const int n_ctas = std::min(n_sm * mss::kProbeCtasPerSm, mss::kProbeMaxCtas);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // iterations sized for a fraction of a millisecond per kind at the
    // expected rates (the multi-function unit and shuffles are 8 and 4 times
    // slower than the fma pipe)
    const int iters[4] = {4096, 4096, 512, 1024};
    std::vector<long long> t0(n_ctas), t1(n_ctas);
    std::vector<int> sm(n_ctas);
    for (int kind = 0; kind < 4 && kind < n_rates; ++kind) {
        int rc = MSS_OK;
        switch (kind) {
            case 0: rc = run_probe<0>(n_ctas, iters[0], st); break;
            case 1: rc = run_probe<1>(n_ctas, iters[1], st); break;
            case 2: rc = run_probe<2>(n_ctas, iters[2], st); break;
            default: rc = run_probe<3>(n_ctas, iters[3], st); break;
        }
        if (rc != MSS_OK) return rc;
        if (cudaStreamSynchronize(st) != cudaSuccess ||
            cudaMemcpyFromSymbol(t0.data(), mss::g_probe_t0, sizeof(long long) * n_ctas) != cudaSuccess ||
            cudaMemcpyFromSymbol(t1.data(), mss::g_probe_t1, sizeof(long long) * n_ctas) != cudaSuccess ||
            cudaMemcpyFromSymbol(sm.data(), mss::g_probe_sm, sizeof(int) * n_ctas) != cudaSuccess)
            return MSS_ERR_CUDA;
        // per SM: threads it ran x operations per thread / (last end - first
        // start); SM ids need not be contiguous
        int n_ids = 0;
        for (int c = 0; c < n_ctas; ++c) n_ids = std::max(n_ids, sm[c] + 1);
        std::vector<long long> first(n_ids, -1), last(n_ids, -1);
        std::vector<int> ctas(n_ids, 0);
        for (int c = 0; c < n_ctas; ++c) {
            const int s = sm[c];
            if (s < 0) continue;
            first[s] = first[s] < 0 ? t0[c] : std::min(first[s], t0[c]);
            last[s] = std::max(last[s], t1[c]);
            ++ctas[s];
        }
        const double ops_per_thread = double(iters[kind]) * mss::kProbeChains * kOpsPerStep[kind];
        double sum = 0.0;
        int used = 0;
        for (int s = 0; s < n_ids; ++s) {
            if (ctas[s] == 0 || last[s] <= first[s]) continue;
            sum += double(ctas[s]) * mss::kProbeThreads * ops_per_thread / double(last[s] - first[s]);
            ++used;
        }
        rates[kind] = used ? sum / used : 0.0;
    }
    for (int kind = 4; kind < n_rates; ++kind) rates[kind] = 0.0;
    return MSS_OK;
}
