// ssd.cu -- host-side launch of the structured-state-space-duality forward
// pass (ssd_mma.cuh).
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "host_common.h"
#include "launch.h"
#include "ssd_chunked.cuh"
#include "ssd_mma.cuh"
#include "ssd_tc.cuh"

namespace mss_host {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 ssd_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// [batch][L][n1][n0] bf16 as a 4-D view (n0 innermost); box = 64 x 1 x 128 x 1
// (128 tokens of 64 elements), 128-byte swizzle.  Tokens past L read as zero
// and are not written by stores.
bool encode_token_major(CUtensorMap* m, const void* base, int64_t batch, int64_t L, int64_t n1, int64_t n0) {
    auto enc = ssd_encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[4] = {cuuint64_t(n0), cuuint64_t(n1), cuuint64_t(L), cuuint64_t(batch)};
    const cuuint64_t strides[3] = {cuuint64_t(n0 * 2), cuuint64_t(n1 * n0 * 2), cuuint64_t(L * n1 * n0 * 2)};
    const cuuint32_t box[4] = {64u, 1u, 128u, 1u};
    const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool kGate, bool kSoftplus>
int launch_ssd_tc_variant(const mss::SsdTcMaps& maps, const mss::SsdParams& p, int64_t unit0, int64_t units,
                          cudaStream_t s) {
    using Ly = mss::SsdTcLayout;
    auto kern = mss::ssd_tc_kernel<kGate, kSoftplus>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Ly::kSmemBytes) != cudaSuccess)
        return MSS_ERR_CUDA;
    if (units <= 0) return MSS_OK;
    if (units > 0x7fffffffLL) return MSS_ERR_SHAPE;
    kern<<<dim3(unsigned(units)), Ly::kThreads, Ly::kSmemBytes, s>>>(maps, p, unit0);
    return launch_status();
}

}  // namespace

// The tcgen05 kernel (dstate 128, headdim 64) on (batch, head) pairs
// unit0 .. unit0 + units - 1.
int launch_ssd_tc(const mss::SsdParams& p, int64_t unit0, int64_t units, cudaStream_t s) {
    if (p.batch > 0x7fffffffLL || p.seqlen > 0x7fffffffLL || p.nheads > 0x7fffffffLL) return MSS_ERR_SHAPE;
    mss::SsdTcMaps maps;
    std::memset(&maps, 0, sizeof(maps));
    if (!encode_token_major(&maps.x, p.x, p.batch, p.seqlen, p.nheads, 64) ||
        !encode_token_major(&maps.B, p.B, p.batch, p.seqlen, p.ngroups, 128) ||
        !encode_token_major(&maps.C, p.C, p.batch, p.seqlen, p.ngroups, 128))
        return MSS_ERR_CUDA;
    if (p.z)
        return p.softplus ? launch_ssd_tc_variant<true, true>(maps, p, unit0, units, s)
                          : launch_ssd_tc_variant<true, false>(maps, p, unit0, units, s);
    return p.softplus ? launch_ssd_tc_variant<false, true>(maps, p, unit0, units, s)
                      : launch_ssd_tc_variant<false, false>(maps, p, unit0, units, s);
}

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

// Cost model for choosing between the two forms, from B200 timings at 4096
// tokens (headdim 64, dstate 128).  The in-order kernel runs one CTA per
// (batch, head), up to two per SM: a wave in which some SM holds two takes
// about 1.24 times as long as one in which none does (460 vs 370 us).  The
// chunk-parallel passes spread every chunk over all SMs and take about 1.28
// of that lone-CTA time per SM's worth of heads (3.2 us per head on 148
// SMs).  Both scale with the sequence length, so the comparison does not.
bool ssd_chunked_pays(int64_t batch, int64_t nheads) {
    static std::mutex mu;
    static int cache[kMaxDevices] = {};
    const int64_t sms = per_device(cache, mu, [](int dev) {
        int n = 0;
        return cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess ? n : 0;
    });
    const int64_t pairs = batch * nheads;
    if (sms <= 0 || pairs <= 0) return false;
    const int64_t full = (pairs - 1) / (2 * sms), rest = pairs - full * 2 * sms;
    const int64_t in_order = full * 124 + (rest > sms ? 124 : 100);  // hundredths of a lone-CTA pass
    const int64_t chunked = 128 * pairs / sms;
    return chunked < in_order;
}

// The same choice against the tcgen05 kernel (dstate 128): one CTA per SM,
// about 0.32 of the warp-level kernel's lone-CTA time per wave of 148
// (118-126 us at 4096 tokens), while the passes take about 25 us plus
// 3.2 us per (batch, head) pair; the passes win up to about 28 pairs on 148
// SMs (B200, 4096 tokens: 61 against 117 us at 4 pairs, 72 against 119 at
// 16, 101 against 126 at 24, 121 against 119 at 32).
bool ssd_chunked_pays_tc(int64_t batch, int64_t nheads) {
    static std::mutex mu;
    static int cache[kMaxDevices] = {};
    const int64_t sms = per_device(cache, mu, [](int dev) {
        int n = 0;
        return cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess ? n : 0;
    });
    const int64_t pairs = batch * nheads;
    if (sms <= 0 || pairs <= 0) return false;
    const int64_t waves = (pairs + sms - 1) / sms;
    return 128 * pairs / sms + 7 < 32 * waves;  // hundredths of a lone warp-level pass
}

int64_t ssd_workspace_bytes(int64_t batch, int64_t seqlen, int64_t nheads, int64_t dstate) {
    const int64_t nc = (seqlen + 63) / 64;
    const int64_t per_chunk = dstate * 64 * (4 + 2) + 4;  // S_local fp32, S_in bf16, decay
    return batch * nheads * nc * per_chunk;
}

template <int NS, bool kGate, bool kSoftplus>
int launch_ssd_chunked_variant(const mss::SsdParams& p, void* workspace, int64_t unit0, int64_t units,
                               cudaStream_t s) {
    using CL = mss::SsdChunkLayout<NS>;
    const int64_t nc = (p.seqlen + 63) / 64, bh = units;
    if (units <= 0) return MSS_OK;
    if (nc > 0x7fffffffLL || units > 65535) return MSS_ERR_SHAPE;
    float* Sl = static_cast<float*>(workspace);
    mss::bf16_t* Sin = reinterpret_cast<mss::bf16_t*>(Sl + bh * nc * NS * 64);
    float* decay = reinterpret_cast<float*>(Sin + bh * nc * NS * 64);
    auto k1 = mss::ssd_chunk_state_kernel<NS, kSoftplus>;
    auto k3 = mss::ssd_chunk_out_kernel<NS, kGate, kSoftplus>;
    if (cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, CL::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(k3, cudaFuncAttributeMaxDynamicSharedMemorySize, CL::kSmemBytes) != cudaSuccess)
        return MSS_ERR_CUDA;
    const dim3 grid{unsigned(nc), unsigned(units), 1u};
    k1<<<grid, 128, CL::kSmemBytes, s>>>(p, Sl, decay, unit0);
    int rc = launch_status();
    if (rc != MSS_OK) return rc;
    mss::ssd_state_pass_kernel<NS><<<dim3(unsigned(bh), unsigned(NS * 64 / 256)), 256, 0, s>>>(p, Sl, decay, Sin, nc,
                                                                                             unit0);
    rc = launch_status();
    if (rc != MSS_OK) return rc;
    k3<<<grid, 128, CL::kSmemBytes, s>>>(p, Sin, unit0);
    return launch_status();
}

template <int NS>
int launch_ssd_chunked_n(const mss::SsdParams& p, void* ws, int64_t unit0, int64_t units, cudaStream_t s) {
    if (p.z)
        return p.softplus ? launch_ssd_chunked_variant<NS, true, true>(p, ws, unit0, units, s)
                          : launch_ssd_chunked_variant<NS, true, false>(p, ws, unit0, units, s);
    return p.softplus ? launch_ssd_chunked_variant<NS, false, true>(p, ws, unit0, units, s)
                      : launch_ssd_chunked_variant<NS, false, false>(p, ws, unit0, units, s);
}

// The chunk-parallel passes on (batch, head) pairs unit0 .. unit0 + units - 1;
// the workspace holds those units' chunk states only.
int launch_ssd_chunked(const mss::SsdParams& p, int dstate, void* workspace, int64_t unit0, int64_t units,
                       cudaStream_t s) {
    return dstate == 64 ? launch_ssd_chunked_n<64>(p, workspace, unit0, units, s)
                        : launch_ssd_chunked_n<128>(p, workspace, unit0, units, s);
}

// For the tcgen05 kernel (one CTA per SM): the (batch, head) pairs past the
// last full wave of CTAs when they are few enough that the chunk-parallel
// passes finish them clearly sooner than a wave of their own (B200, 4096
// tokens: 4 past a wave, 160 against 226 us; 12 past, 201-205 against
// 255 us; 28 past, 238 against 226 us): at most one in nine SMs' worth,
// 16 pairs on 148 SMs; 0 otherwise.
int64_t ssd_tc_tail_units(int64_t batch, int64_t nheads) {
    static std::mutex mu;
    static int cache[kMaxDevices] = {};
    const int64_t sms = per_device(cache, mu, [](int dev) {
        int n = 0;
        return cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess ? n : 0;
    });
    const int64_t pairs = batch * nheads;
    if (sms <= 0 || pairs <= sms) return 0;
    const int64_t tail = pairs % sms;
    return tail > 0 && tail * 9 <= sms ? tail : 0;
}

}  // namespace mss_host
