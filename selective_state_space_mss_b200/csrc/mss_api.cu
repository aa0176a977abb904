// mss_api.cu -- the C ABI of libmss.so (declared in include/mss.h): argument
// checks on the host and dispatch to the launchers of launch.h.  No
// allocation, no host synchronisation on the forward and decode paths.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/mss.h"
#include "host_common.h"
#include "launch.h"
#include "mss_device.cuh"
#include "mss_params.h"

namespace {

using mss::bf16_t;
using namespace mss_host;

constexpr unsigned kScanFlags =
    MSS_FLAG_GENERAL_A | MSS_FLAG_SIMPLE | MSS_FLAG_NO_SPLIT | MSS_FLAG_ZOH_INPUT | MSS_FLAG_SELFTEST_TIMEOUT |
    MSS_FLAG_PAIR_LANES;
constexpr unsigned kBwdFlags = MSS_FLAG_GENERAL_A | MSS_FLAG_SIMPLE | MSS_FLAG_ZOH_INPUT | MSS_FLAG_SAVED_STATES;

// The device error word (one per device, in the library image): kernels
// whose bounded waits give up set it through the address in their
// parameter block; mss_get_device_error reads and clears it.
__device__ unsigned int g_mss_device_error = 0u;

// Address of a __device__ symbol on the current device, looked up once.
template <typename Symbol>
void* symbol_address(const Symbol& sym, void* (&cache)[kMaxDevices], std::mutex& mu) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!cache[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, sym) != cudaSuccess) return nullptr;
        cache[dev] = p;
    }
    return cache[dev];
}

unsigned int* device_error_word() {
    static std::mutex mu;
    static void* cache[kMaxDevices] = {};
    return static_cast<unsigned int*>(symbol_address(g_mss_device_error, cache, mu));
}

// The causal convolution's arguments (mss_scan_fwd_conv).
struct ConvArgs {
    const float* w;
    const float* b;
    int K;
    const void* state_in;
    void* state_out;
};

// The forward pass behind every mss_scan_fwd* entry point; cv = nullptr
// without the convolution; save: also store the backward pass's states
// (mss_scan_fwd_save).
int scan_fwd_impl(const ConvArgs* cv, const void* u, const void* delta, const float* A, const void* B,
                  const void* C, const float* D, const void* z, const float* delta_bias,
                  int softplus_flag, const float* initial_state, void* y, float* last_state,
                  int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                  int dtype, unsigned flags, void* workspace, int64_t workspace_bytes, bool save, void* states,
                  int64_t states_bytes, void* stream) {
    if (dtype != MSS_DTYPE_F32 && dtype != MSS_DTYPE_BF16) return MSS_ERR_DTYPE;
    if (flags & ~kScanFlags) return MSS_ERR_FLAGS;
    if (batch < 0 || dim < 0 || seqlen < 0 || workspace_bytes < 0 || states_bytes < 0) return MSS_ERR_SHAPE;
    if (!valid_n(dstate)) return MSS_ERR_UNSUPPORTED_N;
    const int64_t esz = dtype == MSS_DTYPE_BF16 ? 2 : 4;
    int64_t rows, seq_elems, seq_bytes, bc_elems, bc_bytes, st_elems, st_bytes;
    if (!mul_ok(batch, dim, &rows) || !mul_ok(rows, seqlen, &seq_elems) ||
        !mul_ok(seq_elems, esz, &seq_bytes) || !mul_ok(batch * dstate, seqlen, &bc_elems) ||
        !mul_ok(bc_elems, esz, &bc_bytes) || !mul_ok(rows, dstate, &st_elems) ||
        !mul_ok(st_elems, 4, &st_bytes) || rows > (int64_t(1) << 40))
        return MSS_ERR_SHAPE;
    const int K = cv ? cv->K : 0;
    if (cv && (K < 1 || K > 4)) return MSS_ERR_SHAPE;
    const int64_t cs_bytes = rows * (K > 0 ? K - 1 : 0) * esz;  // conv state, checked with rows below
    if (rows == 0) return MSS_OK;
    // with no tokens the sequence tensors are empty and may be NULL
    if (!A || (seqlen > 0 && (!u || !delta || !B || !C || !y))) return MSS_ERR_NULL;
    if (cv && !cv->w) return MSS_ERR_NULL;
    const void* io[] = {u, delta, B, C, z, y, cv ? cv->state_in : nullptr, cv ? cv->state_out : nullptr};
    for (const void* p : io)
        if (p && !aligned(p, size_t(esz))) return MSS_ERR_ALIGN;
    const void* fp[] = {A, D, delta_bias, last_state, initial_state, workspace, cv ? cv->w : nullptr,
                        cv ? cv->b : nullptr};
    for (const void* p : fp)
        if (p && !aligned(p, 4)) return MSS_ERR_ALIGN;
    // the saved states: the backward pass's workspace size for these arguments
    int64_t need_states = 0;
    if (save) {
        if (cv) return MSS_ERR_PATH;
        need_states = with_n(dstate, [&](auto nc) -> int64_t {
            constexpr int N = decltype(nc)::value;
            return dtype == MSS_DTYPE_BF16 ? backward_workspace_bytes<bf16_t, N>(batch, dim, seqlen, flags)
                                           : backward_workspace_bytes<float, N>(batch, dim, seqlen, flags);
        });
        if (need_states > 0 && (!states || states_bytes < need_states)) return MSS_ERR_WORKSPACE;
        if (states && !aligned(states, 16)) return MSS_ERR_ALIGN;
    }
    // outputs (y, last_state, workspace, states) must not overlap inputs or each other
    const int64_t ws = workspace ? workspace_bytes : 0;
    const int64_t ss = save && states ? states_bytes : 0;
    struct Range { const void* p; int64_t n; };
    const Range outs[] = {{y, seq_bytes}, {last_state, st_bytes}, {workspace, ws},
                          {cv ? cv->state_out : nullptr, cs_bytes}, {save ? states : nullptr, ss}};
    const Range ins[] = {{u, seq_bytes}, {delta, seq_bytes}, {z, seq_bytes}, {B, bc_bytes}, {C, bc_bytes},
                         {A, dim * dstate * 4}, {D, dim * 4}, {delta_bias, dim * 4},
                         {initial_state, st_bytes}, {cv ? cv->w : nullptr, dim * K * 4},
                         {cv ? cv->b : nullptr, dim * 4}, {cv ? cv->state_in : nullptr, cs_bytes}};
    for (const Range& o : outs) {
        for (const Range& i : ins)
            if (overlaps(o.p, o.n, i.p, i.n)) return MSS_ERR_ALIAS;
        for (const Range& o2 : outs)
            if (&o != &o2 && overlaps(o.p, o.n, o2.p, o2.n)) return MSS_ERR_ALIAS;
    }

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (seqlen == 0) {
        // no tokens: the final state is the starting state
        if (last_state) {
            const cudaError_t e = initial_state
                ? cudaMemcpyAsync(last_state, initial_state, size_t(st_bytes), cudaMemcpyDeviceToDevice, s)
                : cudaMemsetAsync(last_state, 0, size_t(st_bytes), s);
            if (e != cudaSuccess) return MSS_ERR_CUDA;
        }
        // and the conv state the one it was handed
        if (cv && cv->state_out && cs_bytes > 0) {
            const cudaError_t e = cv->state_in
                ? cudaMemcpyAsync(cv->state_out, cv->state_in, size_t(cs_bytes), cudaMemcpyDeviceToDevice, s)
                : cudaMemsetAsync(cv->state_out, 0, size_t(cs_bytes), s);
            if (e != cudaSuccess) return MSS_ERR_CUDA;
        }
        return MSS_OK;
    }
    mss::ScanParams p{};
    p.u = u; p.delta = delta; p.A = A; p.B = B; p.C = C; p.D = D; p.z = z; p.delta_bias = delta_bias;
    p.y = y; p.last_state = last_state; p.batch = batch; p.dim = dim; p.seqlen = seqlen;
    p.softplus = softplus_flag ? 1 : 0; p.initial_state = initial_state;
    p.agg = nullptr; p.seg_len = seqlen; p.n_seg = 1;
    p.zoh = (flags & MSS_FLAG_ZOH_INPUT) ? 1 : 0;
    if (cv) {
        p.conv_w = cv->w; p.conv_b = cv->b; p.conv_state_in = cv->state_in; p.conv_state_out = cv->state_out;
        p.conv_width = K;
    }
    // saved states are written by the tiled kernel only
    if (save && !seq_eligible(p, dstate, int(esz), flags)) return MSS_ERR_PATH;
    if (!(p.err = device_error_word())) return MSS_ERR_CUDA;
    return with_n(dstate, [&](auto nc) {
        constexpr int N = decltype(nc)::value;
        float* st = static_cast<float*>(states);
        if (save)
            return dtype == MSS_DTYPE_BF16 ? launch_forward_save<bf16_t, N>(p, flags, workspace, ws, st, s)
                                           : launch_forward_save<float, N>(p, flags, workspace, ws, st, s);
        return dtype == MSS_DTYPE_BF16 ? launch_forward<bf16_t, N>(p, flags, workspace, ws, s)
                                       : launch_forward<float, N>(p, flags, workspace, ws, s);
    });
}

// The decode step behind every mss_state_update* entry point; conv_width 0
// without the convolution.
int state_update_impl(float* state, void* conv_state, const float* conv_w, const float* conv_b, int conv_width,
                      const void* u, const void* delta, const float* A, const void* B, const void* C,
                      const float* D, const void* z, const float* delta_bias, int softplus_flag, void* y,
                      int64_t batch, int64_t dim, int64_t dstate, int dtype, unsigned flags, void* stream) {
    if (dtype != MSS_DTYPE_F32 && dtype != MSS_DTYPE_BF16) return MSS_ERR_DTYPE;
    if (flags & ~unsigned(MSS_FLAG_ZOH_INPUT)) return MSS_ERR_FLAGS;
    if (batch < 0 || dim < 0) return MSS_ERR_SHAPE;
    if (!valid_n(dstate)) return MSS_ERR_UNSUPPORTED_N;
    const int64_t esz = dtype == MSS_DTYPE_BF16 ? 2 : 4;
    int64_t rows, st_elems, st_bytes;
    if (!mul_ok(batch, dim, &rows) || !mul_ok(rows, dstate, &st_elems) ||
        !mul_ok(st_elems, 4, &st_bytes) || rows > (int64_t(1) << 40))
        return MSS_ERR_SHAPE;
    const int K = conv_width;
    if (K < 0 || K > 4) return MSS_ERR_SHAPE;
    const int64_t cs_bytes = rows * (K > 0 ? K - 1 : 0) * esz;
    if (rows == 0) return MSS_OK;
    if (!state || !u || !delta || !A || !B || !C || !y) return MSS_ERR_NULL;
    if (K > 0 && (!conv_w || (K > 1 && !conv_state))) return MSS_ERR_NULL;
    const void* io[] = {u, delta, B, C, z, y, K > 1 ? conv_state : nullptr};
    for (const void* p : io)
        if (p && !aligned(p, size_t(esz))) return MSS_ERR_ALIGN;
    const void* fp[] = {state, A, D, delta_bias, K > 0 ? conv_w : nullptr, K > 0 ? conv_b : nullptr};
    for (const void* p : fp)
        if (p && !aligned(p, 4)) return MSS_ERR_ALIGN;
    const int64_t io_bytes = rows * esz, bc_bytes = batch * dstate * esz;
    const void* in_io[] = {u, delta, z};
    for (const void* p : in_io)
        if (overlaps(y, io_bytes, p, io_bytes) || overlaps(state, st_bytes, p, io_bytes)) return MSS_ERR_ALIAS;
    const void* in_bc[] = {B, C};
    for (const void* p : in_bc)
        if (overlaps(y, io_bytes, p, bc_bytes) || overlaps(state, st_bytes, p, bc_bytes)) return MSS_ERR_ALIAS;
    const void* params[] = {D, delta_bias};
    for (const void* p : params)
        if (overlaps(y, io_bytes, p, dim * 4) || overlaps(state, st_bytes, p, dim * 4)) return MSS_ERR_ALIAS;
    if (overlaps(y, io_bytes, A, dim * dstate * 4) || overlaps(state, st_bytes, A, dim * dstate * 4) ||
        overlaps(y, io_bytes, state, st_bytes))
        return MSS_ERR_ALIAS;
    if (K > 0 && (overlaps(y, io_bytes, conv_w, dim * K * 4) || overlaps(state, st_bytes, conv_w, dim * K * 4) ||
                  overlaps(y, io_bytes, conv_b, dim * 4) || overlaps(state, st_bytes, conv_b, dim * 4)))
        return MSS_ERR_ALIAS;
    if (K > 1) {
        // the conv state is written in place: it must not overlap anything else
        struct Range { const void* p; int64_t n; };
        const Range others[] = {{y, io_bytes}, {state, st_bytes}, {u, io_bytes}, {delta, io_bytes}, {z, io_bytes},
                                {B, bc_bytes}, {C, bc_bytes}, {A, dim * dstate * 4}, {D, dim * 4},
                                {delta_bias, dim * 4}, {conv_w, dim * K * 4}, {conv_b, dim * 4}};
        for (const Range& o : others)
            if (overlaps(conv_state, cs_bytes, o.p, o.n)) return MSS_ERR_ALIAS;
    }

    mss::StepParams p{state, u, delta, A, B, C, D, z, delta_bias, y, batch, dim, softplus_flag ? 1 : 0,
                      (flags & MSS_FLAG_ZOH_INPUT) ? 1 : 0, 0, nullptr, conv_w, conv_b, conv_state, K};
    if (!(p.err = device_error_word())) return MSS_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return with_n(dstate, [&](auto nc) {
        constexpr int N = decltype(nc)::value;
        return dtype == MSS_DTYPE_BF16 ? launch_decode<bf16_t, N>(p, s) : launch_decode<float, N>(p, s);
    });
}

}  // namespace

extern "C" {

int mss_version(void) { return MSS_VERSION; }

const char* mss_strerror(int code) {
    switch (code) {
        case MSS_OK: return "success";
        case MSS_ERR_NULL: return "a required pointer is NULL";
        case MSS_ERR_SHAPE: return "a size is negative or a size product overflows";
        case MSS_ERR_UNSUPPORTED_N: return "dstate must be 1, 2, 4, 8 or 16";
        case MSS_ERR_DTYPE: return "dtype must be MSS_DTYPE_F32 or MSS_DTYPE_BF16";
        case MSS_ERR_ALIGN: return "a pointer is not aligned to its element size";
        case MSS_ERR_CUDA: return "a CUDA call failed";
        case MSS_ERR_DEVICE_TIMEOUT: return "a bounded wait inside a kernel gave up";
        case MSS_ERR_FLAGS: return "unknown bits in flags";
        case MSS_ERR_ALIAS: return "an output overlaps an input";
        case MSS_ERR_SCRATCH: return "the sequence split needs more than the library's fixed scratch holds";
        case MSS_ERR_WORKSPACE: return "no workspace, or a workspace smaller than the call needs";
        case MSS_ERR_PATH: return "saved states need the tiled kernels, which these sizes, flags or alignments do not take";
        default: return "unknown status code";
    }
}

int mss_scan_fwd_ex2(const void* u, const void* delta, const float* A, const void* B,
                     const void* C, const float* D, const void* z, const float* delta_bias,
                     int softplus_flag, const float* initial_state, void* y, float* last_state,
                     int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                     int dtype, unsigned flags, void* workspace, int64_t workspace_bytes, void* stream) {
    return scan_fwd_impl(nullptr, u, delta, A, B, C, D, z, delta_bias, softplus_flag, initial_state, y, last_state,
                         batch, dim, dstate, seqlen, dtype, flags, workspace, workspace_bytes, false, nullptr, 0,
                         stream);
}

int mss_scan_fwd_save(const void* u, const void* delta, const float* A, const void* B,
                      const void* C, const float* D, const void* z, const float* delta_bias,
                      int softplus_flag, const float* initial_state, void* y, float* last_state,
                      int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                      int dtype, unsigned flags, void* workspace, int64_t workspace_bytes,
                      void* states, int64_t states_bytes, void* stream) {
    return scan_fwd_impl(nullptr, u, delta, A, B, C, D, z, delta_bias, softplus_flag, initial_state, y, last_state,
                         batch, dim, dstate, seqlen, dtype, flags, workspace, workspace_bytes, true, states,
                         states_bytes, stream);
}

int mss_scan_fwd_conv(const void* x, const float* conv_w, const float* conv_b, int conv_width,
                      const void* conv_state_in, void* conv_state_out,
                      const void* delta, const float* A, const void* B, const void* C, const float* D,
                      const void* z, const float* delta_bias, int softplus_flag, const float* initial_state,
                      void* y, float* last_state, int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                      int dtype, unsigned flags, void* workspace, int64_t workspace_bytes, void* stream) {
    const ConvArgs cv{conv_w, conv_b, conv_width, conv_state_in, conv_state_out};
    return scan_fwd_impl(&cv, x, delta, A, B, C, D, z, delta_bias, softplus_flag, initial_state, y, last_state,
                         batch, dim, dstate, seqlen, dtype, flags, workspace, workspace_bytes, false, nullptr, 0,
                         stream);
}

int64_t mss_scan_fwd_workspace_size(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen, int dtype,
                                    unsigned flags) {
    if (dtype != MSS_DTYPE_F32 && dtype != MSS_DTYPE_BF16) return MSS_ERR_DTYPE;
    if (flags & ~kScanFlags) return MSS_ERR_FLAGS;
    if (batch < 0 || dim < 0 || seqlen < 0) return MSS_ERR_SHAPE;
    if (!valid_n(dstate)) return MSS_ERR_UNSUPPORTED_N;
    int64_t rows;
    if (!mul_ok(batch, dim, &rows) || rows > (int64_t(1) << 40)) return MSS_ERR_SHAPE;
    const int64_t esz = dtype == MSS_DTYPE_BF16 ? 2 : 4;
    if (rows == 0 || seqlen == 0 || (flags & (MSS_FLAG_SIMPLE | MSS_FLAG_NO_SPLIT)) ||
        (dstate != 4 && dstate != 8 && dstate != 16) || (seqlen * esz) % 16 != 0)
        return 0;
    return with_n(dstate, [&](auto nc) -> int64_t {
        constexpr int N = decltype(nc)::value;
        return dtype == MSS_DTYPE_BF16 ? forward_workspace_bytes<bf16_t, N>(batch, dim, seqlen)
                                       : forward_workspace_bytes<float, N>(batch, dim, seqlen);
    });
}

int mss_scan_fwd_ex(const void* u, const void* delta, const float* A, const void* B,
                    const void* C, const float* D, const void* z, const float* delta_bias,
                    int softplus_flag, void* y, float* last_state,
                    int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                    int dtype, unsigned flags, void* stream) {
    return mss_scan_fwd_ex2(u, delta, A, B, C, D, z, delta_bias, softplus_flag, nullptr, y, last_state,
                            batch, dim, dstate, seqlen, dtype, flags, nullptr, 0, stream);
}

int mss_scan_fwd(const void* u, const void* delta, const float* A, const void* B,
                 const void* C, const float* D, const void* z, const float* delta_bias,
                 int softplus_flag, void* y, float* last_state,
                 int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                 int dtype, void* stream) {
    return mss_scan_fwd_ex2(u, delta, A, B, C, D, z, delta_bias, softplus_flag, nullptr, y, last_state,
                            batch, dim, dstate, seqlen, dtype, 0u, nullptr, 0, stream);
}

int mss_state_update(float* state, const void* u, const void* delta, const float* A,
                     const void* B, const void* C, const float* D, const void* z,
                     const float* delta_bias, int softplus_flag, void* y,
                     int64_t batch, int64_t dim, int64_t dstate, int dtype, void* stream) {
    return mss_state_update_ex(state, u, delta, A, B, C, D, z, delta_bias, softplus_flag, y,
                               batch, dim, dstate, dtype, 0u, stream);
}

int mss_state_update_ex(float* state, const void* u, const void* delta, const float* A,
                        const void* B, const void* C, const float* D, const void* z,
                        const float* delta_bias, int softplus_flag, void* y,
                        int64_t batch, int64_t dim, int64_t dstate, int dtype, unsigned flags, void* stream) {
    return state_update_impl(state, nullptr, nullptr, nullptr, 0, u, delta, A, B, C, D, z, delta_bias,
                             softplus_flag, y, batch, dim, dstate, dtype, flags, stream);
}

int mss_state_update_conv(float* state, void* conv_state, const void* x, const float* conv_w,
                          const float* conv_b, int conv_width, const void* delta, const float* A,
                          const void* B, const void* C, const float* D, const void* z,
                          const float* delta_bias, int softplus_flag, void* y,
                          int64_t batch, int64_t dim, int64_t dstate, int dtype, unsigned flags, void* stream) {
    if (conv_width < 1) return MSS_ERR_SHAPE;
    return state_update_impl(state, conv_state, conv_w, conv_b, conv_width, x, delta, A, B, C, D, z, delta_bias,
                             softplus_flag, y, batch, dim, dstate, dtype, flags, stream);
}

int mss_scan_bwd(const void* u, const void* delta, const float* A, const void* B, const void* C,
                 const float* D, const void* z, const float* delta_bias, int softplus_flag,
                 const float* initial_state, const void* dy, const float* dlast,
                 void* du, void* ddelta, void* dz, float* dA, float* dB, float* dC, float* dD,
                 float* dbias, float* dinit, int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                 int dtype, unsigned flags, void* workspace, int64_t workspace_bytes, void* stream) {
    if (dtype != MSS_DTYPE_F32 && dtype != MSS_DTYPE_BF16) return MSS_ERR_DTYPE;
    if (flags & ~kBwdFlags) return MSS_ERR_FLAGS;
    if (batch < 0 || dim < 0 || seqlen < 0 || workspace_bytes < 0) return MSS_ERR_SHAPE;
    if (!valid_n(dstate)) return MSS_ERR_UNSUPPORTED_N;
    const int64_t esz = dtype == MSS_DTYPE_BF16 ? 2 : 4;
    int64_t rows, seq_elems, seq_bytes, bc_elems, bcf_bytes, bc_bytes, st_elems, st_bytes;
    if (!mul_ok(batch, dim, &rows) || !mul_ok(rows, seqlen, &seq_elems) ||
        !mul_ok(seq_elems, esz, &seq_bytes) || !mul_ok(batch * dstate, seqlen, &bc_elems) ||
        !mul_ok(bc_elems, esz, &bc_bytes) || !mul_ok(bc_elems, 4, &bcf_bytes) || !mul_ok(rows, dstate, &st_elems) ||
        !mul_ok(st_elems, 4, &st_bytes) || rows > (int64_t(1) << 40))
        return MSS_ERR_SHAPE;
    if (rows == 0) return MSS_OK;
    if (!A || !dA || (seqlen > 0 && (!u || !delta || !B || !C || !dy || !du || !ddelta || !dB || !dC)) ||
        (z && seqlen > 0 && !dz))
        return MSS_ERR_NULL;
    const void* io[] = {u, delta, B, C, z, dy, du, ddelta, dz};
    for (const void* p : io)
        if (p && !aligned(p, size_t(esz))) return MSS_ERR_ALIGN;
    const void* fp[] = {A, D, delta_bias, initial_state, dlast, dA, dB, dC, dD, dbias, dinit, workspace};
    for (const void* p : fp)
        if (p && !aligned(p, 4)) return MSS_ERR_ALIGN;
    const int64_t ws = workspace ? workspace_bytes : 0;
    struct Range { const void* p; int64_t n; };
    const Range outs[] = {{du, seq_bytes}, {ddelta, seq_bytes}, {z ? dz : nullptr, seq_bytes}, {dA, dim * dstate * 4},
                          {dB, bcf_bytes}, {dC, bcf_bytes}, {dD, dim * 4}, {dbias, dim * 4}, {dinit, st_bytes},
                          {workspace, ws}};
    const Range ins[] = {{u, seq_bytes}, {delta, seq_bytes}, {z, seq_bytes}, {dy, seq_bytes}, {B, bc_bytes},
                         {C, bc_bytes}, {A, dim * dstate * 4}, {D, dim * 4}, {delta_bias, dim * 4},
                         {initial_state, st_bytes}, {dlast, st_bytes}};
    for (const Range& o : outs) {
        for (const Range& i : ins)
            if (overlaps(o.p, o.n, i.p, i.n)) return MSS_ERR_ALIAS;
        for (const Range& o2 : outs)
            if (&o != &o2 && overlaps(o.p, o.n, o2.p, o2.n)) return MSS_ERR_ALIAS;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (seqlen == 0) {
        // no tokens: nothing flows through the recurrence
        if (cudaMemsetAsync(dA, 0, size_t(dim * dstate * 4), s) != cudaSuccess ||
            (dD && cudaMemsetAsync(dD, 0, size_t(dim * 4), s) != cudaSuccess) ||
            (dbias && cudaMemsetAsync(dbias, 0, size_t(dim * 4), s) != cudaSuccess))
            return MSS_ERR_CUDA;
        if (dinit) {
            const cudaError_t e = dlast ? cudaMemcpyAsync(dinit, dlast, size_t(st_bytes), cudaMemcpyDeviceToDevice, s)
                                        : cudaMemsetAsync(dinit, 0, size_t(st_bytes), s);
            if (e != cudaSuccess) return MSS_ERR_CUDA;
        }
        return MSS_OK;
    }
    mss::ScanParams p{};
    p.u = u; p.delta = delta; p.A = A; p.B = B; p.C = C; p.D = D; p.z = z; p.delta_bias = delta_bias;
    p.batch = batch; p.dim = dim; p.seqlen = seqlen; p.softplus = softplus_flag ? 1 : 0;
    p.initial_state = initial_state; p.seg_len = seqlen; p.n_seg = 1;
    p.zoh = (flags & MSS_FLAG_ZOH_INPUT) ? 1 : 0;
    if (flags & MSS_FLAG_SAVED_STATES) {
        // the saved states are in the tiled kernels' layout: the call must take them
        bool tiled = seq_eligible(p, dstate, int(esz), flags);
        const void* g16[] = {dy, du, ddelta, z ? dz : nullptr, dB, dC};
        for (const void* g : g16)
            if (g && !aligned(g, 16)) tiled = false;
        if (!tiled) return MSS_ERR_PATH;
    }
    if (!(p.err = device_error_word())) return MSS_ERR_CUDA;
    mss::BwdParams q{};
    q.u = u; q.delta = delta; q.A = A; q.B = B; q.C = C; q.D = D; q.z = z; q.delta_bias = delta_bias;
    q.dy = dy; q.dlast = dlast; q.du = du; q.ddelta = ddelta; q.dz = z ? dz : nullptr; q.dA = dA; q.dB = dB;
    q.dC = dC; q.dD = dD; q.dbias = dbias; q.dinit = dinit; q.batch = batch; q.dim = dim; q.seqlen = seqlen;
    q.softplus = p.softplus; q.err = p.err;
    return with_n(dstate, [&](auto nc) {
        constexpr int N = decltype(nc)::value;
        return dtype == MSS_DTYPE_BF16 ? launch_backward<bf16_t, N>(p, q, flags, workspace, ws, s)
                                       : launch_backward<float, N>(p, q, flags, workspace, ws, s);
    });
}

int64_t mss_scan_bwd_workspace_size(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen, int dtype,
                                    unsigned flags) {
    if (dtype != MSS_DTYPE_F32 && dtype != MSS_DTYPE_BF16) return MSS_ERR_DTYPE;
    if (flags & ~kBwdFlags) return MSS_ERR_FLAGS;
    if (batch < 0 || dim < 0 || seqlen < 0) return MSS_ERR_SHAPE;
    if (!valid_n(dstate)) return MSS_ERR_UNSUPPORTED_N;
    int64_t rows, elems;
    if (!mul_ok(batch, dim, &rows) || rows > (int64_t(1) << 40) || !mul_ok(rows, seqlen, &elems) ||
        !mul_ok(elems, dstate * 4, &elems))
        return MSS_ERR_SHAPE;
    return with_n(dstate, [&](auto nc) -> int64_t {
        constexpr int N = decltype(nc)::value;
        return dtype == MSS_DTYPE_BF16 ? backward_workspace_bytes<bf16_t, N>(batch, dim, seqlen, flags)
                                       : backward_workspace_bytes<float, N>(batch, dim, seqlen, flags);
    });
}

int mss_ssd_fwd(const void* x, const void* dt, const float* A, const void* B, const void* C, const float* D,
                const void* z, const float* dt_bias, int softplus_flag, const float* initial_state, void* y,
                float* last_state, int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                int64_t ngroups, int64_t dstate, int dtype, void* stream) {
    return mss_ssd_fwd_ex(x, dt, A, B, C, D, z, dt_bias, softplus_flag, initial_state, y, last_state, batch, seqlen,
                          nheads, headdim, ngroups, dstate, dtype, nullptr, 0, stream);
}

int64_t mss_ssd_fwd_workspace_size(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim, int64_t ngroups,
                                   int64_t dstate) {
    return mss_ssd_fwd_workspace_size_ex(batch, seqlen, nheads, headdim, ngroups, dstate, 0u);
}

int64_t mss_ssd_fwd_workspace_size_ex(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                                      int64_t ngroups, int64_t dstate, unsigned flags) {
    if (flags & ~unsigned(MSS_SSD_FLAG_WARP_MMA)) return MSS_ERR_FLAGS;
    if (batch < 0 || seqlen < 0 || nheads < 1 || ngroups < 1 || nheads % ngroups != 0 || headdim != 64 ||
        (dstate != 64 && dstate != 128))
        return MSS_ERR_SHAPE;
    int64_t bh, tok;
    if (!mul_ok(batch, nheads, &bh) || !mul_ok(bh, seqlen, &tok) || tok > (int64_t(1) << 40)) return MSS_ERR_SHAPE;
    // dstate 128 runs the tcgen05 kernel in order unless the warp-level kernels
    // are asked for, or so few (batch, head) pairs leave most SMs idle that
    // the chunk-parallel passes are faster
    const bool tc = dstate == 128 && !(flags & MSS_SSD_FLAG_WARP_MMA);
    if (seqlen == 0) return 0;
    if (tc ? ssd_chunked_pays_tc(batch, nheads) : ssd_chunked_pays(batch, nheads))
        return ssd_workspace_bytes(batch, seqlen, nheads, dstate);
    // or only the pairs past the tcgen05 kernel's last full wave
    const int64_t tail = tc ? ssd_tc_tail_units(batch, nheads) : 0;
    return tail > 0 ? ssd_workspace_bytes(1, seqlen, tail, dstate) : 0;
}

int mss_ssd_fwd_ex(const void* x, const void* dt, const float* A, const void* B, const void* C, const float* D,
                   const void* z, const float* dt_bias, int softplus_flag, const float* initial_state, void* y,
                   float* last_state, int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                   int64_t ngroups, int64_t dstate, int dtype, void* workspace, int64_t workspace_bytes,
                   void* stream) {
    return mss_ssd_fwd_ex2(x, dt, A, B, C, D, z, dt_bias, softplus_flag, initial_state, y, last_state, batch, seqlen,
                           nheads, headdim, ngroups, dstate, dtype, 0u, workspace, workspace_bytes, stream);
}

int mss_ssd_fwd_ex2(const void* x, const void* dt, const float* A, const void* B, const void* C, const float* D,
                    const void* z, const float* dt_bias, int softplus_flag, const float* initial_state, void* y,
                    float* last_state, int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                    int64_t ngroups, int64_t dstate, int dtype, unsigned flags, void* workspace,
                    int64_t workspace_bytes, void* stream) {
    if (flags & ~unsigned(MSS_SSD_FLAG_WARP_MMA)) return MSS_ERR_FLAGS;
    if (workspace_bytes < 0) return MSS_ERR_SHAPE;
    if (dtype != MSS_DTYPE_BF16) return MSS_ERR_DTYPE;  // the tensor-core path takes bf16 io
    if (batch < 0 || seqlen < 0 || nheads < 1 || ngroups < 1 || nheads % ngroups != 0 || headdim != 64 ||
        (dstate != 64 && dstate != 128))
        return MSS_ERR_SHAPE;
    int64_t tok, xe, xbytes, bce, bcbytes, ste, stbytes, dtbytes;
    if (!mul_ok(batch, seqlen, &tok) || !mul_ok(tok, nheads * headdim, &xe) || !mul_ok(xe, 2, &xbytes) ||
        !mul_ok(tok, ngroups * dstate, &bce) || !mul_ok(bce, 2, &bcbytes) ||
        !mul_ok(batch * nheads, dstate * headdim, &ste) || !mul_ok(ste, 4, &stbytes) ||
        !mul_ok(tok, nheads * 2, &dtbytes) || tok > (int64_t(1) << 40))
        return MSS_ERR_SHAPE;
    if (batch == 0) return MSS_OK;
    if (!A || (seqlen > 0 && (!x || !dt || !B || !C || !y))) return MSS_ERR_NULL;
    const void* v16[] = {x, B, C, y, z};
    for (const void* q : v16)
        if (q && !aligned(q, 16)) return MSS_ERR_ALIGN;
    if (dt && !aligned(dt, 2)) return MSS_ERR_ALIGN;
    const void* fp[] = {A, D, dt_bias, initial_state, last_state};
    for (const void* q : fp)
        if (q && !aligned(q, 4)) return MSS_ERR_ALIGN;
    struct Range { const void* p; int64_t n; };
    const Range outs[] = {{y, xbytes}, {last_state, stbytes}};
    const Range ins[] = {{x, xbytes}, {z, xbytes}, {dt, dtbytes}, {B, bcbytes}, {C, bcbytes}, {A, nheads * 4},
                         {D, nheads * 4}, {dt_bias, nheads * 4}, {initial_state, stbytes}};
    for (const Range& o : outs) {
        for (const Range& r : ins)
            if (overlaps(o.p, o.n, r.p, r.n)) return MSS_ERR_ALIAS;
        for (const Range& o2 : outs)
            if (&o != &o2 && overlaps(o.p, o.n, o2.p, o2.n)) return MSS_ERR_ALIAS;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (seqlen == 0) {
        if (last_state) {
            const cudaError_t e = initial_state
                ? cudaMemcpyAsync(last_state, initial_state, size_t(stbytes), cudaMemcpyDeviceToDevice, s)
                : cudaMemsetAsync(last_state, 0, size_t(stbytes), s);
            if (e != cudaSuccess) return MSS_ERR_CUDA;
        }
        return MSS_OK;
    }
    mss::SsdParams p{x, dt, A, B, C, D, z, dt_bias, initial_state, y, last_state, batch, seqlen, nheads, ngroups,
                     softplus_flag ? 1 : 0};
    if (!(p.err = device_error_word())) return MSS_ERR_CUDA;
    const bool tc = dstate == 128 && !(flags & MSS_SSD_FLAG_WARP_MMA);
    const int64_t pairs = batch * nheads;
    // with a workspace: every pair on the chunk-parallel passes where they
    // pay, or (tcgen05 kernel) only the pairs past its last full wave
    int64_t chunked0 = pairs;  // the first pair the passes take
    if (workspace) {
        if (tc ? ssd_chunked_pays_tc(batch, nheads) : ssd_chunked_pays(batch, nheads))
            chunked0 = 0;
        else if (tc)
            chunked0 = pairs - ssd_tc_tail_units(batch, nheads);
    }
    if (chunked0 < pairs) {
        const int64_t need = ssd_workspace_bytes(1, seqlen, pairs - chunked0, dstate);
        if (need > workspace_bytes || !aligned(workspace, 16)) return MSS_ERR_WORKSPACE;
        const Range ws{workspace, workspace_bytes};
        for (const Range& r : ins)
            if (overlaps(ws.p, ws.n, r.p, r.n)) return MSS_ERR_ALIAS;
        for (const Range& o : outs)
            if (overlaps(ws.p, ws.n, o.p, o.n)) return MSS_ERR_ALIAS;
    }
    if (chunked0 > 0) {
        const int rc = tc ? launch_ssd_tc(p, 0, chunked0, s) : launch_ssd(p, int(dstate), s);
        if (rc != MSS_OK || chunked0 == pairs) return rc;
    }
    return launch_ssd_chunked(p, int(dstate), workspace, chunked0, pairs - chunked0, s);
}

int mss_get_device_error(void* stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return MSS_ERR_CUDA;
    unsigned int word = 0, zero = 0;
    if (cudaMemcpyFromSymbolAsync(&word, g_mss_device_error, sizeof(word), 0,
                                  cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return MSS_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MSS_ERR_CUDA;
    if (word != 0) {
        if (cudaMemcpyToSymbolAsync(g_mss_device_error, &zero, sizeof(zero), 0,
                                    cudaMemcpyHostToDevice, s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return MSS_ERR_CUDA;
        return MSS_ERR_DEVICE_TIMEOUT;
    }
    return MSS_OK;
}

}  // extern "C"


// ---------------------------------------------------------------------------
// Forward pass for callers that cannot allocate device memory.
//
// Some callers have no way to obtain device memory of their own: a plain C
// program that is only handed the input and output buffers, a plug-in whose
// host framework owns every device allocation, a serving loop that must not
// allocate once it has started.  mss_scan_fwd_noalloc gives them the sequence
// split without a workspace argument: its scratch is the fixed array below,
// part of the library image, which every GPU that loads the library holds
// until the process exits.

namespace {

constexpr int64_t kStaticScratchBytes = int64_t(4) << 20;  // 4 MiB per device

// The scratch itself.  In host code this name is only a stand-in for the
// symbol, never a device address: kernels get the address that
// cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) float g_mss_static_scratch[kStaticScratchBytes / sizeof(float)];

// Device address of the scratch on the current device, looked up once per
// device (with that device current) and cached; nullptr on failure.
void* static_scratch_address() {
    static std::mutex mu;
    static void* cache[kMaxDevices] = {};
    return symbol_address(g_mss_static_scratch, cache, mu);
}

}  // namespace

extern "C" {

int mss_scan_fwd_noalloc(const void* u, const void* delta, const float* A, const void* B,
                         const void* C, const float* D, const void* z, const float* delta_bias,
                         int softplus_flag, const float* initial_state, void* y, float* last_state,
                         int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                         int dtype, unsigned flags, void* stream) {
    const int64_t need = mss_scan_fwd_workspace_size(batch, dim, dstate, seqlen, dtype, flags);
    if (need < 0) return int(need);
    if (need > kStaticScratchBytes) return MSS_ERR_SCRATCH;
    void* scratch = nullptr;
    if (need > 0 && !(scratch = static_scratch_address())) return MSS_ERR_CUDA;
    return mss_scan_fwd_ex2(u, delta, A, B, C, D, z, delta_bias, softplus_flag, initial_state, y, last_state,
                            batch, dim, dstate, seqlen, dtype, flags, scratch, need, stream);
}

int64_t mss_scan_fwd_noalloc_scratch_bytes(void) { return kStaticScratchBytes; }

}  // extern "C"
