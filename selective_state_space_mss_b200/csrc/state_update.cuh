// state_update.cuh -- single-token decode update (the recurrent, generation-time
// view: "Exercises -- State-space models (Mamba, S4)", constant-size state,
// O(1) work per token).
//
// The step is bound by HBM: per channel it reads and rewrites N fp32 states
// and touches a handful of other bytes.  Each channel is served by
// TPC = N / SPT threads holding SPT <= 4 consecutive states, so for N >= 4
// every thread moves one 16-byte vector of state in each direction and
// consecutive threads touch consecutive 16-byte pieces: fully coalesced.  The
// read-out sum over the channel's states is finished with TPC-1 xor shuffles.
#pragma once

#include "mss_device.cuh"
#include "mss_params.h"

namespace mss {

template <typename T, int N, bool kVec>
__global__ void __launch_bounds__(256) state_update_kernel(StepParams p) {
    constexpr int SPT = N < 4 ? N : 4;  // states per thread
    constexpr int TPC = N / SPT;        // threads per channel: 1, 2 or 4 (divides 32)
    constexpr bool kFast = sizeof(T) == 2;  // bf16 io: single-instruction exp2

    const int64_t rows = p.batch * p.dim;
    const int64_t gid = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t row = p.row0 + gid / TPC;
    const int q = int(gid % TPC);
    const bool active = row < rows;
    // lanes past the end compute on row row0 (< rows here) so that every lane
    // of a channel group takes part in the shuffles; they store nothing
    const int64_t r = active ? row : p.row0;
    const int64_t b = r / p.dim, d = r % p.dim;

    float h[SPT], a[SPT], Bv[SPT], Cv[SPT];
    float* st = p.state + r * N + q * SPT;
    const float* Ap = p.A + d * N + q * SPT;
    if constexpr (kVec && SPT == 4) {
        const float4 hv = *reinterpret_cast<const float4*>(st);
        const float4 av = __ldg(reinterpret_cast<const float4*>(Ap));
        h[0] = hv.x; h[1] = hv.y; h[2] = hv.z; h[3] = hv.w;
        a[0] = av.x; a[1] = av.y; a[2] = av.z; a[3] = av.w;
    } else {
#pragma unroll
        for (int i = 0; i < SPT; ++i) {
            h[i] = st[i];
            a[i] = __ldg(Ap + i);
        }
    }
    const T* Bp = static_cast<const T*>(p.B) + b * N + q * SPT;
    const T* Cp = static_cast<const T*>(p.C) + b * N + q * SPT;
#pragma unroll
    for (int i = 0; i < SPT; ++i) {
        Bv[i] = ld(Bp + i);
        Cv[i] = ld(Cp + i);
    }

    float ut = ld(static_cast<const T*>(p.u) + r);
    float x_new = 0.f;
    if (p.conv_width > 0) {
        // causal convolution over the stored K-1 inputs and this token's x
        const int K = p.conv_width;
        const T* cs = static_cast<const T*>(p.conv_state) + r * (K - 1);
        float xm[3] = {0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < 3; ++i) {  // slot i holds stored input i - (4 - K)
            const int k = i - (4 - K);
            if (k >= 0) xm[i] = ld(cs + k);
        }
        x_new = ut;
        const float pre = conv_pre(load_conv_taps(p.conv_w, p.conv_b, K, d), xm[0], xm[1], xm[2], x_new);
        ut = kFast ? silu_fast(pre) : silu_precise(pre);
    }
    const float s = ld(static_cast<const T*>(p.delta) + r) + (p.delta_bias ? __ldg(p.delta_bias + d) : 0.f);
    const float dt = p.softplus ? (kFast ? softplus_fast(s) : softplus_precise(s)) : s;
    const float du = dt * ut;
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < SPT; ++i) {
        const float dA = kFast ? ex2_approx(dt * (a[i] * kLog2e)) : expf(dt * a[i]);
        // input weight: Euler Delta, or the zero-order hold (e^{Delta a} - 1)/a
        const float w = p.zoh ? zoh_weight(dt, a[i], dt * a[i], dA) * ut : du;
        h[i] = fmaf(dA, h[i], w * Bv[i]);
        acc = fmaf(Cv[i], h[i], acc);
    }
#pragma unroll
    for (int off = 1; off < TPC; off <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);

    if (!active) return;
    if constexpr (kVec && SPT == 4) {
        *reinterpret_cast<float4*>(st) = make_float4(h[0], h[1], h[2], h[3]);
    } else {
#pragma unroll
        for (int i = 0; i < SPT; ++i) st[i] = h[i];
    }
    if (q == 0 && p.conv_width > 1) {
        // shift the conv state by one token (every lane of the channel has read
        // it: the shuffles above order those reads before this write)
        const int K = p.conv_width;
        T* cs = static_cast<T*>(p.conv_state) + r * (K - 1);
        for (int k = 0; k + 1 < K - 1; ++k) cs[k] = cs[k + 1];
        cs[K - 2] = from_f32<T>(x_new);
    }
    if (q == 0) {
        float out = fmaf(p.D ? __ldg(p.D + d) : 0.f, ut, acc);
        if (p.z) {
            const float zt = ld(static_cast<const T*>(p.z) + r);
            out *= kFast ? silu_fast(zt) : silu_precise(zt);
        }
        static_cast<T*>(p.y)[r] = from_f32<T>(out);
    }
}

}  // namespace mss
