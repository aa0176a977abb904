// scan_bwd_simple.cuh -- reference backward kernel: one thread per
// (batch, channel), full-precision math, any alignment and N.
//
// The same chain rule as scan_bwd.cuh.  The thread runs the forward pass
// once, storing its state every kCk tokens in the caller's workspace, then
// walks those chunks from last to first: it recomputes the chunk's states
// into a local buffer and runs the reverse steps.  dB and dC are summed over
// the channels with one atomic addition per (token, state) and thread; it is
// the parity anchor for the throughput kernel and the path for shapes that
// one does not take, not a fast kernel.
#pragma once

#include "mss_device.cuh"
#include "mss_params.h"

namespace mss {

constexpr int kBwdSimpleChunk = 16;  // tokens between checkpoints

template <typename T, int N>
__global__ void __launch_bounds__(128) scan_bwd_simple_kernel(BwdParams p, const float* initial_state, int zoh,
                                                              float* ckpt) {
    constexpr int K = kBwdSimpleChunk;
    const int64_t rows = p.batch * p.dim;
    const int64_t row = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (row >= rows) return;
    const int64_t b = row / p.dim, d = row % p.dim;
    const int64_t L = p.seqlen;
    const int64_t n_ck = (L + K - 1) / K;
    const T* u = static_cast<const T*>(p.u) + row * L;
    const T* dr_raw = static_cast<const T*>(p.delta) + row * L;
    const T* z = p.z ? static_cast<const T*>(p.z) + row * L : nullptr;
    const T* dy = static_cast<const T*>(p.dy) + row * L;
    const T* Bb = static_cast<const T*>(p.B) + b * N * L;
    const T* Cb = static_cast<const T*>(p.C) + b * N * L;
    float* ck = ckpt + row * n_ck * N;

    float a[N], h[N];
#pragma unroll
    for (int n = 0; n < N; ++n) {
        a[n] = p.A[d * N + n];
        h[n] = initial_state ? initial_state[row * N + n] : 0.f;
    }
    const float bias = p.delta_bias ? p.delta_bias[d] : 0.f;
    const float Dd = p.D ? p.D[d] : 0.f;
    auto step_scalars = [&](int64_t t, float& dt, float& dsp) {
        const float s = ld(dr_raw + t) + bias;
        dt = p.softplus ? softplus_precise(s) : s;
        dsp = p.softplus ? 1.f / (1.f + expf(-s)) : 1.f;
    };
    auto weight = [&](float dt, float an, float e) {
        return zoh ? zoh_weight(dt, an, dt * an, e) : dt;
    };

    // forward, with a checkpoint every K tokens
    for (int64_t t = 0; t < L; ++t) {
        if (t % K == 0) {
#pragma unroll
            for (int n = 0; n < N; ++n) ck[(t / K) * N + n] = h[n];
        }
        float dt, dsp;
        step_scalars(t, dt, dsp);
        const float ut = ld(u + t);
#pragma unroll
        for (int n = 0; n < N; ++n) {
            const float e = expf(dt * a[n]);
            h[n] = fmaf(e, h[n], weight(dt, a[n], e) * ld(Bb + n * L + t) * ut);
        }
    }

    // reverse
    float gh[N], dA_acc[N];
#pragma unroll
    for (int n = 0; n < N; ++n) {
        gh[n] = p.dlast ? p.dlast[row * N + n] : 0.f;
        dA_acc[n] = 0.f;
    }
    float dD_acc = 0.f, dbias_acc = 0.f;
    float hb[K + 1][N];  // hb[0]: chunk start; hb[j + 1]: after the chunk's token j
    for (int64_t c = n_ck - 1; c >= 0; --c) {
        const int64_t t0 = c * K;
        const int cnt = int(min(int64_t(K), L - t0));
#pragma unroll
        for (int n = 0; n < N; ++n) hb[0][n] = ck[c * N + n];
        for (int j = 0; j < cnt; ++j) {
            float dt, dsp;
            step_scalars(t0 + j, dt, dsp);
            const float ut = ld(u + t0 + j);
#pragma unroll
            for (int n = 0; n < N; ++n) {
                const float e = expf(dt * a[n]);
                hb[j + 1][n] = fmaf(e, hb[j][n], weight(dt, a[n], e) * ld(Bb + n * L + t0 + j) * ut);
            }
        }
        for (int j = cnt - 1; j >= 0; --j) {
            const int64_t t = t0 + j;
            float dt, dsp;
            step_scalars(t, dt, dsp);
            const float ut = ld(u + t);
            float dr = ld(dy + t);
            if (z) {
                float r = Dd * ut;
#pragma unroll
                for (int n = 0; n < N; ++n) r = fmaf(ld(Cb + n * L + t), hb[j + 1][n], r);
                const float zt = ld(z + t), sz = 1.f / (1.f + expf(-zt));
                static_cast<T*>(p.dz)[row * L + t] = from_f32<T>(dr * r * (sz * fmaf(zt, 1.f - sz, 1.f)));
                dr *= zt * sz;
            }
            float du = dr * Dd, ddt = 0.f;
#pragma unroll
            for (int n = 0; n < N; ++n) {
                const float Bn = ld(Bb + n * L + t), Cn = ld(Cb + n * L + t);
                const float e = expf(dt * a[n]);
                const float w = weight(dt, a[n], e);
                gh[n] = fmaf(dr, Cn, gh[n]);
                atomicAdd(p.dC + (b * N + n) * L + t, dr * hb[j + 1][n]);
                atomicAdd(p.dB + (b * N + n) * L + t, gh[n] * w * ut);
                du = fmaf(gh[n] * w, Bn, du);
                const float dw = gh[n] * Bn * ut;
                const float da = gh[n] * hb[j][n];
                ddt = fmaf(da * e, a[n], ddt);
                dA_acc[n] = fmaf(da * e, dt, dA_acc[n]);
                if (zoh) {
                    ddt = fmaf(dw, e, ddt);
                    dA_acc[n] = fmaf(dw, zoh_weight_dA(dt, a[n], dt * a[n], e, w), dA_acc[n]);
                } else {
                    ddt += dw;
                }
                gh[n] *= e;
            }
            const float ds = ddt * dsp;
            static_cast<T*>(p.du)[row * L + t] = from_f32<T>(du);
            static_cast<T*>(p.ddelta)[row * L + t] = from_f32<T>(ds);
            dD_acc = fmaf(dr, ut, dD_acc);
            dbias_acc += ds;
        }
    }
    if (p.dinit) {
#pragma unroll
        for (int n = 0; n < N; ++n) p.dinit[row * N + n] = gh[n];
    }
#pragma unroll
    for (int n = 0; n < N; ++n) atomicAdd(p.dA + d * N + n, dA_acc[n]);
    if (p.dD) atomicAdd(p.dD + d, dD_acc);
    if (p.dbias) atomicAdd(p.dbias + d, dbias_acc);
}

}  // namespace mss
