// state_update_tma.cuh -- single-token decode update, staged through shared
// memory with 1-D bulk copies (the streaming form of state_update.cuh).
//
// The step is bound by HBM: per channel it reads and rewrites N fp32 states
// (64 B at N = 16) and moves a few bytes of u, delta, z and y.  Plain loads
// keep one 16-byte vector per thread in flight, which on B200 is not enough
// to cover the memory latency at full bandwidth.  Here a persistent CTA walks
// tiles of 2048/N consecutive channels (8 KB of state) of one batch row
// through a ring of kStages shared-memory stages: one thread issues
// cp.async.bulk loads of the tile's state, u, delta and z a few tiles ahead
// (kStages - 1 tiles, about 9 KB each, in flight per CTA), all threads update
// the state in place in shared memory and write y there, and the same thread
// stores both back with bulk copies, so that neither direction occupies
// registers while in flight.  A B200 sweep of the tile and ring sizes on
// 256 x 5120 x 16 (one token, L2 flushed) picked 8 KB tiles and three stages:
// 38.9 us, against 43.0 us for 4 KB tiles (three or four stages) and 49 us
// or more for 16 KB tiles or two stages.
//
// With the causal convolution in front, the tile's conv state (K-1 inputs per
// channel) travels with it and is shifted in shared memory.
//
// Requirements (checked by the host): N in {4, 8, 16}; dim a multiple of
// 2048/N; state, A, u, delta, z, y and the conv state 16-byte aligned
// (otherwise the host runs state_update_kernel).  Waits on the stage
// barriers are bounded.
#pragma once

#include "mss_device.cuh"
#include "mss_params.h"
#include "tma.cuh"

namespace mss {

template <typename T, int N>
struct DecodeTile {
    static_assert(N == 4 || N == 8 || N == 16, "bulk-staged decode supports N = 4, 8, 16");
    static constexpr int kRows = 2048 / N;                   // channels per tile
    static constexpr int kStateBytes = kRows * N * 4;        // 8 KB
    static constexpr int kIoBytes = kRows * int(sizeof(T));  // one of u, delta, z, y
    static constexpr int kConvOffset = kStateBytes + 4 * kIoBytes;  // conv state: up to 3 inputs per channel
    static constexpr int kStageBytes = kConvOffset + 3 * kIoBytes;
    static constexpr int kStages = 3;
    static constexpr int kThreads = 128;
    static constexpr int kTPC = N / 4;                               // threads per channel
    static constexpr int kSlots = kStateBytes / 16 / kThreads;       // float4 slots per thread per tile
    static constexpr int kBarOffset = kStages * kStageBytes;
    static constexpr int kSmemBytes = kBarOffset + kStages * 8;
    static_assert(kIoBytes % 16 == 0, "bulk copies move multiples of 16 bytes");
    static_assert(kStageBytes % 16 == 0, "stages stay 16-byte aligned");
};

// grid = n_cblocks * bsplit, block = 128 threads, dynamic shared memory
// DecodeTile<T, N>::kSmemBytes.  The channels are cut into n_cblocks =
// dim / kRows blocks; CTA c keeps channel block c % n_cblocks (its A, D and
// bias stay in registers) and serves batch rows c / n_cblocks,
// c / n_cblocks + bsplit, ...  B and C of the next batch row are loaded while
// the current tile is updated.
template <typename T, int N>
__global__ void __launch_bounds__(128) state_update_tma_kernel(StepParams p, int n_cblocks, int bsplit) {
    using Ly = DecodeTile<T, N>;
    constexpr int S = Ly::kStages;
    constexpr int V = Ly::kSlots;
    constexpr bool kFast = sizeof(T) == 2;
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Ly::kBarOffset);
    const int tid = threadIdx.x;

    const int cblock = int(blockIdx.x % unsigned(n_cblocks));
    const int64_t b_first = blockIdx.x / unsigned(n_cblocks);
    const int64_t my_tiles = b_first < p.batch ? (p.batch - 1 - b_first) / bsplit + 1 : 0;
    const int64_t d0 = int64_t(cblock) * Ly::kRows;
    const bool gated = p.z != nullptr;
    const int K = p.conv_width;
    const int conv_bytes = K > 1 ? (K - 1) * Ly::kIoBytes : 0;  // this tile's conv state
    const uint32_t tx = uint32_t(Ly::kStateBytes + (gated ? 3 : 2) * Ly::kIoBytes + conv_bytes);

    if (tid == 0) {
        for (int s = 0; s < S; ++s) mbar_init(bars + s, 1);
        fence_barrier_init();
    }
    __syncthreads();

    auto stage_of = [&](int64_t k) { return smem + int(k % S) * Ly::kStageBytes; };
    auto row0_of = [&](int64_t k) { return (b_first + k * bsplit) * p.dim + d0; };
    auto issue = [&](int64_t k) {
        uint8_t* st = stage_of(k);
        uint64_t* bar = bars + int(k % S);
        const int64_t row0 = row0_of(k);
        mbar_arrive_expect_tx(bar, tx);
        bulk_load(st, p.state + row0 * N, Ly::kStateBytes, bar);
        bulk_load(st + Ly::kStateBytes, static_cast<const T*>(p.u) + row0, Ly::kIoBytes, bar);
        bulk_load(st + Ly::kStateBytes + Ly::kIoBytes, static_cast<const T*>(p.delta) + row0, Ly::kIoBytes, bar);
        if (gated)
            bulk_load(st + Ly::kStateBytes + 2 * Ly::kIoBytes, static_cast<const T*>(p.z) + row0, Ly::kIoBytes, bar);
        if (conv_bytes)
            bulk_load(st + Ly::kConvOffset, static_cast<const T*>(p.conv_state) + row0 * (K - 1), conv_bytes, bar);
    };
    if (tid == 0) {
        for (int64_t k = 0; k < S - 1 && k < my_tiles; ++k) issue(k);
    }

    // per-slot channel constants: A (this thread's 4 states), D, bias, conv taps
    float a[V][4], Dd[V], bias[V];
    ConvTaps taps[V];
#pragma unroll
    for (int v = 0; v < V; ++v) {
        const int slot = tid + v * Ly::kThreads;
        const int64_t d = d0 + slot / Ly::kTPC;
        const float4 av = __ldg(reinterpret_cast<const float4*>(p.A + d * N + (slot % Ly::kTPC) * 4));
        a[v][0] = av.x; a[v][1] = av.y; a[v][2] = av.z; a[v][3] = av.w;
        Dd[v] = p.D ? __ldg(p.D + d) : 0.f;
        bias[v] = p.delta_bias ? __ldg(p.delta_bias + d) : 0.f;
        if (K > 0) taps[v] = load_conv_taps(p.conv_w, p.conv_b, K, d);
    }
    // B and C of a batch row for this thread's states (the same for every slot)
    const int q = tid % Ly::kTPC;  // slot % kTPC == tid % kTPC: kThreads is a multiple of kTPC
    auto load_bc = [&](int64_t b, float (&Bv)[4], float (&Cv)[4]) {
        const T* Bp = static_cast<const T*>(p.B) + b * N + q * 4;
        const T* Cp = static_cast<const T*>(p.C) + b * N + q * 4;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            Bv[i] = ld(Bp + i);
            Cv[i] = ld(Cp + i);
        }
    };
    float Bn[4], Cn[4];
    if (my_tiles > 0) load_bc(b_first, Bn, Cn);

    for (int64_t k = 0; k < my_tiles; ++k) {
        uint8_t* st = stage_of(k);
        float Bv[4], Cv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            Bv[i] = Bn[i];
            Cv[i] = Cn[i];
        }
        if (k + 1 < my_tiles) load_bc(b_first + (k + 1) * bsplit, Bn, Cn);
        const bool landed = mbar_wait_bounded(bars + int(k % S), uint32_t((k / S) & 1), p.err);
        if (!__syncthreads_and(landed)) {
            // give the other loads in flight a bounded chance to land, let the
            // issued stores finish, and stop
            if (tid == 0) {
                for (int64_t k2 = k + 1; k2 < my_tiles && k2 < k + S - 1; ++k2)
                    mbar_wait_bounded(bars + int(k2 % S), uint32_t((k2 / S) & 1), p.err, 100000000ull);
                bulk_wait<0>();
            }
            return;
        }
        const int64_t row0 = row0_of(k);
        float4* hs = reinterpret_cast<float4*>(st);
        const T* us = reinterpret_cast<const T*>(st + Ly::kStateBytes);
        const T* ds = reinterpret_cast<const T*>(st + Ly::kStateBytes + Ly::kIoBytes);
        const T* zs = reinterpret_cast<const T*>(st + Ly::kStateBytes + 2 * Ly::kIoBytes);
        T* ys = reinterpret_cast<T*>(st + Ly::kStateBytes + 3 * Ly::kIoBytes);
        T* cs_tile = reinterpret_cast<T*>(st + Ly::kConvOffset);
#pragma unroll
        for (int v = 0; v < V; ++v) {
            const int slot = tid + v * Ly::kThreads;  // float4 slot of the tile's state
            const int ch = slot / Ly::kTPC;
            const float4 hv = hs[slot];
            float h[4] = {hv.x, hv.y, hv.z, hv.w};
            float ut = to_f32(us[ch]);
            const float x_new = ut;
            if (K > 0) {
                // causal convolution over the stored K-1 inputs and this token's x
                const T* cs = cs_tile + ch * (K - 1);
                float xm[3] = {0.f, 0.f, 0.f};
#pragma unroll
                for (int i = 0; i < 3; ++i) {  // slot i holds stored input i - (4 - K)
                    const int k = i - (4 - K);
                    if (k >= 0) xm[i] = to_f32(cs[k]);
                }
                const float pre = conv_pre(taps[v], xm[0], xm[1], xm[2], x_new);
                ut = kFast ? silu_fast(pre) : silu_precise(pre);
            }
            const float s = to_f32(ds[ch]) + bias[v];
            const float dt = p.softplus ? (kFast ? softplus_fast(s) : softplus_precise(s)) : s;
            const float du = dt * ut;
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float dA = kFast ? ex2_approx(dt * (a[v][i] * kLog2e)) : expf(dt * a[v][i]);
                // input weight: Euler Delta, or the zero-order hold (e^{Delta a} - 1)/a
                const float w = p.zoh ? zoh_weight(dt, a[v][i], dt * a[v][i], dA) * ut : du;
                h[i] = fmaf(dA, h[i], w * Bv[i]);
                acc = fmaf(Cv[i], h[i], acc);
            }
#pragma unroll
            for (int off = 1; off < Ly::kTPC; off <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            hs[slot] = make_float4(h[0], h[1], h[2], h[3]);
            if (q == 0 && K > 1) {
                // shift the conv state (the channel's lanes read it before the shuffles)
                T* cs = cs_tile + ch * (K - 1);
                for (int k = 0; k + 1 < K - 1; ++k) cs[k] = cs[k + 1];
                cs[K - 2] = from_f32<T>(x_new);
            }
            if (q == 0) {
                float out = fmaf(Dd[v], ut, acc);
                if (gated) out *= kFast ? silu_fast(to_f32(zs[ch])) : silu_precise(to_f32(zs[ch]));
                ys[ch] = from_f32<T>(out);
            }
        }
        // make this thread's shared-memory writes visible to the bulk stores
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            bulk_store(p.state + row0 * N, st, Ly::kStateBytes);
            bulk_store(static_cast<T*>(p.y) + row0, ys, Ly::kIoBytes);
            if (conv_bytes)
                bulk_store(static_cast<T*>(p.conv_state) + row0 * (K - 1), cs_tile, uint32_t(conv_bytes));
            bulk_commit();
            if (k + S - 1 < my_tiles) {
                // the stage of tile k-1 is reused once its store has read it
                bulk_wait_read<1>();
                issue(k + S - 1);
            }
        }
    }
    if (tid == 0) bulk_wait<0>();
}

}  // namespace mss
