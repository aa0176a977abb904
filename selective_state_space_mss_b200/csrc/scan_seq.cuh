// scan_seq.cuh -- throughput forward kernel for the selective scan.
//
// Work split.  One lane owns one channel (batch row b, channel d) and keeps its
// N fp32 states in registers for the whole sequence; a warp owns 32
// consecutive channels of one batch row and is its own CTA.  The recurrence
// h_t = Abar_t h_{t-1} + Bbar_t x_t is therefore run in its sequential form:
// per token and state it costs exactly the four fp32 operations the
// definition needs (the transition Abar, the input term Delta*u*B, the state
// update, the read-out C*h), done two states at a time with the packed
// f32x2 instructions.  On B200 those fp32 operations, not HBM, bound this
// kernel at N = 16 (128 fp32 lanes per SM and clock against 8 bytes of
// traffic per channel-token), so no parallel-scan form -- which adds at
// least one more operation per state and token -- is used here.
//
// Data movement.  The sequence is streamed in chunks of 128 bytes per row
// (64 bf16 or 32 fp32 tokens).  Lane 0 stages each chunk with tiled TMA
// copies into a ring of shared-memory stages, one mbarrier per stage:
//   u, delta, z : 32 rows x 128 B boxes of the [batch*dim, L] view, 128-byte
//                 swizzle, so that each lane's 16-byte reads of its own row
//                 are free of bank conflicts;
//   B, C        : N x 128 B boxes of the [batch, N, L] tensor, shared by the
//                 32 channels of the warp.
// After a stage lands, the warp rewrites B and C as one fp32 row of 2N values
// per token (16-byte chunks swizzled by token), so that in the token loop all
// lanes read the same address: broadcast loads, no conversion per use.
// y leaves as one 16-byte store per lane and 8 (bf16) or 4 (fp32) tokens.
// The state never touches HBM; last_state is written once at the end.
//
// Transition.  For bf16 io, Abar_n = exp(Delta A_n) is one ex2 per state, or,
// when every A[d,n] of the warp's channels equals (n+1)*A[d,0] exactly (the
// S4D-Real initialisation A_n = -(n+1) of the pages), Abar_n = r^(n+1) with
// r = exp(Delta A_0): one ex2 per token and one multiply per state.  fp32 io
// uses the full-precision expf for every state.
//
// Waits are bounded: a stage that does not arrive within ~2 s sets the
// device error word (read by mss_get_device_error) and the CTA drains its
// other copies and returns.
#pragma once

#include <cstdint>
#include <cuda.h>

#include "mss_device.cuh"
#include "mss_params.h"
#include "tma.cuh"

namespace mss {

struct SeqMaps {
    CUtensorMap u, delta, z, B, C;
};

template <typename T, int N>
struct SeqLayout {
    static_assert(N == 4 || N == 8 || N == 16, "fast path supports N = 4, 8, 16");
    static constexpr int kRowBytes = 128;                      // one chunk of one row
    static constexpr int kChunk = kRowBytes / int(sizeof(T));  // tokens per chunk
    static constexpr int kVec = 16 / int(sizeof(T));           // tokens per 16-byte vector
    static constexpr int kTile = 32 * kRowBytes;               // 32 rows
    static constexpr int kBCTile = N * kRowBytes;
    static constexpr int kStages = 2;
    static constexpr int kStageBytes = 3 * kTile + 2 * kBCTile;  // multiple of 1024
    static constexpr int kBCfChunks = N / 2;                   // 16-byte (B,B,C,C) chunks per token
    static constexpr int kBCfRow = 2 * N + 4;                  // floats per token row, +16 B padding
    static constexpr int kBCfBytes = kChunk * kBCfRow * 4;
    static constexpr int kBarOffset = kStages * kStageBytes + kBCfBytes;
    static constexpr int kSmemBytes = kBarOffset + kStages * 8 + 1024;  // +1024: base alignment slack
    static_assert(kStageBytes % 1024 == 0, "stage tiles must stay 1024-byte aligned");
};

// Rows of the fp32 B/C buffer are padded to 2N + 4 floats: the 16-byte
// pad spreads the conversion's stores over the banks, and readers, which all
// load the same row, address it with constant offsets.
// Rewrite the staged B and C tiles ([N][chunk] in the io type) as fp32 rows of
// 2N values per token, interleaved by state pair: 16-byte chunk k of token t
// holds (B_2k, B_2k+1, C_2k, C_2k+1).  One broadcast load then feeds both
// packed operands of a state pair.
template <typename T, int N>
__device__ __forceinline__ void convert_bc(const uint8_t* btile, const uint8_t* ctile, float* bcf, int lane) {
    using Ly = SeqLayout<T, N>;
    if constexpr (sizeof(T) == 2) {
        // lane l: tokens 2l and 2l+1 (one 32-bit word of each state row)
        const int t0 = 2 * lane;
        float4* r0 = reinterpret_cast<float4*>(bcf + t0 * Ly::kBCfRow);
        float4* r1 = reinterpret_cast<float4*>(bcf + (t0 + 1) * Ly::kBCfRow);
#pragma unroll
        for (int k = 0; k < N / 2; ++k) {
            const uint32_t b0 = *reinterpret_cast<const uint32_t*>(btile + (2 * k) * Ly::kRowBytes + 4 * lane);
            const uint32_t b1 = *reinterpret_cast<const uint32_t*>(btile + (2 * k + 1) * Ly::kRowBytes + 4 * lane);
            const uint32_t c0 = *reinterpret_cast<const uint32_t*>(ctile + (2 * k) * Ly::kRowBytes + 4 * lane);
            const uint32_t c1 = *reinterpret_cast<const uint32_t*>(ctile + (2 * k + 1) * Ly::kRowBytes + 4 * lane);
            r0[k] = make_float4(bf16_lo(b0), bf16_lo(b1), bf16_lo(c0), bf16_lo(c1));
            r1[k] = make_float4(bf16_hi(b0), bf16_hi(b1), bf16_hi(c0), bf16_hi(c1));
        }
    } else {
        // lane l: token l
        float4* r = reinterpret_cast<float4*>(bcf + lane * Ly::kBCfRow);
#pragma unroll
        for (int k = 0; k < N / 2; ++k) {
            const float* bp = reinterpret_cast<const float*>(btile) + lane;
            const float* cp = reinterpret_cast<const float*>(ctile) + lane;
            constexpr int rs = Ly::kRowBytes / 4;
            r[k] = make_float4(bp[(2 * k) * rs], bp[(2 * k + 1) * rs], cp[(2 * k) * rs], cp[(2 * k + 1) * rs]);
        }
    }
}

// Per-channel constants held in registers.
template <int N>
struct ChanConst {
    float bias, D;
    float a0;          // A[d,0] * log2(e)      (fast transition)
    float2 a2[N / 2];  // A[d,n] * log2(e) pairs (bf16 io) or A[d,n] pairs (fp32 io)
};

// Per-token scalars of one channel, computed ahead of the state updates so
// that the 8 (or 4) tokens of a vector form independent dependency chains.
struct TokenPre {
    float dt;    // step size Delta
    float du;    // Delta * u
    float r;     // exp(Delta * A[d,0]) with the fast transition, else Delta
    float skip;  // D * u
    float gate;  // silu(z), or 1 without a gate
};

template <bool kFast, bool kGeo, bool kGate, bool kSoftplus, int N>
__device__ __forceinline__ TokenPre token_pre(float ut, float dr, float zt, const ChanConst<N>& cc) {
    TokenPre tp;
    const float s = dr + cc.bias;
    tp.dt = s;
    if constexpr (kSoftplus) tp.dt = kFast ? softplus_fast(s) : softplus_precise(s);
    tp.du = tp.dt * ut;
    tp.r = kGeo ? ex2_approx(tp.dt * cc.a0) : tp.dt;
    tp.skip = cc.D * ut;
    tp.gate = kGate ? (kFast ? silu_fast(zt) : silu_precise(zt)) : 1.f;
    return tp;
}

// State update of one token: h <- Abar (.) h + Delta*u*B, returns C . h.
// For the fast transition `rdt` is r = exp(Delta A[d,0]); otherwise it is Delta.
// `row` holds the token's (B_2k, B_2k+1, C_2k, C_2k+1) chunks, already loaded.
template <int N, bool kFast, bool kGeo>
__device__ __forceinline__ float token_states(float2 (&h)[N / 2], const float4 (&row)[N / 2], float du,
                                              float rdt, const ChanConst<N>& cc) {
    const float2 du2 = make_float2(du, du);
    // transition pairs (Abar_{2k}, Abar_{2k+1})
    float2 dA[N / 2];
    if constexpr (kGeo) {
        // Abar_n = r^(n+1): pairs built from r, r^2, r^4, r^8 (depth-3 tree)
        const float r = rdt, r2 = r * r;
        dA[0] = make_float2(r, r2);
        if constexpr (N >= 4) dA[1] = __fmul2_rn(dA[0], make_float2(r2, r2));
        if constexpr (N >= 8) {
            const float r4 = r2 * r2;
            dA[2] = __fmul2_rn(dA[0], make_float2(r4, r4));
            dA[3] = __fmul2_rn(dA[1], make_float2(r4, r4));
            if constexpr (N >= 16) {
                const float r8 = r4 * r4;
#pragma unroll
                for (int k = 0; k < 4; ++k) dA[4 + k] = __fmul2_rn(dA[k], make_float2(r8, r8));
            }
        }
    } else {
#pragma unroll
        for (int k = 0; k < N / 2; ++k) {
            if constexpr (kFast) {
                const float2 arg = __fmul2_rn(make_float2(rdt, rdt), cc.a2[k]);
                dA[k] = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));
            } else {
                dA[k] = make_float2(expf(rdt * cc.a2[k].x), expf(rdt * cc.a2[k].y));
            }
        }
    }
    // two read-out accumulators halve the dependency chain
    float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < N / 2; ++k) {
        const float4 v = row[k];  // (B_2k, B_2k+1, C_2k, C_2k+1)
        h[k] = __ffma2_rn(dA[k], h[k], __fmul2_rn(du2, make_float2(v.x, v.y)));
        if (k & 1)
            acc1 = __ffma2_rn(make_float2(v.z, v.w), h[k], acc1);
        else
            acc0 = __ffma2_rn(make_float2(v.z, v.w), h[k], acc0);
    }
    const float2 acc = __fadd2_rn(acc0, acc1);
    return acc.x + acc.y;
}

template <typename T>
__device__ __forceinline__ void unpack16(const uint4& w, float (&v)[16 / sizeof(T)]) {
    if constexpr (sizeof(T) == 2) {
        const uint32_t a[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = bf16_lo(a[i]);
            v[2 * i + 1] = bf16_hi(a[i]);
        }
    } else {
        v[0] = __uint_as_float(w.x);
        v[1] = __uint_as_float(w.y);
        v[2] = __uint_as_float(w.z);
        v[3] = __uint_as_float(w.w);
    }
}

template <typename T>
__device__ __forceinline__ uint4 pack16(const float (&v)[16 / sizeof(T)]) {
    if constexpr (sizeof(T) == 2) {
        return make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                          pack_bf16x2(v[6], v[7]));
    } else {
        return make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]),
                          __float_as_uint(v[3]));
    }
}

template <typename T, int N, bool kGeo, bool kGate, bool kSoftplus>
__device__ __forceinline__ void scan_seq_body(const SeqMaps& maps, const ScanParams& p, uint8_t* smem,
                                              uint64_t* bars, const ChanConst<N>& cc, bool valid,
                                              int64_t row) {
    using Ly = SeqLayout<T, N>;
    constexpr bool kFast = sizeof(T) == 2;
    constexpr int S = Ly::kStages;
    constexpr int V = Ly::kVec;            // tokens per group (one 16-byte vector per row)
    constexpr int GPC = Ly::kChunk / V;    // groups per chunk
    const int lane = threadIdx.x;
    const int b = blockIdx.y;
    const int row0 = int(int64_t(b) * p.dim + int64_t(blockIdx.x) * 32);
    const int64_t L = p.seqlen;
    const int n_chunks = int((L + Ly::kChunk - 1) / Ly::kChunk);
    const int n_groups = int(L / V);       // L is a multiple of V
    float* bcf = reinterpret_cast<float*>(smem + S * Ly::kStageBytes);
    const uint32_t stage_tx = uint32_t((kGate ? 3 : 2) * Ly::kTile + 2 * Ly::kBCTile);

    auto issue = [&](int chunk) {
        uint8_t* st = smem + (chunk % S) * Ly::kStageBytes;
        uint64_t* bar = bars + chunk % S;
        const int x = chunk * Ly::kChunk;
        mbar_arrive_expect_tx(bar, stage_tx);
        tma_load_2d(st, &maps.u, x, row0, bar);
        tma_load_2d(st + Ly::kTile, &maps.delta, x, row0, bar);
        if constexpr (kGate) tma_load_2d(st + 2 * Ly::kTile, &maps.z, x, row0, bar);
        tma_load_3d(st + 3 * Ly::kTile, &maps.B, x, 0, b, bar);
        tma_load_3d(st + 3 * Ly::kTile + Ly::kBCTile, &maps.C, x, 0, b, bar);
    };
    // Wait (bounded) for chunk c's stage; on timeout give the other copies in
    // flight a bounded chance to land and report failure.
    auto wait_chunk = [&](int c) -> bool {
        const bool landed = mbar_wait_bounded(bars + c % S, uint32_t((c / S) & 1));
        if (__all_sync(0xffffffffu, landed)) return true;
        for (int c2 = c + 1; c2 < n_chunks && c2 < c + S; ++c2)
            mbar_wait_bounded(bars + c2 % S, uint32_t((c2 / S) & 1), 100000000ull);
        return false;
    };
    const int swz = lane & 7;  // 128-byte swizzle: 16-byte chunk j of row r sits at j ^ (r & 7)
    // the V per-token scalars of group g, from the u/delta/z rows of its stage
    auto prologue = [&](int g, TokenPre (&tp)[V]) {
        const int c = g / GPC, j = g % GPC;
        const uint8_t* urow = smem + (c % S) * Ly::kStageBytes + lane * Ly::kRowBytes;
        const int off = ((j ^ swz) << 4);
        float uv[V], dv[V], zv[V];
        unpack16<T>(*reinterpret_cast<const uint4*>(urow + off), uv);
        unpack16<T>(*reinterpret_cast<const uint4*>(urow + Ly::kTile + off), dv);
        if constexpr (kGate) unpack16<T>(*reinterpret_cast<const uint4*>(urow + 2 * Ly::kTile + off), zv);
#pragma unroll
        for (int k = 0; k < V; ++k)
            tp[k] = token_pre<kFast, kGeo, kGate, kSoftplus>(uv[k], dv[k], kGate ? zv[k] : 0.f, cc);
    };

    if (lane == 0) {
        for (int c = 0; c < S && c < n_chunks; ++c) issue(c);
    }
    float2 h[N / 2];
#pragma unroll
    for (int k = 0; k < N / 2; ++k) h[k] = make_float2(0.f, 0.f);
    T* yrow = static_cast<T*>(p.y) + row * L;

    if (!wait_chunk(0)) return;
    convert_bc<T, N>(smem + 3 * Ly::kTile, smem + 3 * Ly::kTile + Ly::kBCTile, bcf, lane);
    __syncwarp();
    TokenPre nxt[V];
    prologue(0, nxt);

#pragma unroll 1
    for (int g = 0; g < n_groups; ++g) {
        const int c = g / GPC, j = g % GPC;
        TokenPre cur[V];
#pragma unroll
        for (int k = 0; k < V; ++k) cur[k] = nxt[k];
        // the next group's scalars are computed while this group's states update:
        // its u/delta/z must have landed when it opens a new chunk
        const bool has_next = g + 1 < n_groups;
        if (has_next && j == GPC - 1 && !wait_chunk(c + 1)) return;
        const int gn = has_next ? g + 1 : g;
        const int cn = gn / GPC, jn = gn % GPC;
        const uint8_t* urow = smem + (cn % S) * Ly::kStageBytes + lane * Ly::kRowBytes;
        const int off = ((jn ^ swz) << 4);
        float uv[V], dv[V], zv[V];
        unpack16<T>(*reinterpret_cast<const uint4*>(urow + off), uv);
        unpack16<T>(*reinterpret_cast<const uint4*>(urow + Ly::kTile + off), dv);
        if constexpr (kGate) unpack16<T>(*reinterpret_cast<const uint4*>(urow + 2 * Ly::kTile + off), zv);

        float yv[V];
        const float* bbase = bcf + (j * V) * Ly::kBCfRow;
#pragma unroll
        for (int k = 0; k < V; ++k) {
            float4 rowv[N / 2];
            const float4* src = reinterpret_cast<const float4*>(bbase + k * Ly::kBCfRow);
#pragma unroll
            for (int q = 0; q < N / 2; ++q) rowv[q] = src[q];
            yv[k] = (token_states<N, kFast, kGeo>(h, rowv, cur[k].du, cur[k].r, cc) + cur[k].skip) * cur[k].gate;
            nxt[k] = token_pre<kFast, kGeo, kGate, kSoftplus>(uv[k], dv[k], kGate ? zv[k] : 0.f, cc);
        }
        if (valid) *reinterpret_cast<uint4*>(yrow + int64_t(g) * V) = pack16<T>(yv);

        if (j == GPC - 1 || !has_next) {
            // chunk c is consumed: convert the next chunk's B/C (its stage was
            // waited for above), then hand chunk c's stage to chunk c + S
            __syncwarp();
            if (has_next) {
                const uint8_t* st = smem + ((c + 1) % S) * Ly::kStageBytes;
                convert_bc<T, N>(st + 3 * Ly::kTile, st + 3 * Ly::kTile + Ly::kBCTile, bcf, lane);
            }
            __syncwarp();
            if (lane == 0 && c + S < n_chunks) {
                fence_proxy_async_smem();
                issue(c + S);
            }
        }
    }
    if (valid && p.last_state) {
        float4* ls = reinterpret_cast<float4*>(p.last_state + row * N);
#pragma unroll
        for (int k = 0; k < N / 4; ++k) ls[k] = make_float4(h[2 * k].x, h[2 * k].y, h[2 * k + 1].x, h[2 * k + 1].y);
    }
}

// grid = (ceil(dim / 32), batch), block = 32 threads, dynamic shared memory
// SeqLayout<T, N>::kSmemBytes.  Requirements checked by the host: N in
// {4, 8, 16}; L * sizeof(T) a multiple of 16; u, delta, z, B, C, y 16-byte
// aligned; last_state 16-byte aligned when given.
template <typename T, int N, bool kGate, bool kSoftplus>
__global__ void __launch_bounds__(32) scan_fwd_seq_kernel(const __grid_constant__ SeqMaps maps, ScanParams p,
                                                          int allow_geo) {
    using Ly = SeqLayout<T, N>;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    // 1024-byte alignment (128-byte swizzle atoms) by pointer arithmetic on the
    // shared array itself, so that every derived pointer stays a shared-memory
    // pointer and its loads compile to shared loads, not generic ones
    uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Ly::kBarOffset);
    const int lane = threadIdx.x;

    const int64_t c = int64_t(blockIdx.x) * 32 + lane;
    const bool valid = c < p.dim;
    const int64_t d = valid ? c : 0;
    const int64_t row = int64_t(blockIdx.y) * p.dim + d;

    if (lane == 0) {
        for (int s = 0; s < Ly::kStages; ++s) mbar_init(bars + s, 1);
        fence_barrier_init();
        prefetch_tensormap(&maps.u);
        prefetch_tensormap(&maps.delta);
        if (kGate) prefetch_tensormap(&maps.z);
        prefetch_tensormap(&maps.B);
        prefetch_tensormap(&maps.C);
    }
    __syncwarp();

    constexpr bool kFast = sizeof(T) == 2;
    ChanConst<N> cc;
    cc.bias = p.delta_bias ? p.delta_bias[d] : 0.f;
    cc.D = p.D ? p.D[d] : 0.f;
    const float* Arow = p.A + d * N;
    const float a_first = Arow[0];
    bool geo = kFast && allow_geo;
#pragma unroll
    for (int k = 0; k < N / 2; ++k) {
        const float x0 = Arow[2 * k], x1 = Arow[2 * k + 1];
        cc.a2[k] = kFast ? make_float2(x0 * kLog2e, x1 * kLog2e) : make_float2(x0, x1);
        geo = geo && x0 == float(2 * k + 1) * a_first && x1 == float(2 * k + 2) * a_first;
    }
    cc.a0 = a_first * kLog2e;
    geo = __all_sync(0xffffffffu, geo || !valid);

    if constexpr (kFast) {
        if (geo) {
            scan_seq_body<T, N, true, kGate, kSoftplus>(maps, p, smem, bars, cc, valid, row);
            return;
        }
    }
    scan_seq_body<T, N, false, kGate, kSoftplus>(maps, p, smem, bars, cc, valid, row);
}

}  // namespace mss
