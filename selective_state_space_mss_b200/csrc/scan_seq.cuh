// scan_seq.cuh -- throughput forward kernel for the selective scan.
//
// Work split.  A CTA is one warp and owns 16 consecutive channels of one
// batch row for the whole sequence.  Each channel is served by a lane pair
// (lane = 2c + h): lane h keeps the N/2 states n = h, h+2, h+4, ... of
// channel c in registers, as N/4 packed pairs.  The recurrence
// h_t = Abar_t h_{t-1} + Bbar_t x_t runs in its sequential form: per token
// and state it costs the four fp32 operations the definition needs (the
// transition Abar, the input term Delta*u*B, the update, the read-out C*h),
// done two states at a time with packed f32x2 instructions.  At N = 16 these
// fp32 operations, not HBM traffic, bound the kernel on B200 (128 fp32 lanes
// per SM and clock against 8 bytes per channel-token), so the parallel-scan
// form, which costs at least one more operation per state and token, is not
// used.  Two lanes per channel give two resident warps per scheduler on the
// large workloads, which hides the latencies a single warp exposes, and
// 16-channel work units keep the SMs evenly loaded.
//
// Per-token scalars.  The step size Delta = softplus(delta + bias), Delta*u,
// r = exp(Delta A[d,0]) (fast transition), D*u and silu(z) of a group of V
// tokens are split between the two lanes of a channel (each computes V/2
// tokens) and swapped with shuffles; they are computed for the next group
// while the current group's states update, so the MUFU work of one overlaps
// the FMA work of the other.  The read-out partial sums of the two lanes are
// combined by a transpose-reduce: each lane finishes V/2 tokens and stores
// them (8 bytes per lane, 16 contiguous bytes per channel).
//
// Data movement.  The sequence is streamed in chunks of 128 bytes per row
// (64 bf16 or 32 fp32 tokens).  Lane 0 stages each chunk with tiled TMA
// copies into a two-deep ring of shared-memory stages, one mbarrier each:
//   u, delta, z : 16 rows x 128 B boxes of the [batch*dim, L] view, 128-byte
//                 swizzle (conflict-free 8-byte reads of each lane's row);
//   B, C        : N x 128 B boxes of the [batch, N, L] tensor.
// When a chunk is due, the warp rewrites its B and C as one fp32 row per
// token: 16-byte chunks (B_n, B_n+2, C_n, C_n+2) for the even states, then
// for the odd states, plus 16 bytes of padding, so that each lane's state
// pairs are four broadcast loads away.  The state never touches HBM;
// last_state is written once at the end.
//
// Transition.  For bf16 io, Abar_n = exp(Delta A_n) is one ex2 per state,
// or, when every A[d,n] of the warp's channels equals (n+1)*A[d,0] exactly
// (the S4D-Real initialisation A_n = -(n+1) of the pages), Abar_n = r^(n+1):
// one ex2 per token and about one multiply per state.  fp32 io uses the
// full-precision expf for every state.
//
// Input matrix.  By default the input term is the Euler Delta*u*B.  With
// the zero-order hold (kZoh) the weight of state n is Delta*phi(Delta A_n),
// phi(x) = (e^x - 1)/x.  On the general path it is formed per state from the
// transition's exponential (zoh_weight: Taylor series near x = 0).  On the
// fast transition A_n = (n+1) A_0 turns it into a geometric sum,
// phi(Delta A_n) = phi(Delta A_0) * S_n / (n+1) with S_n = 1 + r + ... + r^n
// (a sum of positive terms, so no cancellation): phi(Delta A_0) goes into the
// per-token scalar, S_n costs one packed FMA per state pair, and 1/(n+1) is
// folded into the fp32 C rows, the lanes keeping (n+1) h_n instead of h_n.
//
// Waits are bounded: a stage that does not arrive within ~2 s sets the
// device error word (read by mss_get_device_error) and the CTA returns after
// giving its other copies a bounded chance to land.
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
    static constexpr int kRows = 16;                           // channels per CTA
    static constexpr int kRowBytes = 128;                      // one chunk of one row
    static constexpr int kChunk = kRowBytes / int(sizeof(T));  // tokens per chunk
    static constexpr int kVec = 16 / int(sizeof(T));           // tokens per group
    static constexpr int kHalf = kVec / 2;                     // tokens each lane of a pair finishes
    static constexpr int kPairs = N / 4;                       // state pairs per lane
    static constexpr int kTile = kRows * kRowBytes;
    static constexpr int kBCTile = N * kRowBytes;
    static constexpr int kStages = 2;
    static constexpr int kStageBytes = 3 * kTile + 2 * kBCTile;
    static constexpr int kBCfRow = 2 * N + 4;                  // floats per token row, +16 B padding
    static constexpr int kBCfBytes = kChunk * kBCfRow * 4;
    static constexpr int kBarOffset = kStages * kStageBytes + kBCfBytes;
    // one barrier per stage and one for the wait self-test; +1024: base alignment slack
    static constexpr int kSmemBytes = kBarOffset + (kStages + 1) * 8 + 1024;
    static_assert(kStageBytes % 1024 == 0, "stage tiles must stay 1024-byte aligned");
};

// Rewrite the staged B and C tiles ([N][chunk] in the io type) as fp32 rows,
// one per token: chunk p*N/4 + i holds (B_n, B_n+2, C_n, C_n+2) with
// n = p + 4i, for the even (p = 0) and then the odd (p = 1) states.
// kScaleC: C_n is stored as C_n / (n+1) (zero-order hold on the fast
// transition, where the lanes keep (n+1) h_n).
template <typename T, int N, bool kScaleC>
__device__ __forceinline__ void convert_bc(const uint8_t* btile, const uint8_t* ctile, float* bcf, int lane) {
    using Ly = SeqLayout<T, N>;
    constexpr int P = Ly::kPairs;
    auto cs = [](int n) { return kScaleC ? 1.f / float(n + 1) : 1.f; };
    if constexpr (sizeof(T) == 2) {
        // lane l: tokens 2l and 2l+1 (one 32-bit word of each state row)
        float4* r0 = reinterpret_cast<float4*>(bcf + (2 * lane) * Ly::kBCfRow);
        float4* r1 = reinterpret_cast<float4*>(bcf + (2 * lane + 1) * Ly::kBCfRow);
#pragma unroll
        for (int p = 0; p < 2; ++p) {
#pragma unroll
            for (int i = 0; i < P; ++i) {
                const int n = p + 4 * i;
                const uint32_t b0 = *reinterpret_cast<const uint32_t*>(btile + n * Ly::kRowBytes + 4 * lane);
                const uint32_t b2 = *reinterpret_cast<const uint32_t*>(btile + (n + 2) * Ly::kRowBytes + 4 * lane);
                const uint32_t c0 = *reinterpret_cast<const uint32_t*>(ctile + n * Ly::kRowBytes + 4 * lane);
                const uint32_t c2 = *reinterpret_cast<const uint32_t*>(ctile + (n + 2) * Ly::kRowBytes + 4 * lane);
                const float s0 = cs(n), s2 = cs(n + 2);
                r0[p * P + i] = make_float4(bf16_lo(b0), bf16_lo(b2), s0 * bf16_lo(c0), s2 * bf16_lo(c2));
                r1[p * P + i] = make_float4(bf16_hi(b0), bf16_hi(b2), s0 * bf16_hi(c0), s2 * bf16_hi(c2));
            }
        }
    } else {
        // lane l: token l
        constexpr int rs = Ly::kRowBytes / 4;
        const float* bp = reinterpret_cast<const float*>(btile) + lane;
        const float* cp = reinterpret_cast<const float*>(ctile) + lane;
        float4* r = reinterpret_cast<float4*>(bcf + lane * Ly::kBCfRow);
#pragma unroll
        for (int p = 0; p < 2; ++p) {
#pragma unroll
            for (int i = 0; i < P; ++i) {
                const int n = p + 4 * i;
                r[p * P + i] = make_float4(bp[n * rs], bp[(n + 2) * rs], cs(n) * cp[n * rs], cs(n + 2) * cp[(n + 2) * rs]);
            }
        }
    }
}

// Per-lane constants.
template <int N>
struct LaneConst {
    float bias, D;
    float a0;          // A[d,0] * log2(e)                            (fast transition)
    float2 a2[N / 4];  // this lane's state pairs of A (times log2(e) for bf16 io)
    float ia0;         // 1 / A[d,0]                  (zero-order hold, fast transition)
    float2 ia[N / 4];  // 1 / A of this lane's state pairs (zero-order hold, general path)
    ConvTaps conv;     // causal convolution taps (kConv)
};

// Per-token scalars of one channel.
struct TokenPre {
    float dt;    // Delta
    float du;    // Delta * u; zero-order hold on the fast transition: Delta * u * phi(Delta A[d,0])
    float u;     // u (zero-order hold, general path)
    float r;     // exp(Delta * A[d,0]) with the fast transition, else Delta
    float skip;  // D * u
    float gate;  // silu(z), or 1 without a gate
};

// `Consts` carries bias, D, a0 = A[d,0] log2(e) and ia0 = 1 / A[d,0].
template <bool kFast, bool kGeo, bool kGate, bool kSoftplus, bool kZoh, typename Consts>
__device__ __forceinline__ TokenPre token_pre(float ut, float dr, float zt, const Consts& cc) {
    TokenPre tp;
    const float s = dr + cc.bias;
    float dt = s;
    if constexpr (kSoftplus) dt = kFast ? softplus_fast(s) : softplus_precise(s);
    tp.dt = dt;
    tp.du = dt * ut;
    tp.u = ut;
    if constexpr (kGeo) {
        const float arg = dt * cc.a0;
        tp.r = ex2_approx(arg);
        if constexpr (kZoh) {
            const float x0 = arg * kLn2;
            tp.du = fabsf(x0) < kZohTaylorMax ? tp.du * phi_taylor(x0) : ut * ((tp.r - 1.f) * cc.ia0);
        }
    } else {
        tp.r = dt;
    }
    tp.skip = cc.D * ut;
    tp.gate = kGate ? (kFast ? silu_fast(zt) : silu_precise(zt)) : 1.f;
    return tp;
}

// The transition pairs (Abar_n, Abar_n+2) of this lane's states for one
// token; `rdt` is r = exp(Delta A[d,0]) (fast transition) or Delta.
template <int N, bool kFast, bool kGeo>
__device__ __forceinline__ void transition(float2 (&dA)[N / 4], float rdt, int half, const LaneConst<N>& cc) {
    constexpr int P = N / 4;
    if constexpr (kGeo) {
        // states n = half + 4i and n + 2: Abar = (r^(n+1), r^(n+3))
        const float r = rdt, r2 = r * r;
        const float b = half ? r2 : r;
        dA[0] = make_float2(b, b * r2);
        if constexpr (P >= 2) {
            const float r4 = r2 * r2;
            dA[1] = __fmul2_rn(dA[0], make_float2(r4, r4));
            if constexpr (P >= 4) {
                const float r8 = r4 * r4;
                dA[2] = __fmul2_rn(dA[0], make_float2(r8, r8));
                dA[3] = __fmul2_rn(dA[1], make_float2(r8, r8));
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < P; ++i) {
            if constexpr (kFast) {
                const float2 arg = __fmul2_rn(make_float2(rdt, rdt), cc.a2[i]);
                dA[i] = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));
            } else {
                dA[i] = make_float2(expf(rdt * cc.a2[i].x), expf(rdt * cc.a2[i].y));
            }
        }
    }
}

// Zero-order-hold weights of this lane's state pairs, multiplying B.  Fast
// transition: the geometric sums S_n = 1 + r + ... + r^n (the rest of the
// weight is in du and in the scaled C rows), from S_{n+4} = S_n + r^{n+1} S_3
// and S_{n+8} = S_n + r^{n+1} S_7.  General path: Delta*u*phi(Delta A_n) per
// state (du = Delta*u, uu = u, rdt = Delta).
template <int N, bool kFast, bool kGeo>
__device__ __forceinline__ void zoh_weights(float2 (&w)[N / 4], const float2 (&dA)[N / 4], float du, float uu,
                                            float rdt, int half, const LaneConst<N>& cc) {
    constexpr int P = N / 4;
    if constexpr (kGeo) {
        const float r = rdt, r2 = r * r;
        const float s3 = (1.f + r) * (1.f + r2);
        w[0] = half ? make_float2(1.f + r, s3) : make_float2(1.f, fmaf(r, r, 1.f + r));
        if constexpr (P >= 2) w[1] = __ffma2_rn(dA[0], make_float2(s3, s3), w[0]);
        if constexpr (P >= 4) {
            const float s7 = s3 * fmaf(r2, r2, 1.f);
            w[2] = __ffma2_rn(dA[0], make_float2(s7, s7), w[0]);
            w[3] = __ffma2_rn(dA[1], make_float2(s7, s7), w[1]);
        }
    } else {
        const float2 dt2 = make_float2(rdt, rdt), du2 = make_float2(du, du), u2 = make_float2(uu, uu);
#pragma unroll
        for (int i = 0; i < P; ++i) {
            float2 x = __fmul2_rn(dt2, cc.a2[i]);
            if constexpr (kFast) x = __fmul2_rn(x, make_float2(kLn2, kLn2));
            float2 t = __ffma2_rn(x, make_float2(1.f / 120.f, 1.f / 120.f), make_float2(1.f / 24.f, 1.f / 24.f));
            t = __ffma2_rn(t, x, make_float2(1.f / 6.f, 1.f / 6.f));
            t = __ffma2_rn(t, x, make_float2(0.5f, 0.5f));
            t = __fmul2_rn(du2, __ffma2_rn(t, x, make_float2(1.f, 1.f)));
            const float2 big = __fmul2_rn(u2, __fmul2_rn(__fadd2_rn(dA[i], make_float2(-1.f, -1.f)), cc.ia[i]));
            w[i] = make_float2(fabsf(x.x) < kZohTaylorMax ? t.x : big.x, fabsf(x.y) < kZohTaylorMax ? t.y : big.y);
        }
    }
}

// One token for this lane's states: h <- Abar (.) h + Bbar*u, Bbar*u =
// Delta*u*B (Euler) or the zero-order hold (kZoh); with the read-out
// (kReadout) returns the partial C . h over these states.  `row` holds the
// lane's (B_n, B_n+2, C_n, C_n+2) chunks.
template <int N, bool kFast, bool kGeo, bool kZoh, bool kReadout = true>
__device__ __forceinline__ float token_states(float2 (&h)[N / 4], const float4 (&row)[N / 4], float du, float rdt,
                                              float uu, int half, const LaneConst<N>& cc) {
    constexpr int P = N / 4;
    float2 dA[P];
    transition<N, kFast, kGeo>(dA, rdt, half, cc);
    float2 w[P];
    if constexpr (kZoh) zoh_weights<N, kFast, kGeo>(w, dA, du, uu, rdt, half, cc);
    const float2 du2 = make_float2(du, du);
    float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < P; ++i) {
        const float4 v = row[i];  // (B_n, B_n+2, C_n, C_n+2)
        float2 bu;
        if constexpr (!kZoh)
            bu = __fmul2_rn(du2, make_float2(v.x, v.y));
        else if constexpr (kGeo)
            bu = __fmul2_rn(w[i], __fmul2_rn(du2, make_float2(v.x, v.y)));
        else
            bu = __fmul2_rn(w[i], make_float2(v.x, v.y));
        h[i] = __ffma2_rn(dA[i], h[i], bu);
        if constexpr (kReadout) {
            if (i & 1)
                acc1 = __ffma2_rn(make_float2(v.z, v.w), h[i], acc1);
            else
                acc0 = __ffma2_rn(make_float2(v.z, v.w), h[i], acc0);
        }
    }
    if constexpr (kReadout) {
        const float2 acc = __fadd2_rn(acc0, acc1);
        return acc.x + acc.y;
    } else {
        return 0.f;
    }
}

// Unpack the tokens of one 8-byte piece of a row (bf16: 4, fp32: 2).
template <typename T>
__device__ __forceinline__ void unpack8(const uint2& w, float (&v)[8 / sizeof(T)]) {
    if constexpr (sizeof(T) == 2) {
        v[0] = bf16_lo(w.x);
        v[1] = bf16_hi(w.x);
        v[2] = bf16_lo(w.y);
        v[3] = bf16_hi(w.y);
    } else {
        v[0] = __uint_as_float(w.x);
        v[1] = __uint_as_float(w.y);
    }
}

template <typename T>
__device__ __forceinline__ uint2 pack8(const float (&v)[8 / sizeof(T)]) {
    if constexpr (sizeof(T) == 2) {
        return make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
    } else {
        return make_uint2(__float_as_uint(v[0]), __float_as_uint(v[1]));
    }
}

// kFold: the first pass of a split sequence -- run the segment from a zero
// state without read-out and record its aggregates (exp(A * sum of steps) and
// the final state); otherwise the full pass, starting from the caller's state
// carried over the earlier segments' aggregates.  A fold with p.ckpt set is
// the backward pass's checkpoint pass instead: one segment from the caller's
// state, recording the state at the start of every group of V tokens.  kSave:
// a full pass that records those states as well (mss_scan_fwd_save); a
// separate variant, so that the plain full pass carries no code for it.
template <typename T, int N, bool kGeo, bool kGate, bool kSoftplus, bool kFold, bool kZoh, bool kConv,
          bool kSave = false>
__device__ __forceinline__ void scan_seq_body(const SeqMaps& maps, const ScanParams& p, uint8_t* smem,
                                              uint64_t* bars, const LaneConst<N>& cc, bool valid, int64_t row) {
    using Ly = SeqLayout<T, N>;
    constexpr bool kFast = sizeof(T) == 2;
    constexpr int S = Ly::kStages;
    constexpr int V = Ly::kVec;            // tokens per group
    constexpr int HV = Ly::kHalf;          // tokens of a group this lane finishes
    constexpr int P = Ly::kPairs;
    constexpr int GPC = Ly::kChunk / V;    // groups per chunk
    constexpr bool kZG = kZoh && kGeo;     // lanes keep (n+1) h_n, C rows hold C_n / (n+1)
    constexpr bool kZU = kZoh && !kGeo;    // per-state weights need u of every token
    const int lane = threadIdx.x;
    const int half = lane & 1;
    const int ch = lane >> 1;
    const int b = blockIdx.y;
    const int row0 = int(int64_t(b) * p.dim + int64_t(blockIdx.x) * Ly::kRows);
    const int64_t L = p.seqlen;
    const int seg = blockIdx.z;
    const int64_t t_begin = int64_t(seg) * p.seg_len;  // a multiple of the chunk
    const int64_t Ls = (L - t_begin < p.seg_len) ? L - t_begin : p.seg_len;
    const int n_chunks = int((Ls + Ly::kChunk - 1) / Ly::kChunk);
    const int n_groups = int(Ls / V);      // L and seg_len are multiples of V
    const size_t rows_total = size_t(p.batch) * size_t(p.dim);
    float* bcf = reinterpret_cast<float*>(smem + S * Ly::kStageBytes);
    const uint32_t stage_tx = uint32_t((kGate ? 3 : 2) * Ly::kTile + 2 * Ly::kBCTile);

    auto issue = [&](int chunk) {
        uint8_t* st = smem + (chunk % S) * Ly::kStageBytes;
        uint64_t* bar = bars + chunk % S;
        const int x = int(t_begin) + chunk * Ly::kChunk;
        mbar_arrive_expect_tx(bar, stage_tx);
        tma_load_2d(st, &maps.u, x, row0, bar);
        tma_load_2d(st + Ly::kTile, &maps.delta, x, row0, bar);
        if constexpr (kGate) tma_load_2d(st + 2 * Ly::kTile, &maps.z, x, row0, bar);
        tma_load_3d(st + 3 * Ly::kTile, &maps.B, x, 0, b, bar);
        tma_load_3d(st + 3 * Ly::kTile + Ly::kBCTile, &maps.C, x, 0, b, bar);
    };
    // Bounded wait for chunk c's stage; on timeout give the other copies in
    // flight a bounded chance to land and report failure (warp-uniform).
    auto wait_chunk = [&](int c) -> bool {
        const bool landed = mbar_wait_bounded(bars + c % S, uint32_t((c / S) & 1), p.err);
        if (__all_sync(0xffffffffu, landed)) return true;
        for (int c2 = c + 1; c2 < n_chunks && c2 < c + S; ++c2)
            mbar_wait_bounded(bars + c2 % S, uint32_t((c2 / S) & 1), p.err, 100000000ull);
        return false;
    };
    const int swz = ch & 7;  // 128-byte swizzle: 16-byte chunk j of row r sits at j ^ (r & 7)
    // this lane's half of group g's u, delta, z (8 bytes of its channel's row each)
    // causal convolution (kConv): the three inputs before the current group
    float xl[3] = {0.f, 0.f, 0.f};
    auto load_half = [&](int g, float (&uv)[HV], float (&dv)[HV], float (&zv)[HV], bool advance) {
        const int c = g / GPC, j = g % GPC;
        const uint8_t* src = smem + (c % S) * Ly::kStageBytes + ch * Ly::kRowBytes + ((j ^ swz) << 4) + 8 * half;
        if constexpr (kConv) {
            // the whole group of x (both lanes of the pair read the same 16 bytes)
            float xa[HV], xb[HV];
            const uint4 w4 = *reinterpret_cast<const uint4*>(src - 8 * half);
            unpack8<T>(make_uint2(w4.x, w4.y), xa);
            unpack8<T>(make_uint2(w4.z, w4.w), xb);
            float xv[V];
#pragma unroll
            for (int i = 0; i < HV; ++i) {
                xv[i] = xa[i];
                xv[HV + i] = xb[i];
            }
            // this lane's window: inputs half*HV - 3 .. half*HV + HV - 1 of the group
            // (index e of the extended row xl[0..2], xv[0..V-1] is input e - 3)
            auto ext = [&](int e) { return e < 3 ? xl[e] : xv[e - 3]; };
            float win[HV + 3];
#pragma unroll
            for (int i = 0; i < HV + 3; ++i) win[i] = half ? ext(HV + i) : ext(i);
#pragma unroll
            for (int k = 0; k < HV; ++k) {
                const float pre = conv_pre(cc.conv, win[k], win[k + 1], win[k + 2], win[k + 3]);
                uv[k] = kFast ? silu_fast(pre) : silu_precise(pre);
            }
            if (advance) {
                xl[0] = xv[V - 3];
                xl[1] = xv[V - 2];
                xl[2] = xv[V - 1];
            }
        } else {
            unpack8<T>(*reinterpret_cast<const uint2*>(src), uv);
        }
        unpack8<T>(*reinterpret_cast<const uint2*>(src + Ly::kTile), dv);
        if constexpr (kGate) unpack8<T>(*reinterpret_cast<const uint2*>(src + 2 * Ly::kTile), zv);
    };
    if constexpr (kConv) {
        const int K = p.conv_width;
        if (t_begin == 0) {
            if (p.conv_state_in) {
                const T* cs = static_cast<const T*>(p.conv_state_in) + row * (K - 1);
#pragma unroll
                for (int i = 0; i < 3; ++i) {  // slot i holds stored input i - (4 - K)
                    const int k = i - (4 - K);
                    if (k >= 0) xl[i] = ld(cs + k);
                }
            }
        } else {
            // a later segment: the inputs just before it (t_begin >= one chunk > 3)
            const T* xr = static_cast<const T*>(p.u) + row * L + t_begin;
#pragma unroll
            for (int i = 0; i < 3; ++i) xl[i] = ld(xr - 3 + i);
        }
    }

    if (lane == 0) {
        for (int c = 0; c < S && c < n_chunks; ++c) issue(c);
    }
    // starting state: zero for a fold (the caller's state for a checkpoint
    // pass); otherwise the caller's state carried over the aggregates of the
    // earlier segments
    float2 h[P];
#pragma unroll
    for (int i = 0; i < P; ++i) h[i] = make_float2(0.f, 0.f);
    if (!kFold || p.ckpt) {
        if (p.initial_state) {
            const float* h0 = p.initial_state + row * N + half;
#pragma unroll
            for (int i = 0; i < P; ++i) h[i] = make_float2(h0[4 * i], h0[4 * i + 2]);
        }
        for (int s2 = 0; s2 < (kFold ? 0 : seg); ++s2) {
            const float* ga = p.agg + ((size_t(s2) * 2) * rows_total + size_t(row)) * N + half;
            const float* gb = ga + rows_total * N;
#pragma unroll
            for (int i = 0; i < P; ++i)
                h[i] = __ffma2_rn(make_float2(ga[4 * i], ga[4 * i + 2]), h[i], make_float2(gb[4 * i], gb[4 * i + 2]));
        }
        if constexpr (kZG) {
#pragma unroll
            for (int i = 0; i < P; ++i)
                h[i] = __fmul2_rn(h[i], make_float2(float(half + 4 * i + 1), float(half + 4 * i + 3)));
        }
    }
    // the state as h_n (undoing the (n+1) scale of the zero-order hold)
    auto state_out = [&](int i) -> float2 {
        if constexpr (kZG)
            return make_float2(h[i].x / float(half + 4 * i + 1), h[i].y / float(half + 4 * i + 3));
        else
            return h[i];
    };
    // checkpoint pass, or a forward pass that saves the states: the state at
    // the start of every group of V tokens, in h_n form, as [row][group][N]
    // floats over the whole sequence in lane order (lane half h's N/2 floats
    // at h * N/2: its pairs (h_n, h_n+2), n = h + 4i)
    auto store_ckpt = [&](int group) {
        if (!valid) return;
        const size_t g_all = size_t(t_begin / V) + size_t(group);
        float2* ck = reinterpret_cast<float2*>(p.ckpt + (size_t(row) * size_t(L / V) + g_all) * N) + half * P;
#pragma unroll
        for (int i = 0; i < P; i += 2) {
            if (i + 1 < P) {
                const float2 a = state_out(i), b2 = state_out(i + 1);
                *reinterpret_cast<float4*>(ck + i) = make_float4(a.x, a.y, b2.x, b2.y);
            } else {
                ck[i] = state_out(i);
            }
        }
    };
    float dsum = 0.f, dcomp = 0.f;  // fold: compensated sum of this lane's steps
    T* yrow = static_cast<T*>(p.y) + row * L + t_begin + HV * half;
    const float4* my_bcf = reinterpret_cast<const float4*>(bcf) + half * P;  // this lane's chunks of a row
    constexpr int kRowF4 = Ly::kBCfRow / 4;

    if (!wait_chunk(0)) return;
    convert_bc<T, N, kZG>(smem + 3 * Ly::kTile, smem + 3 * Ly::kTile + Ly::kBCTile, bcf, lane);
    __syncwarp();

    // Software pipeline across groups.  Carried into iteration g:
    //   own[]        this lane's scalars of group g's tokens [half*HV, half*HV + HV)
    //   pdu[], prd[] the partner's Delta*u and r (or Delta) of group g
    //   nrow[]       group g's first B/C row
    //   the previous group's transpose-reduce (finished after token 1 of g)
    TokenPre own[HV];
    float pdu[HV], prd[HV], pu[HV];
    {
        float uv[HV], dv[HV], zv[HV];
        load_half(0, uv, dv, zv, true);
#pragma unroll
        for (int k = 0; k < HV; ++k) {
            own[k] = token_pre<kFast, kGeo, kGate, kSoftplus, kZoh>(uv[k], dv[k], kGate ? zv[k] : 0.f, cc);
            pdu[k] = __shfl_xor_sync(0xffffffffu, own[k].du, 1);
            prd[k] = __shfl_xor_sync(0xffffffffu, own[k].r, 1);
            if constexpr (kZU) pu[k] = __shfl_xor_sync(0xffffffffu, own[k].u, 1);
        }
    }
    float4 nrow[P];
#pragma unroll
    for (int i = 0; i < P; ++i) nrow[i] = my_bcf[i];
    float pkeep[HV], precv[HV], pskip[HV], pgate[HV];  // previous group's pending outputs
    int64_t pend_at = -1;                               // its token offset, -1: none

#pragma unroll 1
    for (int g = 0; g < n_groups; ++g) {
        const int c = g / GPC, j = g % GPC;
        const bool has_next = g + 1 < n_groups;
        if constexpr (kFold || kSave) {
            if (p.ckpt) store_ckpt(g);
        }
        // the next group's u/delta/z, first: its stage must have landed when it opens a new chunk
        if (has_next && j == GPC - 1 && !wait_chunk(c + 1)) return;
        float uv[HV], dv[HV], zv[HV];
        load_half(has_next ? g + 1 : g, uv, dv, zv, has_next);

        TokenPre nxt[HV];
        float acc[V];
        const float4* base = my_bcf + (j * V) * kRowF4;
#pragma unroll
        for (int t = 0; t < V; ++t) {
            float4 rowv[P];
#pragma unroll
            for (int i = 0; i < P; ++i) rowv[i] = nrow[i];
            if (t + 1 < V) {
#pragma unroll
                for (int i = 0; i < P; ++i) nrow[i] = base[(t + 1) * kRowF4 + i];
            } else if (j + 1 < GPC) {
                // the next group's first row (same chunk: already converted)
#pragma unroll
                for (int i = 0; i < P; ++i) nrow[i] = base[V * kRowF4 + i];
            }
            // token t belongs to lane half t / HV of the pair
            const bool mine = (t / HV) == half;
            const float du = mine ? own[t % HV].du : pdu[t % HV];
            const float rdt = mine ? own[t % HV].r : prd[t % HV];
            const float uu = kZU ? (mine ? own[t % HV].u : pu[t % HV]) : 0.f;
            acc[t] = token_states<N, kFast, kGeo, kZoh, !kFold>(h, rowv, du, rdt, uu, half, cc);
            // the previous group's outputs, once their shuffles have had time
            if (!kFold && t == 1 && pend_at >= 0) {
                float yv[HV];
#pragma unroll
                for (int k = 0; k < HV; ++k) yv[k] = (pkeep[k] + precv[k] + pskip[k]) * pgate[k];
                if (valid) *reinterpret_cast<uint2*>(yrow + pend_at) = pack8<T>(yv);
            }
            // the next group's scalars, spread over the middle tokens
            constexpr int kPre0 = V >= 8 ? 2 : 0;
            if (t >= kPre0 && t < kPre0 + HV)
                nxt[t - kPre0] = token_pre<kFast, kGeo, kGate, kSoftplus, kZoh>(uv[t - kPre0], dv[t - kPre0],
                                                                                  kGate ? zv[t - kPre0] : 0.f, cc);
        }
        if constexpr (kFold) {
            // compensated (Kahan) sum of this lane's steps
#pragma unroll
            for (int k = 0; k < HV; ++k) {
                const float yk = own[k].dt - dcomp;
                const float tk = dsum + yk;
                dcomp = (tk - dsum) - yk;
                dsum = tk;
            }
        } else {
            // this group's read-out: transpose-reduce (lane half h finishes
            // tokens [h*HV, h*HV + HV)); finished after token 1 of the next group
#pragma unroll
            for (int k = 0; k < HV; ++k) {
                const float send = half ? acc[k] : acc[HV + k];
                pkeep[k] = half ? acc[HV + k] : acc[k];
                precv[k] = __shfl_xor_sync(0xffffffffu, send, 1);
                pskip[k] = own[k].skip;
                pgate[k] = own[k].gate;
            }
            pend_at = int64_t(g) * V;
        }
        // hand over the next group's scalars
#pragma unroll
        for (int k = 0; k < HV; ++k) {
            own[k] = nxt[k];
            pdu[k] = __shfl_xor_sync(0xffffffffu, nxt[k].du, 1);
            prd[k] = __shfl_xor_sync(0xffffffffu, nxt[k].r, 1);
            if constexpr (kZU) pu[k] = __shfl_xor_sync(0xffffffffu, nxt[k].u, 1);
        }

        if (j == GPC - 1 || !has_next) {
            // chunk c is consumed: convert the next chunk's B/C (its stage was
            // waited for above), then hand chunk c's stage to chunk c + S
            __syncwarp();
            if (has_next) {
                const uint8_t* st = smem + ((c + 1) % S) * Ly::kStageBytes;
                convert_bc<T, N, kZG>(st + 3 * Ly::kTile, st + 3 * Ly::kTile + Ly::kBCTile, bcf, lane);
            }
            __syncwarp();
            if (lane == 0 && c + S < n_chunks) {
                fence_proxy_async_smem();
                issue(c + S);
            }
            // the next group's first row, now that its chunk is converted
#pragma unroll
            for (int i = 0; i < P; ++i) nrow[i] = my_bcf[i];
        }
    }
    if constexpr (kFold) {
        // aggregates of this segment: exp(A_n * sum of its steps) and the state
        // it ends in from zero
        const float tot = (dsum + __shfl_xor_sync(0xffffffffu, dsum, 1)) -
                          (dcomp + __shfl_xor_sync(0xffffffffu, dcomp, 1));
        if (valid && p.agg) {
            float* ga = p.agg + ((size_t(seg) * 2) * rows_total + size_t(row)) * N + half;
            float* gb = ga + rows_total * N;
#pragma unroll
            for (int i = 0; i < P; ++i) {
                float2 a;
                if constexpr (kFast)
                    a = make_float2(ex2_approx(cc.a2[i].x * tot), ex2_approx(cc.a2[i].y * tot));
                else
                    a = make_float2(expf(cc.a2[i].x * tot), expf(cc.a2[i].y * tot));
                const float2 hs = state_out(i);
                ga[4 * i] = a.x;
                ga[4 * i + 2] = a.y;
                gb[4 * i] = hs.x;
                gb[4 * i + 2] = hs.y;
            }
        }
        return;
    }
    // the last group's outputs
    if (pend_at >= 0) {
        float yv[HV];
#pragma unroll
        for (int k = 0; k < HV; ++k) yv[k] = (pkeep[k] + precv[k] + pskip[k]) * pgate[k];
        if (valid) *reinterpret_cast<uint2*>(yrow + pend_at) = pack8<T>(yv);
    }
    if constexpr (kConv) {
        // the conv state after the sequence: its last K-1 inputs
        const int K = p.conv_width;
        if (valid && half == 0 && p.conv_state_out && seg == p.n_seg - 1) {
            T* cs = static_cast<T*>(p.conv_state_out) + row * (K - 1);
#pragma unroll
            for (int i = 0; i < 3; ++i) {
                const int k = i - (4 - K);
                if (k >= 0) cs[k] = from_f32<T>(xl[i]);
            }
        }
    }
    if (valid && p.last_state && seg == p.n_seg - 1) {
        float* ls = p.last_state + row * N + half;
#pragma unroll
        for (int i = 0; i < P; ++i) {
            const float2 hs = state_out(i);
            ls[4 * i] = hs.x;
            ls[4 * i + 2] = hs.y;
        }
    }
}

// grid = (ceil(dim / 16), batch, segments), block = 32 threads, dynamic
// shared memory SeqLayout<T, N>::kSmemBytes.  A fold launch covers segments
// 0 .. n_seg-2, the full pass all n_seg (after the fold has completed).
// Requirements checked by the host: N in {4, 8, 16}; L * sizeof(T) a multiple
// of 16; u, delta, z, B, C, y 16-byte aligned; seg_len a multiple of the chunk.
template <typename T, int N, bool kGate, bool kSoftplus, bool kFold, bool kZoh, bool kConv, bool kSave = false>
__global__ void __launch_bounds__(32) scan_fwd_seq_kernel(const __grid_constant__ SeqMaps maps, ScanParams p,
                                                          int allow_geo) {
    using Ly = SeqLayout<T, N>;
    constexpr int P = Ly::kPairs;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    // 1024-byte alignment (128-byte swizzle atoms) by pointer arithmetic on the
    // shared array itself, so that every derived pointer stays a shared-memory
    // pointer and its loads compile to shared loads, not generic ones
    uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Ly::kBarOffset);
    const int lane = threadIdx.x;
    const int half = lane & 1;

    const int64_t c = int64_t(blockIdx.x) * Ly::kRows + (lane >> 1);
    const bool valid = c < p.dim;
    const int64_t d = valid ? c : 0;
    const int64_t row = int64_t(blockIdx.y) * p.dim + d;

    if (lane == 0) {
        for (int s = 0; s <= Ly::kStages; ++s) mbar_init(bars + s, 1);
        fence_barrier_init();
        prefetch_tensormap(&maps.u);
        prefetch_tensormap(&maps.delta);
        if (kGate) prefetch_tensormap(&maps.z);
        prefetch_tensormap(&maps.B);
        prefetch_tensormap(&maps.C);
    }
    __syncwarp();
    if (p.selftest_wait_ns) {
        // wait self-test: barrier kStages never completes (no copy has been
        // issued and nothing arrives), so the bounded wait gives up and sets
        // the error word; the CTA returns with nothing in flight
        mbar_wait_bounded(bars + Ly::kStages, 0u, p.err, p.selftest_wait_ns);
        return;
    }

    constexpr bool kFast = sizeof(T) == 2;
    LaneConst<N> cc;
    cc.bias = p.delta_bias ? p.delta_bias[d] : 0.f;
    cc.D = p.D ? p.D[d] : 0.f;
    const float* Arow = p.A + d * N;
    const float a_first = Arow[0];
    cc.a0 = a_first * kLog2e;
    if constexpr (kZoh) cc.ia0 = 1.f / a_first;  // inf at A = 0, where only the Taylor branch is taken
    if constexpr (kConv) cc.conv = load_conv_taps(p.conv_w, p.conv_b, p.conv_width, d);
    bool geo = kFast && allow_geo;
#pragma unroll
    for (int i = 0; i < P; ++i) {
        const int n = half + 4 * i;
        const float x0 = Arow[n], x1 = Arow[n + 2];
        cc.a2[i] = kFast ? make_float2(x0 * kLog2e, x1 * kLog2e) : make_float2(x0, x1);
        if constexpr (kZoh) cc.ia[i] = make_float2(1.f / x0, 1.f / x1);
        geo = geo && x0 == float(n + 1) * a_first && x1 == float(n + 3) * a_first;
    }
    geo = __all_sync(0xffffffffu, geo || !valid);

    if constexpr (kFast) {
        if (geo) {
            scan_seq_body<T, N, true, kGate, kSoftplus, kFold, kZoh, kConv, kSave>(maps, p, smem, bars, cc, valid, row);
            return;
        }
    }
    scan_seq_body<T, N, false, kGate, kSoftplus, kFold, kZoh, kConv, kSave>(maps, p, smem, bars, cc, valid, row);
}

}  // namespace mss
