// scan_bwd.cuh -- backward pass of the selective scan, with recomputation.
//
// The pages train the model end to end and say the fused kernel recomputes
// the states in the backward pass instead of storing them ("Mamba" paper
// review, section "Selection Mechanism").  This kernel is the chain rule of
// the forward definition walked backwards in time:
//
//   gh = dLoss/dh_t:  gh += dr_t C_t;  dC_t += dr_t h_t;  dB_t += gh w_t u_t;
//   du_t += gh w_t B_t;  dDelta_t += gh (h_{t-1} a_t A + B_t u_t dw/dDelta);
//   dA += gh (h_{t-1} a_t Delta_t + B_t u_t dw/dA);  gh *= a_t,
//
// with dr_t = dy_t silu(z_t), dz_t = dy_t r_t silu'(z_t), ddelta_raw =
// dDelta softplus'(s) and the skip term's du += dr D, dD += dr u.
//
// States.  A checkpoint pass (the forward kernel's fold launch with p.ckpt)
// records the state at the start of every group of V tokens (8 bytes per
// channel and token at N = 16, against the 14 bytes of inputs and gradients
// the pass moves anyway).  This kernel walks the chunks from last to first,
// the group-start states arriving by TMA with the chunk's other tiles, and
// the groups of a chunk from last to first: it recomputes the state in the
// middle of the group, then each half's HV states into registers, and runs
// the HV reverse steps of the half.  A state is recomputed 1.5 times on
// average; none is stored in HBM besides the checkpoints.
//
// Work split and reductions.  As in the forward kernel, a CTA is one warp
// serving 16 channels of a batch row, a lane pair per channel, each lane
// holding N/2 states.  Per-channel sums (dA, dD, dbias) stay in registers and
// are added into HBM once per CTA.  dB and dC are sums over the channels of a
// batch row: each token's 2N per-lane values are reduce-scattered over the
// 16 channels of the warp with shuffles (15 at N = 16), leaving one (state,
// B or C) sum per lane, which is kept for the V tokens of a group and added
// into HBM with one vector reduction (red.global.v4.f32.add) per 4 tokens.
// The float additions of different CTAs land in an unspecified order, so
// dB, dC, dA, dD and dbias are not bitwise reproducible from run to run.
//
// The transition uses the forward kernel's fast form (Abar_n = r^{n+1}) when
// A[d,n] = (n+1) A[d,0] across the warp; the zero-order-hold input rule
// always takes the general form here.  Waits are bounded as in the forward
// kernel.
#pragma once

#include <type_traits>

#include "scan_seq.cuh"

namespace mss {

struct BwdMaps {
    CUtensorMap u, delta, z, dy, B, C, ck;
};

template <typename T, int N>
struct BwdLayout {
    using F = SeqLayout<T, N>;
    static constexpr int kRows = F::kRows;
    static constexpr int kRowBytes = F::kRowBytes;
    static constexpr int kChunk = F::kChunk;
    static constexpr int kVec = F::kVec;
    static constexpr int kGroups = kChunk / kVec;          // groups per chunk
    static constexpr int kPairs = F::kPairs;
    static constexpr int kTile = F::kTile;
    static constexpr int kBCTile = F::kBCTile;
    // the group-start states of the chunk: [16 rows][kGroups][N] floats
    static constexpr int kCkTile = kRows * kGroups * N * 4;
    // one stage: the next chunk's tiles are fetched while the chunk's first
    // group is reversed, once every tile word has been read (B and C are read
    // when the chunk starts); a second stage would cost a CTA per SM
    static constexpr int kStages = 1;
    static constexpr int kCkOffset = 4 * kTile + 2 * kBCTile;
    static constexpr int kStageBytes = kCkOffset + kCkTile;  // u, delta, z, dy, B, C, states
    static constexpr int kBCfRow = F::kBCfRow;
    static constexpr int kBCfBytes = F::kBCfBytes;
    static constexpr int kBCfOffset = kStages * kStageBytes;
    static constexpr int kBarOffset = kBCfOffset + kBCfBytes;
    static constexpr int kSmemBytes = kBarOffset + kStages * 8 + 1024;
    static_assert(kStageBytes % 1024 == 0, "stage tiles must stay 1024-byte aligned");
};

// Per-token scalars of the backward pass.
struct BwdTok {
    float dt;   // Delta
    float du;   // Delta * u
    float rdt;  // r = exp(Delta A[d,0]) (fast transition) or Delta
    float dsp;  // dDelta / ddelta_raw: sigmoid(s) with softplus, else 1
};

// dDelta / ddelta_raw: the slope of the softplus, sigmoid(s), else 1.
template <bool kFast, bool kSoftplus>
__device__ __forceinline__ float softplus_slope(float s) {
    if constexpr (!kSoftplus) return 1.f;
    return kFast ? rcp_approx(1.f + ex2_approx(-s * kLog2e)) : 1.f / (1.f + expf(-s));
}

// Delta, Delta * u and r of one token (dsp is left at 1: the slope is formed
// only for the tokens whose gradient a lane stores).
template <bool kFast, bool kGeo, bool kSoftplus, int N>
__device__ __forceinline__ BwdTok bwd_token(float ut, float dr, const LaneConst<N>& cc) {
    BwdTok tk;
    const float s = dr + cc.bias;
    tk.dt = s;
    tk.dsp = 1.f;
    if constexpr (kSoftplus) tk.dt = kFast ? softplus_fast(s) : softplus_precise(s);
    tk.du = tk.dt * ut;
    tk.rdt = kGeo ? ex2_approx(tk.dt * cc.a0) : tk.dt;
    return tk;
}

// Token t of a 16-byte group held as its raw word (t a compile-time index).
template <typename T>
__device__ __forceinline__ float elem16(const uint4& w, int t) {
    constexpr int per = 4 / int(sizeof(T));  // tokens per 32-bit word
    const int k = t / per;
    const uint32_t word = k == 0 ? w.x : k == 1 ? w.y : k == 2 ? w.z : w.w;
    if constexpr (sizeof(T) == 2)
        return (t & 1) ? bf16_hi(word) : bf16_lo(word);
    else
        return __uint_as_float(word);
}

// The 8 (bf16) or 4 (fp32) tokens of one 16-byte group.
template <typename T>
__device__ __forceinline__ void unpack16(const uint4& w, float (&v)[16 / sizeof(T)]) {
    constexpr int H = 8 / int(sizeof(T));
    float a[H], b[H];
    unpack8<T>(make_uint2(w.x, w.y), a);
    unpack8<T>(make_uint2(w.z, w.w), b);
#pragma unroll
    for (int i = 0; i < H; ++i) {
        v[i] = a[i];
        v[H + i] = b[i];
    }
}

// Sum of the M = 4 * (N/4) values v over the 16 channels of the warp (lane
// bits 1..4), scattered: the lane keeps one sum; returns it.  `index` is the
// value it holds, `writer` whether this lane is the one of its group that
// stores it (for N < 16 the last channel bits are summed by all).
template <int M>
__device__ __forceinline__ float reduce_scatter_channels(float (&v)[M], int lane, int& index, bool& writer) {
    int c = M;
    index = 0;
#pragma unroll
    for (int bit = 1; bit <= 4; ++bit) {
        const int m = 1 << bit;
        const bool up = (lane & m) != 0;
        if (c > 1) {
            const int hcount = c / 2;
#pragma unroll
            for (int j = 0; j < M / 2; ++j) {
                if (j < hcount) {
                    const float send = up ? v[j] : v[j + hcount];
                    const float keep = up ? v[j + hcount] : v[j];
                    v[j] = keep + __shfl_xor_sync(0xffffffffu, send, m);
                }
            }
            if (up) index += hcount;
            c = hcount;
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], m);
        }
    }
    // for M < 16 the bits after the scatter are summed: lanes with those bits
    // clear store
    writer = true;
    int scatter_bits = 0;
    for (int cc = M; cc > 1; cc >>= 1) ++scatter_bits;
#pragma unroll
    for (int bit = 1; bit <= 4; ++bit)
        if (bit > scatter_bits && (lane & (1 << bit))) writer = false;
    return v[0];
}

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
    asm volatile("red.global.v4.f32.add [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

__device__ __forceinline__ void red_add_v2(float* p, float a, float b) {
    asm volatile("red.global.v2.f32.add [%0], {%1, %2};" ::"l"(p), "f"(a), "f"(b) : "memory");
}

template <typename T, int N, bool kGeo, bool kGate, bool kSoftplus, bool kZoh>
__device__ __forceinline__ void scan_bwd_body(const BwdMaps& maps, const BwdParams& p, uint8_t* smem,
                                              uint64_t* bars, const LaneConst<N>& cc, bool valid, int64_t row) {
    using Ly = BwdLayout<T, N>;
    constexpr bool kFast = sizeof(T) == 2;
    constexpr int S = Ly::kStages;
    constexpr int V = Ly::kVec;
    constexpr int HV = V / 2;
    constexpr int P = Ly::kPairs;
    constexpr int GPC = Ly::kGroups;
    constexpr int M = 4 * P;  // dB and dC values of a lane per token
    static_assert(!(kZoh && kGeo), "the zero-order hold takes the general transition here");
    const int lane = threadIdx.x;
    const int half = lane & 1;
    const int ch = lane >> 1;
    const int b = blockIdx.y;
    const int row0 = int(int64_t(b) * p.dim + int64_t(blockIdx.x) * Ly::kRows);
    const int64_t L = p.seqlen;
    const int n_chunks = int((L + Ly::kChunk - 1) / Ly::kChunk);
    const int64_t d = row - int64_t(b) * p.dim;
    float* bcf = reinterpret_cast<float*>(smem + Ly::kBCfOffset);
    const uint32_t stage_tx = uint32_t((kGate ? 4 : 3) * Ly::kTile + 2 * Ly::kBCTile + Ly::kCkTile);

    // the k-th chunk processed is chunk n_chunks - 1 - k
    auto issue = [&](int k) {
        uint8_t* st = smem + (k % S) * Ly::kStageBytes;
        uint64_t* bar = bars + k % S;
        const int x = (n_chunks - 1 - k) * Ly::kChunk;
        mbar_arrive_expect_tx(bar, stage_tx);
        tma_load_2d(st, &maps.u, x, row0, bar);
        tma_load_2d(st + Ly::kTile, &maps.delta, x, row0, bar);
        if constexpr (kGate) tma_load_2d(st + 2 * Ly::kTile, &maps.z, x, row0, bar);
        tma_load_2d(st + 3 * Ly::kTile, &maps.dy, x, row0, bar);
        tma_load_3d(st + 4 * Ly::kTile, &maps.B, x, 0, b, bar);
        tma_load_3d(st + 4 * Ly::kTile + Ly::kBCTile, &maps.C, x, 0, b, bar);
        tma_load_2d(st + Ly::kCkOffset, &maps.ck, (n_chunks - 1 - k) * GPC * N, row0, bar);
    };
    auto wait_chunk = [&](int k) -> bool {
        const bool landed = mbar_wait_bounded(bars + k % S, uint32_t((k / S) & 1), p.err);
        if (__all_sync(0xffffffffu, landed)) return true;
        for (int k2 = k + 1; k2 < n_chunks && k2 < k + S; ++k2)
            mbar_wait_bounded(bars + k2 % S, uint32_t((k2 / S) & 1), p.err, 100000000ull);
        return false;
    };
    if (lane == 0) {
        for (int k = 0; k < S && k < n_chunks; ++k) issue(k);
    }

    const int swz = ch & 7;
    auto group_word = [&](const uint8_t* st, int tile, int g) -> uint4 {
        return *reinterpret_cast<const uint4*>(st + tile * Ly::kTile + ch * Ly::kRowBytes + ((g ^ swz) << 4));
    };
    const float4* my_bcf = reinterpret_cast<const float4*>(bcf) + half * P;
    constexpr int kRowF4 = Ly::kBCfRow / 4;
    // natural A of a state pair
    auto a_nat = [&](int i) { return kFast ? __fmul2_rn(cc.a2[i], make_float2(kLn2, kLn2)) : cc.a2[i]; };

    // adjoint state, per-channel sums
    float2 gh[P], dA_acc[P];
#pragma unroll
    for (int i = 0; i < P; ++i) {
        gh[i] = make_float2(0.f, 0.f);
        dA_acc[i] = make_float2(0.f, 0.f);
    }
    if (p.dlast && valid) {
        const float* dl = p.dlast + row * N + half;
#pragma unroll
        for (int i = 0; i < P; ++i) gh[i] = make_float2(dl[4 * i], dl[4 * i + 2]);
    }
    float dD_acc = 0.f, dbias_acc = 0.f;

    for (int k = 0; k < n_chunks; ++k) {
        const int c = n_chunks - 1 - k;
        if (!wait_chunk(k)) return;
        const uint8_t* st = smem + (k % S) * Ly::kStageBytes;
        convert_bc<T, N, false>(st + 4 * Ly::kTile, st + 4 * Ly::kTile + Ly::kBCTile, bcf, lane);
        __syncwarp();
        const int64_t t_chunk = int64_t(c) * Ly::kChunk;
        const int ng = int(min(int64_t(GPC), (L - t_chunk) / V));

        // groups from last to first; each group in two halves of HV tokens
        // (second half first), so that only HV recomputed states are live
#pragma unroll 1
        for (int g = ng - 1; g >= 0; --g) {
            uint4 zw = make_uint4(0u, 0u, 0u, 0u), yw;
            const uint4 uw = group_word(st, 0, g);
            const uint4 dw = group_word(st, 1, g);
            if constexpr (kGate) zw = group_word(st, 2, g);
            yw = valid ? group_word(st, 3, g) : make_uint4(0u, 0u, 0u, 0u);  // past the last channel: no gradient
            // the group's start state, from the checkpoint pass
            float2 h0[P], hmid[P];
            {
                const float2* ck = reinterpret_cast<const float2*>(st + Ly::kCkOffset) + (ch * GPC + g) * (N / 2) + half * P;
#pragma unroll
                for (int i = 0; i < P; ++i) h0[i] = hmid[i] = ck[i];
            }
            if (g == 0) {
                // every tile word of the chunk has been read: fetch the next chunk
                __syncwarp();
                if (lane == 0 && k + S < n_chunks) {
                    fence_proxy_async_smem();
                    issue(k + S);
                }
            }
            // the group's per-token scalars: Delta and r for all V tokens (each
            // lane of the pair forms them all, which costs less than swapping
            // them), the softplus slope for the HV tokens this lane stores
            // (tokens half * HV ..)
            float dtv[V], rv[V], dspv[HV];
            {
                float uv[V], dv[V];
                unpack16<T>(uw, uv);
                unpack16<T>(dw, dv);
#pragma unroll
                for (int t = 0; t < V; ++t) {
                    const BwdTok tk = bwd_token<kFast, kGeo, kSoftplus>(uv[t], dv[t], cc);
                    dtv[t] = tk.dt;
                    rv[t] = tk.rdt;
                }
#pragma unroll
                for (int k2 = 0; k2 < HV; ++k2)
                    dspv[k2] = softplus_slope<kFast, kSoftplus>((half ? dv[HV + k2] : dv[k2]) + cc.bias);
            }
            const float4* base = my_bcf + (g * V) * kRowF4;
#pragma unroll
            for (int t = 0; t < HV; ++t) {
                float4 rowv[P];
#pragma unroll
                for (int i = 0; i < P; ++i) rowv[i] = base[t * kRowF4 + i];
                const float ut = elem16<T>(uw, t);
                token_states<N, kFast, kGeo, kZoh, false>(hmid, rowv, dtv[t] * ut, rv[t], ut, half, cc);
            }
            const int64_t tg = t_chunk + int64_t(g) * V;
            // the second half, then the first: one copy of the code
#pragma unroll 1
            for (int hf = 1; hf >= 0; --hf) {
                const int T0 = hf * HV;
                BwdTok th[HV];
                float uh[HV], zh[HV], yh[HV];
                // the half's 8 bytes of each group word
                unpack8<T>(hf ? make_uint2(uw.z, uw.w) : make_uint2(uw.x, uw.y), uh);
                unpack8<T>(hf ? make_uint2(yw.z, yw.w) : make_uint2(yw.x, yw.y), yh);
                if constexpr (kGate) unpack8<T>(hf ? make_uint2(zw.z, zw.w) : make_uint2(zw.x, zw.y), zh);
#pragma unroll
                for (int k2 = 0; k2 < HV; ++k2) {
                    th[k2].dt = hf ? dtv[HV + k2] : dtv[k2];
                    th[k2].rdt = hf ? rv[HV + k2] : rv[k2];
                    th[k2].dsp = dspv[k2];  // the right token's on the lane that stores this half
                }
                const float4* hbase = base + T0 * kRowF4;
                float2 hst[P];
#pragma unroll
                for (int i = 0; i < P; ++i) hst[i] = hf ? hmid[i] : h0[i];
                float2 hs[HV][P];
                {
                    float2 hh[P];
#pragma unroll
                    for (int i = 0; i < P; ++i) hh[i] = hst[i];
#pragma unroll
                    for (int t = 0; t < HV; ++t) {
                        float4 rowv[P];
#pragma unroll
                        for (int i = 0; i < P; ++i) rowv[i] = hbase[t * kRowF4 + i];
                        token_states<N, kFast, kGeo, kZoh, false>(hh, rowv, th[t].dt * uh[t], th[t].rdt, uh[t], half, cc);
#pragma unroll
                        for (int i = 0; i < P; ++i) hs[t][i] = hh[i];
                    }
                }
                float red[HV], du_o[HV], ds_o[HV], dz_o[HV];
                int red_index = 0;
                bool red_writer = true;
#pragma unroll
                for (int tt = HV - 1; tt >= 0; --tt) {
                    const BwdTok& tk = th[tt];
                    const float ut = uh[tt];
                    float4 rowv[P];
#pragma unroll
                    for (int i = 0; i < P; ++i) rowv[i] = hbase[tt * kRowF4 + i];
                    // read-out and gate
                    float dr = yh[tt];
                    if constexpr (kGate) {
                        float2 racc2 = make_float2(0.f, 0.f);
#pragma unroll
                        for (int i = 0; i < P; ++i) racc2 = __ffma2_rn(make_float2(rowv[i].z, rowv[i].w), hs[tt][i], racc2);
                        const float racc = racc2.x + racc2.y;
                        const float r = racc + __shfl_xor_sync(0xffffffffu, racc, 1) + cc.D * ut;
                        const float zt = zh[tt];
                        const float sz = kFast ? rcp_approx(1.f + ex2_approx(-zt * kLog2e)) : 1.f / (1.f + expf(-zt));
                        dz_o[tt] = yh[tt] * r * (sz * fmaf(zt, 1.f - sz, 1.f));
                        dr = yh[tt] * (zt * sz);
                    }
                    float2 dA[P];
                    transition<N, kFast, kGeo>(dA, tk.rdt, half, cc);
                    float vals[M];
                    float du_t, ds_t;
                    if constexpr (!kZoh) {
                        // Euler: w_n = Delta for every state, so
                        //   du    = Delta * S1 + dr D,       S1 = sum_n g_n B_n,
                        //   dDelta = u * S1 + S2,            S2 = sum_n q_n A_n,
                        //   dA_n += Delta q_n,  dB_n = Delta u g_n,  dC_n = dr h_n,
                        // with g_n = gh_n + dr C_n and q_n = g_n Abar_n h_{t-1,n} = gh'_n h_{t-1,n}
                        const float2 dr2 = make_float2(dr, dr), dt2 = make_float2(tk.dt, tk.dt);
                        const float2 du2 = make_float2(tk.dt * ut, tk.dt * ut);
                        float2 s1 = make_float2(0.f, 0.f), s2 = make_float2(0.f, 0.f);
#pragma unroll
                        for (int i = 0; i < P; ++i) {
                            const float2 hp = tt > 0 ? hs[tt > 0 ? tt - 1 : 0][i] : hst[i];
                            const float2 g = __ffma2_rn(dr2, make_float2(rowv[i].z, rowv[i].w), gh[i]);
                            const float2 dc = __fmul2_rn(dr2, hs[tt][i]);
                            const float2 db = __fmul2_rn(du2, g);
                            s1 = __ffma2_rn(g, make_float2(rowv[i].x, rowv[i].y), s1);
                            gh[i] = __fmul2_rn(g, dA[i]);
                            const float2 q = __fmul2_rn(gh[i], hp);
                            s2 = __ffma2_rn(q, cc.a2[i], s2);  // A in log2 units for bf16 io
                            dA_acc[i] = __ffma2_rn(q, dt2, dA_acc[i]);
                            vals[2 * i] = db.x;
                            vals[2 * i + 1] = db.y;
                            vals[P * 2 + 2 * i] = dc.x;
                            vals[P * 2 + 2 * i + 1] = dc.y;
                        }
                        float S1 = s1.x + s1.y, S2 = s2.x + s2.y;
                        S1 += __shfl_xor_sync(0xffffffffu, S1, 1);
                        S2 += __shfl_xor_sync(0xffffffffu, S2, 1);
                        if constexpr (kFast) S2 *= kLn2;
                        du_t = fmaf(tk.dt, S1, dr * cc.D);
                        ds_t = fmaf(ut, S1, S2) * tk.dsp;
                    } else {
                        float du_acc = 0.f, ddt = 0.f;
#pragma unroll
                        for (int i = 0; i < P; ++i) {
                            const float2 hp = tt > 0 ? hs[tt > 0 ? tt - 1 : 0][i] : hst[i];
                            const float Bx = rowv[i].x, By = rowv[i].y;
                            const float gx = fmaf(dr, rowv[i].z, gh[i].x), gy = fmaf(dr, rowv[i].w, gh[i].y);
                            vals[P * 2 + 2 * i] = dr * hs[tt][i].x;  // dC
                            vals[P * 2 + 2 * i + 1] = dr * hs[tt][i].y;
                            // w = Delta phi(x), dw/dDelta = a, dw/dA = Delta^2 phi'(x)
                            const float2 an = a_nat(i);
                            const float xx = tk.dt * an.x, xy = tk.dt * an.y;
                            const bool sx = fabsf(xx) < kZohTaylorMax, sy = fabsf(xy) < kZohTaylorMax;
                            const float wx = sx ? tk.dt * phi_taylor(xx) : (dA[i].x - 1.f) * cc.ia[i].x;
                            const float wy = sy ? tk.dt * phi_taylor(xy) : (dA[i].y - 1.f) * cc.ia[i].y;
                            const float dwx = dA[i].x, dwy = dA[i].y;
                            const float dAwx = sx ? tk.dt * tk.dt * dphi_taylor(xx) : fmaf(tk.dt, dA[i].x, -wx) * cc.ia[i].x;
                            const float dAwy = sy ? tk.dt * tk.dt * dphi_taylor(xy) : fmaf(tk.dt, dA[i].y, -wy) * cc.ia[i].y;
                            vals[2 * i] = gx * wx * ut;  // dB
                            vals[2 * i + 1] = gy * wy * ut;
                            du_acc = fmaf(gx * wx, Bx, fmaf(gy * wy, By, du_acc));
                            const float dwsx = gx * Bx * ut, dwsy = gy * By * ut;
                            const float dax = gx * hp.x * dA[i].x, day = gy * hp.y * dA[i].y;
                            ddt = fmaf(dax, an.x, fmaf(day, an.y, ddt));
                            ddt = fmaf(dwsx, dwx, fmaf(dwsy, dwy, ddt));
                            dA_acc[i].x = fmaf(dax, tk.dt, fmaf(dwsx, dAwx, dA_acc[i].x));
                            dA_acc[i].y = fmaf(day, tk.dt, fmaf(dwsy, dAwy, dA_acc[i].y));
                            gh[i] = make_float2(gx * dA[i].x, gy * dA[i].y);
                        }
                        du_t = du_acc + __shfl_xor_sync(0xffffffffu, du_acc, 1) + dr * cc.D;
                        ds_t = (ddt + __shfl_xor_sync(0xffffffffu, ddt, 1)) * tk.dsp;
                    }
                    du_o[tt] = du_t;
                    ds_o[tt] = ds_t;
                    dD_acc = fmaf(dr, ut, dD_acc);
                    if (half == hf) dbias_acc += ds_t;
                    red[tt] = reduce_scatter_channels<M>(vals, lane, red_index, red_writer);
                }
                // this half's per-token gradients: stored by lane half hf
                if (valid && half == hf) {
                    const int64_t at = row * L + tg + T0;
                    *reinterpret_cast<uint2*>(static_cast<T*>(p.du) + at) = pack8<T>(du_o);
                    *reinterpret_cast<uint2*>(static_cast<T*>(p.ddelta) + at) = pack8<T>(ds_o);
                    if constexpr (kGate) *reinterpret_cast<uint2*>(static_cast<T*>(p.dz) + at) = pack8<T>(dz_o);
                }
                // dB / dC of the half's tokens for this lane's (state, B or C)
                if (red_writer) {
                    const int q = red_index / (2 * P);  // 0: dB, 1: dC
                    const int i = red_index % (2 * P);
                    const int n = half + 4 * (i / 2) + 2 * (i % 2);
                    float* dst = (q ? p.dC : p.dB) + (size_t(b) * N + n) * size_t(L) + size_t(tg + T0);
                    if constexpr (HV == 4)
                        red_add_v4(dst, red[0], red[1], red[2], red[3]);
                    else
                        red_add_v2(dst, red[0], red[1]);
                }
            }
        }

        __syncwarp();
    }

    // each lane summed the slopes of the tokens it stored
    dbias_acc += __shfl_xor_sync(0xffffffffu, dbias_acc, 1);
    if (!valid) return;
    if (p.dinit) {
        float* di = p.dinit + row * N + half;
#pragma unroll
        for (int i = 0; i < P; ++i) {
            di[4 * i] = gh[i].x;
            di[4 * i + 2] = gh[i].y;
        }
    }
    float* dA_row = p.dA + d * N + half;
#pragma unroll
    for (int i = 0; i < P; ++i) {
        atomicAdd(dA_row + 4 * i, dA_acc[i].x);
        atomicAdd(dA_row + 4 * i + 2, dA_acc[i].y);
    }
    if (half == 0) {
        if (p.dD) atomicAdd(p.dD + d, dD_acc);
        if (p.dbias) atomicAdd(p.dbias + d, dbias_acc);
    }
}

// grid = (ceil(dim / 16), batch), block = 32 threads, dynamic shared memory
// BwdLayout<T, N>::kSmemBytes.  Requirements as the forward kernel's
// (checked by the host), plus the checkpoints of the same chunking.
template <typename T, int N, bool kGate, bool kSoftplus, bool kZoh>
__global__ void __launch_bounds__(32) scan_bwd_kernel(const __grid_constant__ BwdMaps maps, BwdParams p,
                                                      int allow_geo) {
    using Ly = BwdLayout<T, N>;
    constexpr int P = Ly::kPairs;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Ly::kBarOffset);
    const int lane = threadIdx.x;
    const int half = lane & 1;
    const int64_t c = int64_t(blockIdx.x) * Ly::kRows + (lane >> 1);
    const bool valid = c < p.dim;
    const int64_t d = valid ? c : 0;
    const int64_t row = int64_t(blockIdx.y) * p.dim + d;

    if (lane == 0) {
        for (int s = 0; s < Ly::kStages; ++s) mbar_init(bars + s, 1);
        fence_barrier_init();
        prefetch_tensormap(&maps.u);
        prefetch_tensormap(&maps.delta);
        if (kGate) prefetch_tensormap(&maps.z);
        prefetch_tensormap(&maps.dy);
        prefetch_tensormap(&maps.B);
        prefetch_tensormap(&maps.C);
        prefetch_tensormap(&maps.ck);
    }
    __syncwarp();

    constexpr bool kFast = sizeof(T) == 2;
    LaneConst<N> cc;
    cc.bias = p.delta_bias ? p.delta_bias[d] : 0.f;
    cc.D = p.D ? p.D[d] : 0.f;
    const float* Arow = p.A + d * N;
    const float a_first = Arow[0];
    cc.a0 = a_first * kLog2e;
    bool geo = kFast && !kZoh && allow_geo;
#pragma unroll
    for (int i = 0; i < P; ++i) {
        const int n = half + 4 * i;
        const float x0 = Arow[n], x1 = Arow[n + 2];
        cc.a2[i] = kFast ? make_float2(x0 * kLog2e, x1 * kLog2e) : make_float2(x0, x1);
        if constexpr (kZoh) cc.ia[i] = make_float2(1.f / x0, 1.f / x1);
        geo = geo && x0 == float(n + 1) * a_first && x1 == float(n + 3) * a_first;
    }
    geo = __all_sync(0xffffffffu, geo || !valid);
    if constexpr (kFast && !kZoh) {
        if (geo) {
            scan_bwd_body<T, N, true, kGate, kSoftplus, kZoh>(maps, p, smem, bars, cc, valid, row);
            return;
        }
    }
    scan_bwd_body<T, N, false, kGate, kSoftplus, kZoh>(maps, p, smem, bars, cc, valid, row);
}

}  // namespace mss
