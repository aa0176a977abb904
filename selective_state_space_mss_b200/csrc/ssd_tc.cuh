// ssd_tc.cuh -- forward pass of the structured state space duality (Mamba-2
// layer, scalar A per head) on the fifth-generation tensor cores: TMA-staged
// operands, tcgen05.mma with accumulators in tensor memory (TMEM).
//
// With A = a_h I the map of one head over a chunk of Q tokens is the
// 1-semiseparable matrix M_ij = exp(cs_i - cs_j) (C_i . B_j) Delta_j (j <= i,
// cs the running sum of Delta A over the chunk) plus the state carried in
// from earlier chunks ("NN Lab -- Mamba", Structured State Space Duality;
// "Mamba" paper review, section "Mamba 2").  One CTA of sixteen warps serves
// one (batch, head) and walks its chunks of Q = 128 tokens in order.  Per chunk:
//
//   G   = C B^T                   (128 x 128, K = N)     TMEM columns   0..127
//                                                        (384..511 for odd chunks)
//   dS  = B^T diag(w) X,  w_j = exp(cs_last - cs_j) Delta_j
//                                  (N x P = 128 x 64, K = Q) columns 256..319
//   Yx  = C S_prev                (128 x 64, K = N)      columns 192..255
//   M   = mask(G) . exp(cs_i - cs_j) Delta_j on the CUDA cores, bf16 in smem
//   Ym  = M X                     (128 x 64, K = Q)      columns 128..191
//   S   = exp(cs_last) S_prev + dS        (fp32, registers)
//   y   = (Ym + exp(cs_i) Yx + D x) silu(z)  -> stored from registers
//
// Thread t of the CTA owns TMEM lane (and row) t % 128 and quarter t / 128 of
// the columns of each product it reads (four warps share each 32-lane TMEM
// quarter).  The fp32 state S (N x P) lives in registers (thread t: row
// n = t % 128, columns 16 (t / 128) ..), its bf16 copy in shared memory is the
// B operand of the next chunk's C S_prev.  Sixteen warps (four per scheduler)
// hide the latencies of the TMEM loads, the exponentials and the barriers.
// Operands: C and B tiles [128 tokens][64 state] x 2 and X [128 tokens][64]
// in the 128-byte swizzle TMA writes, double buffered (the next chunk's
// loads run during this one); M, X_w and the state copy are written by the
// threads in the same layout.  One thread issues the MMAs and the TMA copies,
// from a warp whose scores are all masked (it has the least work); the score
// products come from a thread of another such warp.
//
// Order within a chunk, with three CTA barriers: the threads scale X
// (barrier); B^T X_w and C S_prev start, and the threads mask and decay the
// scores, whose C B^T ran during the previous chunk's output step (barrier);
// M X starts (the next chunk's C B^T follows it, issued by a third lightly
// loaded warp once M X is done), while another such warp stores the next
// chunk's step sizes and decay sums (formed during the
// masking, in which its scores are all masked; their raw steps were loaded a
// chunk ahead); the state update waits only for B^T X_w, the output only for
// M X, and y goes straight from registers to memory (barrier); then
// the loads of chunk c + 2.  z is loaded after the first barrier: a proxy
// fence waits for a thread's loads in flight, so z loaded before the scaling
// of X held that fence for the loads' whole latency.  Each thread
// waits on the MMA completion barriers itself; a wait that gives up is
// folded into the next CTA barrier.  Score blocks of 32 x 32 wholly above
// the diagonal are skipped by the warp; blocks wholly below it use
// exp2(cs_i - cs_j) = exp2(cs_i - cs_L) exp2(cs_L - cs_j) (L the block's last
// column), both factors at most one for A <= 0, with the column factor
// shared by every row, so they need no exponential per score.
//
// Waits are bounded (~2 s): on a timeout the CTA sets the device error word,
// gives its copies and products in flight a bounded chance to finish, frees
// its TMEM and returns.
// Requirements (checked by the host): bf16 io, P = 64, N = 128, H a multiple
// of G, x, z, y, B, C 16-byte aligned (row strides are then multiples of 16).
#pragma once

#include <cstdint>
#include <cuda.h>

#include "mss_device.cuh"
#include "mss_params.h"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace mss {

struct SsdTcMaps {
    CUtensorMap x, B, C;  // x: [batch][L][H][64]; B, C: [batch][L][G][128] (4-D views)
};

struct SsdTcLayout {
    static constexpr int kQ = 128, kP = 64, kN = 128;
    static constexpr int kThreads = 512;
    static constexpr int kBox = 16384;  // one [128][64] bf16 tile
    // stage: C (two boxes along N), B (two boxes), X
    static constexpr int kC = 0, kB = 2 * kBox, kX = 4 * kBox;
    static constexpr int kStageBytes = 5 * kBox;
    static constexpr int kM = 2 * kStageBytes;    // masked scores, bf16, two boxes along K
    static constexpr int kXw = kM + 2 * kBox;     // w-scaled X
    static constexpr int kS = kXw + kBox;         // bf16 copy of the state [128 n][64 p]
    // per token of the chunk: Delta (with softplus cs - log2(Delta)), cs in
    // log2 units, and the column factor f_j = exp2(cs_L - cs_j) Delta_j of the
    // masked scores (L the last token of j's 32-token block); read up to the
    // masked scores, then rewritten for the next chunk (each thread keeps the
    // values its output step needs)
    static constexpr int kScal = kS + kBox;
    static constexpr int kBars = kScal + 3 * kQ * 4;
    static constexpr int kTmemSlot = kBars + 5 * 8;
    static constexpr int kSmemBytes = kTmemSlot + 16 + 1024;  // + base alignment slack
    static constexpr uint32_t kTmemCols = 512;
    // scores of even and odd chunks (the next chunk's are computed during this
    // one's output step), M X, C S_prev, B^T X_w
    static constexpr uint32_t kColG = 0, kColYm = 128, kColYx = 192, kColS = 256, kColG2 = 384;
};

template <bool kGate, bool kSoftplus>
__global__ void __launch_bounds__(512, 1) ssd_tc_kernel(const __grid_constant__ SsdTcMaps maps, SsdParams p,
                                                        int64_t unit0) {
    using Ly = SsdTcLayout;
    constexpr int Q = Ly::kQ, P = Ly::kP, NS = Ly::kN;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    float* dts = reinterpret_cast<float*>(smem + Ly::kScal);  // [Q] Delta (0 past the sequence), or with
                                                              // softplus cs - log2(Delta)
    float* css = dts + Q;                                     // [Q] cs * log2(e)
    float* fss = css + Q;                                     // [Q] column factors of the scores
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + Ly::kBars);  // [2] TMA stages
    uint64_t* gbar = full + 2;  // C B^T complete
    uint64_t* mbar = full + 3;  // B^T X_w and C S_prev complete
    uint64_t* ybar = full + 4;  // M X complete
    uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + Ly::kTmemSlot);

    const int tid = threadIdx.x, warp = tid >> 5;
    const int row = tid & 127, qd = tid >> 7;  // TMEM lane / row, column quarter
    // The thread that issues the MMAs and the TMA copies, and the warp that
    // prepares the step sizes, sit in warps whose score blocks are all masked
    // (rows 0..31 against columns 96..127, rows 32..63 against 96..127), so
    // that their extra work does not hold up the CTA barriers.
    constexpr int kCtlWarp = 12, kScanWarp = 13, kScoreWarp = 8;
    const bool ctl = tid == kCtlWarp * 32;
    // the thread that issues the score products C B^T (and commits their
    // barrier), in a third all-masked warp: the next chunk's product waits
    // for this chunk's M X to complete, and the waiting thread must not be the
    // one that issues everything else
    const bool scorer = tid == kScoreWarp * 32;
    const int64_t H = p.nheads, L = p.seqlen;
    // (batch, head) pair unit0 + blockIdx.x
    const int64_t b = (unit0 + blockIdx.x) / H, h = (unit0 + blockIdx.x) % H;
    const int g = int(h / (H / p.ngroups));
    const float A2 = p.A[h] * kLog2e;
    const float bias = p.dt_bias ? p.dt_bias[h] : 0.f;
    const float Dh = p.D ? p.D[h] : 0.f;
    const int n_chunks = int((L + Q - 1) / Q);

    if (tid == 0) {
        for (int k = 0; k < 5; ++k) mbar_init(full + k, 1);
        fence_barrier_init();
        prefetch_tensormap(&maps.x);
        prefetch_tensormap(&maps.B);
        prefetch_tensormap(&maps.C);
    }
    if (warp == 0) {
        tmem_alloc(tslot, Ly::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tslot;
    const uint32_t tlane = tmem + (uint32_t((warp & 3) * 32) << 16);  // this warp's lane quarter

    auto issue_chunk = [&](int c) {
        uint8_t* st = smem + (c & 1) * Ly::kStageBytes;
        uint64_t* bar = full + (c & 1);
        const int t0 = c * Q;
        mbar_arrive_expect_tx(bar, uint32_t(Ly::kStageBytes));
        tma_load_4d(st + Ly::kC, &maps.C, 0, g, t0, int(b), bar);
        tma_load_4d(st + Ly::kC + Ly::kBox, &maps.C, 64, g, t0, int(b), bar);
        tma_load_4d(st + Ly::kB, &maps.B, 0, g, t0, int(b), bar);
        tma_load_4d(st + Ly::kB + Ly::kBox, &maps.B, 64, g, t0, int(b), bar);
        tma_load_4d(st + Ly::kX, &maps.x, 0, int(h), t0, int(b), bar);
    };
    if (ctl) {
        issue_chunk(0);
        if (n_chunks > 1) issue_chunk(1);
    }

    // the state: row n = `row`, columns 16 * qd .. + 15
    float S[16];
    {
        const float* s0 = p.initial_state ? p.initial_state + ((b * H + h) * NS + row) * P + 16 * qd : nullptr;
#pragma unroll
        for (int k = 0; k < 16; ++k) S[k] = s0 ? s0[k] : 0.f;
    }
    auto write_state_copy = [&]() {
        uint8_t* Ss = smem + Ly::kS;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            uint4 v = make_uint4(pack_bf16x2(S[8 * q], S[8 * q + 1]), pack_bf16x2(S[8 * q + 2], S[8 * q + 3]),
                                 pack_bf16x2(S[8 * q + 4], S[8 * q + 5]), pack_bf16x2(S[8 * q + 6], S[8 * q + 7]));
            *reinterpret_cast<uint4*>(Ss + sw128(row, 2 * qd + q)) = v;
        }
    };
    write_state_copy();
    fence_proxy_async_smem();

    bool ok = true;
    constexpr uint32_t idG = idesc_bf16_f32(128, 128, 0, 0);
    constexpr uint32_t idK = idesc_bf16_f32(128, 64, 0, 1);   // K-major A, N-major B
    constexpr uint32_t idMN = idesc_bf16_f32(128, 64, 1, 1);  // M-major A, N-major B
    const uint32_t sbase = smem_addr(smem);
    const bf16_t* dtp = static_cast<const bf16_t*>(p.dt) + b * L * H + h;
    const int lane = tid & 31;

    // The scan warp prepares each chunk's step sizes and their running sum ahead of
    // it: lane l takes tokens 4l .. 4l+3 (raw steps loaded one chunk earlier
    // still), a warp scan adds the lanes' totals.  Results go to the scalar
    // buffer of the chunk's parity.
    float raw[4];
    auto load_raw = [&](int c) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int64_t t = int64_t(c) * Q + 4 * lane + k;
            raw[k] = t < L ? ld(dtp + t * H) : 0.f;
        }
    };
    // scan_compute forms the values into registers, scan_store writes them
    float sd[4], sa[4], sf[4];
    auto scan_compute = [&](int c) {
        float* d = sd;
        float* a = sa;
        float run = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const bool valid = int64_t(c) * Q + 4 * lane + k < L;
            const float s0 = raw[k] + bias;
            d[k] = valid ? (kSoftplus ? softplus_fast(s0) : s0) : 0.f;
            run += d[k] * A2;
            a[k] = run;
        }
        float incl = run;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        const float excl = incl - run;
#pragma unroll
        for (int k = 0; k < 4; ++k) a[k] += excl;
        // the last token of this lane's 32-token block is token 3 of lane 8 (l / 8) + 7
        const float cL = __shfl_sync(0xffffffffu, a[3], (lane & ~7) | 7);
#pragma unroll
        for (int k = 0; k < 4; ++k) sf[k] = ex2_approx(cL - a[k]) * d[k];
    };
    auto scan_store = [&]() {
        if constexpr (kSoftplus) {
            // Delta > 0: the array holds cs_j - log2(Delta_j) instead (+inf
            // where Delta_j is zero), so that exp2(x - it) = exp2(x - cs_j) Delta_j
            // costs one exponential and no multiply
#pragma unroll
            for (int k = 0; k < 4; ++k) sd[k] = sa[k] - lg2_approx(sd[k]);
        }
        reinterpret_cast<float4*>(dts)[lane] = make_float4(sd[0], sd[1], sd[2], sd[3]);
        reinterpret_cast<float4*>(css)[lane] = make_float4(sa[0], sa[1], sa[2], sa[3]);
        reinterpret_cast<float4*>(fss)[lane] = make_float4(sf[0], sf[1], sf[2], sf[3]);
    };
    if (warp == kScanWarp) {
        load_raw(0);
        scan_compute(0);
        scan_store();
        if (n_chunks > 1) load_raw(1);
    }
    __syncthreads();

    // issue C B^T of chunk c once its tiles have landed (thread 0)
    auto issue_scores = [&](int c) -> bool {
        const uint32_t st = sbase + uint32_t((c & 1) * Ly::kStageBytes);
        if (!mbar_wait_bounded(full + (c & 1), uint32_t((c >> 1) & 1), p.err)) return false;
        tc_fence_after_sync();
#pragma unroll
        for (int k = 0; k < NS / 16; ++k) {
            const uint32_t off = uint32_t((k >> 2) * Ly::kBox + (k & 3) * 32);
            umma_bf16(tmem + ((c & 1) ? Ly::kColG2 : Ly::kColG), smem_desc_sw128(st + Ly::kC + off, 16, 1024),
                      smem_desc_sw128(st + Ly::kB + off, 16, 1024), idG, k > 0);
        }
        umma_commit(gbar);
        return true;
    };

    bool abort = false;  // a bounded wait of this thread gave up (folded into the next CTA barrier)
    // the first chunk's scores; each later chunk's start during the previous
    // chunk's output step
    if (scorer && n_chunks > 0) abort |= !issue_scores(0);
    for (int c = 0; c < n_chunks && ok; ++c) {
        const int t0 = c * Q;
        const uint32_t ph = uint32_t(c & 1);  // each completion barrier completes once per chunk
        const uint32_t st = sbase + uint32_t((c & 1) * Ly::kStageBytes);
        const float* dtc = dts;
        const float* csc = css;
        abort |= !mbar_wait_bounded(full + (c & 1), uint32_t((c >> 1) & 1), p.err);
        const float cl = csc[Q - 1];
        const float ci = csc[row];  // kept for the output step (the next chunk's scan rewrites css)
        // X_w = w_j x_j (row j = `row`, this thread's quarter of the 64 columns)
        {
            const float wj = kSoftplus ? ex2_approx(cl - dtc[row]) : ex2_approx(cl - ci) * dtc[row];
            const uint8_t* xs = smem + (c & 1) * Ly::kStageBytes + Ly::kX;
            uint8_t* xw = smem + Ly::kXw;
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const uint32_t off = sw128(row, 2 * qd + q);
                const uint4 v = *reinterpret_cast<const uint4*>(xs + off);
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
                uint32_t o4[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) o4[k] = pack_bf16x2(wj * bf16_lo(w4[k]), wj * bf16_hi(w4[k]));
                *reinterpret_cast<uint4*>(xw + off) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
            }
        }
        fence_proxy_async_smem();
        if (__syncthreads_or(abort)) {
            ok = false;
            break;
        }
        // z of this chunk's rows, in registers until the output step; loaded
        // only now, after the proxy fence above, which would otherwise wait
        // for these loads to land
        uint4 zr[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
        const int64_t tok = int64_t(t0) + row;
        if constexpr (kGate) {
            const bf16_t* zp = static_cast<const bf16_t*>(p.z) + ((b * L + tok) * H + h) * P + 16 * qd;
#pragma unroll
            for (int q = 0; q < 2; ++q)
                if (tok < L) zr[q] = *reinterpret_cast<const uint4*>(zp + 8 * q);
        }
        // dS = B^T X_w and Yx = C S_prev, while the scores are masked
        if (ctl) {
            tc_fence_after_sync();
#pragma unroll
            for (int k = 0; k < Q / 16; ++k) {
                const uint32_t off = uint32_t(k * 2048);
                umma_bf16(tmem + Ly::kColS, smem_desc_sw128(st + Ly::kB + off, Ly::kBox, 1024),
                          smem_desc_sw128(sbase + Ly::kXw + off, 0, 1024), idMN, k > 0);
            }
#pragma unroll
            for (int k = 0; k < NS / 16; ++k) {
                const uint32_t offa = uint32_t((k >> 2) * Ly::kBox + (k & 3) * 32);
                umma_bf16(tmem + Ly::kColYx, smem_desc_sw128(st + Ly::kC + offa, 16, 1024),
                          smem_desc_sw128(sbase + Ly::kS + uint32_t(k * 2048), 0, 1024), idK, k > 0);
            }
            umma_commit(mbar);
        }
        abort |= !mbar_wait_bounded(gbar, ph, p.err);
        tc_fence_after_sync();
        // M_ij = G_ij exp(cs_i - cs_j) Delta_j for j <= i, this thread's 32 columns j
        // (box qd / 2 of the two 64-wide K boxes, pieces 4 (qd % 2) ..).  A
        // warp's 32 rows against a quarter of 32 columns to their right are all
        // masked (rows 32 (warp % 4) .. < columns 32 qd ..): zeros, with no TMEM
        // load and no exponential (a warp-uniform branch).
        {
            uint8_t* Ms = smem + Ly::kM + (qd >> 1) * Ly::kBox;
            if ((warp & 3) < qd) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<uint4*>(Ms + sw128(row, 4 * (qd & 1) + q)) = make_uint4(0u, 0u, 0u, 0u);
            } else {
                float gv[32];
                tmem_ld32(tlane + ((c & 1) ? Ly::kColG2 : Ly::kColG) + uint32_t(32 * qd), gv);
                tmem_wait_ld();
                // A block wholly below the diagonal (every j <= i): exp2(cs_i - cs_j)
                // = exp2(cs_i - cs_L) exp2(cs_L - cs_j) with L = 32 qd + 31 <= i;
                // both exponents are <= 0 for A <= 0, so neither factor overflows,
                // and the column factor (times Delta_j) is shared by every row.
                if ((warp & 3) > qd) {
                    const float ri = ex2_approx(ci - csc[32 * qd + 31]);
                    const float4* f4 = reinterpret_cast<const float4*>(fss + 32 * qd);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4 fa = f4[2 * q], fb = f4[2 * q + 1];
                        const float f[8] = {fa.x, fa.y, fa.z, fa.w, fb.x, fb.y, fb.z, fb.w};
                        uint32_t o4[4];
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            o4[k] = pack_bf16x2(gv[8 * q + 2 * k] * ri * f[2 * k], gv[8 * q + 2 * k + 1] * ri * f[2 * k + 1]);
                        *reinterpret_cast<uint4*>(Ms + sw128(row, 4 * (qd & 1) + q)) =
                            make_uint4(o4[0], o4[1], o4[2], o4[3]);
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t o4[4];
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            float m2[2];
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const int jj = 8 * q + 2 * k + e;  // 0..31 within this quarter
                                const int j = 32 * qd + jj;        // token index in the chunk
                                const float dec = kSoftplus ? ex2_approx(ci - dtc[j])
                                                            : ex2_approx(ci - csc[j]) * dtc[j];
                                m2[e] = j <= row ? gv[jj] * dec : 0.f;
                            }
                            o4[k] = pack_bf16x2(m2[0], m2[1]);
                        }
                        *reinterpret_cast<uint4*>(Ms + sw128(row, 4 * (qd & 1) + q)) =
                            make_uint4(o4[0], o4[1], o4[2], o4[3]);
                    }
                }
            }
        }
        // the scan warp, whose scores are all masked, forms the next chunk's
        // step sizes and decay sums now (stored once every warp has read
        // this chunk's, after the barrier)
        if (warp == kScanWarp && c + 1 < n_chunks) scan_compute(c + 1);
        tc_fence_before_sync();
        fence_proxy_async_smem();
        if (__syncthreads_or(abort)) {
            ok = false;
            break;
        }
        // Ym = M X; meanwhile the scan warp stores the next chunk's step sizes
        if (ctl) {
            tc_fence_after_sync();
#pragma unroll
            for (int k = 0; k < Q / 16; ++k) {
                const uint32_t offa = uint32_t((k >> 2) * Ly::kBox + (k & 3) * 32);
                umma_bf16(tmem + Ly::kColYm, smem_desc_sw128(sbase + Ly::kM + offa, 16, 1024),
                          smem_desc_sw128(st + Ly::kX + uint32_t(k * 2048), 0, 1024), idK, k > 0);
            }
            umma_commit(ybar);
        }
        if (warp == kScanWarp && c + 1 < n_chunks) {
            scan_store();
            if (c + 2 < n_chunks) load_raw(c + 2);
        }
        // the state: S = exp(cs_last) S + dS, and its bf16 copy for the next
        // chunk (C S_prev has read the old copy: it completed with dS)
        abort |= !mbar_wait_bounded(mbar, ph, p.err);
        tc_fence_after_sync();
        {
            float ds[16];
            tmem_ld16(tlane + Ly::kColS + uint32_t(16 * qd), ds);
            tmem_wait_ld();
            const float dec = ex2_approx(cl);
#pragma unroll
            for (int k = 0; k < 16; ++k) S[k] = fmaf(dec, S[k], ds[k]);
            write_state_copy();
        }
        abort |= !mbar_wait_bounded(ybar, ph, p.err);
        tc_fence_after_sync();
        // the next chunk's scores, into the other score buffer (its last
        // reader, the masking of chunk c - 1, finished before this chunk's
        // first barrier), once M X has left the tensor pipe
        if (scorer && c + 1 < n_chunks) abort |= !issue_scores(c + 1);
        // y = (Ym + exp(cs_i) Yx + D x) silu(z) for row i = `row`, this
        // quarter's 16 columns: 32 contiguous bytes of the token's row, stored
        // from registers
        {
            float ym[16], yx[16];
            tmem_ld16(tlane + Ly::kColYm + uint32_t(16 * qd), ym);
            tmem_ld16(tlane + Ly::kColYx + uint32_t(16 * qd), yx);
            tmem_wait_ld();
            const float ei = ex2_approx(ci);
            const uint8_t* xs = smem + (c & 1) * Ly::kStageBytes + Ly::kX;
            bf16_t* yp = static_cast<bf16_t*>(p.y) + ((b * L + tok) * H + h) * P + 16 * qd;
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const uint32_t off = sw128(row, 2 * qd + q);
                const uint4 xv = *reinterpret_cast<const uint4*>(xs + off);
                const uint32_t x4[4] = {xv.x, xv.y, xv.z, xv.w};
                uint32_t z4[4] = {0u, 0u, 0u, 0u};
                if constexpr (kGate) {
                    z4[0] = zr[q].x;
                    z4[1] = zr[q].y;
                    z4[2] = zr[q].z;
                    z4[3] = zr[q].w;
                }
                uint32_t o4[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int i0 = 8 * q + 2 * k;
                    float y0 = fmaf(ei, yx[i0], ym[i0]) + Dh * bf16_lo(x4[k]);
                    float y1 = fmaf(ei, yx[i0 + 1], ym[i0 + 1]) + Dh * bf16_hi(x4[k]);
                    if constexpr (kGate) {
                        y0 *= silu_fast(bf16_lo(z4[k]));
                        y1 *= silu_fast(bf16_hi(z4[k]));
                    }
                    o4[k] = pack_bf16x2(y0, y1);
                }
                if (tok < L) *reinterpret_cast<uint4*>(yp + 8 * q) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
            }
        }
        tc_fence_before_sync();
        if (__syncthreads_or(abort)) {
            ok = false;
            break;
        }
        // every read of chunk c's stage is done: its tiles give way to chunk c + 2
        if (ctl && c + 2 < n_chunks) {
            fence_proxy_async_smem();
            issue_chunk(c + 2);
        }
    }
    if (!ok && ctl) {
        // give the copies and products still in flight a bounded chance to land
        for (int k = 0; k < 5; ++k) {
            mbar_wait_bounded(full + k, 0u, nullptr, 50000000ull);
            mbar_wait_bounded(full + k, 1u, nullptr, 50000000ull);
        }
    }
    if (ok && p.last_state) {
        float* ls = p.last_state + ((b * H + h) * NS + row) * P + 16 * qd;
#pragma unroll
        for (int k = 0; k < 16; k += 4) *reinterpret_cast<float4*>(ls + k) = make_float4(S[k], S[k + 1], S[k + 2], S[k + 3]);
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, Ly::kTmemCols);
    }
}

}  // namespace mss
