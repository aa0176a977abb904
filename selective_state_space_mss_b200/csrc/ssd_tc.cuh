// ssd_tc.cuh -- forward pass of the structured state space duality (Mamba-2
// layer, scalar A per head) on the fifth-generation tensor cores: TMA-staged
// operands, tcgen05.mma with accumulators in tensor memory (TMEM).
//
// With A = a_h I the map of one head over a chunk of Q tokens is the
// 1-semiseparable matrix M_ij = exp(cs_i - cs_j) (C_i . B_j) Delta_j (j <= i,
// cs the running sum of Delta A over the chunk) plus the state carried in
// from earlier chunks ("NN Lab -- Mamba", Structured State Space Duality;
// "Mamba" paper review, section "Mamba 2").  One CTA of eight warps serves one
// (batch, head) and walks its chunks of Q = 128 tokens in order.  Per chunk:
//
//   G   = C B^T                   (128 x 128, K = N)     TMEM columns   0..127
//   dS  = B^T diag(w) X,  w_j = exp(cs_last - cs_j) Delta_j
//                                  (N x P = 128 x 64, K = Q) columns 256..319
//   Yx  = C S_prev                (128 x 64, K = N)      columns 192..255
//   M   = mask(G) . exp(cs_i - cs_j) Delta_j on the CUDA cores, bf16 in smem
//   Ym  = M X                     (128 x 64, K = Q)      columns 128..191
//   S   = exp(cs_last) S_prev + dS        (fp32, registers)
//   y   = (Ym + exp(cs_i) Yx + D x) silu(z)  -> smem -> TMA store
//
// Thread t of the CTA owns TMEM lane (and row) t % 128 and half t / 128 of the
// columns of each product it reads.  The fp32 state S (N x P) lives in
// registers (thread t: row n = t % 128, columns 32 (t / 128) ..), its bf16
// copy in shared memory is the B operand of the next chunk's C S_prev.
// Operands: C and B tiles [128 tokens][64 state] x 2 and X [128 tokens][64]
// in the 128-byte swizzle TMA writes, double buffered (the next chunk's
// loads run during this one); M, X_w and the state copy are written by the
// threads in the same layout.  One thread issues the MMAs and the TMA copies.
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
    CUtensorMap x, z, y, B, C;  // x, y: [batch][L][H][64]; B, C: [batch][L][G][128] (4-D views)
};

struct SsdTcLayout {
    static constexpr int kQ = 128, kP = 64, kN = 128;
    static constexpr int kThreads = 256;
    static constexpr int kBox = 16384;  // one [128][64] bf16 tile
    // stage: C (two boxes along N), B (two boxes), X
    static constexpr int kC = 0, kB = 2 * kBox, kX = 4 * kBox;
    static constexpr int kStageBytes = 5 * kBox;
    static constexpr int kM = 2 * kStageBytes;    // masked scores, bf16, two boxes along K
    static constexpr int kXw = kM + 2 * kBox;     // w-scaled X; then the y tile of the same chunk
    static constexpr int kS = kXw + kBox;         // bf16 copy of the state [128 n][64 p]
    static constexpr int kScal = kS + kBox;       // per token: Delta, cs (log2 units); warp sums
    static constexpr int kBars = kScal + 2 * kQ * 4 + 64;
    static constexpr int kTmemSlot = kBars + 4 * 8;
    static constexpr int kSmemBytes = kTmemSlot + 16 + 1024;  // + base alignment slack
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColG = 0, kColYm = 128, kColYx = 192, kColS = 256;
};

template <bool kGate, bool kSoftplus>
__global__ void __launch_bounds__(256, 1) ssd_tc_kernel(const __grid_constant__ SsdTcMaps maps, SsdParams p) {
    using Ly = SsdTcLayout;
    constexpr int Q = Ly::kQ, P = Ly::kP, NS = Ly::kN;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    float* dts = reinterpret_cast<float*>(smem + Ly::kScal);  // Delta (0 past the sequence)
    float* css = dts + Q;                                     // cs * log2(e)
    float* wsum = css + Q;                                    // warp totals of the scan
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + Ly::kBars);  // [2] TMA stages
    uint64_t* mbar = full + 2;                                       // MMA completion
    uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + Ly::kTmemSlot);

    const int tid = threadIdx.x, warp = tid >> 5;
    const int row = tid & 127, half = tid >> 7;
    const int64_t H = p.nheads, L = p.seqlen;
    const int64_t b = blockIdx.x / H, h = blockIdx.x % H;
    const int g = int(h / (H / p.ngroups));
    const float A2 = p.A[h] * kLog2e;
    const float bias = p.dt_bias ? p.dt_bias[h] : 0.f;
    const float Dh = p.D ? p.D[h] : 0.f;
    const int n_chunks = int((L + Q - 1) / Q);

    if (tid == 0) {
        mbar_init(full, 1);
        mbar_init(full + 1, 1);
        mbar_init(mbar, 1);
        fence_barrier_init();
        prefetch_tensormap(&maps.x);
        prefetch_tensormap(&maps.B);
        prefetch_tensormap(&maps.C);
        prefetch_tensormap(&maps.y);
        if (kGate) prefetch_tensormap(&maps.z);
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
    if (tid == 0) {
        issue_chunk(0);
        if (n_chunks > 1) issue_chunk(1);
    }

    // the state: row n = `row`, columns 32 * half .. + 31
    float S[32];
    {
        const float* s0 = p.initial_state ? p.initial_state + ((b * H + h) * NS + row) * P + 32 * half : nullptr;
#pragma unroll
        for (int k = 0; k < 32; ++k) S[k] = s0 ? s0[k] : 0.f;
    }
    auto write_state_copy = [&]() {
        uint8_t* Ss = smem + Ly::kS;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint4 v = make_uint4(pack_bf16x2(S[8 * q], S[8 * q + 1]), pack_bf16x2(S[8 * q + 2], S[8 * q + 3]),
                                 pack_bf16x2(S[8 * q + 4], S[8 * q + 5]), pack_bf16x2(S[8 * q + 6], S[8 * q + 7]));
            *reinterpret_cast<uint4*>(Ss + sw128(row, 4 * half + q)) = v;
        }
    };
    write_state_copy();
    fence_proxy_async_smem();

    bool ok = true;
    uint32_t mphase = 0;
    constexpr uint32_t idG = idesc_bf16_f32(128, 128, 0, 0);
    constexpr uint32_t idK = idesc_bf16_f32(128, 64, 0, 1);   // K-major A, N-major B
    constexpr uint32_t idMN = idesc_bf16_f32(128, 64, 1, 1);  // M-major A, N-major B
    const uint32_t sbase = smem_addr(smem);

    for (int c = 0; c < n_chunks && ok; ++c) {
        const int t0 = c * Q;
        const uint32_t st = sbase + uint32_t((c & 1) * Ly::kStageBytes);
        // the previous chunk's y store must have read its tile (the X_w bytes)
        if (tid == 0) bulk_wait_read<0>();
        // step sizes and their running sum over the chunk (log2 units)
        if (tid < Q) {
            float d = 0.f;
            if (t0 + tid < L) {
                const float raw = ld(static_cast<const bf16_t*>(p.dt) + ((b * L + t0 + tid) * H + h)) + bias;
                d = kSoftplus ? softplus_fast(raw) : raw;
            }
            float a = d * A2;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float v = __shfl_up_sync(0xffffffffu, a, o);
                if ((tid & 31) >= o) a += v;
            }
            dts[tid] = d;
            css[tid] = a;
            if ((tid & 31) == 31) wsum[warp] = a;
        }
        const bool landed = mbar_wait_bounded(full + (c & 1), uint32_t((c >> 1) & 1), p.err);
        if (__syncthreads_or(!landed)) {
            ok = false;
            break;
        }
        if (tid < Q) {
            float off = 0.f;
            for (int w = 0; w < (tid >> 5); ++w) off += wsum[w];
            css[tid] += off;
        }
        __syncthreads();
        const float cl = css[Q - 1];
        // X_w = w_j x_j (row j = `row`, this thread's half of the 64 columns)
        {
            const float wj = ex2_approx(cl - css[row]) * dts[row];
            const uint8_t* xs = smem + (c & 1) * Ly::kStageBytes + Ly::kX;
            uint8_t* xw = smem + Ly::kXw;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t off = sw128(row, 4 * half + q);
                const uint4 v = *reinterpret_cast<const uint4*>(xs + off);
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
                uint32_t o4[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) o4[k] = pack_bf16x2(wj * bf16_lo(w4[k]), wj * bf16_hi(w4[k]));
                *reinterpret_cast<uint4*>(xw + off) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
            }
        }
        fence_proxy_async_smem();
        __syncthreads();
        // G = C B^T, dS = B^T X_w, Yx = C S_prev
        if (tid == 0) {
            tc_fence_after_sync();
#pragma unroll
            for (int k = 0; k < NS / 16; ++k) {
                const uint32_t off = uint32_t((k >> 2) * Ly::kBox + (k & 3) * 32);
                umma_bf16(tmem + Ly::kColG, smem_desc_sw128(st + Ly::kC + off, 16, 1024),
                          smem_desc_sw128(st + Ly::kB + off, 16, 1024), idG, k > 0);
            }
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
        if (__syncthreads_or(!mbar_wait_bounded(mbar, mphase, p.err))) {
            ok = false;
            break;
        }
        mphase ^= 1u;
        tc_fence_after_sync();
        // M_ij = G_ij exp(cs_i - cs_j) Delta_j for j <= i, this thread's 64 columns j
        {
            const float ci = css[row];
            uint8_t* Ms = smem + Ly::kM + half * Ly::kBox;
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                float gv[32];
                tmem_ld32(tlane + Ly::kColG + uint32_t(64 * half + 32 * part), gv);
                tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t o4[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        float m2[2];
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int jj = 8 * q + 2 * k + e;          // 0..31 within this part
                            const int j = 64 * half + 32 * part + jj;  // token index in the chunk
                            m2[e] = j <= row ? gv[jj] * ex2_approx(ci - css[j]) * dts[j] : 0.f;
                        }
                        o4[k] = pack_bf16x2(m2[0], m2[1]);
                    }
                    *reinterpret_cast<uint4*>(Ms + sw128(row, 4 * part + q)) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
                }
            }
        }
        tc_fence_before_sync();
        fence_proxy_async_smem();
        __syncthreads();
        // Ym = M X
        if (tid == 0) {
            tc_fence_after_sync();
#pragma unroll
            for (int k = 0; k < Q / 16; ++k) {
                const uint32_t offa = uint32_t((k >> 2) * Ly::kBox + (k & 3) * 32);
                umma_bf16(tmem + Ly::kColYm, smem_desc_sw128(sbase + Ly::kM + offa, 16, 1024),
                          smem_desc_sw128(st + Ly::kX + uint32_t(k * 2048), 0, 1024), idK, k > 0);
            }
            umma_commit(mbar);
        }
        if (__syncthreads_or(!mbar_wait_bounded(mbar, mphase, p.err))) {
            ok = false;
            break;
        }
        mphase ^= 1u;
        tc_fence_after_sync();
        // the state: S = exp(cs_last) S + dS, and its bf16 copy for the next chunk
        {
            float ds[32];
            tmem_ld32(tlane + Ly::kColS + uint32_t(32 * half), ds);
            tmem_wait_ld();
            const float dec = ex2_approx(cl);
#pragma unroll
            for (int k = 0; k < 32; ++k) S[k] = fmaf(dec, S[k], ds[k]);
            write_state_copy();
        }
        // y = (Ym + exp(cs_i) Yx + D x) silu(z) for row i = `row`, this half's 32 columns
        {
            float ym[32], yx[32];
            tmem_ld32(tlane + Ly::kColYm + uint32_t(32 * half), ym);
            tmem_ld32(tlane + Ly::kColYx + uint32_t(32 * half), yx);
            tmem_wait_ld();
            const float ei = ex2_approx(css[row]);
            const int64_t tok = t0 + row;
            const bool valid = tok < L;
            const uint8_t* xs = smem + (c & 1) * Ly::kStageBytes + Ly::kX;
            uint8_t* ys = smem + Ly::kXw;
            const bf16_t* zr = kGate && valid ? static_cast<const bf16_t*>(p.z) + ((b * L + tok) * H + h) * P + 32 * half
                                              : nullptr;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t off = sw128(row, 4 * half + q);
                const uint4 xv = *reinterpret_cast<const uint4*>(xs + off);
                const uint32_t x4[4] = {xv.x, xv.y, xv.z, xv.w};
                uint4 zv = make_uint4(0u, 0u, 0u, 0u);
                if (kGate && valid) zv = *reinterpret_cast<const uint4*>(zr + 8 * q);
                const uint32_t z4[4] = {zv.x, zv.y, zv.z, zv.w};
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
                *reinterpret_cast<uint4*>(ys + off) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
            }
        }
        tc_fence_before_sync();
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            tma_store_4d(&maps.y, smem + Ly::kXw, 0, int(h), t0, int(b));
            bulk_commit();
            if (c + 2 < n_chunks) issue_chunk(c + 2);
        }
    }
    if (!ok && tid == 0) {
        // give the copies and products still in flight a bounded chance to land
        for (int s = 0; s < 2; ++s) mbar_wait_bounded(full + s, 0u, nullptr, 100000000ull);
        mbar_wait_bounded(mbar, mphase, nullptr, 100000000ull);
    }
    if (tid == 0) bulk_wait<0>();
    if (ok && p.last_state) {
        float* ls = p.last_state + ((b * H + h) * NS + row) * P + 32 * half;
#pragma unroll
        for (int k = 0; k < 32; k += 4) *reinterpret_cast<float4*>(ls + k) = make_float4(S[k], S[k + 1], S[k + 2], S[k + 3]);
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, Ly::kTmemCols);
    }
}

}  // namespace mss
