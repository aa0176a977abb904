// ssd_mma.cuh -- forward pass of the structured state space duality (Mamba-2
// layer with a scalar A per head) on the tensor cores.
//
// With A = a_h I the map of one head over a chunk of Q tokens is the
// 1-semiseparable matrix M_ij = exp(cs_i - cs_j) (C_i . B_j) Delta_j (j <= i,
// cs the running sum of Delta A over the chunk) plus the state carried in
// from earlier chunks ("NN Lab -- Mamba", Structured State Space Duality;
// "Mamba" paper review, section "Mamba 2": quadratic form inside chunks,
// linear recurrence across them).  Per chunk of 64 tokens one CTA of four
// warps computes, with bf16 tensor-core products (fp32 accumulation):
//
//   G = C B^T (64 x 64, K = N),  masked and decayed in registers into M;
//   Y = M X + diag(exp(cs)) C S_prev  (64 x P, K = 64 and K = N);
//   S = exp(cs_last) S_prev + B^T diag(exp(cs_last - cs_j) Delta_j) X
//       (N x P, K = 64),
//
// then y = Y + D x, gated by silu(z).  The CTA serves one (batch, head) and
// walks its chunks in order; the N x P fp32 state stays in the accumulator
// registers of the state product from chunk to chunk (its bf16 copy in shared
// memory feeds the next chunk's C S_prev).  Operands reach the tensor cores
// through ldmatrix from padded shared-memory rows (conflict-free), and the
// masked G is reused from the accumulator registers as the A operand of M X.
//
// This first version uses the warp-level mma.sync path; the tcgen05 form
// (TMA-staged operands, TMEM accumulators) is the next step for this row.
// Requirements (checked by the host): bf16 io, P = 64, N in {64, 128},
// H a multiple of G.
#pragma once

#include <cstdint>

#include "mss_device.cuh"
#include "mss_params.h"

namespace mss {

template <int NS>
struct SsdLayout {
    static_assert(NS == 64 || NS == 128, "SSD state size 64 or 128");
    static constexpr int kQ = 64;                      // tokens per chunk
    static constexpr int kP = 64;                      // head dimension
    static constexpr int kThreads = 128;
    static constexpr int kXStride = kP + 8;            // bf16 per padded row of X (144 B)
    static constexpr int kBStride = NS + 8;            // bf16 per padded row of B, C
    static constexpr int kSStride = kP + 8;            // bf16 per padded row of the state copy
    static constexpr int kXBytes = kQ * kXStride * 2;
    static constexpr int kBBytes = kQ * kBStride * 2;
    static constexpr int kSBytes = NS * kSStride * 2;
    // two buffers of X, B, C: the next chunk's copies run during this one
    static constexpr int kBufBytes = kXBytes + 2 * kBBytes;
    static constexpr int kBuf = 0;                     // [2] x (X, B, C)
    // the state's bf16 copy, read by C S_prev; then, in the same bytes, X
    // scaled by exp(cs_last - cs_j) Delta_j for the state product
    static constexpr int kSs = 2 * kBufBytes;
    static constexpr int kXw = kSs;
    static_assert(kXBytes <= kSBytes, "X fits where the state copy was");
    static constexpr int kScal = kSs + kSBytes;        // per token: Delta, cs (fp32)
    // z of the current chunk, 128-byte rows with 16-byte pieces swizzled
    // (piece k of row r at k ^ (r & 7)); each warp copies and reads its own 16 rows
    static constexpr int kZ = kScal + 2 * kQ * 4;
    static constexpr int kZBytes = kQ * kP * 2;
    static constexpr int kSmemBytes = kZ + kZBytes;    // 115,200 B at N = 128: two CTAs per SM
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}

// D += A B for one m16n8k16 tile, bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) { return pack_bf16x2(lo, hi); }

// 16-byte asynchronous copy global -> shared; src_bytes = 0 writes zeros.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int kPending>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(kPending) : "memory"); }

// grid = batch * nheads, block = 128 threads, dynamic shared memory
// SsdLayout<NS>::kSmemBytes.
template <int NS, bool kGate, bool kSoftplus>
__global__ void __launch_bounds__(128) ssd_fwd_kernel(SsdParams p) {
    using Ly = SsdLayout<NS>;
    constexpr int Q = Ly::kQ, P = Ly::kP;
    constexpr int MS = NS / 64;  // 16-row state tiles per warp (the state is NS rows over 4 warps)
    extern __shared__ __align__(16) uint8_t smem[];
    bf16_t* Xw = reinterpret_cast<bf16_t*>(smem + Ly::kXw);
    bf16_t* Ss = reinterpret_cast<bf16_t*>(smem + Ly::kSs);
    float* dts = reinterpret_cast<float*>(smem + Ly::kScal);
    float* css = dts + Q;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gq = lane >> 2, tq = lane & 3;  // mma fragment row group / column pair
    const int64_t H = p.nheads, L = p.seqlen;
    const int64_t b = blockIdx.x / H, h = blockIdx.x % H;
    const int64_t g = h / (H / p.ngroups);
    const float Ah = p.A[h];
    const float bias = p.dt_bias ? p.dt_bias[h] : 0.f;
    const float Dh = p.D ? p.D[h] : 0.f;
    const bf16_t* x = static_cast<const bf16_t*>(p.x);
    const bf16_t* zp = static_cast<const bf16_t*>(p.z);
    const bf16_t* dtp = static_cast<const bf16_t*>(p.dt);
    const bf16_t* Bg = static_cast<const bf16_t*>(p.B);
    const bf16_t* Cg = static_cast<const bf16_t*>(p.C);
    bf16_t* y = static_cast<bf16_t*>(p.y);

    // the state, in the accumulator layout of the state product: warp w holds
    // rows n in [w * 16 * MS, (w + 1) * 16 * MS), every p
    float s[MS][P / 8][4];
#pragma unroll
    for (int m = 0; m < MS; ++m)
#pragma unroll
        for (int pt = 0; pt < P / 8; ++pt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int n = (warp * MS + m) * 16 + gq + (e >> 1) * 8, pc = pt * 8 + 2 * tq + (e & 1);
                s[m][pt][e] = p.initial_state ? p.initial_state[((b * H + h) * NS + n) * P + pc] : 0.f;
            }

    const int64_t n_chunks = (L + Q - 1) / Q;
    auto buf_x = [&](int64_t c) { return reinterpret_cast<bf16_t*>(smem + Ly::kBuf + (c & 1) * Ly::kBufBytes); };
    auto buf_b = [&](int64_t c) { return buf_x(c) + Q * Ly::kXStride; };
    auto buf_c = [&](int64_t c) { return buf_b(c) + Q * Ly::kBStride; };
    // X, B, C rows of chunk c (16-byte pieces) into its buffer, zero past the sequence
    auto issue = [&](int64_t c) {
        const int64_t t0 = c * Q;
        const int q = int(min(int64_t(Q), L - t0));
        bf16_t* X_ = buf_x(c);
        bf16_t* B_ = buf_b(c);
        bf16_t* C_ = buf_c(c);
        for (int i = tid; i < Q * (P / 8); i += Ly::kThreads) {
            const int r = i / (P / 8), k8 = i % (P / 8);
            const int rr = r < q ? r : 0;  // a row inside the sequence, copied as zeros
            cp_async16(X_ + r * Ly::kXStride + k8 * 8, x + ((b * L + t0 + rr) * H + h) * P + k8 * 8, r < q ? 16u : 0u);
        }
        for (int i = tid; i < Q * (NS / 8); i += Ly::kThreads) {
            const int r = i / (NS / 8), k8 = i % (NS / 8);
            const int rr = r < q ? r : 0;
            const int64_t off = ((b * L + t0 + rr) * p.ngroups + g) * NS + k8 * 8;
            cp_async16(B_ + r * Ly::kBStride + k8 * 8, Bg + off, r < q ? 16u : 0u);
            cp_async16(C_ + r * Ly::kBStride + k8 * 8, Cg + off, r < q ? 16u : 0u);
        }
        cp_async_commit();
    };
    // raw step inputs of chunk c's tokens, two a lane of warp 0 (read one chunk
    // ahead; the softplus is taken when they are used)
    auto load_dt = [&](int64_t c, bf16_t (&dv)[2]) {
        const int64_t t0 = c * Q;
        const int q = int(min(int64_t(Q), L - t0));
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int r = 2 * lane + k;
            dv[k] = r < q ? dtp[(b * L + t0 + r) * H + h] : bf16_t{0};
        }
    };
    // this warp's 16 rows of z for chunk c: four 16-byte pieces a lane
    bf16_t* Zs = reinterpret_cast<bf16_t*>(smem + Ly::kZ) + warp * 16 * P;
    auto issue_z = [&](int64_t c) {
        const int64_t t0 = c * Q;
        const int q = int(min(int64_t(Q), L - t0));
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int piece = lane + 32 * k, r = piece >> 3, k8 = piece & 7;
            const int i = warp * 16 + r, ii = i < q ? i : 0;
            cp_async16(Zs + r * P + ((k8 ^ (r & 7)) << 3), zp + ((b * L + t0 + ii) * H + h) * P + k8 * 8,
                       i < q ? 16u : 0u);
        }
    };
    bf16_t dnext[2] = {bf16_t{0}, bf16_t{0}};
    if (n_chunks > 0) {
        issue(0);
        if (warp == 0) load_dt(0, dnext);
    }
    for (int64_t c = 0; c < n_chunks; ++c) {
        const int64_t t0 = c * Q;
        const int q = int(min(int64_t(Q), L - t0));
        __syncthreads();  // the previous chunk's reads of shared memory are done
        // this chunk's z (read by the output) and the next chunk's X, B, C
        // run during this chunk; two commit groups every chunk (the second
        // may be empty), so the waits below count the same way each time
        if constexpr (kGate) issue_z(c);
        cp_async_commit();
        if (c + 1 < n_chunks)
            issue(c + 1);
        else
            cp_async_commit();
        const bf16_t* Xs = buf_x(c);
        const bf16_t* Bs = buf_b(c);
        const bf16_t* Cs = buf_c(c);
        // the incoming state as bf16, [n][p]
#pragma unroll
        for (int m = 0; m < MS; ++m)
#pragma unroll
            for (int pt = 0; pt < P / 8; ++pt)
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {
                    const int n = (warp * MS + m) * 16 + gq + hr * 8, pc = pt * 8 + 2 * tq;
                    *reinterpret_cast<uint32_t*>(Ss + n * Ly::kSStride + pc) =
                        pack_bf16(s[m][pt][2 * hr], s[m][pt][2 * hr + 1]);
                }
        // step sizes and the running sum of Delta A (warp 0: two tokens a lane);
        // the next chunk's step sizes are read now, used then
        if (warp == 0) {
            float dv[2], cv[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const float sraw = to_f32(dnext[k]) + bias;
                dv[k] = 2 * lane + k < q ? (kSoftplus ? softplus_fast(sraw) : sraw) : 0.f;
            }
            if (c + 1 < n_chunks) load_dt(c + 1, dnext);
            cv[0] = dv[0] * Ah;
            cv[1] = cv[0] + dv[1] * Ah;
            float run = cv[1];
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float o = __shfl_up_sync(0xffffffffu, run, off);
                if (lane >= off) run += o;
            }
            const float before = run - cv[1];  // sum over the lanes before this one
            dts[2 * lane] = dv[0];
            dts[2 * lane + 1] = dv[1];
            css[2 * lane] = before + cv[0];
            css[2 * lane + 1] = before + cv[1];
        }
        // this chunk's X, B, C have landed (its z and the next chunk's copies may still run)
        cp_async_wait<2>();
        __syncthreads();
        const float cs_last = css[Q - 1];

        // G = C B^T for rows i in [16 warp, 16 warp + 16), all 64 columns j
        float gacc[Q / 8][4];
#pragma unroll
        for (int jt = 0; jt < Q / 8; ++jt)
#pragma unroll
            for (int e = 0; e < 4; ++e) gacc[jt][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < NS / 16; ++kk) {
            uint32_t a[4];
            ldsm_x4(a, Cs + (warp * 16 + (lane & 15)) * Ly::kBStride + kk * 16 + (lane >> 4) * 8);
#pragma unroll
            for (int jp = 0; jp < Q / 16; ++jp) {
                // B operand for two 8-column tiles: rows j of B, k = n contiguous
                uint32_t bb[4];
                ldsm_x4(bb, Bs + (jp * 16 + (lane & 7) + ((lane >> 4) << 3)) * Ly::kBStride + kk * 16 +
                                ((lane >> 3) & 1) * 8);
                mma_bf16(gacc[2 * jp], a, bb[0], bb[1]);
                mma_bf16(gacc[2 * jp + 1], a, bb[2], bb[3]);
            }
        }
        // mask and decay: M_ij = G_ij exp(cs_i - cs_j) Delta_j for j <= i
        const int i0 = warp * 16 + gq, i1 = i0 + 8;
        const float csi0 = css[i0], csi1 = css[i1];
        uint32_t ma[Q / 16][4];  // M as A fragments of the next product
#pragma unroll
        for (int jt = 0; jt < Q / 8; ++jt) {
            const int j0 = jt * 8 + 2 * tq, j1 = j0 + 1;
            const float cj0 = css[j0], cj1 = css[j1], dj0 = dts[j0], dj1 = dts[j1];
            const float m00 = j0 <= i0 ? gacc[jt][0] * __expf(csi0 - cj0) * dj0 : 0.f;
            const float m01 = j1 <= i0 ? gacc[jt][1] * __expf(csi0 - cj1) * dj1 : 0.f;
            const float m10 = j0 <= i1 ? gacc[jt][2] * __expf(csi1 - cj0) * dj0 : 0.f;
            const float m11 = j1 <= i1 ? gacc[jt][3] * __expf(csi1 - cj1) * dj1 : 0.f;
            const int kt = jt >> 1, hi = jt & 1;
            ma[kt][hi * 2 + 0] = pack_bf16(m00, m01);
            ma[kt][hi * 2 + 1] = pack_bf16(m10, m11);
        }
        // Y = M X (K = j) and C S_prev (K = n), rows i of this warp, every p
        float yi[P / 8][4], ye[P / 8][4];
#pragma unroll
        for (int pt = 0; pt < P / 8; ++pt)
#pragma unroll
            for (int e = 0; e < 4; ++e) yi[pt][e] = ye[pt][e] = 0.f;
#pragma unroll
        for (int kt = 0; kt < Q / 16; ++kt) {
            // A fragment order: (rows g, k 0-7), (rows g+8, k 0-7), (rows g, k 8-15), (rows g+8, k 8-15)
            const uint32_t a[4] = {ma[kt][0], ma[kt][1], ma[kt][2], ma[kt][3]};
#pragma unroll
            for (int pp = 0; pp < P / 16; ++pp) {
                uint32_t bb[4];
                ldsm_x4_t(bb, Xs + (kt * 16 + (lane & 15)) * Ly::kXStride + pp * 16 + (lane >> 4) * 8);
                mma_bf16(yi[2 * pp], a, bb[0], bb[1]);
                mma_bf16(yi[2 * pp + 1], a, bb[2], bb[3]);
            }
        }
#pragma unroll
        for (int kk = 0; kk < NS / 16; ++kk) {
            uint32_t a[4];
            ldsm_x4(a, Cs + (warp * 16 + (lane & 15)) * Ly::kBStride + kk * 16 + (lane >> 4) * 8);
#pragma unroll
            for (int pp = 0; pp < P / 16; ++pp) {
                uint32_t bb[4];
                ldsm_x4_t(bb, Ss + (kk * 16 + (lane & 15)) * Ly::kSStride + pp * 16 + (lane >> 4) * 8);
                mma_bf16(ye[2 * pp], a, bb[0], bb[1]);
                mma_bf16(ye[2 * pp + 1], a, bb[2], bb[3]);
            }
        }
        // output: y = Y_intra + exp(cs_i) C S_prev + D x, gated
        if constexpr (kGate) {
            cp_async_wait<1>();  // this lane's pieces of z
            __syncwarp();        // and its warp's
        }
        {
            const float e0 = __expf(csi0), e1 = __expf(csi1);
#pragma unroll
            for (int pt = 0; pt < P / 8; ++pt) {
                const int pc = pt * 8 + 2 * tq;
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {
                    const int i = hr ? i1 : i0;
                    if (i >= q) continue;
                    const float ex = hr ? e1 : e0;
                    const uint32_t xw = *reinterpret_cast<const uint32_t*>(Xs + i * Ly::kXStride + pc);
                    float o0 = yi[pt][2 * hr] + ex * ye[pt][2 * hr] + Dh * bf16_lo(xw);
                    float o1 = yi[pt][2 * hr + 1] + ex * ye[pt][2 * hr + 1] + Dh * bf16_hi(xw);
                    const int64_t off = ((b * L + t0 + i) * H + h) * P + pc;
                    if constexpr (kGate) {
                        const int r = gq + 8 * hr;  // row in the warp's z rows; r & 7 = gq
                        const uint32_t zw =
                            *reinterpret_cast<const uint32_t*>(Zs + r * P + ((pt ^ gq) << 3) + 2 * tq);
                        o0 *= silu_fast(bf16_lo(zw));
                        o1 *= silu_fast(bf16_hi(zw));
                    }
                    *reinterpret_cast<uint32_t*>(y + off) = pack_bf16(o0, o1);
                }
            }
        }
        // X scaled by w_j = exp(cs_last - cs_j) Delta_j for the state product,
        // where the state copy was (every warp is done reading it)
        __syncthreads();
        for (int i = tid; i < Q * (P / 2); i += Ly::kThreads) {
            const int r = i / (P / 2), k2 = i % (P / 2);
            const float w = __expf(cs_last - css[r]) * dts[r];
            const uint32_t v = *reinterpret_cast<const uint32_t*>(Xs + r * Ly::kXStride + 2 * k2);
            *reinterpret_cast<uint32_t*>(Xw + r * Ly::kXStride + 2 * k2) = pack_bf16(w * bf16_lo(v), w * bf16_hi(v));
        }
        __syncthreads();
        // S = exp(cs_last) S + B^T Xw (rows n of this warp, K = j)
        const float dec = __expf(cs_last);
#pragma unroll
        for (int m = 0; m < MS; ++m)
#pragma unroll
            for (int pt = 0; pt < P / 8; ++pt)
#pragma unroll
                for (int e = 0; e < 4; ++e) s[m][pt][e] *= dec;
#pragma unroll
        for (int kt = 0; kt < Q / 16; ++kt) {
#pragma unroll
            for (int m = 0; m < MS; ++m) {
                // A = B^T: rows n, k = j; from Bs [j][n] transposed
                uint32_t a[4];
                const int n0 = (warp * MS + m) * 16;
                ldsm_x4_t(a, Bs + (kt * 16 + (lane & 7) + ((lane >> 4) << 3)) * Ly::kBStride + n0 +
                                 ((lane >> 3) & 1) * 8);
                // ldmatrix.trans gives the 8x8 blocks as (n 0-7, j 0-7), (n 8-15, j 0-7),
                // (n 0-7, j 8-15), (n 8-15, j 8-15): the A fragment order
#pragma unroll
                for (int pp = 0; pp < P / 16; ++pp) {
                    uint32_t bb[4];
                    ldsm_x4_t(bb, Xw + (kt * 16 + (lane & 15)) * Ly::kXStride + pp * 16 + (lane >> 4) * 8);
                    mma_bf16(s[m][2 * pp], a, bb[0], bb[1]);
                    mma_bf16(s[m][2 * pp + 1], a, bb[2], bb[3]);
                }
            }
        }
    }
    if (p.last_state) {
#pragma unroll
        for (int m = 0; m < MS; ++m)
#pragma unroll
            for (int pt = 0; pt < P / 8; ++pt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int n = (warp * MS + m) * 16 + gq + (e >> 1) * 8, pc = pt * 8 + 2 * tq + (e & 1);
                    p.last_state[((b * H + h) * NS + n) * P + pc] = s[m][pt][e];
                }
    }
}

}  // namespace mss
