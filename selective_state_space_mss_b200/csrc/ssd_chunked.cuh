// ssd_chunked.cuh -- the structured-state-space-duality forward pass with
// every chunk in parallel (three passes), for callers that give a workspace.
//
// ssd_mma.cuh walks the chunks of a (batch, head) in order inside one CTA,
// which leaves a B200 with 1.7 CTAs per SM on a 4 x 64-head layer.  Here the
// chunks of every head run at once ("Mamba" paper review, section "Mamba 2":
// chunks in the quadratic form, the linear recurrence applied to the
// processed chunks):
//
//   1. chunk states: per (batch, head, chunk), the state the chunk would end
//      in from zero, B^T diag(exp(cs_last - cs_j) Delta_j) X (N x P, fp32),
//      and the chunk's decay exp(cs_last);
//   2. state pass: per (batch, head) and state element, the state entering
//      each chunk, S_in[c + 1] = decay[c] S_in[c] + S_local[c] (stored in bf16
//      as the next pass's tensor-core operand), and the final state;
//   3. chunk outputs: per (batch, head, chunk), y = M X + diag(exp(cs)) C S_in
//      + D x, gated, with M the masked, decayed C B^T of the chunk.
//
// Same arithmetic and operand rounding as ssd_mma.cuh; the chunk products
// use the same mma.sync tiles and ldmatrix layouts.
#pragma once

#include "ssd_mma.cuh"

namespace mss {

template <int NS>
struct SsdChunkLayout {
    using S = SsdLayout<NS>;
    static constexpr int kQ = S::kQ, kP = S::kP, kThreads = 128;
    static constexpr int kX = 0;                          // X (padded rows)
    static constexpr int kB = kX + S::kXBytes;            // B
    static constexpr int kC = kB + S::kBBytes;            // C (pass 3)
    static constexpr int kS = kC + S::kBBytes;            // S_in bf16 [n][p] (pass 3) / scaled X (pass 1)
    static constexpr int kScal = kS + S::kSBytes;         // Delta, cs
    static constexpr int kSmemBytes = kScal + 2 * kQ * 4;
};

// Delta and the running sum of Delta A of one chunk into dts/css (warp 0).
__device__ __forceinline__ void ssd_chunk_scalars(const SsdParams& p, int64_t b, int64_t h, int64_t t0, int q,
                                                  float Ah, float bias, bool softplus, float* dts, float* css,
                                                  int lane) {
    const bf16_t* dtp = static_cast<const bf16_t*>(p.dt);
    const int64_t H = p.nheads, L = p.seqlen;
    float dv[2], cv[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int r = 2 * lane + k;
        float d = 0.f;
        if (r < q) {
            const float sraw = to_f32(dtp[(b * L + t0 + r) * H + h]) + bias;
            d = softplus ? softplus_fast(sraw) : sraw;
        }
        dv[k] = d;
    }
    cv[0] = dv[0] * Ah;
    cv[1] = cv[0] + dv[1] * Ah;
    float run = cv[1];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float o = __shfl_up_sync(0xffffffffu, run, off);
        if (lane >= off) run += o;
    }
    const float before = run - cv[1];
    dts[2 * lane] = dv[0];
    dts[2 * lane + 1] = dv[1];
    css[2 * lane] = before + cv[0];
    css[2 * lane + 1] = before + cv[1];
}

// Rows of one chunk into padded shared memory (16-byte copies, zeros past q).
template <int NS>
__device__ __forceinline__ void ssd_load_rows(const SsdParams& p, int64_t b, int64_t h, int64_t g, int64_t t0, int q,
                                              bf16_t* Xs, bf16_t* Bs, bf16_t* Cs, int tid) {
    using Ly = SsdLayout<NS>;
    constexpr int Q = Ly::kQ, P = Ly::kP;
    const int64_t H = p.nheads, L = p.seqlen;
    const bf16_t* x = static_cast<const bf16_t*>(p.x);
    const bf16_t* Bg = static_cast<const bf16_t*>(p.B);
    const bf16_t* Cg = static_cast<const bf16_t*>(p.C);
    for (int i = tid; i < Q * (P / 8); i += 128) {
        const int r = i / (P / 8), k8 = i % (P / 8);
        const int rr = r < q ? r : 0;
        cp_async16(Xs + r * Ly::kXStride + k8 * 8, x + ((b * L + t0 + rr) * H + h) * P + k8 * 8, r < q ? 16u : 0u);
    }
    for (int i = tid; i < Q * (NS / 8); i += 128) {
        const int r = i / (NS / 8), k8 = i % (NS / 8);
        const int rr = r < q ? r : 0;
        const int64_t off = ((b * L + t0 + rr) * p.ngroups + g) * NS + k8 * 8;
        cp_async16(Bs + r * Ly::kBStride + k8 * 8, Bg + off, r < q ? 16u : 0u);
        if (Cs) cp_async16(Cs + r * Ly::kBStride + k8 * 8, Cg + off, r < q ? 16u : 0u);
    }
    cp_async_commit();
}

// Pass 1.  grid = (n_chunks, units), block = 128: (batch, head) pairs
// unit0 .. unit0 + units - 1 (pair u = batch index * nheads + head).
// Sl: [units][n_chunks][NS][P] fp32; decay: [units][n_chunks].
template <int NS, bool kSoftplus>
__global__ void __launch_bounds__(128) ssd_chunk_state_kernel(SsdParams p, float* Sl, float* decay, int64_t unit0) {
    using Ly = SsdLayout<NS>;
    using CL = SsdChunkLayout<NS>;
    constexpr int Q = Ly::kQ, P = Ly::kP, MS = NS / 64;
    extern __shared__ __align__(16) uint8_t smem[];
    bf16_t* Xs = reinterpret_cast<bf16_t*>(smem + CL::kX);
    bf16_t* Bs = reinterpret_cast<bf16_t*>(smem + CL::kB);
    bf16_t* Xw = reinterpret_cast<bf16_t*>(smem + CL::kS);
    float* dts = reinterpret_cast<float*>(smem + CL::kScal);
    float* css = dts + Q;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gq = lane >> 2, tq = lane & 3;
    // (batch, head) unit unit0 + blockIdx.y; the workspace holds this launch's units only
    const int64_t c = blockIdx.x, ul = blockIdx.y, H = p.nheads, L = p.seqlen, n_chunks = gridDim.x;
    const int64_t h = (unit0 + ul) % H, b = (unit0 + ul) / H;
    const int64_t g = h / (H / p.ngroups);
    const int64_t t0 = c * Q;
    const int q = int(min(int64_t(Q), L - t0));
    ssd_load_rows<NS>(p, b, h, g, t0, q, Xs, Bs, nullptr, tid);
    if (warp == 0)
        ssd_chunk_scalars(p, b, h, t0, q, p.A[h], p.dt_bias ? p.dt_bias[h] : 0.f, kSoftplus, dts, css, lane);
    cp_async_wait<0>();
    __syncthreads();
    const float cs_last = css[Q - 1];
    for (int i = tid; i < Q * (P / 2); i += 128) {
        const int r = i / (P / 2), k2 = i % (P / 2);
        const float w = __expf(cs_last - css[r]) * dts[r];
        const uint32_t v = *reinterpret_cast<const uint32_t*>(Xs + r * Ly::kXStride + 2 * k2);
        *reinterpret_cast<uint32_t*>(Xw + r * Ly::kXStride + 2 * k2) = pack_bf16(w * bf16_lo(v), w * bf16_hi(v));
    }
    __syncthreads();
    float s[MS][P / 8][4];
#pragma unroll
    for (int m = 0; m < MS; ++m)
#pragma unroll
        for (int pt = 0; pt < P / 8; ++pt)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[m][pt][e] = 0.f;
#pragma unroll
    for (int kt = 0; kt < Q / 16; ++kt) {
#pragma unroll
        for (int m = 0; m < MS; ++m) {
            uint32_t a[4];
            const int n0 = (warp * MS + m) * 16;
            ldsm_x4_t(a, Bs + (kt * 16 + (lane & 7) + ((lane >> 4) << 3)) * Ly::kBStride + n0 + ((lane >> 3) & 1) * 8);
#pragma unroll
            for (int pp = 0; pp < P / 16; ++pp) {
                uint32_t bb[4];
                ldsm_x4_t(bb, Xw + (kt * 16 + (lane & 15)) * Ly::kXStride + pp * 16 + (lane >> 4) * 8);
                mma_bf16(s[m][2 * pp], a, bb[0], bb[1]);
                mma_bf16(s[m][2 * pp + 1], a, bb[2], bb[3]);
            }
        }
    }
    float* out = Sl + ((ul * n_chunks + c) * NS) * P;
#pragma unroll
    for (int m = 0; m < MS; ++m)
#pragma unroll
        for (int pt = 0; pt < P / 8; ++pt)
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                const int n = (warp * MS + m) * 16 + gq + hr * 8, pc = pt * 8 + 2 * tq;
                *reinterpret_cast<float2*>(out + n * P + pc) = make_float2(s[m][pt][2 * hr], s[m][pt][2 * hr + 1]);
            }
    if (tid == 0) decay[ul * n_chunks + c] = __expf(cs_last);
}

// Pass 2.  grid = (units, NS * P / 256), block = 256: one state element per
// thread, the chunks in order.  Sin: [units][n_chunks][NS][P] bf16.
template <int NS>
__global__ void __launch_bounds__(256) ssd_state_pass_kernel(SsdParams p, const float* Sl, const float* decay,
                                                             bf16_t* Sin, int64_t n_chunks, int64_t unit0) {
    constexpr int P = SsdLayout<NS>::kP;
    const int64_t ul = blockIdx.x, bh = unit0 + ul;  // the launch's unit, the (batch, head) pair
    const int e = blockIdx.y * 256 + threadIdx.x;  // n * P + p
    float S = p.initial_state ? p.initial_state[bh * NS * P + e] : 0.f;
    const float* sl = Sl + ul * n_chunks * NS * P + e;
    const float* dc = decay + ul * n_chunks;
    bf16_t* si = Sin + ul * n_chunks * NS * P + e;
    for (int64_t c = 0; c < n_chunks; ++c) {
        si[c * NS * P] = from_f32<bf16_t>(S);
        S = fmaf(dc[c], S, sl[c * NS * P]);
    }
    if (p.last_state) p.last_state[bh * NS * P + e] = S;
}

// Pass 3.  grid = (n_chunks, units), block = 128.
template <int NS, bool kGate, bool kSoftplus>
__global__ void __launch_bounds__(128) ssd_chunk_out_kernel(SsdParams p, const bf16_t* Sin, int64_t unit0) {
    using Ly = SsdLayout<NS>;
    using CL = SsdChunkLayout<NS>;
    constexpr int Q = Ly::kQ, P = Ly::kP;
    extern __shared__ __align__(16) uint8_t smem[];
    bf16_t* Xs = reinterpret_cast<bf16_t*>(smem + CL::kX);
    bf16_t* Bs = reinterpret_cast<bf16_t*>(smem + CL::kB);
    bf16_t* Cs = reinterpret_cast<bf16_t*>(smem + CL::kC);
    bf16_t* Ss = reinterpret_cast<bf16_t*>(smem + CL::kS);
    float* dts = reinterpret_cast<float*>(smem + CL::kScal);
    float* css = dts + Q;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gq = lane >> 2, tq = lane & 3;
    // (batch, head) unit unit0 + blockIdx.y; the workspace holds this launch's units only
    const int64_t c = blockIdx.x, ul = blockIdx.y, H = p.nheads, L = p.seqlen, n_chunks = gridDim.x;
    const int64_t h = (unit0 + ul) % H, b = (unit0 + ul) / H;
    const int64_t g = h / (H / p.ngroups);
    const int64_t t0 = c * Q;
    const int q = int(min(int64_t(Q), L - t0));
    const float Dh = p.D ? p.D[h] : 0.f;
    ssd_load_rows<NS>(p, b, h, g, t0, q, Xs, Bs, Cs, tid);
    {
        // the state entering the chunk, [n][p] bf16 into padded rows
        const bf16_t* si = Sin + ((ul * n_chunks + c) * NS) * P;
        for (int i = tid; i < NS * (P / 8); i += 128) {
            const int r = i / (P / 8), k8 = i % (P / 8);
            cp_async16(Ss + r * Ly::kSStride + k8 * 8, si + r * P + k8 * 8, 16u);
        }
        cp_async_commit();
    }
    if (warp == 0)
        ssd_chunk_scalars(p, b, h, t0, q, p.A[h], p.dt_bias ? p.dt_bias[h] : 0.f, kSoftplus, dts, css, lane);
    cp_async_wait<0>();
    __syncthreads();

    // G = C B^T, masked and decayed into M (rows i of this warp)
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
            uint32_t bb[4];
            ldsm_x4(bb, Bs + (jp * 16 + (lane & 7) + ((lane >> 4) << 3)) * Ly::kBStride + kk * 16 + ((lane >> 3) & 1) * 8);
            mma_bf16(gacc[2 * jp], a, bb[0], bb[1]);
            mma_bf16(gacc[2 * jp + 1], a, bb[2], bb[3]);
        }
    }
    const int i0 = warp * 16 + gq, i1 = i0 + 8;
    const float csi0 = css[i0], csi1 = css[i1];
    uint32_t ma[Q / 16][4];
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
    float yi[P / 8][4], ye[P / 8][4];
#pragma unroll
    for (int pt = 0; pt < P / 8; ++pt)
#pragma unroll
        for (int e = 0; e < 4; ++e) yi[pt][e] = ye[pt][e] = 0.f;
#pragma unroll
    for (int kt = 0; kt < Q / 16; ++kt) {
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
    const bf16_t* zp = static_cast<const bf16_t*>(p.z);
    bf16_t* y = static_cast<bf16_t*>(p.y);
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
                const uint32_t zw = *reinterpret_cast<const uint32_t*>(zp + off);
                o0 *= silu_fast(bf16_lo(zw));
                o1 *= silu_fast(bf16_hi(zw));
            }
            *reinterpret_cast<uint32_t*>(y + off) = pack_bf16(o0, o1);
        }
    }
}

}  // namespace mss
