// mss_device.cuh -- device-side helpers shared by the selective-scan kernels:
// element loads/stores for float and bf16, the step-size and gate functions,
// and thin wrappers over single sm_100a instructions.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace mss {

// ---------------------------------------------------------------------------
// Element types.  bf16 travels as its 16-bit pattern; widening is exact
// (the pattern is the top half of an fp32), narrowing rounds to nearest even
// with the hardware conversion instruction.

struct bf16_t {
    uint16_t bits;
};

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(bf16_t x) { return __uint_as_float(uint32_t(x.bits) << 16); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16_t from_f32<bf16_t>(float x) {
    uint16_t r;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(x));
    return bf16_t{r};
}

// Two fp32 values -> one 32-bit word of two bf16 (lo in the low half).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

template <typename T> __device__ __forceinline__ float ld(const T* p) { return to_f32(*p); }

// ---------------------------------------------------------------------------
// Single-instruction approximations (MUFU).  Their accuracy is the PTX ISA's
// documented bound for each instruction; callers that need the full-precision
// library function use expf / log1pf instead.

__device__ __forceinline__ float ex2_approx(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ float rcp_approx(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

constexpr float kLog2e = 1.4426950408889634f;  // 1 / ln 2

// ---------------------------------------------------------------------------
// Step size and gate.
//
// softplus(s) = ln(1 + e^s) ("Exercises -- State-space models (Mamba, S4)",
// softplus exercise).  Above s = 20 the correction ln(1 + e^{-s}) < 2.1e-9 is
// below half an ulp of s in fp32, so s itself is the correctly rounded result.

// Full precision: the CUDA math library's expf and log1pf.
__device__ __forceinline__ float softplus_precise(float s) {
    return s > 20.f ? s : log1pf(expf(s));
}

__device__ __forceinline__ float lg2_approx(float x) {
    float r;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// Fast form for bf16 io: softplus(s) = max(s, 0) + ln 2 * log2(1 + e^{-|s|}),
// two MUFU instructions and three fp32 operations.  The single-instruction
// log2 has an absolute error near 2^-22 on (1, 2], so Delta carries an
// absolute error of about 2e-7 (relative 2e-4 at Delta = 1e-3, less for
// larger steps): ten times below the rounding of a bf16 output.  fp32 io uses
// softplus_precise.
__device__ __forceinline__ float softplus_fast(float s) {
    const float e = ex2_approx(-fabsf(s) * kLog2e);
    const float r = fmaf(0.69314718f, lg2_approx(1.f + e), fmaxf(s, 0.f));
    return s > 20.f ? s : r;
}

// silu(z) = z * sigmoid(z) = z / (1 + e^{-z}).
__device__ __forceinline__ float silu_precise(float z) { return z / (1.f + expf(-z)); }
__device__ __forceinline__ float silu_fast(float z) {
    // e^{-z} overflows to +inf for z < -88: rcp(inf) = 0 gives the right limit
    return z * rcp_approx(1.f + ex2_approx(-z * kLog2e));
}

// ---------------------------------------------------------------------------
// Zero-order-hold input weight.  The exact discretisation of the input term
// ("Mamba" paper review, section "SSM") is Bbar = (e^{Delta a} - 1)/a * B per
// state, i.e. Delta * phi(Delta a) * B with phi(x) = (e^x - 1)/x.  Formed from
// the already computed e = e^x as (e - 1)/a it loses |x|^-1 ulps to
// cancellation, so below |x| = 1/8 the kernels use the Taylor series of phi
// instead, 1 + x/2 + x^2/6 + x^3/24 + x^4/120, whose first omitted term is
// under 5e-8 there; above it the cancellation costs less than 3 bits.  phi is
// finite and positive everywhere and phi(0) = 1 gives the Euler weight Delta
// at a = 0.

constexpr float kZohTaylorMax = 0.125f;
constexpr float kLn2 = 0.69314718055994531f;

__device__ __forceinline__ float phi_taylor(float x) {
    return fmaf(fmaf(fmaf(fmaf(x, 1.f / 120.f, 1.f / 24.f), x, 1.f / 6.f), x, 0.5f), x, 1.f);
}

// Delta * phi(x) with x = Delta * a and e = e^x: the weight of B * u.
__device__ __forceinline__ float zoh_weight(float dt, float a, float x, float e) {
    return fabsf(x) < kZohTaylorMax ? dt * phi_taylor(x) : (e - 1.f) / a;
}

// d/da of the weight Delta * phi(Delta a) (the backward pass):
// Delta^2 phi'(x), phi'(x) = 1/2 + x/3 + x^2/8 + x^3/30 + x^4/144 + ... below
// |x| = 1/8 (first omitted term under 2e-7 of the sum), else (Delta e - w)/a.
__device__ __forceinline__ float dphi_taylor(float x) {
    return fmaf(fmaf(fmaf(fmaf(x, 1.f / 144.f, 1.f / 30.f), x, 1.f / 8.f), x, 1.f / 3.f), x, 0.5f);
}

__device__ __forceinline__ float zoh_weight_dA(float dt, float a, float x, float e, float w) {
    return fabsf(x) < kZohTaylorMax ? dt * dt * dphi_taylor(x) : (dt * e - w) / a;
}

// ---------------------------------------------------------------------------
// Causal convolution in front of the scan ("Mamba" paper review, section
// "SSM", block description: a convolution and non-linearity before the SSM
// bank).  The K <= 4 taps of a channel are kept right-aligned in four slots,
// so that slot j multiplies x_{t-3+j} and slots below 4-K hold zero; the
// window is the three previous inputs and the current one.

struct ConvTaps {
    float w[4];
    float b;
};

__device__ __forceinline__ ConvTaps load_conv_taps(const float* conv_w, const float* conv_b, int K, int64_t d) {
    ConvTaps c;
#pragma unroll
    for (int j = 0; j < 4; ++j) c.w[j] = j >= 4 - K ? __ldg(conv_w + d * K + (j - (4 - K))) : 0.f;
    c.b = conv_b ? __ldg(conv_b + d) : 0.f;
    return c;
}

// Pre-activation cb + sum_j w[j] x_{t-3+j} for the window (x_{t-3}, x_{t-2}, x_{t-1}, x_t).
__device__ __forceinline__ float conv_pre(const ConvTaps& c, float xm3, float xm2, float xm1, float x0) {
    return fmaf(c.w[3], x0, fmaf(c.w[2], xm1, fmaf(c.w[1], xm2, fmaf(c.w[0], xm3, c.b))));
}

// ---------------------------------------------------------------------------
// Device error word: set by kernels whose bounded waits give up, read and
// cleared by mss_get_device_error.  It is one word per device defined in
// mss_api.cu; every launch receives its address in its parameter block.
constexpr unsigned int kDeviceErrTimeout = 1u;

__device__ __forceinline__ void raise_device_error(unsigned int* err, unsigned int code) {
    if (err) atomicOr(err, code);
}

}  // namespace mss
