// mss_params.h -- kernel argument blocks (passed by value to every launch).
#pragma once

#include <cstdint>

namespace mss {

struct ScanParams {
    const void* u;
    const void* delta;
    const float* A;
    const void* B;
    const void* C;
    const float* D;           // may be null
    const void* z;            // may be null
    const float* delta_bias;  // may be null
    void* y;
    float* last_state;        // may be null
    int64_t batch, dim, seqlen;
    int softplus;
    const float* initial_state;  // [batch, dim, N] state before the first token, or null (zero)
    // Sequence split: n_seg segments of seg_len tokens (the last may be
    // shorter); agg holds the per-segment aggregates [n_seg-1][2][batch*dim][N]
    // (exp(A * sum of steps), then the segment's final state from zero).
    float* agg;
    int64_t seg_len;
    int n_seg;
    int zoh;  // input matrix: 0 Euler Delta*B, 1 zero-order hold (e^{Delta A} - 1)/A * B
    unsigned int* err;  // device error word (bounded waits that give up set it)
    // Causal convolution in front of the scan (conv_width > 0): u holds x and
    // the scan input is silu(conv_b + sum_k conv_w[d,k] x_{t-(K-1)+k}).
    const float* conv_w;         // [dim, K]
    const float* conv_b;         // [dim], may be null
    const void* conv_state_in;   // [batch, dim, K-1] io type: x before the first token, or null (zeros)
    void* conv_state_out;        // [batch, dim, K-1] io type: the last K-1 inputs, may be null
    int conv_width;              // K in 1..4, or 0 without the convolution
    // Checkpoint pass of the backward pass (fold launches only): the state at
    // the start of every group of V tokens, [batch * dim, seqlen / V, N], each
    // group's N floats in lane order (lane half h: pairs (h_n, h_n+2), n = h + 4i).
    float* ckpt;
    // Self-test of the bounded waits (MSS_FLAG_SELFTEST_TIMEOUT): nonzero makes
    // every CTA of the tiled kernel wait this many nanoseconds on a barrier no
    // copy completes, then return; 0 otherwise.
    unsigned long long selftest_wait_ns;
};

// Backward pass (scan_bwd.cuh).  Inputs as ScanParams; dy is the gradient
// with respect to y, dlast with respect to last_state (may be null).  The
// per-token gradients du, ddelta (with respect to delta_raw) and dz have the
// io type; dB, dC [batch, N, L], dA [dim, N], dD, dbias [dim] are fp32 sums
// (zeroed by the host, accumulated with atomics); dinit [batch, dim, N] is
// the gradient with respect to the starting state (may be null).
struct BwdParams {
    const void* u;
    const void* delta;
    const float* A;
    const void* B;
    const void* C;
    const float* D;           // may be null
    const void* z;            // may be null
    const float* delta_bias;  // may be null
    const void* dy;
    const float* dlast;       // may be null
    const float* ckpt;        // [batch * dim, seqlen / V, N] states at the start of each group of V tokens
    void* du;
    void* ddelta;
    void* dz;                 // null when z is null
    float* dA;
    float* dB;
    float* dC;
    float* dD;
    float* dbias;
    float* dinit;             // may be null
    int64_t batch, dim, seqlen;
    int softplus;
    unsigned int* err;
};

// Structured state space duality (ssd_mma.cuh): x, z, y [batch, L, H, P];
// dt [batch, L, H]; B, C [batch, L, G, N]; A, D, dt_bias [H] fp32;
// initial_state, last_state [batch, H, N, P] fp32.
struct SsdParams {
    const void* x;
    const void* dt;
    const float* A;
    const void* B;
    const void* C;
    const float* D;        // may be null
    const void* z;         // may be null
    const float* dt_bias;  // may be null
    const float* initial_state;  // may be null
    void* y;
    float* last_state;     // may be null
    int64_t batch, seqlen, nheads, ngroups;
    int softplus;
    unsigned int* err;     // device error word (the tcgen05 kernel's bounded waits)
};

struct StepParams {
    float* state;
    const void* u;
    const void* delta;
    const float* A;
    const void* B;
    const void* C;
    const float* D;
    const void* z;
    const float* delta_bias;
    void* y;
    int64_t batch, dim;
    int softplus;
    int zoh;       // as in ScanParams
    int64_t row0;  // first (batch * dim + channel) row this launch serves
    unsigned int* err;  // as in ScanParams
    // Causal convolution in front (conv_width > 0): u holds this token's x;
    // conv_state [batch, dim, K-1] (io type, oldest first) is read and shifted.
    const float* conv_w;  // [dim, K]
    const float* conv_b;  // [dim], may be null
    void* conv_state;
    int conv_width;
};

}  // namespace mss
