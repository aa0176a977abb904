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
};

}  // namespace mss
