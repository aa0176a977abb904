// launch.h -- the kernel launchers behind the C ABI, one explicit
// instantiation per (io type, N), compiled in separate translation units
// (fwd_*.cu, decode.cu) so that the library builds in parallel.
#pragma once

#include <cstdint>

#include <cuda_runtime.h>

#include "mss_device.cuh"
#include "mss_params.h"

namespace mss_host {

// Forward pass over validated arguments (p.err set): picks the throughput
// kernel or the scalar one and, with a workspace, the sequence split.
template <typename T, int N>
int launch_forward(mss::ScanParams p, unsigned flags, void* workspace, int64_t workspace_bytes,
                   cudaStream_t stream);

// The same through the tiled kernel only, also storing the backward pass's
// group-start states; MSS_ERR_PATH when the tiled kernel does not take it.
template <typename T, int N>
int launch_forward_save(mss::ScanParams p, unsigned flags, void* workspace, int64_t workspace_bytes, float* states,
                        cudaStream_t stream);

// Workspace bytes the forward pass would use to split the sequence (0: none).
template <typename T, int N>
int64_t forward_workspace_bytes(int64_t batch, int64_t dim, int64_t seqlen);

// Backward pass over validated arguments: fp holds the forward arguments
// (with p.err), bp the gradients; the workspace holds the checkpoints (with
// MSS_FLAG_SAVED_STATES already written by the saving forward pass).
template <typename T, int N>
int launch_backward(mss::ScanParams fp, mss::BwdParams bp, unsigned flags, void* workspace, int64_t workspace_bytes,
                    cudaStream_t stream);

template <typename T, int N>
int64_t backward_workspace_bytes(int64_t batch, int64_t dim, int64_t seqlen, unsigned flags);

// Decode update over validated arguments (p.err set).
template <typename T, int N>
int launch_decode(mss::StepParams p, cudaStream_t stream);

// Structured-state-space-duality forward pass over validated arguments
// (bf16 io, P = 64, dstate 64 or 128): the warp-level (mma.sync) kernel.
int launch_ssd(const mss::SsdParams& p, int dstate, cudaStream_t stream);

// The same on the tcgen05 tensor cores (dstate 128; x, z, y, B, C 16-byte
// aligned).
int launch_ssd_tc(const mss::SsdParams& p, int64_t unit0, int64_t units, cudaStream_t stream);

// The same with every chunk in parallel (three passes) over a workspace of
// ssd_workspace_bytes (16-byte aligned).
int launch_ssd_chunked(const mss::SsdParams& p, int dstate, void* workspace, int64_t unit0, int64_t units,
                       cudaStream_t stream);
int64_t ssd_workspace_bytes(int64_t batch, int64_t seqlen, int64_t nheads, int64_t dstate);
// Whether the chunk-parallel passes beat the in-order kernel for this many
// (batch, head) pairs on the current device.
bool ssd_chunked_pays(int64_t batch, int64_t nheads);
// The same against the tcgen05 kernel (dstate 128).
bool ssd_chunked_pays_tc(int64_t batch, int64_t nheads);
// The pairs past the tcgen05 kernel's last full wave that the chunk-parallel
// passes should take (0: none).
int64_t ssd_tc_tail_units(int64_t batch, int64_t nheads);

#define MSS_DECLARE_LAUNCHERS(T, N)                                                                      \
    extern template int launch_forward<T, N>(mss::ScanParams, unsigned, void*, int64_t, cudaStream_t); \
    extern template int launch_forward_save<T, N>(mss::ScanParams, unsigned, void*, int64_t, float*,    \
                                                  cudaStream_t);                                         \
    extern template int64_t forward_workspace_bytes<T, N>(int64_t, int64_t, int64_t);                   \
    extern template int launch_decode<T, N>(mss::StepParams, cudaStream_t);                              \
    extern template int launch_backward<T, N>(mss::ScanParams, mss::BwdParams, unsigned, void*, int64_t,   \
                                              cudaStream_t);                                             \
    extern template int64_t backward_workspace_bytes<T, N>(int64_t, int64_t, int64_t, unsigned);

MSS_DECLARE_LAUNCHERS(mss::bf16_t, 1)
MSS_DECLARE_LAUNCHERS(mss::bf16_t, 2)
MSS_DECLARE_LAUNCHERS(mss::bf16_t, 4)
MSS_DECLARE_LAUNCHERS(mss::bf16_t, 8)
MSS_DECLARE_LAUNCHERS(mss::bf16_t, 16)
MSS_DECLARE_LAUNCHERS(float, 1)
MSS_DECLARE_LAUNCHERS(float, 2)
MSS_DECLARE_LAUNCHERS(float, 4)
MSS_DECLARE_LAUNCHERS(float, 8)
MSS_DECLARE_LAUNCHERS(float, 16)

#undef MSS_DECLARE_LAUNCHERS

}  // namespace mss_host
