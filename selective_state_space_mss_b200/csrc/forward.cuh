// forward.cuh -- host-side launch of the forward pass (included by the
// fwd_*.cu translation units, each instantiating a few (io type, N) pairs):
// tensor maps for the TMA loads, the choice between the throughput and the
// scalar kernel, and the sequence split.
#pragma once

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "host_common.h"
#include "launch.h"
#include "scan_seq.cuh"
#include "scan_seq4.cuh"
#include "scan_simple.cuh"

namespace mss_host {

// cuTensorMapEncodeTiled, resolved once through the runtime so that the
// library does not link the driver library itself.
inline PFN_cuTensorMapEncodeTiled_v12000 encode_tiled_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// [rows, L] row-major view, box = box_rows rows x 128 bytes, 128-byte swizzle.
inline bool encode_rows(CUtensorMap* m, const void* base, int64_t rows, int64_t L, int esz, int box_rows) {
    auto enc = encode_tiled_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cuuint64_t(L), cuuint64_t(rows)};
    const cuuint64_t strides[1] = {cuuint64_t(L * esz)};
    const cuuint32_t box[2] = {cuuint32_t(128 / esz), cuuint32_t(box_rows)};
    const cuuint32_t estr[2] = {1u, 1u};
    return enc(m, esz == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
               const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [batch, N, L] view, box = 1 x N x 128 bytes, no swizzle.
inline bool encode_bc(CUtensorMap* m, const void* base, int64_t batch, int64_t N, int64_t L, int esz) {
    auto enc = encode_tiled_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {cuuint64_t(L), cuuint64_t(N), cuuint64_t(batch)};
    const cuuint64_t strides[2] = {cuuint64_t(L * esz), cuuint64_t(N * L * esz)};
    const cuuint32_t box[3] = {cuuint32_t(128 / esz), cuuint32_t(N), 1u};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    return enc(m, esz == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
               const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T, int N>
int launch_simple(const mss::ScanParams& p, cudaStream_t stream) {
    const int64_t rows = p.batch * p.dim;
    const int threads = 128;
    const int64_t blocks = (rows + threads - 1) / threads;
    if (blocks > 0x7fffffffLL) return MSS_ERR_SHAPE;
    mss::scan_fwd_simple_kernel<T, N><<<dim3(unsigned(blocks)), threads, 0, stream>>>(p);
    return launch_status();
}

template <typename T, int N, bool kGate, bool kSoftplus, bool kFold, bool kZoh, bool kConv, bool kSave = false>
int launch_seq_variant(const mss::SeqMaps& maps, const mss::ScanParams& p, unsigned flags, int segs,
                       cudaStream_t stream) {
    auto kern = mss::scan_fwd_seq_kernel<T, N, kGate, kSoftplus, kFold, kZoh, kConv, kSave>;
    const int smem = mss::SeqLayout<T, N>::kSmemBytes;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return MSS_ERR_CUDA;
    constexpr int rows = mss::SeqLayout<T, N>::kRows;
    const dim3 grid(unsigned((p.dim + rows - 1) / rows), unsigned(p.batch), unsigned(segs));
    kern<<<grid, 32, smem, stream>>>(maps, p, (flags & MSS_FLAG_GENERAL_A) ? 0 : 1);
    return launch_status();
}

// Resident blocks of the throughput kernel (all its variants share the
// layout) on the current device, looked up once per device.
template <typename T, int N>
int seq_slots() {
    static std::mutex mu;
    static int cache[kMaxDevices] = {};
    return per_device(cache, mu, [](int dev) {
        return resident_blocks(mss::scan_fwd_seq_kernel<T, N, true, true, false, false, false>, 32,
                               mss::SeqLayout<T, N>::kSmemBytes, dev);
    });
}

// Sequence split for workloads with too few channels to occupy the GPU:
// segments per sequence so that the full pass has about two warps per
// scheduler without exceeding one wave.  1 = no split.
template <typename T, int N>
int choose_segments(int64_t batch, int64_t dim, int64_t seqlen) {
    using Ly = mss::SeqLayout<T, N>;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 1;
    const int64_t slots = seq_slots<T, N>();
    if (slots <= 0) return 1;
    const int64_t ctas = batch * ((dim + Ly::kRows - 1) / Ly::kRows);
    const int64_t target = 2 * 4 * int64_t(sms);  // two warps per scheduler
    const int64_t n_chunks = (seqlen + Ly::kChunk - 1) / Ly::kChunk;
    int64_t n = std::min<int64_t>(slots / ctas, (target + ctas - 1) / ctas);
    n = std::min<int64_t>(std::min<int64_t>(n, n_chunks), 64);
    if (n < 2) return 1;
    // Measured against one pass (L = 4096, B200), where one pass wins: bf16
    // at N = 16 with two segments (263-267 against 285-291 us at 384-512
    // units of 16 channels: the fold re-runs half the sequence to double the
    // warps), fp32 at N = 8 or 16 above 384 units, where the one pass runs
    // four lanes per channel (646 against 797 us at N = 16, 461 against 483 at
    // N = 8).  bf16 at N = 8 keeps the split up to 512 units (226 against
    // 240 us), fp32 up to 384 (607 against 646, 370 against 461 us).
    if constexpr (sizeof(T) == 2 && N == 16) {
        if (n == 2) return 1;
    }
    if constexpr (sizeof(T) == 4 && N >= 8) {
        if (ctas > 384) return 1;
    }
    // equal segments of whole chunks
    const int64_t seg_chunks = (n_chunks + n - 1) / n;
    return int((n_chunks + seg_chunks - 1) / seg_chunks);
}

template <typename T, int N>
int64_t seg_len_for(int64_t seqlen, int n_seg) {
    using Ly = mss::SeqLayout<T, N>;
    const int64_t n_chunks = (seqlen + Ly::kChunk - 1) / Ly::kChunk;
    return ((n_chunks + n_seg - 1) / n_seg) * Ly::kChunk;
}

inline int64_t agg_bytes(int n_seg, int64_t rows, int64_t N) { return n_seg > 1 ? int64_t(n_seg - 1) * 2 * rows * N * 4 : 0; }

// The fold pass (split sequences only), then the full pass.
template <typename T, int N, bool kZoh, bool kConv>
int launch_seq_passes(const mss::SeqMaps& maps, const mss::ScanParams& p, unsigned flags, cudaStream_t stream) {
    if (p.n_seg > 1) {
        // first pass: each segment but the last folds to its aggregates (from
        // a zero state: its states are not the sequence's, so it stores none)
        mss::ScanParams pf = p;
        pf.ckpt = nullptr;
        const int rc = p.softplus
                           ? launch_seq_variant<T, N, false, true, true, kZoh, kConv>(maps, pf, flags, p.n_seg - 1, stream)
                           : launch_seq_variant<T, N, false, false, true, kZoh, kConv>(maps, pf, flags, p.n_seg - 1, stream);
        if (rc != MSS_OK) return rc;
    }
    if constexpr (!kConv) {
        // the full pass that also stores the states (mss_scan_fwd_save)
        if (p.ckpt) {
            if (p.z)
                return p.softplus
                           ? launch_seq_variant<T, N, true, true, false, kZoh, false, true>(maps, p, flags, p.n_seg, stream)
                           : launch_seq_variant<T, N, true, false, false, kZoh, false, true>(maps, p, flags, p.n_seg, stream);
            return p.softplus
                       ? launch_seq_variant<T, N, false, true, false, kZoh, false, true>(maps, p, flags, p.n_seg, stream)
                       : launch_seq_variant<T, N, false, false, false, kZoh, false, true>(maps, p, flags, p.n_seg, stream);
        }
    }
    if (p.z)
        return p.softplus ? launch_seq_variant<T, N, true, true, false, kZoh, kConv>(maps, p, flags, p.n_seg, stream)
                          : launch_seq_variant<T, N, true, false, false, kZoh, kConv>(maps, p, flags, p.n_seg, stream);
    return p.softplus ? launch_seq_variant<T, N, false, true, false, kZoh, kConv>(maps, p, flags, p.n_seg, stream)
                      : launch_seq_variant<T, N, false, false, false, kZoh, kConv>(maps, p, flags, p.n_seg, stream);
}

// Every pass of one convolution setting; the variants with the convolution
// can be compiled in a translation unit of their own (extern template).
template <typename T, int N, bool kConv>
int launch_seq_conv(const mss::SeqMaps& maps, const mss::ScanParams& p, unsigned flags, cudaStream_t stream) {
    return p.zoh ? launch_seq_passes<T, N, true, kConv>(maps, p, flags, stream)
                 : launch_seq_passes<T, N, false, kConv>(maps, p, flags, stream);
}

// The four-lane kernel (one pass, Euler input rule, no convolution, no
// checkpoints).  With bf16 io it is taken for grids of at most this many
// 16-channel units (2.6 per SM on 148 SMs).
constexpr int64_t kFourLaneBf16MaxUnits = 384;

template <typename T, int N, bool kGate, bool kSoftplus>
int launch_seq4_variant(const mss::SeqMaps& maps, const mss::ScanParams& p, unsigned flags, cudaStream_t stream) {
    using Ly = mss::Seq4Layout<T, N>;
    auto kern = mss::scan_fwd_seq4_kernel<T, N, kGate, kSoftplus>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Ly::kSmemBytes) != cudaSuccess)
        return MSS_ERR_CUDA;
    const dim3 grid(unsigned((p.dim + Ly::kRows - 1) / Ly::kRows), unsigned(p.batch), 1u);
    kern<<<grid, Ly::kThreads, Ly::kSmemBytes, stream>>>(maps, p, (flags & MSS_FLAG_GENERAL_A) ? 0 : 1);
    return launch_status();
}

template <typename T, int N>
int launch_seq4(const mss::SeqMaps& maps, const mss::ScanParams& p, unsigned flags, cudaStream_t stream) {
    if (p.z)
        return p.softplus ? launch_seq4_variant<T, N, true, true>(maps, p, flags, stream)
                          : launch_seq4_variant<T, N, true, false>(maps, p, flags, stream);
    return p.softplus ? launch_seq4_variant<T, N, false, true>(maps, p, flags, stream)
                      : launch_seq4_variant<T, N, false, false>(maps, p, flags, stream);
}

template <typename T, int N>
int launch_seq(mss::ScanParams p, unsigned flags, void* workspace, int64_t workspace_bytes, cudaStream_t stream) {
    constexpr int esz = int(sizeof(T));
    mss::SeqMaps maps;
    std::memset(&maps, 0, sizeof(maps));
    const int64_t rows = p.batch * p.dim;
    constexpr int br = mss::SeqLayout<T, N>::kRows;
    if (!encode_rows(&maps.u, p.u, rows, p.seqlen, esz, br) ||
        !encode_rows(&maps.delta, p.delta, rows, p.seqlen, esz, br) ||
        (p.z && !encode_rows(&maps.z, p.z, rows, p.seqlen, esz, br)) ||
        !encode_bc(&maps.B, p.B, p.batch, N, p.seqlen, esz) || !encode_bc(&maps.C, p.C, p.batch, N, p.seqlen, esz))
        return MSS_ERR_CUDA;
    p.n_seg = 1;
    p.seg_len = p.seqlen;
    p.agg = nullptr;
    if (!(flags & (MSS_FLAG_NO_SPLIT | MSS_FLAG_SELFTEST_TIMEOUT)) && workspace) {
        const int n_seg = choose_segments<T, N>(p.batch, p.dim, p.seqlen);
        if (n_seg > 1 && agg_bytes(n_seg, rows, N) <= workspace_bytes) {
            p.n_seg = n_seg;
            p.seg_len = seg_len_for<T, N>(p.seqlen, n_seg);
            p.agg = static_cast<float*>(workspace);
        }
    }
    if constexpr (N == 8 || N == 16) {
        // one pass without the convolution, the zero-order hold or stored
        // states: four lanes per channel, twice the warps of the pair kernel.
        // fp32 io always; bf16 io only on small grids, where the doubled warps
        // outweigh its extra shuffles and selects (measured on B200: 0.78x the
        // pair kernel's time at 128 and 256 units of 16 channels, 1.05x at
        // 512, 1.27x at 1024)
        const int64_t units = p.batch * ((p.dim + br - 1) / br);
        if (p.n_seg == 1 && p.conv_width == 0 && !p.zoh && !p.ckpt && !(flags & MSS_FLAG_PAIR_LANES) &&
            (sizeof(T) == 4 || units <= kFourLaneBf16MaxUnits))
            return launch_seq4<T, N>(maps, p, flags, stream);
    }
    return p.conv_width > 0 ? launch_seq_conv<T, N, true>(maps, p, flags, stream)
                            : launch_seq_conv<T, N, false>(maps, p, flags, stream);
}

template <typename T, int N>
int launch_forward(mss::ScanParams p, unsigned flags, void* workspace, int64_t workspace_bytes,
                   cudaStream_t stream) {
    if constexpr (N == 4 || N == 8 || N == 16) {
        if (seq_eligible(p, N, int(sizeof(T)), flags)) {
            p.selftest_wait_ns = (flags & MSS_FLAG_SELFTEST_TIMEOUT) ? 1000000ull : 0ull;
            return launch_seq<T, N>(p, flags, workspace, workspace_bytes, stream);
        }
    }
    if (flags & MSS_FLAG_SELFTEST_TIMEOUT) return MSS_ERR_FLAGS;  // only the tiled kernel has the self-test
    return launch_simple<T, N>(p, stream);
}

// The forward pass that also stores the backward pass's group-start states
// (mss_scan_fwd_save): the tiled kernel only, whose full pass writes them.
template <typename T, int N>
int launch_forward_save(mss::ScanParams p, unsigned flags, void* workspace, int64_t workspace_bytes, float* states,
                        cudaStream_t stream) {
    if constexpr (N == 4 || N == 8 || N == 16) {
        if (seq_eligible(p, N, int(sizeof(T)), flags)) {
            p.selftest_wait_ns = (flags & MSS_FLAG_SELFTEST_TIMEOUT) ? 1000000ull : 0ull;
            p.ckpt = states;
            return launch_seq<T, N>(p, flags, workspace, workspace_bytes, stream);
        }
    }
    return MSS_ERR_PATH;
}

template <typename T, int N>
int64_t forward_workspace_bytes(int64_t batch, int64_t dim, int64_t seqlen) {
    if constexpr (N == 4 || N == 8 || N == 16)
        return agg_bytes(choose_segments<T, N>(batch, dim, seqlen), batch * dim, N);
    return 0;
}

#define MSS_INSTANTIATE_FORWARD(T, N)                                                                     \
    template int launch_forward<T, N>(mss::ScanParams, unsigned, void*, int64_t, cudaStream_t);          \
    template int launch_forward_save<T, N>(mss::ScanParams, unsigned, void*, int64_t, float*, cudaStream_t); \
    template int64_t forward_workspace_bytes<T, N>(int64_t, int64_t, int64_t);

// The convolution variants of (T, N) live in another translation unit.
#define MSS_EXTERN_SEQ_CONV(T, N) \
    extern template int launch_seq_conv<T, N, true>(const mss::SeqMaps&, const mss::ScanParams&, unsigned, cudaStream_t);
#define MSS_INSTANTIATE_SEQ_CONV(T, N) \
    template int launch_seq_conv<T, N, true>(const mss::SeqMaps&, const mss::ScanParams&, unsigned, cudaStream_t);

}  // namespace mss_host
