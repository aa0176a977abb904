// backward.cuh -- host-side launch of the backward pass (included by the
// bwd_*.cu translation units): zeroing of the summed gradients, the
// checkpoint pass (the forward kernel's fold launch recording the state at
// every group start), then the backward kernel; or the scalar reference
// kernel for the shapes the throughput kernels do not take.
#pragma once

#include "forward.cuh"
#include "scan_bwd.cuh"
#include "scan_bwd_simple.cuh"

namespace mss_host {

// Workspace bytes of the backward pass: the checkpoints of the throughput
// kernels (one state per group of 16 bytes of a row: 8 bf16 or 4 fp32 tokens)
// when the sizes can take them (the same test as the launch, for
// 16-byte-aligned tensors), else those of the scalar kernel (one per 16
// tokens).
template <typename T, int N>
int64_t backward_workspace_bytes(int64_t batch, int64_t dim, int64_t seqlen, unsigned flags) {
    const int64_t rows = batch * dim;
    if (rows == 0 || seqlen == 0) return 0;
    const bool fast = seq_shape_ok(batch, dim, seqlen, N, int(sizeof(T)), flags);
    const int64_t every = fast ? mss::SeqLayout<T, (N >= 4 ? N : 4)>::kVec : mss::kBwdSimpleChunk;
    return rows * ((seqlen + every - 1) / every) * N * 4;
}

// [rows, seqlen / V * N] fp32 view of the group-start states, box = 16 rows x
// the chunk's groups.
template <typename T, int N>
bool encode_ckpt(CUtensorMap* m, const void* base, int64_t rows, int64_t seqlen) {
    using Ly = mss::BwdLayout<T, N>;
    auto enc = encode_tiled_fn();
    if (!enc) return false;
    const int64_t width = seqlen / Ly::kVec * N;
    const cuuint64_t dims[2] = {cuuint64_t(width), cuuint64_t(rows)};
    const cuuint64_t strides[1] = {cuuint64_t(width * 4)};
    const cuuint32_t box[2] = {cuuint32_t(Ly::kGroups * N), cuuint32_t(Ly::kRows)};
    const cuuint32_t estr[2] = {1u, 1u};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T, int N, bool kGate, bool kSoftplus, bool kZoh>
int launch_bwd_variant(const mss::BwdMaps& maps, const mss::BwdParams& p, unsigned flags, cudaStream_t s) {
    using Ly = mss::BwdLayout<T, N>;
    auto kern = mss::scan_bwd_kernel<T, N, kGate, kSoftplus, kZoh>;
    if (Ly::kSmemBytes > 48 * 1024 &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Ly::kSmemBytes) != cudaSuccess)
        return MSS_ERR_CUDA;
    const dim3 grid(unsigned((p.dim + Ly::kRows - 1) / Ly::kRows), unsigned(p.batch));
    kern<<<grid, 32, Ly::kSmemBytes, s>>>(maps, p, (flags & MSS_FLAG_GENERAL_A) ? 0 : 1);
    return launch_status();
}

template <typename T, int N, bool kZoh>
int launch_bwd_fast(mss::ScanParams fp, const mss::BwdParams& bp, unsigned flags, cudaStream_t s) {
    const bool saved = (flags & MSS_FLAG_SAVED_STATES) != 0;
    constexpr int esz = int(sizeof(T));
    const int64_t rows = fp.batch * fp.dim;
    constexpr int br = mss::SeqLayout<T, N>::kRows;
    // checkpoint pass, unless the forward pass saved the states
    if (!saved) {
        mss::SeqMaps fm;
        std::memset(&fm, 0, sizeof(fm));
        if (!encode_rows(&fm.u, fp.u, rows, fp.seqlen, esz, br) ||
            !encode_rows(&fm.delta, fp.delta, rows, fp.seqlen, esz, br) ||
            !encode_bc(&fm.B, fp.B, fp.batch, N, fp.seqlen, esz) || !encode_bc(&fm.C, fp.C, fp.batch, N, fp.seqlen, esz))
            return MSS_ERR_CUDA;
        fp.n_seg = 1;
        fp.seg_len = fp.seqlen;
        fp.agg = nullptr;
        fp.y = nullptr;
        fp.last_state = nullptr;
        fp.z = nullptr;
        const int rc = fp.softplus ? launch_seq_variant<T, N, false, true, true, kZoh, false>(fm, fp, flags, 1, s)
                                   : launch_seq_variant<T, N, false, false, true, kZoh, false>(fm, fp, flags, 1, s);
        if (rc != MSS_OK) return rc;
    }
    // backward
    mss::BwdMaps bm;
    std::memset(&bm, 0, sizeof(bm));
    if (!encode_rows(&bm.u, bp.u, rows, bp.seqlen, esz, br) || !encode_rows(&bm.delta, bp.delta, rows, bp.seqlen, esz, br) ||
        (bp.z && !encode_rows(&bm.z, bp.z, rows, bp.seqlen, esz, br)) ||
        !encode_rows(&bm.dy, bp.dy, rows, bp.seqlen, esz, br) ||
        !encode_bc(&bm.B, bp.B, bp.batch, N, bp.seqlen, esz) || !encode_bc(&bm.C, bp.C, bp.batch, N, bp.seqlen, esz) ||
        !encode_ckpt<T, N>(&bm.ck, bp.ckpt, rows, bp.seqlen))
        return MSS_ERR_CUDA;
    if (bp.z)
        return bp.softplus ? launch_bwd_variant<T, N, true, true, kZoh>(bm, bp, flags, s)
                           : launch_bwd_variant<T, N, true, false, kZoh>(bm, bp, flags, s);
    return bp.softplus ? launch_bwd_variant<T, N, false, true, kZoh>(bm, bp, flags, s)
                       : launch_bwd_variant<T, N, false, false, kZoh>(bm, bp, flags, s);
}

// fp: the forward arguments (initial_state, zoh, softplus, error word set);
// bp: the backward arguments (ckpt filled in here).
template <typename T, int N>
int launch_backward(mss::ScanParams fp, mss::BwdParams bp, unsigned flags, void* workspace, int64_t workspace_bytes,
                    cudaStream_t s) {
    const int64_t rows = bp.batch * bp.dim, L = bp.seqlen;
    // the summed gradients are accumulated with atomics
    const size_t bc_bytes = size_t(bp.batch) * N * size_t(L) * 4;
    if (cudaMemsetAsync(bp.dA, 0, size_t(bp.dim) * N * 4, s) != cudaSuccess ||
        cudaMemsetAsync(bp.dB, 0, bc_bytes, s) != cudaSuccess || cudaMemsetAsync(bp.dC, 0, bc_bytes, s) != cudaSuccess ||
        (bp.dD && cudaMemsetAsync(bp.dD, 0, size_t(bp.dim) * 4, s) != cudaSuccess) ||
        (bp.dbias && cudaMemsetAsync(bp.dbias, 0, size_t(bp.dim) * 4, s) != cudaSuccess))
        return MSS_ERR_CUDA;
    if constexpr (N == 4 || N == 8 || N == 16) {
        const void* v16[] = {bp.dy, bp.du, bp.ddelta, bp.dz, bp.dB, bp.dC};
        bool fast = seq_eligible(fp, N, int(sizeof(T)), flags);
        for (const void* q : v16)
            if (q && !aligned(q, 16)) fast = false;
        if (fast) {
            const int64_t need = backward_workspace_bytes<T, N>(bp.batch, bp.dim, L, flags);
            if (!workspace || need > workspace_bytes || !aligned(workspace, 16)) return MSS_ERR_WORKSPACE;
            bp.ckpt = static_cast<const float*>(workspace);
            fp.ckpt = static_cast<float*>(workspace);
            return fp.zoh ? launch_bwd_fast<T, N, true>(fp, bp, flags, s) : launch_bwd_fast<T, N, false>(fp, bp, flags, s);
        }
    }
    // saved states are in the tiled kernels' layout
    if (flags & MSS_FLAG_SAVED_STATES) return MSS_ERR_PATH;
    const int64_t need = rows * ((L + mss::kBwdSimpleChunk - 1) / mss::kBwdSimpleChunk) * N * 4;
    if (!workspace || need > workspace_bytes || !aligned(workspace, 4)) return MSS_ERR_WORKSPACE;
    const int64_t blocks = (rows + 127) / 128;
    if (blocks > 0x7fffffffLL) return MSS_ERR_SHAPE;
    mss::scan_bwd_simple_kernel<T, N><<<dim3(unsigned(blocks)), 128, 0, s>>>(bp, fp.initial_state, fp.zoh,
                                                                            static_cast<float*>(workspace));
    return launch_status();
}

#define MSS_INSTANTIATE_BACKWARD(T, N)                                                                            \
    template int launch_backward<T, N>(mss::ScanParams, mss::BwdParams, unsigned, void*, int64_t, cudaStream_t); \
    template int64_t backward_workspace_bytes<T, N>(int64_t, int64_t, int64_t, unsigned);

}  // namespace mss_host
