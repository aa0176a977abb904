// mss_api.cu -- the C ABI of libmss.so (declared in include/mss.h): argument
// checks on the host, kernel choice, launches.  No allocation, no host
// synchronisation on the forward and decode paths.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <type_traits>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "../../include/mss.h"
#include "mss_device.cuh"
#include "mss_params.h"
#include "scan_seq.cuh"
#include "scan_simple.cuh"
#include "state_update.cuh"
#include "state_update_tma.cuh"

namespace {

using mss::bf16_t;

inline bool mul_ok(int64_t a, int64_t b, int64_t* out) { return !__builtin_mul_overflow(a, b, out); }

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline bool valid_n(int64_t n) { return n == 1 || n == 2 || n == 4 || n == 8 || n == 16; }

// [p, p + bytes) and [q, q + qbytes) overlap (null or empty ranges never do)
inline bool overlaps(const void* p, int64_t bytes, const void* q, int64_t qbytes) {
    if (!p || !q || bytes <= 0 || qbytes <= 0) return false;
    const uintptr_t a = reinterpret_cast<uintptr_t>(p), b = reinterpret_cast<uintptr_t>(q);
    return a < b + uint64_t(qbytes) && b < a + uint64_t(bytes);
}

// Dispatch on N: calls f(std::integral_constant<int, N>).
template <typename F>
int with_n(int64_t n, F&& f) {
    switch (n) {
        case 1: return f(std::integral_constant<int, 1>{});
        case 2: return f(std::integral_constant<int, 2>{});
        case 4: return f(std::integral_constant<int, 4>{});
        case 8: return f(std::integral_constant<int, 8>{});
        case 16: return f(std::integral_constant<int, 16>{});
        default: return MSS_ERR_UNSUPPORTED_N;
    }
}

inline int launch_status() { return cudaGetLastError() == cudaSuccess ? MSS_OK : MSS_ERR_CUDA; }

// cuTensorMapEncodeTiled, resolved once through the runtime so that the
// library does not link the driver library itself.
PFN_cuTensorMapEncodeTiled_v12000 encode_tiled_fn() {
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
bool encode_rows(CUtensorMap* m, const void* base, int64_t rows, int64_t L, int esz, int box_rows) {
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
bool encode_bc(CUtensorMap* m, const void* base, int64_t batch, int64_t N, int64_t L, int esz) {
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

// The throughput kernel's requirements; otherwise the scalar kernel runs.
bool seq_eligible(const mss::ScanParams& p, int64_t N, int esz, unsigned flags) {
    if (flags & MSS_FLAG_SIMPLE) return false;
    if (N != 4 && N != 8 && N != 16) return false;
    if ((p.seqlen * esz) % 16 != 0) return false;
    if (p.batch * p.dim >= (int64_t(1) << 31) || p.seqlen >= (int64_t(1) << 31)) return false;
    if ((p.dim + 15) / 16 > 0x7fffffffLL || p.batch > 65535) return false;
    const void* v[] = {p.u, p.delta, p.z, p.B, p.C, p.y};
    for (const void* q : v)
        if (q && !aligned(q, 16)) return false;
    return true;
}

template <typename T, int N, bool kGate, bool kSoftplus, bool kFold, bool kZoh>
int launch_seq_variant(const mss::SeqMaps& maps, const mss::ScanParams& p, unsigned flags, int segs,
                       cudaStream_t stream) {
    auto kern = mss::scan_fwd_seq_kernel<T, N, kGate, kSoftplus, kFold, kZoh>;
    const int smem = mss::SeqLayout<T, N>::kSmemBytes;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return MSS_ERR_CUDA;
    constexpr int rows = mss::SeqLayout<T, N>::kRows;
    const dim3 grid(unsigned((p.dim + rows - 1) / rows), unsigned(p.batch), unsigned(segs));
    kern<<<grid, 32, smem, stream>>>(maps, p, (flags & MSS_FLAG_GENERAL_A) ? 0 : 1);
    return launch_status();
}

// Sequence split for workloads with too few channels to occupy the GPU:
// segments per sequence so that the full pass has about two warps per
// scheduler without exceeding one wave.  1 = no split.
template <typename T, int N>
int choose_segments(int64_t batch, int64_t dim, int64_t seqlen) {
    using Ly = mss::SeqLayout<T, N>;
    int dev = 0, sms = 0, occ = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 1;
    auto kern = mss::scan_fwd_seq_kernel<T, N, true, true, false, false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Ly::kSmemBytes) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, 32, Ly::kSmemBytes) != cudaSuccess || occ < 1)
        return 1;
    const int64_t ctas = batch * ((dim + Ly::kRows - 1) / Ly::kRows);
    const int64_t slots = int64_t(occ) * sms;
    const int64_t target = 2 * 4 * int64_t(sms);  // two warps per scheduler
    const int64_t n_chunks = (seqlen + Ly::kChunk - 1) / Ly::kChunk;
    int64_t n = std::min<int64_t>(slots / ctas, (target + ctas - 1) / ctas);
    n = std::min<int64_t>(std::min<int64_t>(n, n_chunks), 64);
    if (n < 2) return 1;
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

// Resident CTAs of the bulk-staged decode kernel on the current device
// (SMs x CTAs per SM), looked up once per device; 0 if the query fails.
template <typename T, int N>
int decode_tma_slots() {
    constexpr int kMaxDev = 64;
    static std::mutex mu;
    static int slots[kMaxDev] = {};
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return 0;
    std::lock_guard<std::mutex> lock(mu);
    if (slots[dev] == 0) {
        int sms = 0, occ = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, mss::state_update_tma_kernel<T, N>,
                                                          mss::DecodeTile<T, N>::kThreads,
                                                          mss::DecodeTile<T, N>::kSmemBytes) != cudaSuccess ||
            occ < 1)
            return 0;
        slots[dev] = sms * occ;
    }
    return slots[dev];
}

constexpr unsigned kScanFlags = MSS_FLAG_GENERAL_A | MSS_FLAG_SIMPLE | MSS_FLAG_NO_SPLIT | MSS_FLAG_ZOH_INPUT;

int64_t agg_bytes(int n_seg, int64_t rows, int64_t N) { return n_seg > 1 ? int64_t(n_seg - 1) * 2 * rows * N * 4 : 0; }

// The fold pass (split sequences only), then the full pass.
template <typename T, int N, bool kZoh>
int launch_seq_passes(const mss::SeqMaps& maps, const mss::ScanParams& p, unsigned flags, cudaStream_t stream) {
    if (p.n_seg > 1) {
        // first pass: each segment but the last folds to its aggregates
        const int rc = p.softplus
                           ? launch_seq_variant<T, N, false, true, true, kZoh>(maps, p, flags, p.n_seg - 1, stream)
                           : launch_seq_variant<T, N, false, false, true, kZoh>(maps, p, flags, p.n_seg - 1, stream);
        if (rc != MSS_OK) return rc;
    }
    if (p.z)
        return p.softplus ? launch_seq_variant<T, N, true, true, false, kZoh>(maps, p, flags, p.n_seg, stream)
                          : launch_seq_variant<T, N, true, false, false, kZoh>(maps, p, flags, p.n_seg, stream);
    return p.softplus ? launch_seq_variant<T, N, false, true, false, kZoh>(maps, p, flags, p.n_seg, stream)
                      : launch_seq_variant<T, N, false, false, false, kZoh>(maps, p, flags, p.n_seg, stream);
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
    if (!(flags & MSS_FLAG_NO_SPLIT) && workspace) {
        const int n_seg = choose_segments<T, N>(p.batch, p.dim, p.seqlen);
        if (n_seg > 1 && agg_bytes(n_seg, rows, N) <= workspace_bytes) {
            p.n_seg = n_seg;
            p.seg_len = seg_len_for<T, N>(p.seqlen, n_seg);
            p.agg = static_cast<float*>(workspace);
        }
    }
    return p.zoh ? launch_seq_passes<T, N, true>(maps, p, flags, stream)
                 : launch_seq_passes<T, N, false>(maps, p, flags, stream);
}

template <typename T, int N>
int launch_scan(const mss::ScanParams& p, unsigned flags, void* workspace, int64_t workspace_bytes,
                cudaStream_t stream) {
    if constexpr (N == 4 || N == 8 || N == 16) {
        if (seq_eligible(p, N, int(sizeof(T)), flags)) return launch_seq<T, N>(p, flags, workspace, workspace_bytes, stream);
    }
    return launch_simple<T, N>(p, stream);
}

}  // namespace

extern "C" {

int mss_version(void) { return MSS_VERSION; }

const char* mss_strerror(int code) {
    switch (code) {
        case MSS_OK: return "success";
        case MSS_ERR_NULL: return "a required pointer is NULL";
        case MSS_ERR_SHAPE: return "a size is negative or a size product overflows";
        case MSS_ERR_UNSUPPORTED_N: return "dstate must be 1, 2, 4, 8 or 16";
        case MSS_ERR_DTYPE: return "dtype must be MSS_DTYPE_F32 or MSS_DTYPE_BF16";
        case MSS_ERR_ALIGN: return "a pointer is not aligned to its element size";
        case MSS_ERR_CUDA: return "a CUDA call failed";
        case MSS_ERR_DEVICE_TIMEOUT: return "a bounded wait inside a kernel gave up";
        case MSS_ERR_FLAGS: return "unknown bits in flags";
        case MSS_ERR_ALIAS: return "an output overlaps an input";
        case MSS_ERR_SCRATCH: return "the sequence split needs more than the library's fixed scratch holds";
        default: return "unknown status code";
    }
}

int mss_scan_fwd_ex2(const void* u, const void* delta, const float* A, const void* B,
                     const void* C, const float* D, const void* z, const float* delta_bias,
                     int softplus_flag, const float* initial_state, void* y, float* last_state,
                     int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                     int dtype, unsigned flags, void* workspace, int64_t workspace_bytes, void* stream) {
    if (dtype != MSS_DTYPE_F32 && dtype != MSS_DTYPE_BF16) return MSS_ERR_DTYPE;
    if (flags & ~kScanFlags) return MSS_ERR_FLAGS;
    if (batch < 0 || dim < 0 || seqlen < 0 || workspace_bytes < 0) return MSS_ERR_SHAPE;
    if (!valid_n(dstate)) return MSS_ERR_UNSUPPORTED_N;
    const int64_t esz = dtype == MSS_DTYPE_BF16 ? 2 : 4;
    int64_t rows, seq_elems, seq_bytes, bc_elems, bc_bytes, st_elems, st_bytes;
    if (!mul_ok(batch, dim, &rows) || !mul_ok(rows, seqlen, &seq_elems) ||
        !mul_ok(seq_elems, esz, &seq_bytes) || !mul_ok(batch * dstate, seqlen, &bc_elems) ||
        !mul_ok(bc_elems, esz, &bc_bytes) || !mul_ok(rows, dstate, &st_elems) ||
        !mul_ok(st_elems, 4, &st_bytes) || rows > (int64_t(1) << 40))
        return MSS_ERR_SHAPE;
    if (rows == 0) return MSS_OK;
    // with no tokens the sequence tensors are empty and may be NULL
    if (!A || (seqlen > 0 && (!u || !delta || !B || !C || !y))) return MSS_ERR_NULL;
    const void* io[] = {u, delta, B, C, z, y};
    for (const void* p : io)
        if (p && !aligned(p, size_t(esz))) return MSS_ERR_ALIGN;
    const void* fp[] = {A, D, delta_bias, last_state, initial_state, workspace};
    for (const void* p : fp)
        if (p && !aligned(p, 4)) return MSS_ERR_ALIGN;
    // outputs (y, last_state, workspace) must not overlap inputs or each other
    const int64_t ws = workspace ? workspace_bytes : 0;
    struct Range { const void* p; int64_t n; };
    const Range outs[] = {{y, seq_bytes}, {last_state, st_bytes}, {workspace, ws}};
    const Range ins[] = {{u, seq_bytes}, {delta, seq_bytes}, {z, seq_bytes}, {B, bc_bytes}, {C, bc_bytes},
                         {A, dim * dstate * 4}, {D, dim * 4}, {delta_bias, dim * 4},
                         {initial_state, st_bytes}};
    for (const Range& o : outs) {
        for (const Range& i : ins)
            if (overlaps(o.p, o.n, i.p, i.n)) return MSS_ERR_ALIAS;
        for (const Range& o2 : outs)
            if (&o != &o2 && overlaps(o.p, o.n, o2.p, o2.n)) return MSS_ERR_ALIAS;
    }

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (seqlen == 0) {
        // no tokens: the final state is the starting state
        if (last_state) {
            const cudaError_t e = initial_state
                ? cudaMemcpyAsync(last_state, initial_state, size_t(st_bytes), cudaMemcpyDeviceToDevice, s)
                : cudaMemsetAsync(last_state, 0, size_t(st_bytes), s);
            if (e != cudaSuccess) return MSS_ERR_CUDA;
        }
        return MSS_OK;
    }
    mss::ScanParams p{};
    p.u = u; p.delta = delta; p.A = A; p.B = B; p.C = C; p.D = D; p.z = z; p.delta_bias = delta_bias;
    p.y = y; p.last_state = last_state; p.batch = batch; p.dim = dim; p.seqlen = seqlen;
    p.softplus = softplus_flag ? 1 : 0; p.initial_state = initial_state;
    p.agg = nullptr; p.seg_len = seqlen; p.n_seg = 1;
    p.zoh = (flags & MSS_FLAG_ZOH_INPUT) ? 1 : 0;
    return with_n(dstate, [&](auto nc) {
        constexpr int N = decltype(nc)::value;
        return dtype == MSS_DTYPE_BF16 ? launch_scan<bf16_t, N>(p, flags, workspace, ws, s)
                                       : launch_scan<float, N>(p, flags, workspace, ws, s);
    });
}

int64_t mss_scan_fwd_workspace_size(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen, int dtype,
                                    unsigned flags) {
    if (dtype != MSS_DTYPE_F32 && dtype != MSS_DTYPE_BF16) return MSS_ERR_DTYPE;
    if (flags & ~kScanFlags) return MSS_ERR_FLAGS;
    if (batch < 0 || dim < 0 || seqlen < 0) return MSS_ERR_SHAPE;
    if (!valid_n(dstate)) return MSS_ERR_UNSUPPORTED_N;
    int64_t rows;
    if (!mul_ok(batch, dim, &rows) || rows > (int64_t(1) << 40)) return MSS_ERR_SHAPE;
    const int64_t esz = dtype == MSS_DTYPE_BF16 ? 2 : 4;
    if (rows == 0 || seqlen == 0 || (flags & (MSS_FLAG_SIMPLE | MSS_FLAG_NO_SPLIT)) ||
        (dstate != 4 && dstate != 8 && dstate != 16) || (seqlen * esz) % 16 != 0)
        return 0;
    return with_n(dstate, [&](auto nc) -> int64_t {
        constexpr int N = decltype(nc)::value;
        if constexpr (N == 4 || N == 8 || N == 16) {
            const int n_seg = dtype == MSS_DTYPE_BF16 ? choose_segments<bf16_t, N>(batch, dim, seqlen)
                                                      : choose_segments<float, N>(batch, dim, seqlen);
            return agg_bytes(n_seg, rows, N);
        }
        return 0;
    });
}

int mss_scan_fwd_ex(const void* u, const void* delta, const float* A, const void* B,
                    const void* C, const float* D, const void* z, const float* delta_bias,
                    int softplus_flag, void* y, float* last_state,
                    int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                    int dtype, unsigned flags, void* stream) {
    return mss_scan_fwd_ex2(u, delta, A, B, C, D, z, delta_bias, softplus_flag, nullptr, y, last_state,
                            batch, dim, dstate, seqlen, dtype, flags, nullptr, 0, stream);
}

int mss_scan_fwd(const void* u, const void* delta, const float* A, const void* B,
                 const void* C, const float* D, const void* z, const float* delta_bias,
                 int softplus_flag, void* y, float* last_state,
                 int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                 int dtype, void* stream) {
    return mss_scan_fwd_ex2(u, delta, A, B, C, D, z, delta_bias, softplus_flag, nullptr, y, last_state,
                            batch, dim, dstate, seqlen, dtype, 0u, nullptr, 0, stream);
}

int mss_state_update(float* state, const void* u, const void* delta, const float* A,
                     const void* B, const void* C, const float* D, const void* z,
                     const float* delta_bias, int softplus_flag, void* y,
                     int64_t batch, int64_t dim, int64_t dstate, int dtype, void* stream) {
    return mss_state_update_ex(state, u, delta, A, B, C, D, z, delta_bias, softplus_flag, y,
                               batch, dim, dstate, dtype, 0u, stream);
}

int mss_state_update_ex(float* state, const void* u, const void* delta, const float* A,
                        const void* B, const void* C, const float* D, const void* z,
                        const float* delta_bias, int softplus_flag, void* y,
                        int64_t batch, int64_t dim, int64_t dstate, int dtype, unsigned flags, void* stream) {
    if (dtype != MSS_DTYPE_F32 && dtype != MSS_DTYPE_BF16) return MSS_ERR_DTYPE;
    if (flags & ~unsigned(MSS_FLAG_ZOH_INPUT)) return MSS_ERR_FLAGS;
    if (batch < 0 || dim < 0) return MSS_ERR_SHAPE;
    if (!valid_n(dstate)) return MSS_ERR_UNSUPPORTED_N;
    const int64_t esz = dtype == MSS_DTYPE_BF16 ? 2 : 4;
    int64_t rows, st_elems, st_bytes;
    if (!mul_ok(batch, dim, &rows) || !mul_ok(rows, dstate, &st_elems) ||
        !mul_ok(st_elems, 4, &st_bytes) || rows > (int64_t(1) << 40))
        return MSS_ERR_SHAPE;
    if (rows == 0) return MSS_OK;
    if (!state || !u || !delta || !A || !B || !C || !y) return MSS_ERR_NULL;
    const void* io[] = {u, delta, B, C, z, y};
    for (const void* p : io)
        if (p && !aligned(p, size_t(esz))) return MSS_ERR_ALIGN;
    const void* fp[] = {state, A, D, delta_bias};
    for (const void* p : fp)
        if (p && !aligned(p, 4)) return MSS_ERR_ALIGN;
    const int64_t io_bytes = rows * esz, bc_bytes = batch * dstate * esz;
    const void* in_io[] = {u, delta, z};
    for (const void* p : in_io)
        if (overlaps(y, io_bytes, p, io_bytes) || overlaps(state, st_bytes, p, io_bytes)) return MSS_ERR_ALIAS;
    const void* in_bc[] = {B, C};
    for (const void* p : in_bc)
        if (overlaps(y, io_bytes, p, bc_bytes) || overlaps(state, st_bytes, p, bc_bytes)) return MSS_ERR_ALIAS;
    const void* params[] = {D, delta_bias};
    for (const void* p : params)
        if (overlaps(y, io_bytes, p, dim * 4) || overlaps(state, st_bytes, p, dim * 4)) return MSS_ERR_ALIAS;
    if (overlaps(y, io_bytes, A, dim * dstate * 4) || overlaps(state, st_bytes, A, dim * dstate * 4) ||
        overlaps(y, io_bytes, state, st_bytes))
        return MSS_ERR_ALIAS;

    mss::StepParams p{state, u, delta, A, B, C, D, z, delta_bias, y, batch, dim, softplus_flag ? 1 : 0,
                      (flags & MSS_FLAG_ZOH_INPUT) ? 1 : 0, 0};
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool vec = aligned(state, 16) && aligned(A, 16);
    // bulk-staged kernel when every streamed tensor is 16-byte aligned and
    // dim is a whole number of tiles; otherwise the per-thread kernel
    const bool bulk_ok = vec && aligned(u, 16) && aligned(delta, 16) && aligned(y, 16) && (!z || aligned(z, 16));
    return with_n(dstate, [&](auto nc) {
        constexpr int N = decltype(nc)::value;
        if constexpr (N == 4 || N == 8 || N == 16) {
            if (bulk_ok) {
                auto go_tma = [&](auto tag) -> int {
                    using T = decltype(tag);
                    using Ly = mss::DecodeTile<T, N>;
                    if (dim % Ly::kRows != 0 || batch > 0x7fffffffLL) return 1;  // not handled here
                    const int64_t n_cblocks = dim / Ly::kRows;
                    const int slots = decode_tma_slots<T, N>();
                    if (slots <= 0) return int(MSS_ERR_CUDA);
                    // batch rows per channel block served by separate CTAs
                    const int64_t bsplit = std::max<int64_t>(1, std::min<int64_t>(batch, slots / n_cblocks));
                    const int64_t grid = n_cblocks * bsplit;
                    if (grid > 0x7fffffffLL) return 1;
                    mss::state_update_tma_kernel<T, N><<<dim3(unsigned(grid)), Ly::kThreads, Ly::kSmemBytes, s>>>(
                        p, int(n_cblocks), int(bsplit));
                    return launch_status();
                };
                const int rc = dtype == MSS_DTYPE_BF16 ? go_tma(bf16_t{}) : go_tma(float{});
                if (rc <= 0) return rc;  // done (MSS_OK) or failed
            }
        }
        constexpr int TPC = N < 4 ? 1 : N / 4;
        const int threads = 256;
        const int64_t blocks = ((rows - p.row0) * TPC + threads - 1) / threads;
        if (blocks > 0x7fffffffLL) return int(MSS_ERR_SHAPE);
        auto go = [&](auto kern) {
            kern<<<dim3(unsigned(blocks)), threads, 0, s>>>(p);
            return launch_status();
        };
        if (dtype == MSS_DTYPE_BF16)
            return vec ? go(mss::state_update_kernel<bf16_t, N, true>)
                       : go(mss::state_update_kernel<bf16_t, N, false>);
        return vec ? go(mss::state_update_kernel<float, N, true>)
                   : go(mss::state_update_kernel<float, N, false>);
    });
}

int mss_get_device_error(void* stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return MSS_ERR_CUDA;
    unsigned int word = 0, zero = 0;
    if (cudaMemcpyFromSymbolAsync(&word, mss::g_mss_device_error, sizeof(word), 0,
                                  cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return MSS_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MSS_ERR_CUDA;
    if (word != 0) {
        if (cudaMemcpyToSymbolAsync(mss::g_mss_device_error, &zero, sizeof(zero), 0,
                                    cudaMemcpyHostToDevice, s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return MSS_ERR_CUDA;
        return MSS_ERR_DEVICE_TIMEOUT;
    }
    return MSS_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Forward pass for callers that cannot allocate device memory.
//
// Some callers have no way to obtain device memory of their own: a plain C
// program that is only handed the input and output buffers, a plug-in whose
// host framework owns every device allocation, a serving loop that must not
// allocate once it has started.  mss_scan_fwd_noalloc gives them the sequence
// split without a workspace argument: its scratch is the fixed array below,
// part of the library image, which every GPU that loads the library holds
// until the process exits.

namespace {

constexpr int64_t kStaticScratchBytes = int64_t(4) << 20;  // 4 MiB per device
constexpr int kMaxDevices = 64;

// The scratch itself.  In host code this name is only a stand-in for the
// symbol, never a device address: kernels get the address that
// cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) float g_mss_static_scratch[kStaticScratchBytes / sizeof(float)];

// Device address of the scratch on the current device, looked up once per
// device (with that device current) and cached; nullptr on failure.
void* static_scratch_address() {
    static std::mutex mu;
    static void* addr[kMaxDevices] = {};
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_mss_static_scratch) != cudaSuccess) return nullptr;
        addr[dev] = p;
    }
    return addr[dev];
}

}  // namespace

extern "C" {

int mss_scan_fwd_noalloc(const void* u, const void* delta, const float* A, const void* B,
                         const void* C, const float* D, const void* z, const float* delta_bias,
                         int softplus_flag, const float* initial_state, void* y, float* last_state,
                         int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                         int dtype, unsigned flags, void* stream) {
    const int64_t need = mss_scan_fwd_workspace_size(batch, dim, dstate, seqlen, dtype, flags);
    if (need < 0) return int(need);
    if (need > kStaticScratchBytes) return MSS_ERR_SCRATCH;
    void* scratch = nullptr;
    if (need > 0 && !(scratch = static_scratch_address())) return MSS_ERR_CUDA;
    return mss_scan_fwd_ex2(u, delta, A, B, C, D, z, delta_bias, softplus_flag, initial_state, y, last_state,
                            batch, dim, dstate, seqlen, dtype, flags, scratch, need, stream);
}

int64_t mss_scan_fwd_noalloc_scratch_bytes(void) { return kStaticScratchBytes; }

}  // extern "C"
