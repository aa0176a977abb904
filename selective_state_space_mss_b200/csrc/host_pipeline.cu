// host_pipeline.cu -- the forward pass over inputs and outputs in host
// memory (mss_scan_fwd_host).
//
// The rows are cut into pieces: parts of one batch row when a row holds more
// than the piece target, else groups of whole batch rows.  Each piece is
// staged through one of up to kSlots slots of a caller-owned device workspace: its inputs are copied in
// on one stream, the forward kernel runs on one of two compute streams, and
// y and the final state are copied out on a third stream.  Events order the
// three stages of a piece and hand a slot to the next piece only once its
// outputs have left, so the host-to-device copy of piece i + 1, the kernel
// of piece i and the device-to-host copy of piece i - 1 run at the same time.
// PCIe moves the two directions concurrently, so the call takes about as
// long as the larger direction, instead of the sum of both directions plus
// the kernels.
#include <algorithm>
#include <mutex>

#include <cuda_runtime.h>

#include "host_common.h"

namespace mss_host {
namespace {

constexpr int kSlots = 3;
constexpr int64_t kPieceInputBytes = int64_t(64) << 20;  // about this much of u, delta, z per piece
constexpr int64_t kAlign = 256;
constexpr unsigned kHostFlags = MSS_FLAG_GENERAL_A | MSS_FLAG_SIMPLE | MSS_FLAG_NO_SPLIT | MSS_FLAG_ZOH_INPUT;

inline int64_t round_up(int64_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Piece size and workspace layout for one call's sizes and optional inputs.
// A batch row larger than the piece target is cut into pieces of whole
// 16-channel groups; smaller rows are grouped, several whole batch rows to a
// piece (their rows are contiguous, so a piece is still one copy per tensor).
struct Plan {
    int64_t piece_batches = 0;  // batch rows per piece (1 when rows are cut)
    int64_t piece_dim = 0;      // channels per piece and batch row (dim when rows are whole)
    int64_t row_pieces = 0;     // pieces per batch row (1 when rows are whole)
    int64_t n_pieces = 0;
    int slots = 0;              // staging slots in the workspace (at most kSlots)
    // parameter block: A, D, bias, B, C
    int64_t off_A = 0, off_D = 0, off_bias = 0, off_B = 0, off_C = 0;
    // one slot: u, delta, z, y, initial state, last state
    int64_t slot0 = 0, slot_bytes = 0;
    int64_t off_u = 0, off_delta = 0, off_z = 0, off_y = 0, off_h0 = 0, off_last = 0;
    int64_t total = 0;
};

Plan make_plan(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen, int64_t esz, bool gated, bool has_D,
               bool has_bias, bool has_h0, bool has_last) {
    Plan pl;
    const int64_t row_in = seqlen * esz * (gated ? 3 : 2);  // input bytes of one channel
    const int64_t batch_row_in = dim * row_in;              // of one batch row
    if (batch_row_in <= kPieceInputBytes) {
        int64_t nb = batch_row_in > 0 ? std::max<int64_t>(1, kPieceInputBytes / batch_row_in) : batch;
        nb = std::min<int64_t>(nb, batch);
        const int64_t pieces = (batch + nb - 1) / nb;
        pl.piece_batches = (batch + pieces - 1) / pieces;  // equal pieces
        pl.piece_dim = dim;
        pl.row_pieces = 1;
        pl.n_pieces = (batch + pl.piece_batches - 1) / pl.piece_batches;
    } else {
        int64_t k = (batch_row_in + kPieceInputBytes - 1) / kPieceInputBytes;
        k = std::max<int64_t>(1, std::min<int64_t>(k, (dim + 15) / 16));
        // equal pieces of whole 16-channel groups (the forward kernel's CTA)
        pl.piece_batches = 1;
        pl.piece_dim = std::min<int64_t>(dim, ((dim + k - 1) / k + 15) / 16 * 16);
        pl.row_pieces = (dim + pl.piece_dim - 1) / pl.piece_dim;
        pl.n_pieces = batch * pl.row_pieces;
    }
    pl.slots = int(std::min<int64_t>(kSlots, pl.n_pieces));
    const int64_t slot_rows = pl.piece_batches * pl.piece_dim;
    int64_t o = 0;
    pl.off_A = o;    o += round_up(dim * dstate * 4);
    pl.off_D = o;    o += has_D ? round_up(dim * 4) : 0;
    pl.off_bias = o; o += has_bias ? round_up(dim * 4) : 0;
    pl.off_B = o;    o += round_up(batch * dstate * seqlen * esz);
    pl.off_C = o;    o += round_up(batch * dstate * seqlen * esz);
    pl.slot0 = o;
    const int64_t seq = slot_rows * seqlen * esz, st = slot_rows * dstate * 4;
    int64_t s = 0;
    pl.off_u = s;     s += round_up(seq);
    pl.off_delta = s; s += round_up(seq);
    pl.off_z = s;     s += gated ? round_up(seq) : 0;
    pl.off_y = s;     s += round_up(seq);
    pl.off_h0 = s;    s += has_h0 ? round_up(st) : 0;
    pl.off_last = s;  s += has_last ? round_up(st) : 0;
    pl.slot_bytes = s;
    pl.total = pl.slot0 + pl.slots * s;
    return pl;
}

// Three streams per device (copies in, copies out, and two for kernels),
// created on first use and kept for the life of the process, and a mutex
// that keeps the enqueue of concurrent calls on one device from interleaving.
struct DeviceStreams {
    std::mutex enqueue;
    cudaStream_t h2d = nullptr, d2h = nullptr, comp[2] = {nullptr, nullptr};
    bool ready = false;
};

DeviceStreams* streams_for_current_device() {
    static std::mutex mu;
    static DeviceStreams per_dev[kMaxDevices];
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    DeviceStreams& d = per_dev[dev];
    if (!d.ready) {
        cudaStream_t* all[] = {&d.h2d, &d.d2h, &d.comp[0], &d.comp[1]};
        for (cudaStream_t* s : all)
            if (!*s && cudaStreamCreateWithFlags(s, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
        d.ready = true;
    }
    return &d;
}

// Events of one call, destroyed when the call returns (a pending event is
// released once it completes).
struct CallEvents {
    cudaEvent_t start = nullptr, end = nullptr, in[kSlots] = {}, done[kSlots] = {}, freed[kSlots] = {};
    bool ok = true;
    CallEvents() {
        cudaEvent_t* all[] = {&start, &end, &in[0], &in[1], &in[2], &done[0], &done[1], &done[2],
                              &freed[0], &freed[1], &freed[2]};
        for (cudaEvent_t* e : all)
            ok = ok && cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
    }
    ~CallEvents() {
        cudaEvent_t all[] = {start, end, in[0], in[1], in[2], done[0], done[1], done[2], freed[0], freed[1], freed[2]};
        for (cudaEvent_t e : all)
            if (e) cudaEventDestroy(e);
    }
};

// On a failure after work was queued, the caller's stream still waits for
// everything already queued on the library's streams, so that the caller
// does not release the workspace or the host buffers under copies in flight.
struct JoinOnFailure {
    DeviceStreams* ds;
    cudaStream_t caller;
    bool armed = true;
    ~JoinOnFailure() {
        if (!armed) return;
        cudaStream_t all[] = {ds->h2d, ds->d2h, ds->comp[0], ds->comp[1]};
        for (cudaStream_t h : all) {
            cudaEvent_t e;
            if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) continue;
            if (cudaEventRecord(e, h) == cudaSuccess) cudaStreamWaitEvent(caller, e, 0);
            cudaEventDestroy(e);
        }
    }
};

inline bool copy(void* dst, const void* src, int64_t bytes, cudaMemcpyKind kind, cudaStream_t s) {
    return bytes <= 0 || cudaMemcpyAsync(dst, src, size_t(bytes), kind, s) == cudaSuccess;
}

}  // namespace
}  // namespace mss_host

using namespace mss_host;

extern "C" {

int64_t mss_scan_fwd_host_workspace_size(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen, int dtype,
                                         int with_z, int with_D, int with_delta_bias, int with_initial_state,
                                         int with_last_state) {
    if (dtype != MSS_DTYPE_F32 && dtype != MSS_DTYPE_BF16) return MSS_ERR_DTYPE;
    if (batch < 0 || dim < 0 || seqlen < 0) return MSS_ERR_SHAPE;
    if (!valid_n(dstate)) return MSS_ERR_UNSUPPORTED_N;
    const int64_t esz = dtype == MSS_DTYPE_BF16 ? 2 : 4;
    int64_t rows, elems, bytes;
    if (!mul_ok(batch, dim, &rows) || !mul_ok(rows, seqlen, &elems) || !mul_ok(elems, 4 * esz, &bytes) ||
        rows > (int64_t(1) << 40))
        return MSS_ERR_SHAPE;
    if (rows == 0) return 0;
    return make_plan(batch, dim, dstate, seqlen, esz, with_z != 0, with_D != 0, with_delta_bias != 0,
                     with_initial_state != 0, with_last_state != 0)
        .total;
}

int mss_scan_fwd_host(const void* u, const void* delta, const float* A, const void* B, const void* C,
                      const float* D, const void* z, const float* delta_bias, int softplus_flag,
                      const float* initial_state, void* y, float* last_state, int64_t batch, int64_t dim,
                      int64_t dstate, int64_t seqlen, int dtype, unsigned flags, void* workspace,
                      int64_t workspace_bytes, void* stream) {
    if (dtype != MSS_DTYPE_F32 && dtype != MSS_DTYPE_BF16) return MSS_ERR_DTYPE;
    if (flags & ~kHostFlags) return MSS_ERR_FLAGS;
    if (batch < 0 || dim < 0 || seqlen < 0 || workspace_bytes < 0) return MSS_ERR_SHAPE;
    if (!valid_n(dstate)) return MSS_ERR_UNSUPPORTED_N;
    const int64_t esz = dtype == MSS_DTYPE_BF16 ? 2 : 4;
    int64_t rows, seq_elems, seq_bytes, bc_bytes, st_bytes;
    if (!mul_ok(batch, dim, &rows) || !mul_ok(rows, seqlen, &seq_elems) || !mul_ok(seq_elems, 4 * esz, &seq_bytes) ||
        !mul_ok(batch * dstate, seqlen * esz, &bc_bytes) || !mul_ok(rows, dstate * 4, &st_bytes) ||
        rows > (int64_t(1) << 40))
        return MSS_ERR_SHAPE;
    seq_bytes /= 4;  // one [batch][dim][seqlen] tensor (checked with room for four)
    if (rows == 0) return MSS_OK;
    if (!A || (seqlen > 0 && (!u || !delta || !B || !C || !y))) return MSS_ERR_NULL;
    if (!workspace) return MSS_ERR_NULL;
    const void* io[] = {u, delta, B, C, z, y};
    for (const void* p : io)
        if (p && !aligned(p, size_t(esz))) return MSS_ERR_ALIGN;
    const void* fp[] = {A, D, delta_bias, last_state, initial_state};
    for (const void* p : fp)
        if (p && !aligned(p, 4)) return MSS_ERR_ALIGN;
    if (!aligned(workspace, kAlign)) return MSS_ERR_ALIGN;
    // host outputs must not overlap host inputs or each other
    struct Range { const void* p; int64_t n; };
    const Range outs[] = {{y, seq_bytes}, {last_state, st_bytes}};
    const Range ins[] = {{u, seq_bytes}, {delta, seq_bytes}, {z, seq_bytes}, {B, bc_bytes}, {C, bc_bytes},
                         {A, dim * dstate * 4}, {D, dim * 4}, {delta_bias, dim * 4}, {initial_state, st_bytes}};
    for (const Range& o : outs)
        for (const Range& i : ins)
            if (overlaps(o.p, o.n, i.p, i.n)) return MSS_ERR_ALIAS;
    if (overlaps(y, seq_bytes, last_state, st_bytes)) return MSS_ERR_ALIAS;
    const Plan pl = make_plan(batch, dim, dstate, seqlen, esz, z != nullptr, D != nullptr, delta_bias != nullptr,
                              initial_state != nullptr, last_state != nullptr);
    if (workspace_bytes < pl.total) return MSS_ERR_WORKSPACE;

    DeviceStreams* ds = streams_for_current_device();
    if (!ds) return MSS_ERR_CUDA;
    std::lock_guard<std::mutex> lock(ds->enqueue);
    CallEvents ev;
    if (!ev.ok) return MSS_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    JoinOnFailure join{ds, s};
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const cudaMemcpyKind H2D = cudaMemcpyHostToDevice, D2H = cudaMemcpyDeviceToHost;

    // everything waits for the work already on the caller's stream (an
    // earlier call on the same workspace, say)
    if (cudaEventRecord(ev.start, s) != cudaSuccess || cudaStreamWaitEvent(ds->h2d, ev.start, 0) != cudaSuccess ||
        cudaStreamWaitEvent(ds->d2h, ev.start, 0) != cudaSuccess)
        return MSS_ERR_CUDA;
    for (cudaStream_t c : ds->comp)
        if (cudaStreamWaitEvent(c, ev.start, 0) != cudaSuccess) return MSS_ERR_CUDA;
    // the parameters and every batch's B and C, once (ahead of the first piece on the same stream)
    float* A_d = reinterpret_cast<float*>(ws + pl.off_A);
    float* D_d = D ? reinterpret_cast<float*>(ws + pl.off_D) : nullptr;
    float* bias_d = delta_bias ? reinterpret_cast<float*>(ws + pl.off_bias) : nullptr;
    uint8_t* B_d = ws + pl.off_B;
    uint8_t* C_d = ws + pl.off_C;
    if (!copy(A_d, A, dim * dstate * 4, H2D, ds->h2d) || (D && !copy(D_d, D, dim * 4, H2D, ds->h2d)) ||
        (delta_bias && !copy(bias_d, delta_bias, dim * 4, H2D, ds->h2d)) ||
        (seqlen > 0 && (!copy(B_d, B, bc_bytes, H2D, ds->h2d) || !copy(C_d, C, bc_bytes, H2D, ds->h2d))))
        return MSS_ERR_CUDA;

    for (int64_t i = 0; i < pl.n_pieces; ++i) {
        const int slot = int(i % pl.slots);
        // piece i: batch rows [b, b + nb), channels [d0, d0 + nd) of each
        const int64_t b = pl.row_pieces > 1 ? i / pl.row_pieces : i * pl.piece_batches;
        const int64_t nb = std::min<int64_t>(pl.piece_batches, batch - b);
        const int64_t d0 = pl.row_pieces > 1 ? (i % pl.row_pieces) * pl.piece_dim : 0;
        const int64_t nd = std::min<int64_t>(pl.piece_dim, dim - d0);
        const int64_t row0 = b * dim + d0, rows_n = nb * nd;  // contiguous rows (nb > 1 only with nd = dim)
        const int64_t seq_off = row0 * seqlen * esz, seq_n = rows_n * seqlen * esz;
        const int64_t st_off = row0 * dstate * 4, st_n = rows_n * dstate * 4;
        uint8_t* sl = ws + pl.slot0 + slot * pl.slot_bytes;
        uint8_t* u_d = sl + pl.off_u;
        uint8_t* delta_d = sl + pl.off_delta;
        uint8_t* z_d = z ? sl + pl.off_z : nullptr;
        uint8_t* y_d = sl + pl.off_y;
        float* h0_d = initial_state ? reinterpret_cast<float*>(sl + pl.off_h0) : nullptr;
        float* last_d = last_state ? reinterpret_cast<float*>(sl + pl.off_last) : nullptr;
        // in: once the slot's previous piece has left
        if (i >= pl.slots && cudaStreamWaitEvent(ds->h2d, ev.freed[slot], 0) != cudaSuccess) return MSS_ERR_CUDA;
        if (seqlen > 0 &&
            (!copy(u_d, static_cast<const uint8_t*>(u) + seq_off, seq_n, H2D, ds->h2d) ||
             !copy(delta_d, static_cast<const uint8_t*>(delta) + seq_off, seq_n, H2D, ds->h2d) ||
             (z && !copy(z_d, static_cast<const uint8_t*>(z) + seq_off, seq_n, H2D, ds->h2d))))
            return MSS_ERR_CUDA;
        if (initial_state && !copy(h0_d, reinterpret_cast<const uint8_t*>(initial_state) + st_off, st_n, H2D, ds->h2d))
            return MSS_ERR_CUDA;
        if (cudaEventRecord(ev.in[slot], ds->h2d) != cudaSuccess) return MSS_ERR_CUDA;
        // the kernel, on alternating streams so that small pieces overlap
        cudaStream_t cs = ds->comp[i & 1];
        if (cudaStreamWaitEvent(cs, ev.in[slot], 0) != cudaSuccess) return MSS_ERR_CUDA;
        const int rc = mss_scan_fwd_ex2(
            seqlen > 0 ? u_d : nullptr, seqlen > 0 ? delta_d : nullptr, A_d + d0 * dstate,
            seqlen > 0 ? B_d + b * dstate * seqlen * esz : nullptr, seqlen > 0 ? C_d + b * dstate * seqlen * esz : nullptr,
            D_d ? D_d + d0 : nullptr, z_d, bias_d ? bias_d + d0 : nullptr, softplus_flag, h0_d,
            seqlen > 0 ? y_d : nullptr, last_d, nb, nd, dstate, seqlen, dtype, flags | MSS_FLAG_NO_SPLIT, nullptr, 0,
            cs);
        if (rc != MSS_OK) return rc;
        if (cudaEventRecord(ev.done[slot], cs) != cudaSuccess) return MSS_ERR_CUDA;
        // out
        if (cudaStreamWaitEvent(ds->d2h, ev.done[slot], 0) != cudaSuccess) return MSS_ERR_CUDA;
        if (seqlen > 0 && !copy(static_cast<uint8_t*>(y) + seq_off, y_d, seq_n, D2H, ds->d2h)) return MSS_ERR_CUDA;
        if (last_state && !copy(reinterpret_cast<uint8_t*>(last_state) + st_off, last_d, st_n, D2H, ds->d2h))
            return MSS_ERR_CUDA;
        if (cudaEventRecord(ev.freed[slot], ds->d2h) != cudaSuccess) return MSS_ERR_CUDA;
    }
    // the caller's stream resumes once the last output has left (the copies
    // out run in order on one stream, and each follows its piece's kernel)
    if (cudaEventRecord(ev.end, ds->d2h) != cudaSuccess || cudaStreamWaitEvent(s, ev.end, 0) != cudaSuccess)
        return MSS_ERR_CUDA;
    join.armed = false;
    return MSS_OK;
}

}  // extern "C"
