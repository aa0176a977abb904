/*
 * mss.h -- C ABI of libmss.so, the B200 (sm_100a) selective scan (S6).
 *
 * The library computes, per channel d of batch row b and token t, a diagonal
 * real state-space model discretised per token:
 *
 *   Delta_t  = softplus(delta[b,d,t] + delta_bias[d])   (or without softplus)
 *   Abar_t,n = exp(Delta_t * A[d,n])                     zero-order hold
 *   h_t,n    = Abar_t,n * h_{t-1},n + Delta_t * B[b,n,t] * u[b,d,t]
 *   y[b,d,t] = (sum_n C[b,n,t] * h_t,n + D[d] * u[b,d,t]) * silu(z[b,d,t])
 *
 * with h_{-1} = 0 and silu(z) = z / (1 + e^{-z}).  Sources: the continuous
 * SSM, the zero-order-hold transition exp(Delta A) and the discrete
 * recurrence ("Mamba" paper review, section "SSM"); token-dependent B, C and
 * step ("Mamba" paper review, section "Selection Mechanism"); softplus for the
 * step ("Exercises -- State-space models (Mamba, S4)", softplus exercise);
 * the Euler input rule Bbar = Delta B, listed beside zero-order hold on the
 * "Paper: Mamba" course page (Objectives, Math & data structures); the gate
 * and skip term of the block ("Mamba" paper review, section "SSM", block
 * description; the pages print no formula for them, the form above is the
 * library's definition).
 *
 * Conventions shared by every entry point:
 *   - Every tensor pointer is a DEVICE pointer owned by the caller, C-contiguous
 *     in the layout given below (mss_scan_fwd_host alone takes HOST tensors).
 *     The library never allocates memory on the forward or decode path and
 *     never frees caller memory.
 *   - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL means
 *     the legacy default stream) and is asynchronous: a return of MSS_OK means
 *     the launch was accepted, not that it has finished.
 *   - Argument errors are detected on the host before any launch; the outputs
 *     are then left untouched.
 *   - Optional pointers: z == NULL means no gate, D == NULL means D = 0,
 *     delta_bias == NULL means bias 0, last_state == NULL means not written.
 *   - `dtype` selects the element type of u, delta, z, B, C and y:
 *     MSS_DTYPE_F32 (float) or MSS_DTYPE_BF16 (bfloat16, round-to-nearest-even
 *     on store).  A, D, delta_bias, last_state and the decode state are always
 *     float.  All arithmetic is fp32.
 *   - dstate (N) must be 1, 2, 4, 8 or 16.
 *   - Outputs must not overlap inputs (the decode state is in/out by design).
 *   - Thread safety: the library's only host state is looked up or created
 *     once per device on first use and then kept: a driver entry point,
 *     occupancy figures, and for mss_scan_fwd_host four streams.  Calls from
 *     several host threads are safe.
 */
#ifndef MSS_H
#define MSS_H

#include <stdint.h>

#if defined(__GNUC__)
#define MSS_API __attribute__((visibility("default")))
#else
#define MSS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define MSS_VERSION 10500 /* major*10000 + minor*100 + patch: 1.5.0 */

enum mss_dtype {
    MSS_DTYPE_F32 = 0,
    MSS_DTYPE_BF16 = 1
};

enum mss_status {
    MSS_OK = 0,
    MSS_ERR_NULL = -1,           /* a required pointer is NULL */
    MSS_ERR_SHAPE = -2,          /* a size is negative or out of range (conv_width), or a product overflows */
    MSS_ERR_UNSUPPORTED_N = -3,  /* dstate is not 1, 2, 4, 8 or 16 */
    MSS_ERR_DTYPE = -4,          /* dtype is not an mss_dtype */
    MSS_ERR_ALIGN = -5,          /* a pointer is not aligned to its element size */
    MSS_ERR_CUDA = -6,           /* a CUDA call failed (launch or device query) */
    MSS_ERR_DEVICE_TIMEOUT = -7, /* a bounded wait inside a kernel gave up */
    MSS_ERR_FLAGS = -8,          /* unknown bits in `flags` */
    MSS_ERR_ALIAS = -9,          /* an output overlaps an input */
    MSS_ERR_SCRATCH = -10,       /* mss_scan_fwd_noalloc: the split needs more than its fixed scratch */
    MSS_ERR_WORKSPACE = -11,     /* mss_scan_bwd: no workspace, or smaller than it needs */
    MSS_ERR_PATH = -12           /* saved states: the sizes, flags or alignments take the scalar kernels */
};

/* Flags of mss_scan_fwd_ex / mss_scan_fwd_ex2 / mss_scan_fwd_noalloc
 * (MSS_FLAG_ZOH_INPUT also of mss_state_update_ex). */
#define MSS_FLAG_GENERAL_A 0x1u /* never use the fast path for A[d,n] = (n+1)*A[d,0] */
#define MSS_FLAG_SIMPLE 0x2u    /* run the one-thread-per-channel reference kernel */
#define MSS_FLAG_NO_SPLIT 0x4u  /* never split the sequence, even with a workspace */
/* Input matrix by the exact zero-order hold instead of the Euler rule:
 * Bbar x = (exp(Delta A[d,n]) - 1) / A[d,n] * B[n] * u per state, with its
 * limit Delta * B[n] * u at A[d,n] = 0 ("Mamba" paper review, section "SSM";
 * "Paper: Mamba", Objectives).  The transition Abar = exp(Delta A) is the
 * same under both rules. */
#define MSS_FLAG_ZOH_INPUT 0x8u
/* Self-test of the kernels' bounded waits (for tests of the failure path):
 * every CTA of the tiled forward kernel (two or four lanes per channel,
 * whichever the call takes) first waits on a barrier that no copy
 * will ever complete -- none has been issued yet -- with a limit of 1 ms.  The
 * wait gives up, sets the device error word (mss_get_device_error then
 * returns MSS_ERR_DEVICE_TIMEOUT, once) and the CTA returns; y, last_state and
 * the workspace are not written.  The CUDA context stays usable and later
 * calls are unaffected.  The flag needs a call that takes the tiled kernel
 * (16-byte-aligned rows, dstate 4, 8 or 16, no MSS_FLAG_SIMPLE); otherwise the
 * call returns MSS_ERR_FLAGS and launches nothing.  The sequence is not
 * split. */
#define MSS_FLAG_SELFTEST_TIMEOUT 0x10u
/* mss_scan_bwd (and mss_scan_bwd_workspace_size): the workspace already holds
 * the states that mss_scan_fwd_save wrote for the same inputs, so the call
 * skips its checkpoint pass.  See mss_scan_fwd_save. */
#define MSS_FLAG_SAVED_STATES 0x20u
/* Forward passes: run the two-lanes-per-channel kernel where the four-lane
 * one would (N = 8 or 16, one pass over the sequence, Euler input rule, no
 * convolution; fp32 io on any grid, bf16 io when batch * ceil(dim / 16) is
 * at most 384); for testing and measurement, the results agree within the
 * io type's rounding. */
#define MSS_FLAG_PAIR_LANES 0x40u

/*
 * mss_scan_fwd -- selective-scan forward pass over whole sequences.
 *
 *   u, delta, z : [batch][dim][seqlen]  dtype     (z may be NULL)
 *   A           : [dim][dstate]         float     (negative for a stable system)
 *   B, C        : [batch][dstate][seqlen] dtype   (shared by all channels of a row)
 *   D, delta_bias: [dim]                float     (each may be NULL)
 *   softplus_flag: nonzero -> Delta = softplus(delta + bias), else delta + bias
 *   y           : [batch][dim][seqlen]  dtype     output
 *   last_state  : [batch][dim][dstate]  float     output h_{seqlen-1} (may be NULL)
 *
 * Any seqlen >= 0 works (a ragged tail is masked); seqlen == 0 writes
 * last_state = 0 and then u, delta, z, B, C and y may be NULL.  batch * dim == 0 launches nothing.  The fp32 state stays
 * on chip; only last_state is written.  Any pointer alignment that matches
 * the element size is accepted: 16-byte aligned rows take the vectorised
 * kernel, others a scalar one.
 *
 * Returns MSS_OK or a negative mss_status.
 */
MSS_API int mss_scan_fwd(const void *u, const void *delta, const float *A, const void *B,
                 const void *C, const float *D, const void *z, const float *delta_bias,
                 int softplus_flag, void *y, float *last_state,
                 int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                 int dtype, void *stream);

/* mss_scan_fwd with `flags` (MSS_FLAG_*): the same computation, with a choice
 * of kernel for testing and measurement.  flags == 0 is mss_scan_fwd. */
MSS_API int mss_scan_fwd_ex(const void *u, const void *delta, const float *A, const void *B,
                    const void *C, const float *D, const void *z, const float *delta_bias,
                    int softplus_flag, void *y, float *last_state,
                    int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                    int dtype, unsigned flags, void *stream);

/*
 * mss_scan_fwd_ex2 -- the forward pass with a starting state and an optional
 * caller-owned workspace.
 *
 *   initial_state : [batch][dim][dstate] float, the state before the first
 *                   token (NULL: zero, the pages' convention).  With it, a
 *                   sequence can be run in pieces: passing one call's
 *                   last_state as the next call's initial_state gives the
 *                   same outputs as one call over the whole sequence.  It
 *                   must not overlap last_state.
 *   workspace, workspace_bytes : device memory the call may use for a
 *                   sequence split (NULL / 0: none).  When the batch has too
 *                   few channels to occupy the GPU (long sequences), the
 *                   sequence is cut into segments that run in parallel: a
 *                   first kernel reduces every segment but the last to its
 *                   aggregate (the product of its transitions and its final
 *                   state from zero, 2 * dstate floats per channel), a second
 *                   runs all segments from their carried-in states.  The
 *                   size the call would use is mss_scan_fwd_workspace_size;
 *                   a smaller or NULL workspace disables the split.  The
 *                   library never allocates; the contents of the workspace
 *                   on return are unspecified.  Calls that share a workspace
 *                   must not overlap in time.
 *
 * Every other argument, flag and rule is that of mss_scan_fwd_ex.
 * seqlen == 0 copies initial_state (or zero) to last_state.
 */
MSS_API int mss_scan_fwd_ex2(const void *u, const void *delta, const float *A, const void *B,
                             const void *C, const float *D, const void *z, const float *delta_bias,
                             int softplus_flag, const float *initial_state, void *y, float *last_state,
                             int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                             int dtype, unsigned flags, void *workspace, int64_t workspace_bytes,
                             void *stream);

/*
 * mss_scan_fwd_save -- mss_scan_fwd_ex2 for a training step: the forward pass
 * that also stores the states mss_scan_bwd would otherwise recompute in its
 * checkpoint pass.  The pages train the model end to end and have the fused
 * kernel keep the states out of HBM except where the backward pass needs them
 * ("Mamba" paper review, section "Selection Mechanism"); the forward pass is
 * where those states are formed anyway, so storing them costs writes only.
 *
 *   every argument of mss_scan_fwd_ex2, with the same meaning, then
 *   states       : device memory of at least states_bytes =
 *                  mss_scan_bwd_workspace_size(batch, dim, dstate, seqlen,
 *                  dtype, flags) bytes, 16-byte aligned, owned by the caller:
 *                  the state at the start of every group of 16 bytes of a row
 *                  (8 bf16 or 4 fp32 tokens), written in full by the call and
 *                  read by mss_scan_bwd with MSS_FLAG_SAVED_STATES.  Its layout
 *                  is private to the library.
 *
 * Then call mss_scan_bwd with the same forward inputs, the same flags plus
 * MSS_FLAG_SAVED_STATES, and `states` as its workspace (not modified between
 * the two calls).  The call needs the tiled kernels: dstate 4, 8 or 16,
 * 16-byte-aligned rows and tensors, no MSS_FLAG_SIMPLE; otherwise it returns
 * MSS_ERR_PATH and launches nothing (use mss_scan_fwd_ex2 and mss_scan_bwd
 * without the flag).  y and last_state are those of mss_scan_fwd_ex2, bit for
 * bit.  MSS_ERR_WORKSPACE when states is NULL or too small; MSS_ERR_ALIAS when
 * it overlaps another argument; otherwise the errors of mss_scan_fwd_ex2.
 */
MSS_API int mss_scan_fwd_save(const void *u, const void *delta, const float *A, const void *B,
                              const void *C, const float *D, const void *z, const float *delta_bias,
                              int softplus_flag, const float *initial_state, void *y, float *last_state,
                              int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                              int dtype, unsigned flags, void *workspace, int64_t workspace_bytes,
                              void *states, int64_t states_bytes, void *stream);

/*
 * mss_scan_fwd_workspace_size -- bytes of workspace mss_scan_fwd_ex2 would use
 * for these sizes on the current device (0: the sequence is not split), or a
 * negative mss_status for invalid arguments.  Assumes 16-byte aligned rows.
 */
MSS_API int64_t mss_scan_fwd_workspace_size(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                                            int dtype, unsigned flags);

/*
 * mss_scan_fwd_host -- mss_scan_fwd_ex2 over inputs and outputs in HOST
 * memory: u, delta, A, B, C, D, z, delta_bias, initial_state are read from
 * the host, y and last_state written to the host, with the layouts of
 * mss_scan_fwd.  The channels are cut into pieces of whole batch rows or
 * parts of them.  Each piece is staged through a caller-owned device
 * workspace.  The library's own streams on the current device then overlap
 * the host-to-device copies of one piece, the kernel of the one before it,
 * and the device-to-host copies of the one before that.
 *
 *   workspace, workspace_bytes : device memory on the current device,
 *       256-byte aligned, at least mss_scan_fwd_host_workspace_size bytes
 *       for the same sizes and the same optional arguments (else
 *       MSS_ERR_NULL / MSS_ERR_ALIGN / MSS_ERR_WORKSPACE).  Its contents on
 *       return are unspecified.
 *   stream : the call is asynchronous on it like every other entry point.
 *       The copies wait for the work already queued on it, and work queued
 *       on it later waits for the last copy out.  The host buffers must
 *       stay valid and untouched until then.  Page-locked (pinned) host
 *       memory is needed for the copies to overlap.  Pageable memory works
 *       but is copied synchronously.
 *
 * The kernels run with MSS_FLAG_NO_SPLIT added to flags (the pieces, not a
 * sequence split, fill the GPU).  y and last_state must not overlap the host
 * inputs.  Returns MSS_OK or a negative mss_status; argument errors are
 * found before anything is queued.
 */
MSS_API int mss_scan_fwd_host(const void *u, const void *delta, const float *A, const void *B,
                              const void *C, const float *D, const void *z, const float *delta_bias,
                              int softplus_flag, const float *initial_state, void *y, float *last_state,
                              int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                              int dtype, unsigned flags, void *workspace, int64_t workspace_bytes,
                              void *stream);

/* Device workspace bytes mss_scan_fwd_host needs for these sizes, with z, D,
 * delta_bias, initial_state and last_state present (nonzero) or NULL (0);
 * 0 when batch * dim == 0, or a negative mss_status. */
MSS_API int64_t mss_scan_fwd_host_workspace_size(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                                                 int dtype, int with_z, int with_D, int with_delta_bias,
                                                 int with_initial_state, int with_last_state);

/*
 * mss_scan_fwd_conv -- the forward pass with a causal convolution and SiLU
 * in front of the scan.  The pages put "a convolution and non-linearity"
 * between the input projection and the bank of SSMs ("Mamba" paper review,
 * section "SSM", block description) and fuse the causal 1D convolution into
 * the scan kernel ("NN Lab -- Mamba"); read as a per-channel causal
 * convolution of width K followed by SiLU:
 *
 *   u[b,d,t] = silu(conv_b[d] + sum_{k<K} conv_w[d,k] * x[b,d,t-(K-1)+k])
 *
 * and u drives the scan exactly as in mss_scan_fwd_ex2 (both the input term
 * and the skip term D*u).  x is read once; u never goes to memory.
 *
 *   x             : [batch][dim][seqlen] dtype  (takes the place of u)
 *   conv_w        : [dim][K] float; tap k multiplies x_{t-(K-1)+k}
 *   conv_b        : [dim] float (NULL: no bias)
 *   conv_width    : K, 1..4 (else MSS_ERR_SHAPE)
 *   conv_state_in : [batch][dim][K-1] dtype, the K-1 inputs before the first
 *                   token, oldest first (NULL: zeros)
 *   conv_state_out: [batch][dim][K-1] dtype, written with the last K-1 inputs
 *                   of the history followed by x (NULL: not written); pass it
 *                   to mss_state_update_conv or to the next call
 *
 * The other arguments, the sequence split and the errors are those of
 * mss_scan_fwd_ex2 (the workspace size does not depend on the convolution);
 * conv_state_out must not overlap any other argument.  seqlen == 0 copies
 * conv_state_in (or zeros) to conv_state_out.
 */
MSS_API int mss_scan_fwd_conv(const void *x, const float *conv_w, const float *conv_b, int conv_width,
                      const void *conv_state_in, void *conv_state_out,
                      const void *delta, const float *A, const void *B, const void *C, const float *D,
                      const void *z, const float *delta_bias, int softplus_flag, const float *initial_state,
                      void *y, float *last_state, int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                      int dtype, unsigned flags, void *workspace, int64_t workspace_bytes, void *stream);

/*
 * mss_scan_fwd_noalloc -- mss_scan_fwd_ex2 for callers that cannot allocate
 * device memory.  The pages have no counterpart: this is an interface
 * convenience.
 *
 * Some callers have no way to get device memory of their own -- a C program
 * that is only handed its input and output buffers, a plug-in whose host
 * framework owns all device allocations, a serving loop that must not
 * allocate after start-up -- and so cannot pass mss_scan_fwd_ex2 a
 * workspace.  This entry point takes no workspace: when the sequence is
 * split, the aggregates live in a fixed scratch array of
 * mss_scan_fwd_noalloc_scratch_bytes() bytes (4 MiB) that is part of the
 * library image; every GPU that loads the library holds it until the process
 * exits.  Nothing here allocates (no cudaMalloc, no allocating library call).
 *
 *   - Sizes whose split would need more scratch than that are rejected with
 *     MSS_ERR_SCRATCH before anything is launched (mss_scan_fwd_workspace_size
 *     gives the need; MSS_FLAG_NO_SPLIT avoids it).
 *   - The first call on a device looks up the scratch's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it; make
 *     that first call before any stream capture on that device.
 *   - Every call on a device shares the one array, which keeps the last
 *     call's contents.  Nothing in it needs to start at zero: each call's
 *     first kernel writes every aggregate its second kernel reads.  Calls that
 *     overlap on the GPU (other streams, other threads) race on it and must be
 *     serialised by the caller.
 *
 * Arguments, flags and results are those of mss_scan_fwd_ex2 without the
 * workspace pair.
 */
MSS_API int mss_scan_fwd_noalloc(const void *u, const void *delta, const float *A, const void *B,
                                 const void *C, const float *D, const void *z, const float *delta_bias,
                                 int softplus_flag, const float *initial_state, void *y, float *last_state,
                                 int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                                 int dtype, unsigned flags, void *stream);

/* Size in bytes of mss_scan_fwd_noalloc's fixed scratch (per device). */
MSS_API int64_t mss_scan_fwd_noalloc_scratch_bytes(void);

/*
 * mss_scan_bwd -- backward pass of mss_scan_fwd_ex2 (without the convolution):
 * the gradients of a loss with respect to every input, given its gradients
 * with respect to y and last_state.  The pages train the model end to end
 * and have the fused kernel recompute the states in the backward pass rather
 * than store them ("Mamba" paper review, section "Selection Mechanism"); they
 * print no gradient, so this is the chain rule of the forward definition.
 * The states are recomputed from checkpoints (one state per channel every
 * 16 bytes of a row, i.e. 8 bf16 or 4 fp32 tokens, or every 16 tokens on the
 * scalar path) that the call writes into the caller's workspace; nothing
 * else is stored.
 *
 *   forward inputs: u, delta, A, B, C, D, z, delta_bias, softplus_flag,
 *                   initial_state, with the layouts of mss_scan_fwd_ex2, and
 *                   flags (MSS_FLAG_ZOH_INPUT, MSS_FLAG_GENERAL_A,
 *                   MSS_FLAG_SIMPLE) as used by the forward pass, plus
 *                   MSS_FLAG_SAVED_STATES when the workspace holds the states
 *                   of mss_scan_fwd_save (the checkpoint pass is skipped; the
 *                   call then needs the tiled kernels, else MSS_ERR_PATH)
 *   dy      : [batch][dim][seqlen] dtype, dLoss/dy
 *   dlast   : [batch][dim][dstate] float, dLoss/dlast_state (NULL: zero)
 *   du, ddelta : [batch][dim][seqlen] dtype out (ddelta: with respect to
 *                the raw delta, i.e. through softplus and the bias)
 *   dz      : [batch][dim][seqlen] dtype out, required when z is given
 *   dA      : [dim][dstate] float out
 *   dB, dC  : [batch][dstate][seqlen] float out (sums over the channels)
 *   dD, dbias : [dim] float out (NULL: not computed)
 *   dinit   : [batch][dim][dstate] float out, dLoss/dinitial_state (NULL: not written)
 *   workspace : at least mss_scan_bwd_workspace_size bytes of device memory,
 *               16-byte aligned, owned by the caller; its contents on entry
 *               do not matter, except with MSS_FLAG_SAVED_STATES, where they
 *               are read and not written
 *
 * dA, dB, dC, dD and dbias are zeroed and then accumulated with float atomics
 * on the stream, so they are not bitwise reproducible between runs.  No
 * output may overlap an input, another output or the workspace.  Errors as
 * mss_scan_fwd_ex2, plus MSS_ERR_WORKSPACE.  seqlen == 0: the per-token and
 * summed gradients are empty or zero and dinit = dlast.
 */
MSS_API int mss_scan_bwd(const void *u, const void *delta, const float *A, const void *B, const void *C,
                 const float *D, const void *z, const float *delta_bias, int softplus_flag,
                 const float *initial_state, const void *dy, const float *dlast,
                 void *du, void *ddelta, void *dz, float *dA, float *dB, float *dC, float *dD,
                 float *dbias, float *dinit, int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                 int dtype, unsigned flags, void *workspace, int64_t workspace_bytes, void *stream);

/* Workspace bytes mss_scan_bwd needs for these sizes and flags, assuming
 * 16-byte aligned tensors (with unaligned ones it takes the scalar path: ask
 * with MSS_FLAG_SIMPLE for that size).  Sizes the tiled kernels cannot take
 * (batch > 65535, batch * dim >= 2^31, seqlen >= 2^31) get the scalar path's
 * size here, as they get its kernel.  Negative mss_status on bad arguments;
 * 0 when there is nothing to do. */
MSS_API int64_t mss_scan_bwd_workspace_size(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                                    int dtype, unsigned flags);

/*
 * mss_ssd_fwd -- forward pass of the structured state space duality layer
 * (Mamba-2): A is a scalar per head, each head carries an N x P state, and
 * the heads of a group share B and C ("NN Lab -- Mamba", Structured State
 * Space Duality; "Mamba" paper review, section "Mamba 2").  Per (batch, head):
 *
 *   Delta_t = softplus(dt_t + dt_bias_h) (or dt_t + dt_bias_h),
 *   S_t = exp(Delta_t A_h) S_{t-1} + Delta_t B_t x_t^T,
 *   y_t = S_t^T C_t + D_h x_t, times silu(z_t) when z is given,
 *
 * computed chunk by chunk with tensor-core matrix products: the masked
 * quadratic form within a chunk plus the state carried across (chunks of 128
 * tokens on the tcgen05 kernel for dstate 128, 64 on the warp-level kernels;
 * see mss_ssd_fwd_ex2).
 *
 *   x, z, y  : [batch][seqlen][nheads][headdim]  bf16 (z may be NULL)
 *   dt       : [batch][seqlen][nheads]           bf16
 *   A, D, dt_bias : [nheads] float (D and dt_bias may be NULL)
 *   B, C     : [batch][seqlen][ngroups][dstate]   bf16; head h reads group
 *              h / (nheads / ngroups)
 *   initial_state, last_state : [batch][nheads][dstate][headdim] float
 *              (NULL: zero / not written)
 *
 * Supported: dtype MSS_DTYPE_BF16 (else MSS_ERR_DTYPE); headdim 64, dstate
 * 64 or 128, nheads a multiple of ngroups (else MSS_ERR_SHAPE); x, B, C, y,
 * z 16-byte aligned (else MSS_ERR_ALIGN).  Outputs must not overlap inputs.
 * The intermediate products round to bf16 (the masked score matrix, the
 * state as read by the next chunk), as tensor-core operands do.
 */
MSS_API int mss_ssd_fwd(const void *x, const void *dt, const float *A, const void *B, const void *C,
                const float *D, const void *z, const float *dt_bias, int softplus_flag,
                const float *initial_state, void *y, float *last_state, int64_t batch, int64_t seqlen,
                int64_t nheads, int64_t headdim, int64_t ngroups, int64_t dstate, int dtype, void *stream);

/* mss_ssd_fwd with a caller-owned workspace (device memory, 16-byte aligned,
 * at least mss_ssd_fwd_workspace_size bytes, not overlapping any argument).
 * When batch * nheads leaves the in-order kernel's last wave of CTAs (one
 * per (batch, head): up to two per SM for dstate 64, one for the tcgen05
 * kernel of dstate 128) short enough, the chunks of every head then run in
 * parallel in three passes (chunk states, the recurrence of chunk states,
 * chunk outputs; warp-level kernels) instead of one CTA walking a head's
 * chunks in order; otherwise the workspace is not used (the passes' extra
 * state traffic would cost more than they gain).  On a 148-SM B200 the
 * passes run for up to 115 pairs at dstate 64 and up to 28 at dstate 128.
 * At dstate 128 they also take the pairs past the tcgen05 kernel's last full
 * wave (one CTA per SM) when those are at most one in nine SMs' worth (16 on
 * 148 SMs), the whole waves staying on the tcgen05 kernel, and the
 * workspace then holds only those pairs' chunk states;
 * mss_ssd_fwd_workspace_size returns 0 where the workspace goes unused.
 * Same result up to rounding; a NULL workspace is mss_ssd_fwd.
 * MSS_ERR_WORKSPACE if it is too small. */
MSS_API int mss_ssd_fwd_ex(const void *x, const void *dt, const float *A, const void *B, const void *C,
                   const float *D, const void *z, const float *dt_bias, int softplus_flag,
                   const float *initial_state, void *y, float *last_state, int64_t batch, int64_t seqlen,
                   int64_t nheads, int64_t headdim, int64_t ngroups, int64_t dstate, int dtype,
                   void *workspace, int64_t workspace_bytes, void *stream);

/* Workspace bytes mss_ssd_fwd_ex would use for these sizes on the current
 * device (0: the in-order kernel, or no tokens), or a negative mss_status
 * (MSS_ERR_SHAPE for unsupported sizes). */
MSS_API int64_t mss_ssd_fwd_workspace_size(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                                   int64_t ngroups, int64_t dstate);

/* Flags of mss_ssd_fwd_ex2. */
#define MSS_SSD_FLAG_WARP_MMA 0x1u /* the warp-level (mma.sync) kernels instead of the tcgen05 one */

/*
 * mss_ssd_fwd_ex2 -- mss_ssd_fwd_ex with `flags`, for testing and measurement.
 *
 * With flags == 0 (this is then mss_ssd_fwd_ex): dstate 128 runs the tcgen05
 * kernel -- one CTA per (batch, head) walking chunks of 128 tokens in order,
 * operands staged by TMA in shared memory, the four chunk products
 * (C B^T, B^T diag(w) X, C S_prev, M X) on the fifth-generation tensor cores
 * with fp32 accumulators in tensor memory -- unless a workspace is given
 * and there are so few (batch, head) pairs that the chunk-parallel passes
 * are faster (see mss_ssd_fwd_ex); dstate 64 runs the warp-level kernels as
 * described at mss_ssd_fwd_ex.
 * MSS_SSD_FLAG_WARP_MMA: the warp-level kernels for both dstate (in order,
 * or the chunk-parallel passes with a workspace where they pay).  Other
 * bits: MSS_ERR_FLAGS.  Same results up to rounding; the tcgen05 kernel's
 * bounded waits report through mss_get_device_error.
 */
MSS_API int mss_ssd_fwd_ex2(const void *x, const void *dt, const float *A, const void *B, const void *C,
                    const float *D, const void *z, const float *dt_bias, int softplus_flag,
                    const float *initial_state, void *y, float *last_state, int64_t batch, int64_t seqlen,
                    int64_t nheads, int64_t headdim, int64_t ngroups, int64_t dstate, int dtype,
                    unsigned flags, void *workspace, int64_t workspace_bytes, void *stream);

/* Workspace bytes mss_ssd_fwd_ex2 would use with these flags (as
 * mss_ssd_fwd_workspace_size, which is flags == 0). */
MSS_API int64_t mss_ssd_fwd_workspace_size_ex(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                                      int64_t ngroups, int64_t dstate, unsigned flags);

/*
 * mss_state_update -- one decode token for every (batch, channel):
 * the recurrence above applied once to a caller-held state
 * (the generation-time view of "Exercises -- State-space models (Mamba, S4)":
 * O(1) work and O(N) memory per token).
 *
 *   state       : [batch][dim][dstate] float, read and overwritten in place
 *   u, delta, z : [batch][dim]         dtype (z may be NULL)
 *   A           : [dim][dstate]        float
 *   B, C        : [batch][dstate]      dtype
 *   D, delta_bias: [dim]               float (each may be NULL)
 *   y           : [batch][dim]         dtype output
 *
 * Returns MSS_OK or a negative mss_status.
 */
MSS_API int mss_state_update(float *state, const void *u, const void *delta, const float *A,
                     const void *B, const void *C, const float *D, const void *z,
                     const float *delta_bias, int softplus_flag, void *y,
                     int64_t batch, int64_t dim, int64_t dstate, int dtype, void *stream);

/* mss_state_update with `flags`: 0, or MSS_FLAG_ZOH_INPUT for the
 * zero-order-hold input matrix (the rule the forward pass that produced the
 * state used).  Other bits: MSS_ERR_FLAGS.  flags == 0 is mss_state_update. */
MSS_API int mss_state_update_ex(float *state, const void *u, const void *delta, const float *A,
                        const void *B, const void *C, const float *D, const void *z,
                        const float *delta_bias, int softplus_flag, void *y,
                        int64_t batch, int64_t dim, int64_t dstate, int dtype,
                        unsigned flags, void *stream);

/*
 * mss_state_update_conv -- one decode token with the causal convolution of
 * mss_scan_fwd_conv in front: u = silu(conv_b + sum_k conv_w[d,k] * window_k)
 * over the window (conv_state[b,d,0..K-2], x[b,d]); then conv_state is
 * shifted by one token in place (it ends with x) and the state update runs
 * on u as in mss_state_update_ex.
 *
 *   conv_state : [batch][dim][K-1] dtype, read and overwritten in place
 *                (may be NULL when K == 1); must not overlap anything else
 *   x          : [batch][dim] dtype (takes the place of u)
 *   conv_w, conv_b, conv_width: as in mss_scan_fwd_conv
 *
 * The other arguments and the errors are those of mss_state_update_ex.
 */
MSS_API int mss_state_update_conv(float *state, void *conv_state, const void *x, const float *conv_w,
                          const float *conv_b, int conv_width, const void *delta, const float *A,
                          const void *B, const void *C, const float *D, const void *z,
                          const float *delta_bias, int softplus_flag, void *y,
                          int64_t batch, int64_t dim, int64_t dstate, int dtype, unsigned flags,
                          void *stream);

/*
 * mss_get_device_error -- synchronises `stream`, then reports and clears the
 * device error word that kernels set when a bounded wait gives up
 * (MSS_ERR_DEVICE_TIMEOUT), or MSS_ERR_CUDA if the stream itself reports an
 * error.  Returns MSS_OK when neither happened.  The error word is one
 * word of device memory per device, defined in the library image; nothing
 * is allocated.
 */
MSS_API int mss_get_device_error(void *stream);

/*
 * mss_probe_pipe_rates -- a measurement aid, not part of the scan: the
 * throughput of the pipes the scan kernels are bound by, on the current
 * device, in operations per SM and SM clock cycle.  The scan's arithmetic
 * roof is stated from unit counts (128 fp32 lanes per SM); this call
 * measures what those units deliver.
 *
 *   rates   HOST array of n_rates doubles, written:
 *             [0] fp32 fma lane operations (scalar fma)
 *             [1] fp32 fma lane operations with the packed two-wide fma
 *             [2] ex2.approx results (multi-function unit)
 *             [3] warp-shuffle results (one per lane)
 *           entries past [3] are set to 0
 *   stream  the stream the four loops run on; the call synchronises it
 *
 * Each loop runs 8 CTAs of 256 threads per SM, every thread 8 independent
 * chains of one instruction; a rate is the operations an SM's CTAs executed
 * over the SM clock cycles from their first start to their last end (the
 * per-SM cycle counter), averaged over the SMs.  Uses four fixed device
 * arrays in the library image; allocates nothing.  Not safe to call
 * concurrently from several host threads on one device.
 * Errors: MSS_ERR_NULL (rates NULL), MSS_ERR_SHAPE (n_rates < 0),
 * MSS_ERR_CUDA (launch, copy or synchronisation failed).
 */
MSS_API int mss_probe_pipe_rates(double *rates, int n_rates, void *stream);

/* Human-readable text for a status code (static storage, never NULL). */
MSS_API const char *mss_strerror(int code);

/* MSS_VERSION of the library that was loaded. */
MSS_API int mss_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MSS_H */
