/*
 * sscan.h -- C ABI of libsscan, a B200 (sm_100a) implementation of the selective
 * state-space scan (S6) from "Mamba: Linear-Time Sequence Modeling with Selective
 * State Spaces" (Gu & Dao, 2023).
 *
 * The operation (technical summary page "Mamba 状态空间模型原理与 Transformer 对比",
 * kb.agiseed.tech, sec. 2.1 eqs. (2), (3a), (3b); sec. 3.2; sec. 4.1; Fig. 3):
 *   delta_t = softplus(delta_raw_t + delta_bias_d)     (flag SSCAN_DELTA_SOFTPLUS,
 *                                                        else delta_raw_t + bias_d)
 *   Abar_tn = exp(delta_t A_dn)                          eq. (2)
 *   Bbar_tn = expm1(delta_t A_dn) / A_dn * B_tn          eq. (2), diagonal A;
 *                                                        the limit delta_t B_tn at A_dn = 0
 *   h_tn    = Abar_tn h_{t-1,n} + Bbar_tn x_t            eq. (3a), x = u
 *   y_t     = sum_n C_tn h_tn + D_skip_d x_t             eq. (3b) plus a skip term
 *   out_t   = y_t * SiLU(z_t)                            Fig. 3 gate (when z is given)
 * for every batch b and channel d independently; h_{-1} = h0 (zero when NULL).
 * The (batch, L, D, N) state is never written to memory (sec. 4.1).
 *
 * Layouts (dense, row-major, no padding):
 *   u, delta_raw, z, out, du, ddelta_raw, dz, dout : (batch, L, D)
 *   B, C, dB, dC                                    : (batch, L, N), shared by all D channels
 *   A, dA                                           : (D, N)
 *   delta_bias, D_skip, ddelta_bias, dD             : (D)
 *   h0, h_last, dh0                                 : (batch, D, N)
 * Element types: the tensors in the first two rows (and their gradients) use
 * problem->io_dtype (fp32 or bf16); A, delta_bias, D_skip, states and their
 * gradients are always fp32.  All arithmetic is fp32; bf16 results are rounded
 * to nearest-even once.
 *
 * Ownership and execution: every pointer is a device pointer owned by the caller
 * (except `problem`, a host pointer read during the call).  The library never
 * allocates device memory, frees or synchronises; it enqueues its kernels on
 * `stream` (a cudaStream_t, NULL = legacy default stream) and returns.  (The only
 * CUDA objects it creates -- once per device, kept for the process -- are the
 * auxiliary stream and two events of sscan_bwd, described there.)  Outputs are
 * overwritten, never accumulated into.  Inputs must not alias outputs.
 *
 * Errors: arguments are checked on the host before anything is launched; a
 * rejected call returns a non-zero status and enqueues nothing.  Launch failures
 * return SSCAN_ERR_CUDA.  sscan_last_error() gives a one-line reason for the most
 * recent failure on the calling thread.
 */
#ifndef SSCAN_H
#define SSCAN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SSCAN_API __attribute__((visibility("default")))
#else
#define SSCAN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum sscan_status {
    SSCAN_OK = 0,
    SSCAN_ERR_INVALID_ARG = 1, /* NULL required pointer, negative size, unknown dtype or flag */
    SSCAN_ERR_UNSUPPORTED = 2, /* a well-formed problem this build does not handle (dstate > 16) */
    SSCAN_ERR_WORKSPACE = 3,   /* workspace NULL or smaller than sscan_workspace_size() */
    SSCAN_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed */
    SSCAN_ERR_TIMEOUT = 5      /* sscan_device_status: a kernel's bounded wait gave up */
} sscan_status;

typedef enum sscan_dtype { SSCAN_F32 = 0, SSCAN_BF16 = 1 } sscan_dtype;

/* problem->flags */
#define SSCAN_DELTA_SOFTPLUS 1u
/* The scan's input is x_t = SiLU(u_t) instead of u_t, in the state update and the
 * skip term alike: the activation of the block's input branch ahead of the SSM
 * (Fig. 3 caption: the block replaces its first multiplicative gate with an
 * activation, sigma = SiLU).  Backward: du receives dL/dx * SiLU'(u). */
#define SSCAN_INPUT_SILU 2u

typedef struct sscan_problem {
    int64_t batch;    /* >= 0 */
    int64_t seqlen;   /* L >= 0 */
    int64_t dim;      /* D >= 0, channels */
    int64_t dstate;   /* N, 1..16 */
    int32_t io_dtype; /* sscan_dtype of the (batch,L,D) and (batch,L,N) tensors */
    uint32_t flags;   /* OR of SSCAN_DELTA_SOFTPLUS, SSCAN_INPUT_SILU, or 0 */
} sscan_problem;

typedef enum sscan_op {
    SSCAN_OP_FWD = 0,
    SSCAN_OP_LAST_STATE = 1,
    SSCAN_OP_BWD = 2,
    SSCAN_OP_SUMMARY = 3,
    SSCAN_OP_BWD_COMPLEX = 4
} sscan_op;

/* Bytes of device workspace the operation needs for this problem (0 when none).
 * The size depends only on the problem and the op.  Returns 0 for an invalid
 * problem (the operation itself then reports the error). */
SSCAN_API size_t sscan_workspace_size(const sscan_problem* problem, int op);

/*
 * Forward scan: writes out (batch, L, D) in io_dtype and, when h_last is not
 * NULL, the final state h_{L-1} (batch, D, N) fp32.  delta_bias, D_skip, z and h0
 * may be NULL (zero bias, no skip term, no gate, zero initial state).  out may be
 * NULL only if h_last is not (that is the last-state operation).
 * Sec. 2.1 eqs. (2)-(3), sec. 3.2, sec. 4.1, Fig. 3 of the page cited above.
 */
SSCAN_API sscan_status sscan_fwd(const sscan_problem* problem, const void* u, const void* delta_raw,
                       const float* delta_bias, const float* A, const void* B, const void* C,
                       const float* D_skip, const void* z, const float* h0, void* out,
                       float* h_last, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Final state only: h_last = h_{L-1} (batch, D, N) fp32, without reading C or z
 * and without writing any (batch, L, D) output.  With h0 this chains sequence
 * segments: running [0,k) then [k,L) from its h_last equals one run over [0,L)
 * (eq. (3a) is a recurrence; sec. 5: constant-size state for generation).
 */
SSCAN_API sscan_status sscan_last_state(const sscan_problem* problem, const void* u, const void* delta_raw,
                              const float* delta_bias, const float* A, const void* B,
                              const float* h0, float* h_last, void* workspace,
                              size_t workspace_bytes, void* stream);

/*
 * Forward scan without a caller workspace (the paper has no counterpart: this
 * is plumbing for callers that cannot allocate device memory).  Same arguments
 * and results as sscan_fwd, minus workspace / workspace_bytes.
 *
 * Who needs it: code that may not call cudaMalloc or any allocator -- a plugin
 * hosted by a framework that owns every byte of device memory and forbids
 * outside allocations, or a latency-critical caller that cannot afford
 * cudaMalloc's implicit device synchronisation.  Such callers still pass their
 * own inputs and outputs; only the scratch moves inside the library.
 *
 * Scratch: a fixed 4 MiB array in the library's device memory (every GPU that
 * loads libsscan holds it until the process exits).  It covers every problem
 * whose (batch, L, D) tensors have 16-byte aligned bases and row pitches (the
 * TMA-tiled path needs at most 3.8 MB: this entry point splits a long sequence into
 * fewer, longer chunks than sscan_fwd does, one wave of CTAs instead of several, so a
 * split sequence can take somewhat longer here; results agree with sscan_fwd to the
 * rounding of the chunk carries).  A call whose path needs more scratch
 * than that (possible only on the general path for unaligned tensors) returns
 * SSCAN_ERR_WORKSPACE before anything is launched.  The first call on each
 * device looks up the array's device address (cudaGetSymbolAddress, with that
 * device current) and caches it for the process; make that first call before any
 * stream capture.  A cudaDeviceReset between calls is not supported (the cached
 * address would be stale).  All calls share the one array and it keeps the last call's
 * contents; the kernels overwrite every scratch byte they later read, so nothing
 * needs clearing.  Calls whose work overlaps on the GPU (different streams, or
 * different host threads without ordering) race on the scratch: serialise them.
 * No allocation or free of any kind happens in this call.
 */
SSCAN_API sscan_status sscan_fwd_noalloc(const sscan_problem* problem, const void* u, const void* delta_raw,
                                         const float* delta_bias, const float* A, const void* B, const void* C,
                                         const float* D_skip, const void* z, const float* h0, void* out,
                                         float* h_last, void* stream);

/*
 * Backward scan: gradients of sum(out * dout) with respect to every input of
 * sscan_fwd, recomputing the states on chip instead of storing them (sec. 4.1,
 * item 3).  du, ddelta_raw, dB, dC (and dz) are in io_dtype; dA, ddelta_bias, dD,
 * dh0 are fp32.  ddelta_bias, dD, dz and dh0 may be NULL when not wanted; dz must
 * be given exactly when z is, dD only when D_skip is.  The argument list of the
 * forward pass must be repeated exactly as it was given to sscan_fwd.
 * Streams: when the reverse sweep is split into sequence segments (few batch x
 * channel blocks, long L), the segment summaries run on a second stream while the
 * checkpoint pass runs on `stream`; the call forks to it and joins back with an
 * event record / wait pair, so all work is still ordered after earlier work on
 * `stream` and before later work on it (and stream capture records the fork as
 * graph edges).  That stream and its two events are created once per device on
 * first use and kept for the process (no device memory is allocated).
 */
SSCAN_API sscan_status sscan_bwd(const sscan_problem* problem, const void* u, const void* delta_raw,
                       const float* delta_bias, const float* A, const void* B, const void* C,
                       const float* D_skip, const void* z, const float* h0, const void* dout,
                       void* du, void* ddelta_raw, float* ddelta_bias, float* dA, void* dB,
                       void* dC, float* dD, void* dz, float* dh0, void* workspace,
                       size_t workspace_bytes, void* stream);

/*
 * One recurrence step for autoregressive generation: every (batch, channel)
 * advances its state by one token, h <- Abar h + Bbar x, and emits
 * out = (C.h + D_skip x) SiLU(z) -- constant time and memory per token with no
 * cache that grows with the context (sec. 5; sec. 2.1 eqs. (2), (3a), (3b) at one t).
 * problem->seqlen must be 1; u, delta_raw, z, out are (batch, D) and B, C are
 * (batch, N) in io_dtype; state (batch, D, N) fp32 is read and overwritten in
 * place.  The result equals sscan_fwd with seqlen 1, h0 = state, h_last = state.
 * delta_bias, D_skip and z may be NULL.  No workspace.
 */
SSCAN_API sscan_status sscan_step(const sscan_problem* problem, const void* u, const void* delta_raw,
                                  const float* delta_bias, const float* A, const void* B, const void* C,
                                  const float* D_skip, const void* z, float* state, void* out, void* stream);

/*
 * Summary of one stretch of the sequence, for splitting a long sequence across
 * devices (sec. 4.1 / sec. 5: the recurrence is linear in the state, so a stretch
 * acts on its initial state as the affine map h -> P h + H):
 *   P = prod_t Abar_t = exp(A * sum_t delta_t)   (batch, D, N) fp32
 *   H = the final state of the stretch started from zero   (batch, D, N) fp32
 * C, z and D_skip are not needed.  Workspace: sscan_workspace_size(problem,
 * SSCAN_OP_SUMMARY) bytes.  seqlen 0 gives the identity (P = 1, H = 0).
 */
SSCAN_API sscan_status sscan_chunk_summary(const sscan_problem* problem, const void* u, const void* delta_raw,
                                           const float* delta_bias, const float* A, const void* B, float* P,
                                           float* H, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Compose the summaries of nchunks consecutive stretches, in order, starting from
 * h0 (NULL = zero): carry_in[k] = the state entering stretch k, h_final = the state
 * after the last (a warp-shuffle scan of the affine pairs, 32 stretches at a time).  P, H, carry_in: (nchunks, batch, D, N) fp32, chunk-major;
 * h0, h_final: (batch, D, N).  Running sscan_fwd on stretch k with
 * h0 = carry_in[k] reproduces the unsplit scan.  carry_in or h_final may be NULL.
 * Only problem->batch, dim, dstate are read.
 */
SSCAN_API sscan_status sscan_carry(const sscan_problem* problem, int64_t nchunks, const float* P, const float* H,
                                   const float* h0, float* carry_in, float* h_final, void* stream);

/*
 * Forward scan with a complex diagonal A: the complex initialisation A_n = -1/2 + n i
 * of the A-init ablation table (sec. 6.5), with eqs. (2) and (3) of sec. 2.1 taken in
 * complex arithmetic:
 *   Abar = exp(delta a),  Bbar = (exp(delta a) - 1) / a * B  (delta B at a = 0),
 *   h_t  = Abar h_{t-1} + Bbar x_t   (complex state),
 *   out  = (Re(sum_n C_tn h_tn) + D_skip x_t) * SiLU(z_t).
 * B and C are the real (batch, L, N) input projections of sec. 3.2, as in sscan_fwd.
 * A: (D, N, 2) fp32, (re, im) pairs.  h0 (may be NULL = zero) and h_last (may be
 * NULL): (batch, D, N, 2) fp32 pairs.  out (batch, L, D) in io_dtype is required.
 * No workspace; the whole sequence of a (batch, channel block) runs in one CTA (no
 * sequence split).  seqlen 0 copies h0 (or zero) to h_last.  Errors as sscan_fwd.
 */
SSCAN_API sscan_status sscan_fwd_complex(const sscan_problem* problem, const void* u, const void* delta_raw,
                                         const float* delta_bias, const float* A, const void* B, const void* C,
                                         const float* D_skip, const void* z, const float* h0, void* out,
                                         float* h_last, void* stream);

/*
 * Backward of sscan_fwd_complex: gradients of sum(out * dout), the states
 * recomputed on chip from checkpoints of every 8th step (sec. 4.1 item 3).  The
 * gradient with respect to a complex quantity (dA, dh0) is the pair
 * (dL/dRe, dL/dIm) in the same (re, im) layout as the quantity.  du, ddelta_raw, dB,
 * dC, dz in io_dtype; dA (D, N, 2), ddelta_bias, dD, dh0 (batch, D, N, 2) fp32.
 * NULL rules as sscan_bwd.  Workspace: sscan_workspace_size(problem,
 * SSCAN_OP_BWD_COMPLEX) bytes (fp32 dB, dC accumulators and the checkpoints).
 */
SSCAN_API sscan_status sscan_bwd_complex(const sscan_problem* problem, const void* u, const void* delta_raw,
                                         const float* delta_bias, const float* A, const void* B, const void* C,
                                         const float* D_skip, const void* z, const float* h0, const void* dout,
                                         void* du, void* ddelta_raw, float* ddelta_bias, float* dA, void* dB,
                                         void* dC, float* dD, void* dz, float* dh0, void* workspace,
                                         size_t workspace_bytes, void* stream);

/* Static, human-readable name of a status code. */
SSCAN_API const char* sscan_status_string(sscan_status status);

/* One-line reason for the most recent failed call on this thread ("" if none). */
SSCAN_API const char* sscan_last_error(void);

/* Number of kernels the most recent sscan_fwd / sscan_fwd_noalloc /
 * sscan_last_state / sscan_bwd call on this thread enqueued (memsets and copies
 * not counted). */
SSCAN_API int sscan_last_launch_count(void);

/* 1 in the debug build of the library (libsscan_debug.so), whose kernels check every
 * index they compute into a workspace, parameter or state array and report a bad one
 * through bit 3 of sscan_device_status (skipping the access) instead of touching the
 * memory; 0 in the release build, where those checks are compiled out. */
SSCAN_API int sscan_debug_bounds(void);

/*
 * Device-side status of the library's kernels on the current device: *flags
 * receives the OR of every error bit raised since the last clear (bit 0: in a
 * forward kernel, bit 1: in the backward kernel, a bounded wait for an
 * asynchronous tile copy gave up, so that kernel stopped early and its outputs
 * are incomplete; bit 2: sscan_probe_wait_timeout's wait ran out, as it is meant
 * to; bit 3, debug build only: an index out of its array's range was caught and the
 * access skipped).  Returns SSCAN_ERR_TIMEOUT when any bit is set, SSCAN_OK when none is.
 * clear != 0 resets the word after reading.  Synchronous: it waits for work
 * already submitted to the device.  Every wait in the library's kernels is
 * bounded, so a failed copy surfaces here instead of hanging the device.
 */
SSCAN_API sscan_status sscan_device_status(int clear, unsigned int* flags);

/* Library version, major * 10000 + minor * 100 + patch. */
SSCAN_API int sscan_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SSCAN_H */
