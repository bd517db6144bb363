// sscan_launch.h -- launchers of the fast (tiled) kernels, called by sscan_api.cu.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace sscan {

// Scalar arguments and small parameter tensors of the tiled forward kernel.
struct TiledArgs {
    int64_t batch, L, D;
    int N;
    int softplus;
    int input_silu;       // the scan's input is SiLU(u)
    int has_z;
    int bc_tma;           // set by the launcher: B and C tiles travel by TMA
    const float* bias;    // (D) or null
    const float* A;       // (D, N)
    const float* Dskip;   // (D) or null
    const float* h0;      // (batch, D, N) or null
    const void* B;        // (batch, L, N)
    const void* C;        // (batch, L, N) or null (aggregate / last-state modes)
    float* h_last;        // (batch, D, N) or null
    int64_t chunk_len;    // sequence split, as in the general kernels
    int64_t nchunks;
    float* ws_state;      // [batch][nchunks][D][N]
    float* ws_dsum;       // [batch][nchunks][D]
    float* ws_ckpt;       // [batch][nck][D][N]: state before every 8th step (checkpoint mode)
    int64_t nck;          // ceil(L / 8)
};

// The (batch, L, D) tensors, reached through TMA tensor maps built per call.
struct TiledPtrs {
    const void* u;
    const void* delta_raw;
    const void* z;        // or null
    void* out;            // or null
};

enum { kTiledOut = 0, kTiledAgg = 1, kTiledLast = 2, kTiledCkpt = 3 };

// Lane geometry of the tiled kernel: NG lanes per channel, G states per lane,
// DC channels per CTA (its TMA box width).  A pure function of the problem.
constexpr int kMaxDevices = 64;  // per-device caches of the host code

struct TiledGeom {
    int NG, G, DC;
};
TiledGeom tiled_geometry(int64_t batch, int64_t L, int64_t D, int64_t N);

cudaError_t launch_fwd_tiled(const TiledArgs& a, const TiledPtrs& p, const TiledGeom& geo, int io_bf16, int mode,
                             cudaStream_t st);

// One recurrence step (autoregressive generation): tensors of one time step.
struct StepArgs {
    int64_t batch, D;
    int N;
    int softplus;
    int input_silu;         // the scan's input is SiLU(u)
    const void* u;          // (batch, D)
    const void* delta_raw;  // (batch, D)
    const float* bias;      // (D) or null
    const float* A;         // (D, N)
    const void* B;          // (batch, N)
    const void* C;          // (batch, N)
    const float* Dskip;     // (D) or null
    const void* z;          // (batch, D) or null
    float* state;           // (batch, D, N), updated in place
    void* out;              // (batch, D)
};

cudaError_t launch_step(const StepArgs& a, int io_bf16, cudaStream_t st);

// Forward scan with a complex diagonal A (sscan_complex.cu).
struct ComplexArgs {
    int64_t batch, L, D;
    int N;
    int softplus;
    int input_silu;         // the scan's input is SiLU(u)
    const void* u;          // (batch, L, D)
    const void* delta_raw;  // (batch, L, D)
    const float* bias;      // (D) or null
    const float* A;         // (D, N, 2): (re, im) pairs
    const void* B;          // (batch, L, N), real
    const void* C;          // (batch, L, N), real
    const float* Dskip;     // (D) or null
    const void* z;          // (batch, L, D) or null
    const float* h0;        // (batch, D, N, 2) or null
    void* out;              // (batch, L, D), or null when only checkpoints are wanted
    float* h_last;          // (batch, D, N, 2) or null
};

// ckpt: null for the forward with outputs; else [batch][nck][D][N][2] receives the
// state before every 8th step (the backward's checkpoint pass, a.out unused).  Kept
// out of ComplexArgs: the kernel's parameter block stays as small as the forward needs.
cudaError_t launch_fwd_complex(const ComplexArgs& a, float* ckpt, int64_t nck, int io_bf16, cudaStream_t st);
// Read (and optionally clear) the complex forward kernel's error word (bit 0: a bounded
// wait for a TMA tile copy gave up).  Synchronous.
cudaError_t read_device_error_cx(unsigned int* value, int clear);

// Backward of the complex-A scan (sscan_complex_bwd.cu).
struct ComplexBwdArgs {
    ComplexArgs f;          // forward inputs
    const float* ckpt;      // [batch][nck][D][N][2], written by the checkpoint pass
    int64_t nck;
    const void* dout;       // (batch, L, D)
    void* du;               // (batch, L, D)
    void* ddelta_raw;       // (batch, L, D)
    void* dz;               // (batch, L, D) or null
    float* dA;              // (D, N, 2), pre-zeroed
    float* dB32;            // (batch, L, N) fp32, pre-zeroed
    float* dC32;            // (batch, L, N) fp32, pre-zeroed
    float* dD;              // (D) or null, pre-zeroed
    float* dbias;           // (D) or null, pre-zeroed
    float* dh0;             // (batch, D, N, 2) or null
};

cudaError_t launch_bwd_complex(const ComplexBwdArgs& a, int io_bf16, cudaStream_t st);

// Backward of the tiled path: scalars, small tensors and gradient accumulators.
struct BwdTiledArgs {
    int64_t batch, L, D;
    int N;
    int softplus;
    int input_silu;      // the scan's input is SiLU(u); du gets the SiLU' factor
    int has_z;
    const float* bias;   // (D) or null
    const float* A;      // (D, N)
    const float* Dskip;  // (D) or null
    const float* ws_ckpt;  // [batch][nck][D][N] from the forward checkpoint pass
    int64_t nck;
    float* dB32;         // (batch, L, N) fp32, pre-zeroed
    float* dC32;         // (batch, L, N) fp32, pre-zeroed
    float* dA;           // (D, N), pre-zeroed
    float* dD;           // (D) or null, pre-zeroed
    float* dbias;        // (D) or null, pre-zeroed
    float* dh0;          // (batch, D, N) or null
    // sequence split of the reverse sweep: segment s covers steps
    // [s * seg_len, min(L, (s + 1) * seg_len)), seg_len a multiple of 8
    int64_t seg_len, nseg;
    float* ws_lam;       // [batch][nseg][D][N]: segment adjoint summaries, then carry-ins
    float* ws_dsum;      // [batch][nseg][D]: sum of delta over each segment
};

enum { kBwdFull = 0, kBwdSummary = 1 };

struct BwdTiledPtrs {
    const void* u;
    const void* delta_raw;
    const void* z;       // or null
    const void* dout;
    const void* B;
    const void* C;
    void* du;
    void* ddelta_raw;
    void* dz;            // or null
};

// kBwdFull: the gradients of every segment (adjoint state entering each segment from
// ws_lam when nseg > 1).  kBwdSummary: for segments 1 .. nseg-1 only, the adjoint
// state a segment passes to its left from zero and its sum of delta.
cudaError_t launch_bwd_tiled(const BwdTiledArgs& a, const BwdTiledPtrs& p, int io_bf16, int mode, cudaStream_t st);
// Turn the segment summaries in ws_lam into each segment's entering adjoint state.
cudaError_t launch_bwd_carry(const BwdTiledArgs& a, cudaStream_t st);
cudaError_t read_device_error_bwd(unsigned int* value, int clear);

// Read (and optionally clear) the library's device error word; nonzero means a
// bounded wait in a kernel gave up.  Synchronous.
cudaError_t read_device_error(unsigned int* value, int clear);

// One thread waits, with the kernels' bounded wait cut to `polls` polls, on an
// mbarrier that nothing arrives on, then raises bit 2 of the device error word.
cudaError_t launch_wait_probe(unsigned int polls, cudaStream_t st);

}  // namespace sscan
