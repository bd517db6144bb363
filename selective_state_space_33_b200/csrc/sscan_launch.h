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
    int has_z;
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
};

// The (batch, L, D) tensors, reached through TMA tensor maps built per call.
struct TiledPtrs {
    const void* u;
    const void* delta_raw;
    const void* z;        // or null
    void* out;            // or null
};

enum { kTiledOut = 0, kTiledAgg = 1, kTiledLast = 2 };

// Channels one CTA covers for a given state count (its TMA box width).
int tiled_channels_per_cta(int64_t N);

cudaError_t launch_fwd_tiled(const TiledArgs& a, const TiledPtrs& p, int io_bf16, int mode, cudaStream_t st);

// Read (and optionally clear) the library's device error word; nonzero means a
// bounded wait in a kernel gave up.  Synchronous.
cudaError_t read_device_error(unsigned int* value, int clear);

}  // namespace sscan
