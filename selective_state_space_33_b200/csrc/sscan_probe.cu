// sscan_probe.cu -- MUFU ex2 throughput probe (include/sscan_probe.h).
#include <cuda_runtime.h>

#include "sscan_launch.h"
#include "sscan_math.cuh"
#include "sscan_probe.h"

namespace {

// Eight independent chains per thread keep the pipe full; the inputs stay in
// [-1, 0) so no result is denormal or saturates.
__global__ void ex2_probe_kernel(float* sink, int64_t iters) {
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = -0.001f * (float)(threadIdx.x + j);
    for (int64_t i = 0; i < iters; ++i) {
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = sscan::ex2(v[j]) - 1.0f;
    }
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) s += v[j];
    sink[(int64_t)blockIdx.x * blockDim.x + threadIdx.x] = s;
}

}  // namespace

extern "C" sscan_status sscan_probe_ex2(float* sink, int64_t iters, int blocks, int threads, void* stream) {
    if (!sink || iters <= 0 || blocks <= 0 || threads <= 0 || threads > 1024) return SSCAN_ERR_INVALID_ARG;
    ex2_probe_kernel<<<blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(sink, iters);
    return cudaGetLastError() == cudaSuccess ? SSCAN_OK : SSCAN_ERR_CUDA;
}

extern "C" sscan_status sscan_probe_wait_timeout(unsigned int polls, void* stream) {
    if (polls == 0 || polls > (1u << 20)) return SSCAN_ERR_INVALID_ARG;
    return sscan::launch_wait_probe(polls, static_cast<cudaStream_t>(stream)) == cudaSuccess ? SSCAN_OK
                                                                                            : SSCAN_ERR_CUDA;
}
