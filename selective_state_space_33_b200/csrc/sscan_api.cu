// sscan_api.cu -- the C ABI of libsscan (declared in include/sscan.h): argument
// checks, workspace planning and kernel dispatch.  Everything is enqueued on the
// caller's stream; nothing here allocates, frees or synchronises.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <mutex>

#include "sscan.h"
#include "sscan_generic.cuh"
#include "sscan_generic_bwd.cuh"
#include "sscan_launch.h"
#include "sscan_plan.h"

namespace {

thread_local char g_err[256] = "";
thread_local int g_launches = 0;  // kernels the most recent call on this thread enqueued

sscan_status fail(sscan_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return s;
}

sscan_status cuda_check(const char* what) {
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(SSCAN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return SSCAN_OK;
}

sscan_status check_problem(const sscan_problem* p) {
    if (!p) return fail(SSCAN_ERR_INVALID_ARG, "problem is NULL");
    if (p->batch < 0 || p->seqlen < 0 || p->dim < 0)
        return fail(SSCAN_ERR_INVALID_ARG, "negative size (batch %lld, seqlen %lld, dim %lld)",
                    (long long)p->batch, (long long)p->seqlen, (long long)p->dim);
    if (p->dstate < 1) return fail(SSCAN_ERR_INVALID_ARG, "dstate must be >= 1");
    if (p->dstate > sscan::kMaxState)
        return fail(SSCAN_ERR_UNSUPPORTED, "dstate %lld > %d", (long long)p->dstate, sscan::kMaxState);
    if (p->io_dtype != SSCAN_F32 && p->io_dtype != SSCAN_BF16)
        return fail(SSCAN_ERR_INVALID_ARG, "unknown io_dtype %d", (int)p->io_dtype);
    if (p->flags & ~(SSCAN_DELTA_SOFTPLUS | SSCAN_INPUT_SILU))
        return fail(SSCAN_ERR_INVALID_ARG, "unknown flag bits 0x%x",
                    (unsigned)(p->flags & ~(SSCAN_DELTA_SOFTPLUS | SSCAN_INPUT_SILU)));
    return SSCAN_OK;
}

sscan_status check_workspace(size_t need, const void* ws, size_t bytes) {
    if (need == 0) return SSCAN_OK;
    if (!ws || bytes < need)
        return fail(SSCAN_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given%s", need, bytes,
                    ws ? "" : " (NULL)");
    if (reinterpret_cast<uintptr_t>(ws) % 256 != 0)
        return fail(SSCAN_ERR_WORKSPACE, "workspace must be 256-byte aligned");
    return SSCAN_OK;
}

inline unsigned blocks_for(int64_t n, int threads) { return (unsigned)((n + threads - 1) / threads); }

template <typename T, int NMAX>
void launch_fwd_rows(const sscan::ScanArgs& a, int mode, cudaStream_t st) {
    const int64_t n = a.batch * a.D * a.nchunks;
    if (mode == sscan::kModeOutput)
        sscan::fwd_rows_kernel<T, NMAX, sscan::kModeOutput><<<blocks_for(n, 128), 128, 0, st>>>(a);
    else
        sscan::fwd_rows_kernel<T, NMAX, sscan::kModeAggregate><<<blocks_for(n, 128), 128, 0, st>>>(a);
}

template <typename T>
void dispatch_fwd_rows(const sscan::ScanArgs& a, int mode, cudaStream_t st) {
    if (a.N <= 4) launch_fwd_rows<T, 4>(a, mode, st);
    else if (a.N <= 8) launch_fwd_rows<T, 8>(a, mode, st);
    else launch_fwd_rows<T, 16>(a, mode, st);
}

void fwd_rows(const sscan::ScanArgs& a, int io, int mode, cudaStream_t st) {
    ++g_launches;
    if (io == SSCAN_BF16) dispatch_fwd_rows<__nv_bfloat16>(a, mode, st);
    else dispatch_fwd_rows<float>(a, mode, st);
}

// L == 0: no steps, h_last = h0 (or zero); nothing else to write.
sscan_status empty_sequence(const sscan_problem* p, const float* h0, float* h_last, cudaStream_t st) {
    if (!h_last) return SSCAN_OK;
    const size_t bytes = (size_t)(p->batch * p->dim * p->dstate) * sizeof(float);
    if (bytes == 0) return SSCAN_OK;
    const cudaError_t e = h0 ? cudaMemcpyAsync(h_last, h0, bytes, cudaMemcpyDeviceToDevice, st)
                             : cudaMemsetAsync(h_last, 0, bytes, st);
    if (e != cudaSuccess) return fail(SSCAN_ERR_CUDA, "copying h0 to h_last: %s", cudaGetErrorString(e));
    return SSCAN_OK;
}

sscan::ScanArgs make_args(const sscan_problem* p, const void* u, const void* delta_raw,
                          const float* delta_bias, const float* A, const void* B, const void* C,
                          const float* D_skip, const void* z, const float* h0, void* out,
                          float* h_last) {
    sscan::ScanArgs a{};
    a.batch = p->batch;
    a.L = p->seqlen;
    a.D = p->dim;
    a.N = p->dstate;
    a.u = u;
    a.delta_raw = delta_raw;
    a.bias = delta_bias;
    a.A = A;
    a.B = B;
    a.C = C;
    a.Dskip = D_skip;
    a.z = z;
    a.h0 = h0;
    a.out = out;
    a.h_last = h_last;
    a.softplus = (p->flags & SSCAN_DELTA_SOFTPLUS) ? 1 : 0;
    a.input_silu = (p->flags & SSCAN_INPUT_SILU) ? 1 : 0;
    a.chunk_len = p->seqlen;
    a.nchunks = 1;
    return a;
}

// Forward or last-state through the row kernels, split along L when there are
// too few rows to fill the GPU (chunk aggregates, carry, then the chunk outputs).
sscan_status run_rows(const sscan_problem* p, sscan::ScanArgs a, void* ws, cudaStream_t st) {
    const sscan::FwdPlan plan = sscan::plan_fwd(p->batch, p->seqlen, p->dim, p->dstate);
    a.nchunks = plan.nchunks;
    a.chunk_len = plan.chunk_len;
    const bool want_out = a.out != nullptr;
    if (plan.nchunks > 1) {
        a.ws_state = static_cast<float*>(ws);
        a.ws_dsum = a.ws_state + plan.state_floats;
        fwd_rows(a, p->io_dtype, sscan::kModeAggregate, st);
        if (sscan_status s = cuda_check("chunk aggregate kernel")) return s;
        sscan::ScanArgs c = a;
        if (want_out) c.h_last = nullptr;  // the output pass writes h_last itself
        const int W = sscan::affine_lanes(c.nchunks);
        sscan::carry_kernel<<<blocks_for(p->batch * p->dim * p->dstate * W, 128), 128, 0, st>>>(c, W);
        ++g_launches;
        if (sscan_status s = cuda_check("carry kernel")) return s;
        if (!want_out) return SSCAN_OK;
    }
    fwd_rows(a, p->io_dtype, sscan::kModeOutput, st);
    return cuda_check("forward kernel");
}

bool aligned16(const void* q) { return q == nullptr || reinterpret_cast<uintptr_t>(q) % 16 == 0; }

// The tiled kernel reads rows of the (batch, L, D) tensors through TMA, which needs
// 16-byte aligned bases and row pitches.
bool tiled_ok(const sscan_problem* p, const sscan::ScanArgs& a) {
    const int64_t es = p->io_dtype == SSCAN_BF16 ? 2 : 4;
    return (p->dim * es) % 16 == 0 && aligned16(a.u) && aligned16(a.delta_raw) && aligned16(a.z) &&
           aligned16(a.out) && p->seqlen < (int64_t(1) << 31) && p->dim < (int64_t(1) << 31);
}

sscan_status run_tiled(const sscan_problem* p, const sscan::ScanArgs& a, void* ws, cudaStream_t st,
                       int64_t target) {
    const sscan::TiledGeom geo = sscan::tiled_geometry(p->batch, p->seqlen, p->dim, p->dstate);
    const sscan::FwdPlan plan = sscan::plan_tiled(p->batch, p->seqlen, p->dim, p->dstate, geo.DC, target);
    sscan::TiledArgs t{};
    t.batch = p->batch;
    t.L = p->seqlen;
    t.D = p->dim;
    t.N = (int)p->dstate;
    t.softplus = a.softplus;
    t.input_silu = a.input_silu;
    t.has_z = a.z != nullptr;
    t.bias = a.bias;
    t.A = a.A;
    t.Dskip = a.Dskip;
    t.h0 = a.h0;
    t.B = a.B;
    t.C = a.C;
    t.h_last = a.h_last;
    t.chunk_len = plan.chunk_len;
    t.nchunks = plan.nchunks;
    sscan::TiledPtrs ptr{a.u, a.delta_raw, a.z, a.out};
    const int bf16 = p->io_dtype == SSCAN_BF16;
    const bool want_out = a.out != nullptr;
    cudaError_t e;
    if (plan.nchunks > 1) {
        t.ws_state = static_cast<float*>(ws);
        t.ws_dsum = t.ws_state + plan.state_floats;
        e = sscan::launch_fwd_tiled(t, ptr, geo, bf16, sscan::kTiledAgg, st);
        ++g_launches;
        if (e != cudaSuccess) return fail(SSCAN_ERR_CUDA, "chunk aggregate kernel: %s", cudaGetErrorString(e));
        sscan::ScanArgs c = a;
        c.nchunks = plan.nchunks;
        c.chunk_len = plan.chunk_len;
        c.ws_state = t.ws_state;
        c.ws_dsum = t.ws_dsum;
        if (want_out) c.h_last = nullptr;
        const int W = sscan::affine_lanes(c.nchunks);
        sscan::carry_kernel<<<blocks_for(p->batch * p->dim * p->dstate * W, 128), 128, 0, st>>>(c, W);
        ++g_launches;
        if (sscan_status s = cuda_check("carry kernel")) return s;
        if (!want_out) return SSCAN_OK;
    }
    ++g_launches;
    e = sscan::launch_fwd_tiled(t, ptr, geo, bf16, want_out ? sscan::kTiledOut : sscan::kTiledLast, st);
    if (e != cudaSuccess) return fail(SSCAN_ERR_CUDA, "tiled forward kernel: %s", cudaGetErrorString(e));
    return SSCAN_OK;
}

// The tiled backward reads and writes every (batch, L, D) tensor and the B, C rows
// through TMA: 16-byte aligned bases, row pitches and B/C rows.
bool bwd_tiled_ok(const sscan_problem* p, const void* u, const void* dr, const void* z, const void* dout,
                  const void* B, const void* C, const void* du, const void* ddr, const void* dz) {
    const int64_t es = p->io_dtype == SSCAN_BF16 ? 2 : 4;
    return (p->dim * es) % 16 == 0 && (p->dstate * es) % 16 == 0 && aligned16(u) && aligned16(dr) &&
           aligned16(z) && aligned16(dout) && aligned16(B) && aligned16(C) && aligned16(du) && aligned16(ddr) &&
           aligned16(dz) && p->seqlen < (int64_t(1) << 31) && p->dim < (int64_t(1) << 31);
}

// A second stream per device on which the backward runs its segment summaries while
// the caller's stream runs the checkpoint pass (the two read the same inputs and
// write disjoint workspace).  Created on first use and kept for the process; the
// fork / join events are recorded under a mutex so that concurrent callers do not
// interleave them.  The fork and join are event record / wait pairs, which stream
// capture turns into graph edges.
struct AuxStream {
    cudaStream_t stream = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};
std::mutex g_aux_mutex;
AuxStream g_aux[64];

cudaError_t aux_stream(AuxStream** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    AuxStream& a = g_aux[dev];
    if (!a.stream) {
        if ((e = cudaStreamCreateWithFlags(&a.stream, cudaStreamNonBlocking)) != cudaSuccess) return e;
        if ((e = cudaEventCreateWithFlags(&a.fork, cudaEventDisableTiming)) != cudaSuccess) return e;
        if ((e = cudaEventCreateWithFlags(&a.join, cudaEventDisableTiming)) != cudaSuccess) return e;
    }
    *out = &a;
    return cudaSuccess;
}

// target: the split's target CTA count (kTiledTargetCtasCompact for the fixed scratch).
sscan_status run_fwd(const sscan_problem* p, const sscan::ScanArgs& a, void* ws, cudaStream_t st,
                     int64_t target = sscan::kTiledTargetCtas) {
    if (tiled_ok(p, a)) return run_tiled(p, a, ws, st, target);
    return run_rows(p, a, ws, st);
}

template <typename T, int NMAX>
void launch_bwd_rows(const sscan::BwdArgs& g, cudaStream_t st) {
    ++g_launches;
    sscan::bwd_rows_kernel<T, NMAX><<<blocks_for(g.f.batch * g.f.D, 128), 128, 0, st>>>(g);
}

template <typename T>
void dispatch_bwd_rows(const sscan::BwdArgs& g, cudaStream_t st) {
    if (g.f.N <= 4) launch_bwd_rows<T, 4>(g, st);
    else if (g.f.N <= 8) launch_bwd_rows<T, 8>(g, st);
    else launch_bwd_rows<T, 16>(g, st);
}

template <typename T>
void cast_out(const float* src, void* dst, int64_t n, cudaStream_t st) {
    if (n > 0) {
        sscan::cast_kernel<T><<<blocks_for(n, 256), 256, 0, st>>>(src, static_cast<T*>(dst), n);
        ++g_launches;
    }
}

// Fixed device scratch for sscan_fwd_noalloc.  Every GPU that loads this library
// holds these bytes until the process exits.  In host code the array's name is
// only a host-side stand-in; its device address comes from cudaGetSymbolAddress.
// 4 MiB covers every plan of the tiled path as this entry point plans it (with the
// one-wave target kTiledTargetCtasCompact): fewer than kTiledMinCols CTA columns times at
// most ceil(kTiledTargetCtasCompact / cols) chunks bounds the chunk states by
// 1480 * DC * (N + 1) floats, at most 3.8 MB for N <= 16.
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// The bound above, from plan_tiled's own constants: a split plan has cols < kTiledMinCols
// CTA columns of DC channels and ceil(kTiledTargetCtasCompact / cols) chunks, i.e. fewer than
// kTiledTargetCtasCompact + kTiledMinCols column-chunks, each holding DC * (N + 1) floats
// (the chunk's end states and delta sum); DC * (N + 1) is largest at N = 4 (DC = 128).
constexpr size_t tiled_scratch_bound() {
    size_t worst = 0;
    for (int n = 1; n <= sscan::kMaxState; ++n) {
        const size_t dc = n <= 4 ? 128 : (n <= 8 ? 64 : 32);
        const size_t b = (size_t)(sscan::kTiledTargetCtasCompact + sscan::kTiledMinCols - 1) * dc * (n + 1) * 4 + 255;
        worst = b > worst ? b : worst;
    }
    return worst;
}
static_assert(tiled_scratch_bound() <= kNoAllocScratchBytes,
              "the static scratch must hold every plan of the tiled forward path");

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch on the current device, looked up once per device
// (with that device current) and cached for the process.  A cudaDeviceReset between
// calls would leave a stale address behind, so it is not supported.
sscan_status noalloc_scratch(void** ptr) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(SSCAN_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return fail(SSCAN_ERR_UNSUPPORTED, "device ordinal %d >= %d", dev, kMaxDevices);
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p)
            return fail(SSCAN_ERR_CUDA, "cudaGetSymbolAddress of the static scratch: %s", cudaGetErrorString(e));
        g_noalloc_ptr[dev] = p;
    }
    *ptr = g_noalloc_ptr[dev];
    return SSCAN_OK;
}

}  // namespace

extern "C" {

size_t sscan_workspace_size(const sscan_problem* p, int op) {
    if (check_problem(p) != SSCAN_OK) return 0;
    switch (op) {
        case SSCAN_OP_FWD:
        case SSCAN_OP_LAST_STATE: {
            // enough for either path (the choice also depends on pointer alignment)
            const size_t g = sscan::plan_fwd(p->batch, p->seqlen, p->dim, p->dstate).workspace_bytes;
            const size_t t = sscan::plan_tiled(p->batch, p->seqlen, p->dim, p->dstate,
                                               sscan::tiled_geometry(p->batch, p->seqlen, p->dim, p->dstate).DC)
                                 .workspace_bytes;
            return g > t ? g : t;
        }
        case SSCAN_OP_BWD:
            return sscan::plan_bwd(p->batch, p->seqlen, p->dim, p->dstate).workspace_bytes;
        case SSCAN_OP_SUMMARY:
            return (p->batch * p->dim > 0 && p->seqlen > 0)
                       ? sscan::align256((size_t)(p->batch * p->dim) * sizeof(float))
                       : 0;
        case SSCAN_OP_BWD_COMPLEX: {
            // fp32 dB, dC accumulators, then the complex state before every 8th step
            if (p->batch * p->dim <= 0 || p->seqlen <= 0) return 0;
            const int64_t nck = (p->seqlen + 7) / 8;
            const size_t floats = (size_t)(2 * p->batch * p->seqlen * p->dstate) +
                                  (size_t)(p->batch * nck * p->dim * p->dstate * 2);
            return sscan::align256(floats * sizeof(float));
        }
        default:
            return 0;
    }
}

sscan_status sscan_fwd(const sscan_problem* p, const void* u, const void* delta_raw,
                       const float* delta_bias, const float* A, const void* B, const void* C,
                       const float* D_skip, const void* z, const float* h0, void* out,
                       float* h_last, void* workspace, size_t workspace_bytes, void* stream) {
    g_err[0] = 0;
    g_launches = 0;
    if (sscan_status s = check_problem(p)) return s;
    const bool any = p->batch * p->dim > 0;
    if (any && p->seqlen > 0) {
        if (!out && !h_last) return fail(SSCAN_ERR_INVALID_ARG, "out and h_last are both NULL");
        if (!u || !delta_raw || !A || !B) return fail(SSCAN_ERR_INVALID_ARG, "u, delta_raw, A, B are required");
        if (out && !C) return fail(SSCAN_ERR_INVALID_ARG, "C is required when out is written");
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (!any) return SSCAN_OK;
    if (p->seqlen == 0) return empty_sequence(p, h0, h_last, st);
    if (sscan_status s = check_workspace(sscan_workspace_size(p, SSCAN_OP_FWD), workspace, workspace_bytes))
        return s;
    return run_fwd(p, make_args(p, u, delta_raw, delta_bias, A, B, C, D_skip, z, h0, out, h_last),
                   workspace, st);
}

sscan_status sscan_last_state(const sscan_problem* p, const void* u, const void* delta_raw,
                              const float* delta_bias, const float* A, const void* B,
                              const float* h0, float* h_last, void* workspace,
                              size_t workspace_bytes, void* stream) {
    g_err[0] = 0;
    g_launches = 0;
    if (sscan_status s = check_problem(p)) return s;
    const bool any = p->batch * p->dim > 0;
    if (any && !h_last) return fail(SSCAN_ERR_INVALID_ARG, "h_last is required");
    if (any && p->seqlen > 0 && (!u || !delta_raw || !A || !B))
        return fail(SSCAN_ERR_INVALID_ARG, "u, delta_raw, A, B are required");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (!any) return SSCAN_OK;
    if (p->seqlen == 0) return empty_sequence(p, h0, h_last, st);
    if (sscan_status s = check_workspace(sscan_workspace_size(p, SSCAN_OP_LAST_STATE), workspace,
                                         workspace_bytes))
        return s;
    return run_fwd(p, make_args(p, u, delta_raw, delta_bias, A, B, nullptr, nullptr, nullptr, h0,
                                nullptr, h_last),
                   workspace, st);
}

sscan_status sscan_fwd_noalloc(const sscan_problem* p, const void* u, const void* delta_raw,
                               const float* delta_bias, const float* A, const void* B, const void* C,
                               const float* D_skip, const void* z, const float* h0, void* out,
                               float* h_last, void* stream) {
    g_err[0] = 0;
    g_launches = 0;
    if (sscan_status s = check_problem(p)) return s;
    const bool any = p->batch * p->dim > 0;
    if (any && p->seqlen > 0) {
        if (!out && !h_last) return fail(SSCAN_ERR_INVALID_ARG, "out and h_last are both NULL");
        if (!u || !delta_raw || !A || !B) return fail(SSCAN_ERR_INVALID_ARG, "u, delta_raw, A, B are required");
        if (out && !C) return fail(SSCAN_ERR_INVALID_ARG, "C is required when out is written");
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (!any) return SSCAN_OK;
    if (p->seqlen == 0) return empty_sequence(p, h0, h_last, st);
    const sscan::ScanArgs a = make_args(p, u, delta_raw, delta_bias, A, B, C, D_skip, z, h0, out, h_last);
    // scratch of the path this call takes (run_fwd makes the same choice)
    const size_t need =
        tiled_ok(p, a) ? sscan::plan_tiled(p->batch, p->seqlen, p->dim, p->dstate,
                                           sscan::tiled_geometry(p->batch, p->seqlen, p->dim, p->dstate).DC,
                                           sscan::kTiledTargetCtasCompact)
                             .workspace_bytes
                       : sscan::plan_fwd(p->batch, p->seqlen, p->dim, p->dstate).workspace_bytes;
    if (need > kNoAllocScratchBytes)
        return fail(SSCAN_ERR_WORKSPACE, "problem needs %zu bytes of scratch; the static scratch holds %zu", need,
                    kNoAllocScratchBytes);
    void* ws = nullptr;
    if (need > 0) {
        if (sscan_status s = noalloc_scratch(&ws)) return s;
    }
    return run_fwd(p, a, ws, st, sscan::kTiledTargetCtasCompact);
}

sscan_status sscan_bwd(const sscan_problem* p, const void* u, const void* delta_raw,
                       const float* delta_bias, const float* A, const void* B, const void* C,
                       const float* D_skip, const void* z, const float* h0, const void* dout,
                       void* du, void* ddelta_raw, float* ddelta_bias, float* dA, void* dB,
                       void* dC, float* dD, void* dz, float* dh0, void* workspace,
                       size_t workspace_bytes, void* stream) {
    g_err[0] = 0;
    g_launches = 0;
    if (sscan_status s = check_problem(p)) return s;
    if ((z == nullptr) != (dz == nullptr)) return fail(SSCAN_ERR_INVALID_ARG, "dz must be given exactly when z is");
    if (dD && !D_skip) return fail(SSCAN_ERR_INVALID_ARG, "dD needs D_skip");
    const int64_t rows = p->batch * p->dim;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (rows > 0 && p->seqlen > 0 &&
        (!u || !delta_raw || !A || !B || !C || !dout || !du || !ddelta_raw || !dB || !dC))
        return fail(SSCAN_ERR_INVALID_ARG, "u, delta_raw, A, B, C, dout, du, ddelta_raw, dB, dC are required");
    if (p->dim > 0 && !dA) return fail(SSCAN_ERR_INVALID_ARG, "dA is required");
    const size_t need = sscan_workspace_size(p, SSCAN_OP_BWD);
    if (sscan_status s = check_workspace(need, workspace, workspace_bytes)) return s;
    const int64_t DN = p->dim * p->dstate, BLN = p->batch * p->seqlen * p->dstate;
    // parameter gradients are sums: start them at zero
    cudaError_t e = cudaSuccess;
    if (DN > 0) e = cudaMemsetAsync(dA, 0, (size_t)DN * sizeof(float), st);
    if (e == cudaSuccess && dD && p->dim > 0) e = cudaMemsetAsync(dD, 0, (size_t)p->dim * sizeof(float), st);
    if (e == cudaSuccess && ddelta_bias && p->dim > 0)
        e = cudaMemsetAsync(ddelta_bias, 0, (size_t)p->dim * sizeof(float), st);
    if (e != cudaSuccess) return fail(SSCAN_ERR_CUDA, "zeroing gradients: %s", cudaGetErrorString(e));
    if (rows == 0) {
        // no channels (D = 0) with batch * L * N > 0: dB and dC are sums over nothing
        const size_t bytes = (size_t)BLN * (p->io_dtype == SSCAN_BF16 ? 2 : 4);
        if (bytes > 0 && dB) e = cudaMemsetAsync(dB, 0, bytes, st);
        if (e == cudaSuccess && bytes > 0 && dC) e = cudaMemsetAsync(dC, 0, bytes, st);
        if (e != cudaSuccess) return fail(SSCAN_ERR_CUDA, "zeroing dB, dC: %s", cudaGetErrorString(e));
        return SSCAN_OK;
    }
    if (p->seqlen == 0) {
        if (dh0) {
            e = cudaMemsetAsync(dh0, 0, (size_t)(rows * p->dstate) * sizeof(float), st);
            if (e != cudaSuccess) return fail(SSCAN_ERR_CUDA, "zeroing dh0: %s", cudaGetErrorString(e));
        }
        return SSCAN_OK;
    }
    const sscan::BwdPlan plan = sscan::plan_bwd(p->batch, p->seqlen, p->dim, p->dstate);
    float* ws = static_cast<float*>(workspace);
    e = cudaMemsetAsync(ws, 0, (size_t)(2 * BLN) * sizeof(float), st);
    if (e != cudaSuccess) return fail(SSCAN_ERR_CUDA, "zeroing workspace: %s", cudaGetErrorString(e));
    if (bwd_tiled_ok(p, u, delta_raw, z, dout, B, C, du, ddelta_raw, dz)) {
        // checkpoint pass: the state before every 8th step, by the tiled forward kernel
        const sscan::TiledGeom geo = sscan::tiled_geometry(p->batch, p->seqlen, p->dim, p->dstate);
        sscan::TiledArgs t{};
        t.batch = p->batch;
        t.L = p->seqlen;
        t.D = p->dim;
        t.N = (int)p->dstate;
        t.softplus = (p->flags & SSCAN_DELTA_SOFTPLUS) ? 1 : 0;
        t.input_silu = (p->flags & SSCAN_INPUT_SILU) ? 1 : 0;
        t.has_z = 0;
        t.bias = delta_bias;
        t.A = A;
        t.h0 = h0;
        t.B = B;
        t.chunk_len = p->seqlen;
        t.nchunks = 1;
        t.ws_ckpt = ws + 2 * BLN;
        t.nck = (p->seqlen + sscan::kBwdTiledSeg - 1) / sscan::kBwdTiledSeg;
        sscan::TiledPtrs tp{u, delta_raw, nullptr, nullptr};
        const int bf16 = p->io_dtype == SSCAN_BF16;
        sscan::BwdTiledArgs ba{};
        ba.batch = p->batch;
        ba.L = p->seqlen;
        ba.D = p->dim;
        ba.N = (int)p->dstate;
        ba.softplus = t.softplus;
        ba.input_silu = t.input_silu;
        ba.has_z = z != nullptr;
        ba.bias = delta_bias;
        ba.A = A;
        ba.Dskip = D_skip;
        ba.ws_ckpt = t.ws_ckpt;
        ba.nck = t.nck;
        ba.dB32 = ws;
        ba.dC32 = ws + BLN;
        ba.dA = dA;
        ba.dD = dD;
        ba.dbias = ddelta_bias;
        ba.dh0 = dh0;
        ba.seg_len = plan.seg_len;
        ba.nseg = plan.nsegs;
        ba.ws_lam = ws + 2 * BLN + plan.ck_floats;
        ba.ws_dsum = ba.ws_lam + p->batch * plan.nsegs * p->dim * p->dstate;
        sscan::BwdTiledPtrs bp{u, delta_raw, z, dout, B, C, du, ddelta_raw, dz};
        if (plan.nsegs > 1) {
            // the reverse sweep split in time: segment summaries and their carry on the
            // second stream, the checkpoint pass on the caller's, joined before the
            // reverse kernel.  The checkpoint pass, the longer of the two, is launched
            // first so that its CTAs are placed before the summaries fill the SMs.
            std::lock_guard<std::mutex> lock(g_aux_mutex);
            AuxStream* ax = nullptr;
            if ((e = aux_stream(&ax)) != cudaSuccess || (e = cudaEventRecord(ax->fork, st)) != cudaSuccess ||
                (e = cudaStreamWaitEvent(ax->stream, ax->fork, 0)) != cudaSuccess)
                return fail(SSCAN_ERR_CUDA, "backward stream fork: %s", cudaGetErrorString(e));
            ++g_launches;
            e = sscan::launch_fwd_tiled(t, tp, geo, bf16, sscan::kTiledCkpt, st);
            if (e != cudaSuccess) return fail(SSCAN_ERR_CUDA, "checkpoint kernel: %s", cudaGetErrorString(e));
            ++g_launches;
            e = sscan::launch_bwd_tiled(ba, bp, bf16, sscan::kBwdSummary, ax->stream);
            if (e != cudaSuccess) return fail(SSCAN_ERR_CUDA, "backward summary kernel: %s", cudaGetErrorString(e));
            ++g_launches;
            e = sscan::launch_bwd_carry(ba, ax->stream);
            if (e != cudaSuccess) return fail(SSCAN_ERR_CUDA, "backward carry kernel: %s", cudaGetErrorString(e));
            if ((e = cudaEventRecord(ax->join, ax->stream)) != cudaSuccess ||
                (e = cudaStreamWaitEvent(st, ax->join, 0)) != cudaSuccess)
                return fail(SSCAN_ERR_CUDA, "backward stream join: %s", cudaGetErrorString(e));
        } else {
            ++g_launches;
            e = sscan::launch_fwd_tiled(t, tp, geo, bf16, sscan::kTiledCkpt, st);
            if (e != cudaSuccess) return fail(SSCAN_ERR_CUDA, "checkpoint kernel: %s", cudaGetErrorString(e));
        }
        ++g_launches;
        e = sscan::launch_bwd_tiled(ba, bp, bf16, sscan::kBwdFull, st);
        if (e != cudaSuccess) return fail(SSCAN_ERR_CUDA, "backward kernel: %s", cudaGetErrorString(e));
        if (bf16) {
            cast_out<__nv_bfloat16>(ws, dB, BLN, st);
            cast_out<__nv_bfloat16>(ws + BLN, dC, BLN, st);
        } else {
            cast_out<float>(ws, dB, BLN, st);
            cast_out<float>(ws + BLN, dC, BLN, st);
        }
        return cuda_check("gradient cast kernel");
    }
    sscan::BwdArgs g{};
    g.f = make_args(p, u, delta_raw, delta_bias, A, B, C, D_skip, z, h0, nullptr, nullptr);
    g.dout = dout;
    g.du = du;
    g.ddelta_raw = ddelta_raw;
    g.dbias = ddelta_bias;
    g.dA = dA;
    g.dD = dD;
    g.dz = dz;
    g.dh0 = dh0;
    g.nseg = plan.nseg;
    g.dB32 = ws;
    g.dC32 = ws + BLN;
    g.ckpt = ws + 2 * BLN;
    if (p->io_dtype == SSCAN_BF16) dispatch_bwd_rows<__nv_bfloat16>(g, st);
    else dispatch_bwd_rows<float>(g, st);
    if (sscan_status s = cuda_check("backward kernel")) return s;
    if (p->io_dtype == SSCAN_BF16) {
        cast_out<__nv_bfloat16>(g.dB32, dB, BLN, st);
        cast_out<__nv_bfloat16>(g.dC32, dC, BLN, st);
    } else {
        cast_out<float>(g.dB32, dB, BLN, st);
        cast_out<float>(g.dC32, dC, BLN, st);
    }
    return cuda_check("gradient cast kernel");
}

sscan_status sscan_fwd_complex(const sscan_problem* p, const void* u, const void* delta_raw,
                               const float* delta_bias, const float* A, const void* B, const void* C,
                               const float* D_skip, const void* z, const float* h0, void* out, float* h_last,
                               void* stream) {
    g_err[0] = 0;
    g_launches = 0;
    if (sscan_status s = check_problem(p)) return s;
    const int64_t rows = p->batch * p->dim;
    if (rows == 0) return SSCAN_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t state_bytes = (size_t)(rows * p->dstate * 2) * sizeof(float);
    if (p->seqlen == 0) {
        if (!h_last) return SSCAN_OK;
        const cudaError_t e = h0 ? cudaMemcpyAsync(h_last, h0, state_bytes, cudaMemcpyDeviceToDevice, st)
                                 : cudaMemsetAsync(h_last, 0, state_bytes, st);
        return e == cudaSuccess ? SSCAN_OK : fail(SSCAN_ERR_CUDA, "empty sequence: %s", cudaGetErrorString(e));
    }
    if (!u || !delta_raw || !A || !B || !C || !out)
        return fail(SSCAN_ERR_INVALID_ARG, "u, delta_raw, A, B, C and out are required");
    sscan::ComplexArgs a{};
    a.batch = p->batch;
    a.L = p->seqlen;
    a.D = p->dim;
    a.N = (int)p->dstate;
    a.softplus = (p->flags & SSCAN_DELTA_SOFTPLUS) ? 1 : 0;
    a.input_silu = (p->flags & SSCAN_INPUT_SILU) ? 1 : 0;
    a.u = u;
    a.delta_raw = delta_raw;
    a.bias = delta_bias;
    a.A = A;
    a.B = B;
    a.C = C;
    a.Dskip = D_skip;
    a.z = z;
    a.h0 = h0;
    a.out = out;
    a.h_last = h_last;
    ++g_launches;
    const cudaError_t e = sscan::launch_fwd_complex(a, nullptr, 0, p->io_dtype == SSCAN_BF16, st);
    if (e != cudaSuccess) return fail(SSCAN_ERR_CUDA, "complex forward kernel: %s", cudaGetErrorString(e));
    return SSCAN_OK;
}

sscan_status sscan_bwd_complex(const sscan_problem* p, const void* u, const void* delta_raw,
                               const float* delta_bias, const float* A, const void* B, const void* C,
                               const float* D_skip, const void* z, const float* h0, const void* dout, void* du,
                               void* ddelta_raw, float* ddelta_bias, float* dA, void* dB, void* dC, float* dD,
                               void* dz, float* dh0, void* workspace, size_t workspace_bytes, void* stream) {
    g_err[0] = 0;
    g_launches = 0;
    if (sscan_status s = check_problem(p)) return s;
    if ((z == nullptr) != (dz == nullptr)) return fail(SSCAN_ERR_INVALID_ARG, "dz must be given exactly when z is");
    if (dD && !D_skip) return fail(SSCAN_ERR_INVALID_ARG, "dD needs D_skip");
    const int64_t rows = p->batch * p->dim;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (rows > 0 && p->seqlen > 0 &&
        (!u || !delta_raw || !A || !B || !C || !dout || !du || !ddelta_raw || !dB || !dC))
        return fail(SSCAN_ERR_INVALID_ARG, "u, delta_raw, A, B, C, dout, du, ddelta_raw, dB, dC are required");
    if (p->dim > 0 && !dA) return fail(SSCAN_ERR_INVALID_ARG, "dA is required");
    if (sscan_status s = check_workspace(sscan_workspace_size(p, SSCAN_OP_BWD_COMPLEX), workspace, workspace_bytes))
        return s;
    const int64_t DN = p->dim * p->dstate, BLN = p->batch * p->seqlen * p->dstate;
    cudaError_t e = cudaSuccess;
    if (DN > 0) e = cudaMemsetAsync(dA, 0, (size_t)(2 * DN) * sizeof(float), st);
    if (e == cudaSuccess && dD && p->dim > 0) e = cudaMemsetAsync(dD, 0, (size_t)p->dim * sizeof(float), st);
    if (e == cudaSuccess && ddelta_bias && p->dim > 0)
        e = cudaMemsetAsync(ddelta_bias, 0, (size_t)p->dim * sizeof(float), st);
    if (e == cudaSuccess && rows > 0 && p->seqlen == 0 && dh0)
        e = cudaMemsetAsync(dh0, 0, (size_t)(2 * rows * p->dstate) * sizeof(float), st);
    if (rows == 0 && BLN > 0) {
        // no channels (D = 0) with batch * L * N > 0: dB and dC are sums over nothing
        const size_t bytes = (size_t)BLN * (p->io_dtype == SSCAN_BF16 ? 2 : 4);
        if (e == cudaSuccess && dB) e = cudaMemsetAsync(dB, 0, bytes, st);
        if (e == cudaSuccess && dC) e = cudaMemsetAsync(dC, 0, bytes, st);
    }
    if (e != cudaSuccess) return fail(SSCAN_ERR_CUDA, "zeroing gradients: %s", cudaGetErrorString(e));
    if (rows == 0 || p->seqlen == 0) return SSCAN_OK;
    float* ws = static_cast<float*>(workspace);
    e = cudaMemsetAsync(ws, 0, (size_t)(2 * BLN) * sizeof(float), st);
    if (e != cudaSuccess) return fail(SSCAN_ERR_CUDA, "zeroing workspace: %s", cudaGetErrorString(e));
    sscan::ComplexBwdArgs g{};
    sscan::ComplexArgs& a = g.f;
    a.batch = p->batch;
    a.L = p->seqlen;
    a.D = p->dim;
    a.N = (int)p->dstate;
    a.softplus = (p->flags & SSCAN_DELTA_SOFTPLUS) ? 1 : 0;
    a.input_silu = (p->flags & SSCAN_INPUT_SILU) ? 1 : 0;
    a.u = u;
    a.delta_raw = delta_raw;
    a.bias = delta_bias;
    a.A = A;
    a.B = B;
    a.C = C;
    a.Dskip = D_skip;
    a.z = z;
    a.h0 = h0;
    a.out = nullptr;
    a.h_last = nullptr;
    float* ckpt = ws + 2 * BLN;
    g.ckpt = ckpt;
    g.nck = (p->seqlen + 7) / 8;
    const int bf16 = p->io_dtype == SSCAN_BF16;
    // checkpoint pass: the complex forward kernel storing the state before every 8th step
    ++g_launches;
    e = sscan::launch_fwd_complex(a, ckpt, g.nck, bf16, st);
    if (e != cudaSuccess) return fail(SSCAN_ERR_CUDA, "complex checkpoint kernel: %s", cudaGetErrorString(e));
    g.dout = dout;
    g.du = du;
    g.ddelta_raw = ddelta_raw;
    g.dz = dz;
    g.dA = dA;
    g.dB32 = ws;
    g.dC32 = ws + BLN;
    g.dD = dD;
    g.dbias = ddelta_bias;
    g.dh0 = dh0;
    ++g_launches;
    e = sscan::launch_bwd_complex(g, bf16, st);
    if (e != cudaSuccess) return fail(SSCAN_ERR_CUDA, "complex backward kernel: %s", cudaGetErrorString(e));
    if (bf16) {
        cast_out<__nv_bfloat16>(ws, dB, BLN, st);
        cast_out<__nv_bfloat16>(ws + BLN, dC, BLN, st);
    } else {
        cast_out<float>(ws, dB, BLN, st);
        cast_out<float>(ws + BLN, dC, BLN, st);
    }
    return cuda_check("gradient cast kernel");
}

sscan_status sscan_step(const sscan_problem* p, const void* u, const void* delta_raw, const float* delta_bias,
                        const float* A, const void* B, const void* C, const float* D_skip, const void* z,
                        float* state, void* out, void* stream) {
    g_err[0] = 0;
    g_launches = 0;
    if (sscan_status s = check_problem(p)) return s;
    if (p->seqlen != 1) return fail(SSCAN_ERR_INVALID_ARG, "sscan_step takes seqlen == 1, got %lld", (long long)p->seqlen);
    if (p->batch * p->dim == 0) return SSCAN_OK;
    if (!u || !delta_raw || !A || !B || !C || !state || !out)
        return fail(SSCAN_ERR_INVALID_ARG, "u, delta_raw, A, B, C, state, out are required");
    sscan::StepArgs a{};
    a.batch = p->batch;
    a.D = p->dim;
    a.N = (int)p->dstate;
    a.softplus = (p->flags & SSCAN_DELTA_SOFTPLUS) ? 1 : 0;
    a.input_silu = (p->flags & SSCAN_INPUT_SILU) ? 1 : 0;
    a.u = u;
    a.delta_raw = delta_raw;
    a.bias = delta_bias;
    a.A = A;
    a.B = B;
    a.C = C;
    a.Dskip = D_skip;
    a.z = z;
    a.state = state;
    a.out = out;
    ++g_launches;
    const cudaError_t e = sscan::launch_step(a, p->io_dtype == SSCAN_BF16, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(SSCAN_ERR_CUDA, "step kernel: %s", cudaGetErrorString(e));
    return SSCAN_OK;
}

sscan_status sscan_chunk_summary(const sscan_problem* p, const void* u, const void* delta_raw,
                                 const float* delta_bias, const float* A, const void* B, float* P, float* H,
                                 void* workspace, size_t workspace_bytes, void* stream) {
    g_err[0] = 0;
    g_launches = 0;
    if (sscan_status s = check_problem(p)) return s;
    const int64_t BD = p->batch * p->dim, BDN = BD * p->dstate;
    if (BD == 0) return SSCAN_OK;
    if (!P || !H) return fail(SSCAN_ERR_INVALID_ARG, "P and H are required");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (p->seqlen == 0) {  // the identity map
        cudaError_t e = cudaMemsetAsync(H, 0, (size_t)BDN * sizeof(float), st);
        if (e != cudaSuccess) return fail(SSCAN_ERR_CUDA, "zeroing H: %s", cudaGetErrorString(e));
        sscan::fill_kernel<<<blocks_for(BDN, 256), 256, 0, st>>>(P, 1.f, BDN);
        ++g_launches;
        return cuda_check("fill kernel");
    }
    if (!u || !delta_raw || !A || !B) return fail(SSCAN_ERR_INVALID_ARG, "u, delta_raw, A, B are required");
    if (sscan_status s = check_workspace(sscan_workspace_size(p, SSCAN_OP_SUMMARY), workspace, workspace_bytes))
        return s;
    // one aggregate pass over the whole sequence: H = end state from zero, dsum = sum of delta
    sscan::ScanArgs a = make_args(p, u, delta_raw, delta_bias, A, B, nullptr, nullptr, nullptr, nullptr, nullptr,
                                  nullptr);
    a.nchunks = 1;
    a.chunk_len = p->seqlen;
    a.ws_state = H;
    a.ws_dsum = static_cast<float*>(workspace);
    if (tiled_ok(p, a)) {
        const sscan::TiledGeom geo = sscan::tiled_geometry(p->batch, p->seqlen, p->dim, p->dstate);
        sscan::TiledArgs t{};
        t.batch = p->batch;
        t.L = p->seqlen;
        t.D = p->dim;
        t.N = (int)p->dstate;
        t.softplus = a.softplus;
        t.input_silu = a.input_silu;
        t.bias = delta_bias;
        t.A = A;
        t.B = B;
        t.chunk_len = p->seqlen;
        t.nchunks = 1;
        t.ws_state = H;
        t.ws_dsum = a.ws_dsum;
        sscan::TiledPtrs tp{u, delta_raw, nullptr, nullptr};
        ++g_launches;
        const cudaError_t e = sscan::launch_fwd_tiled(t, tp, geo, p->io_dtype == SSCAN_BF16, sscan::kTiledAgg, st);
        if (e != cudaSuccess) return fail(SSCAN_ERR_CUDA, "aggregate kernel: %s", cudaGetErrorString(e));
    } else {
        fwd_rows(a, p->io_dtype, sscan::kModeAggregate, st);
        if (sscan_status s = cuda_check("aggregate kernel")) return s;
    }
    sscan::decay_kernel<<<blocks_for(BDN, 128), 128, 0, st>>>(a.ws_dsum, A, P, p->batch, p->dim, p->dstate);
    ++g_launches;
    return cuda_check("decay kernel");
}

sscan_status sscan_carry(const sscan_problem* p, int64_t nchunks, const float* P, const float* H, const float* h0,
                         float* carry_in, float* h_final, void* stream) {
    g_err[0] = 0;
    g_launches = 0;
    if (sscan_status s = check_problem(p)) return s;
    if (nchunks < 0) return fail(SSCAN_ERR_INVALID_ARG, "nchunks must be >= 0");
    const int64_t BDN = p->batch * p->dim * p->dstate;
    if (BDN == 0 || (!carry_in && !h_final)) return SSCAN_OK;
    if (nchunks > 0 && (!P || !H)) return fail(SSCAN_ERR_INVALID_ARG, "P and H are required");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int W = sscan::affine_lanes(nchunks);
    sscan::compose_kernel<<<blocks_for(BDN * W, 128), 128, 0, st>>>(P, H, h0, carry_in, h_final, nchunks, BDN, W);
    ++g_launches;
    return cuda_check("compose kernel");
}

const char* sscan_status_string(sscan_status s) {
    switch (s) {
        case SSCAN_OK: return "SSCAN_OK";
        case SSCAN_ERR_INVALID_ARG: return "SSCAN_ERR_INVALID_ARG";
        case SSCAN_ERR_UNSUPPORTED: return "SSCAN_ERR_UNSUPPORTED";
        case SSCAN_ERR_WORKSPACE: return "SSCAN_ERR_WORKSPACE";
        case SSCAN_ERR_CUDA: return "SSCAN_ERR_CUDA";
        case SSCAN_ERR_TIMEOUT: return "SSCAN_ERR_TIMEOUT";
        default: return "SSCAN_ERR_UNKNOWN";
    }
}

const char* sscan_last_error(void) { return g_err; }

int sscan_last_launch_count(void) { return g_launches; }

int sscan_debug_bounds(void) {
#ifdef SSCAN_DEBUG_BOUNDS
    return 1;
#else
    return 0;
#endif
}

sscan_status sscan_device_status(int clear, unsigned int* flags) {
    g_err[0] = 0;
    if (!flags) return fail(SSCAN_ERR_INVALID_ARG, "flags is NULL");
    unsigned int f1 = 0, f2 = 0, f3 = 0;
    cudaError_t e = sscan::read_device_error(&f1, clear);
    if (e == cudaSuccess) e = sscan::read_device_error_bwd(&f2, clear);
    if (e == cudaSuccess) e = sscan::read_device_error_cx(&f3, clear);
    if (e != cudaSuccess) return fail(SSCAN_ERR_CUDA, "reading the device error word: %s", cudaGetErrorString(e));
    *flags = f1 | f2 | f3;
    return *flags ? SSCAN_ERR_TIMEOUT : SSCAN_OK;
}

int sscan_version(void) { return 100; }

}  // extern "C"
