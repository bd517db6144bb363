// sscan_plan.h -- host-side planning: how a problem is split across the GPU and
// how much workspace each operation needs.  Pure integer arithmetic, identical
// for sscan_workspace_size() and the operations themselves.
#pragma once

#include <cstddef>
#include <cstdint>

namespace sscan {

constexpr int kMaxState = 16;
constexpr int kSmCount = 148;               // B200
constexpr int64_t kSmemPerSm = 228 * 1024;  // shared memory per SM (B200)
constexpr int64_t kSmemPerCtaReserved = 1024;  // reserved by the system per resident CTA
constexpr int64_t kRowsFillGpu = 16384;     // rows that keep every sub-partition busy
constexpr int64_t kTargetThreads = (int64_t)kSmCount * 4 * 32 * 4;  // 4 warps per sub-partition
constexpr int64_t kMinChunk = 512;          // shortest sequence chunk worth a carry
constexpr int kBwdSeg = 16;                 // steps between backward checkpoints

inline size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

struct FwdPlan {
    int64_t nchunks;
    int64_t chunk_len;
    int64_t state_floats;  // floats of chunk end states (then carry-ins)
    size_t workspace_bytes;
};

// Split L into chunks only when the rows alone cannot fill the GPU; each extra
// chunk costs one more pass over its steps (the chunk aggregate), so chunks are
// kept long.
inline FwdPlan plan_fwd(int64_t batch, int64_t L, int64_t D, int64_t N) {
    FwdPlan p{1, L, 0, 0};
    const int64_t rows = batch * D;
    if (rows <= 0 || L <= 0 || rows >= kRowsFillGpu) return p;
    int64_t want = (kTargetThreads + rows - 1) / rows;
    const int64_t most = L / kMinChunk;
    if (want > most) want = most;
    if (want <= 1) return p;
    p.chunk_len = (L + want - 1) / want;
    p.nchunks = (L + p.chunk_len - 1) / p.chunk_len;
    if (p.nchunks <= 1) return FwdPlan{1, L, 0, 0};
    p.state_floats = batch * p.nchunks * D * N;
    const int64_t dsum_floats = batch * p.nchunks * D;
    p.workspace_bytes = align256((size_t)(p.state_floats + dsum_floats) * sizeof(float));
    return p;
}

// Plan of the tiled forward kernel: CTAs cover DC channels of one batch; the
// sequence is split only when there are too few CTA columns to occupy the GPU.
constexpr int64_t kTiledMinCols = 2 * kSmCount;     // below this, split the sequence
// Target CTA count of a split: chunks enough for several waves of 8 CTAs per SM.  The CTAs
// of an SM finish in launch order, so a single wave of long chunks leaves the SMs short of
// work for its last ~30%; shorter chunks over more waves keep them fed at the cost of a
// longer carry (at the million-step shape: 8 per SM 19.50 ms, 16 17.49, 32 16.58, 64 16.28,
// 128 16.26).  The fixed-scratch entry point plans with the one-wave target, which bounds
// its chunk states (see kTiledTargetCtasCompact).
constexpr int64_t kTiledTargetCtas = 64 * kSmCount;
constexpr int64_t kTiledTargetCtasCompact = 8 * kSmCount;
constexpr int64_t kTiledMinChunk = 1024;            // steps
constexpr int64_t kTiledStep = 64;                  // chunk lengths are whole tiles of any length

inline FwdPlan plan_tiled(int64_t batch, int64_t L, int64_t D, int64_t N, int64_t DC,
                          int64_t target = kTiledTargetCtas) {
    FwdPlan p{1, L, 0, 0};
    const int64_t cols = batch * ((D + DC - 1) / DC);
    if (cols <= 0 || L <= 0 || cols >= kTiledMinCols) return p;
    int64_t want = (target + cols - 1) / cols;
    const int64_t most = L / kTiledMinChunk;
    if (want > most) want = most;
    if (want <= 1) return p;
    int64_t len = (L + want - 1) / want;
    len = (len + kTiledStep - 1) / kTiledStep * kTiledStep;
    p.chunk_len = len;
    p.nchunks = (L + len - 1) / len;
    if (p.nchunks <= 1) return FwdPlan{1, L, 0, 0};
    p.state_floats = batch * p.nchunks * D * N;
    p.workspace_bytes = align256((size_t)(p.state_floats + batch * p.nchunks * D) * sizeof(float));
    return p;
}

struct BwdPlan {
    int64_t nseg;           // general kernel: checkpoint segments per row
    int64_t ck_floats;      // checkpoint floats (general or tiled layout, the larger)
    int64_t seg_len;        // tiled kernel: steps per reverse-sweep segment
    int64_t nsegs;          // tiled kernel: reverse-sweep segments
    size_t workspace_bytes;
};

// The tiled backward gives every channel 1, 2 or 4 lanes (4 states each), so a CTA
// of 4 warps holds 128, 64 or 32 channels of one batch, and 5 CTAs fit an SM.
// When batch x channel blocks leave the GPU short of that, the reverse sweep is
// split in time into segments, each started from the adjoint state its right
// neighbours pass in (one summary pass over all but the first segment, plus a
// carry).  The segment count fills the resident slots best over whole waves (up to
// kBwdMaxSegs); segments are whole checkpoint tiles of at least kBwdMinSeg steps.
constexpr int kBwdTiledSeg = 8;
constexpr int64_t kBwdSlots = 5 * kSmCount;
constexpr int64_t kBwdMinSeg = 128;
constexpr int64_t kBwdMaxSegs = 8;

inline int64_t bwd_tiled_channels(int64_t N) {
    const int64_t ng = N <= 4 ? 1 : (N <= 8 ? 2 : 4);
    return 4 * (32 / ng);
}

// fp32 accumulators for dB and dC (batch, L, N); checkpointed states (one every
// kBwdSeg steps of every row for the general kernel, one every kBwdTiledSeg steps
// for the tiled kernel; the workspace covers either); then, for the tiled kernel's
// segments, their adjoint summaries [batch][nsegs][D][N] and delta sums
// [batch][nsegs][D].
inline BwdPlan plan_bwd(int64_t batch, int64_t L, int64_t D, int64_t N) {
    BwdPlan p{0, 0, 0, 1, 0};
    if (batch * D <= 0 || L <= 0) return p;
    p.nseg = (L + kBwdSeg - 1) / kBwdSeg;
    const int64_t nck = (L + kBwdTiledSeg - 1) / kBwdTiledSeg;
    p.ck_floats = (batch * D * p.nseg * N > batch * nck * D * N) ? batch * D * p.nseg * N : batch * nck * D * N;
    p.seg_len = L;
    const int64_t cols = batch * ((D + bwd_tiled_channels(N) - 1) / bwd_tiled_channels(N));
    int64_t want = 1;
    if (cols < kBwdSlots) {
        // fraction of slot-time used over whole waves: cols n / (waves * slots)
        double best = (double)cols / (double)kBwdSlots;
        const int64_t most = L / kBwdMinSeg < kBwdMaxSegs ? L / kBwdMinSeg : kBwdMaxSegs;
        for (int64_t n = 2; n <= most; ++n) {
            const int64_t ctas = cols * n, waves = (ctas + kBwdSlots - 1) / kBwdSlots;
            const double eff = (double)ctas / (double)(waves * kBwdSlots);
            if (eff > best * 1.05) {
                best = eff;
                want = n;
            }
        }
    }
    if (want > 1) {
        int64_t len = (L + want - 1) / want;
        len = (len + kBwdTiledSeg - 1) / kBwdTiledSeg * kBwdTiledSeg;
        p.seg_len = len;
        p.nsegs = (L + len - 1) / len;
    }
    const int64_t seg_floats = p.nsegs > 1 ? batch * p.nsegs * D * (N + 1) : 0;
    const size_t floats = (size_t)(2 * batch * L * N) + (size_t)p.ck_floats + (size_t)seg_floats;
    p.workspace_bytes = align256(floats * sizeof(float));
    return p;
}

}  // namespace sscan
