/*
 * sscan_probe.h -- diagnostics shipped with libsscan: a throughput probe for the
 * MUFU ex2 pipe, the unit that bounds the selective-scan forward pass (N
 * exponentials per element for Abar = exp(delta A), eq. (2) of the Mamba technical
 * summary page, sec. 2.1), and a self-test of the kernels' bounded-wait failure
 * reporting.  Neither computes anything of the scan; neither has a counterpart on
 * the pages.
 */
#ifndef SSCAN_PROBE_H
#define SSCAN_PROBE_H

#include <stdint.h>

#include "sscan.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Enqueue `blocks` x `threads` threads, each issuing `iters` rounds of 8
 * independent ex2.approx.ftz.f32 (8 * iters exponentials per thread), and store
 * one float per thread to `sink` (device, blocks * threads floats, caller-owned)
 * so the work is not removed.  Returns SSCAN_ERR_INVALID_ARG for non-positive
 * sizes or a NULL sink, SSCAN_ERR_CUDA if the launch fails.
 */
SSCAN_API sscan_status sscan_probe_ex2(float* sink, int64_t iters, int blocks, int threads, void* stream);

/*
 * Exercise the failure path of the kernels' bounded waits: enqueue one thread that
 * waits, polling at most `polls` times (1 .. 2^20), on a shared-memory mbarrier
 * that nothing arrives on, then sets bit 2 of the device status word read by
 * sscan_device_status.  Nothing is in flight on the barrier, so the kernel simply
 * returns and the context stays usable.  Returns SSCAN_ERR_INVALID_ARG for polls
 * out of range, SSCAN_ERR_CUDA if the launch fails.
 */
SSCAN_API sscan_status sscan_probe_wait_timeout(unsigned int polls, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SSCAN_PROBE_H */
