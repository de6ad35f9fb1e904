/*
 * ssm_testing.h -- testing hooks of libssm for the failure path of the
 * kernels' bounded waits.
 *
 * The pipelined kernels (the tensor-core ssd_chunk_scan and the bulk-copy
 * ring of causal_conv1d_fwd) wait on mbarriers that a producer thread arms
 * with TMA or bulk copies.  Every such wait is bounded (2 s of wall time by
 * default).  When one expires, the CTA raises an abort flag in shared
 * memory, its producer stops issuing loads and MMAs, the other threads skip
 * their remaining waits, the producer waits (again bounded) for the copies
 * and MMAs it had already issued, and the kernel writes SSM_ERR_TIMEOUT to
 * the status word and exits with nothing left in flight.  The context stays
 * usable.
 *
 * These two entry points run those kernels with their producer disabled (it
 * issues no load and no MMA) and a caller-chosen short wait limit, so that
 * the first wait of every CTA expires: a test then checks that the call
 * returns, that *status_dev reads SSM_ERR_TIMEOUT and that the device still
 * runs later work.  They are not part of the scan's interface; the outputs
 * they write are meaningless.  The operation itself has no counterpart in
 * the pages the library follows: it exists to exercise the timeout path
 * without faulting or hanging a GPU.
 *
 * ssm_testing_balanced_runs exposes, for host-only tests, the rule by which
 * ssd_chunk_scan_workspace_size decides whether a fixed-length batch gets
 * the balanced schedule, for a device of a given SM count.
 */
#ifndef LIBSSM_SSM_TESTING_H
#define LIBSSM_SSM_TESTING_H

#include "ssm.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * ssm_testing_scan_stalled -- the tensor-core ssd_chunk_scan kernel with a
 * stalled producer, on nseq sequences of seqlen tokens (no cu_seqlens).
 *   x [T][nheads][64] bf16, dt [T][nheads] fp32, A [nheads] fp32,
 *   B, C [T][ngroups][128] bf16, y [T][nheads][64] bf16 (written with
 *   meaningless values): device pointers, 16-byte aligned.
 *   nheads / ngroups must be even (the tensor-core kernel's shape rule).
 *   wait_ns: limit of each bounded wait, in [1e3, 1e10] ns.
 *   status_dev: device int32, required; zeroed by the caller, set to
 *   SSM_ERR_TIMEOUT by the kernel.
 * Returns SSM_ERR_INVALID_ARG / SSM_ERR_MISALIGNED / SSM_ERR_UNSUPPORTED
 * before launching anything when an argument is wrong, else the launch status.
 */
SSM_API int ssm_testing_scan_stalled(int nseq, int seqlen, int nheads, int ngroups,
                                     const void *x, const float *dt, const float *A,
                                     const void *B, const void *C, void *y,
                                     unsigned long long wait_ns, int *status_dev,
                                     cudaStream_t stream);

/*
 * ssm_testing_conv1d_stalled -- the bulk-copy ring kernel of
 * causal_conv1d_fwd with a stalled producer, on nseq sequences of seqlen
 * tokens, bf16 x and y [T][dim] (dim a multiple of 8), fp32 weight
 * [dim][width] (width 1..8), no conv state, no bias, no activation.
 * wait_ns and status_dev as above.
 */
/*
 * ssm_testing_balanced_runs -- the number of runs (one per SM) into which
 * ssd_chunk_scan cuts the (sequence, head pair) chains of a fixed-length
 * batch of nseq sequences of seqlen tokens and nheads heads on a device of
 * `sms` SMs, or 0 when it keeps one CTA per chain: with no more chains than
 * SMs, or when the last wave of chains fills at least nine tenths of the
 * SMs.  Host arithmetic only; no device is used.
 */
SSM_API int ssm_testing_balanced_runs(int nseq, int seqlen, int nheads, int sms);

SSM_API int ssm_testing_conv1d_stalled(int nseq, int seqlen, int dim, int width,
                                       const void *x, const float *weight, void *y,
                                       unsigned long long wait_ns, int *status_dev,
                                       cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* LIBSSM_SSM_TESTING_H */
