// ssm_internal.h -- argument bundles passed from the C ABI layer (abi.cu),
// which has already validated them, to the kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace ssm {

struct StateUpdateArgs {
    int batch, nheads, head_dim, d_state, ngroups;
    int in_dtype, y_dtype;        // 0 = fp32, 1 = bf16
    void *state;                  // fp32, or fp16 when rp.f16
    const void *x;
    const float *dt, *A;
    const void *B, *C;
    const float *D;
    void *y;
    // slot-indexed state pool (nullptr: row b of the state is batch row b)
    const int32_t *slot_idx;      // device [batch]; < 0 skips the row
    int max_slots;
    int *status_dev;
    DtParams dtp;                 // transform of dt (identity when all off)
    RoundParams rp;               // state storage (fp32, or fp16 and its rounding)
};

// Speculative (multi-token) decode: ntok draft tokens per batch row, in
// order, from the row's state; optional outputs per token.
struct MultiUpdateArgs {
    int batch, ntok, nheads, head_dim, d_state, ngroups;
    int in_dtype, y_dtype;
    float *state;                 // [rows][H][P][N] (rows = batch, or max_slots)
    const int32_t *slot_idx;      // device [batch] or nullptr; < 0 = padding
    int max_slots;
    const void *x;                // [batch][ntok][H][P]
    const float *dt, *A;          // dt [batch][ntok][H]
    const void *B, *C;            // [batch][ntok][G][N]
    const float *D;
    DtParams dtp;
    const int32_t *accept_len;    // device [batch] or nullptr (state not written)
    float *inter;                 // [batch][ntok][H][P][N] or nullptr
    void *y;                      // [batch][ntok][H][P] or nullptr
    int *status_dev;
};

// Scatter of accepted intermediate states into the state rows.
struct CommitArgs {
    int batch, ntok, nheads, head_dim, d_state;
    const float *inter;           // [batch][ntok][H][P][N]
    const int32_t *accept_len;    // device [batch]
    float *state;
    const int32_t *slot_idx;
    int max_slots;
    int *status_dev;
};

struct ScanArgs {
    int nseq, seqlen;             // seqlen = T when cu_seqlens is given
    const int32_t *cu_seqlens;    // device [nseq+1] or nullptr
    int nheads, head_dim, d_state, ngroups, chunk_size;
    int in_dtype, y_dtype;
    const void *x;
    const float *dt, *A;
    const void *B, *C;
    const float *D;
    const void *initial_state;    // nullptr = zero; fp32, or fp16 when rp.f16
    void *y;
    void *final_state;            // nullptr = not written; same storage type
    int *status_dev;              // nullptr = not reported
    // slot-indexed state pool: sequence s reads and writes state row
    // slot_idx[s] of initial_state / final_state (the same pool); nullptr
    // means row s.  has_initial[s] == 0 starts sequence s from zero.
    const int32_t *slot_idx;
    const int32_t *has_initial;
    int max_slots;
    DtParams dtp;
    RoundParams rp;
    // Failure-path testing only (both 0 in every entry point but the
    // testing hooks of ssm_testing.h): limit of the bounded waits in ns
    // (0 = the 2 s default), and a producer that issues no load or MMA.
    unsigned long long wait_ns;
    int stall_producer;
    // Balanced schedule of the tensor-core scan (fixed-length batches only):
    // `runs` CTAs split the chains (sequence, head pair) laid end to end into
    // runs of equal chunk counts, handing the carried state across each cut
    // through `handoff` (runs slots of 2 x head_dim x d_state fp32) and
    // `handoff_flags` (runs ints, zeroed before the launch).  runs == 0: one
    // CTA per chain.
    int runs;
    float *handoff;
    int *handoff_flags;
};

// Causal depthwise conv1d (prefill over packed sequences, or one decode token
// per batch row when update != 0; then nseq is the batch).
struct ConvArgs {
    int update;
    // decode only: ntok tokens per row (x, y [batch][ntok][dim]); the state
    // row is rewritten after accept_len[b] tokens, after all of them when
    // commit_all is set, or not at all.
    int ntok, commit_all;
    const int32_t *accept_len;
    int nseq, seqlen;             // seqlen = T when cu_seqlens is given
    const int32_t *cu_seqlens;
    int dim, width, activation;   // activation: 0 none, 1 SiLU
    int in_dtype, y_dtype;
    const void *x;
    const float *weight;          // [dim][width]
    const float *bias;            // [dim] or nullptr
    void *state;                  // [rows][dim][width-1], in_dtype, or nullptr
    const int32_t *slot_idx;      // rows map, or nullptr
    const int32_t *has_initial;
    int max_slots;
    void *y;
    int *status_dev;
    // Failure-path testing only, as for ScanArgs (the pipelined prefill kernel).
    unsigned long long wait_ns;
    int stall_producer;
};

cudaError_t launch_state_update(const StateUpdateArgs &a, cudaStream_t stream);
cudaError_t launch_conv1d(const ConvArgs &a, cudaStream_t stream);
cudaError_t launch_state_update_multi(const MultiUpdateArgs &a, cudaStream_t stream);
cudaError_t launch_state_commit(const CommitArgs &a, cudaStream_t stream);

// Gated group RMSNorm (gate first): out = g / sqrt(mean_group(g^2) + eps) * w,
// g = y * silu(z), over groups of group_size channels of each row.
struct GatedNormArgs {
    int rows, dim, group_size;
    int y_dtype, z_dtype, out_dtype;
    const void *y, *z;
    const float *weight;
    float eps;
    void *out;
};
cudaError_t launch_gated_rmsnorm(const GatedNormArgs &a, cudaStream_t stream);

// General chunked scan on the CUDA cores: any supported shape and dtype.
cudaError_t launch_scan_simt(const ScanArgs &a, cudaStream_t stream);

// Tensor-core (tcgen05 / TMEM / TMA) chunked scan.  Returns
// cudaErrorNotSupported, launching nothing, for shapes it does not cover.
bool scan_tc_supports(const ScanArgs &a);
bool scan_tc_shape(int head_dim, int d_state, int chunk_size, int nheads, int ngroups);
cudaError_t launch_scan_tc(const ScanArgs &a, cudaStream_t stream);
// Balanced schedule: the number of runs (CTAs) for fixed-length sequences of
// these sizes on the current device (0: one CTA per chain), and the hand-off
// workspace it needs.
int scan_tc_balanced_runs(int nseq, int seqlen, int nheads);
// The same decision for a device of `sms` SMs (pure host arithmetic).
int scan_tc_balanced_runs_for(int nseq, int seqlen, int nheads, int sms);
size_t scan_tc_handoff_bytes(int runs);

}  // namespace ssm
