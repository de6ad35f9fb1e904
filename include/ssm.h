/*
 * ssm.h -- C ABI of libssm, the B200 (sm_100a) Mamba-2 selective state-space
 * scan.
 *
 * The operation (the selective-SSM recurrence of the note "Mamba 与 Nemotron
 * 系列模型深度调研", section "1. Selective SSM 的直觉"; its decode form in the
 * modeling_nemotron_h.py walk-through, section "Decode 阶段"): for every
 * sequence, head h (group g = h / (nheads / ngroups)) and token t in order,
 *
 *     state[p][n] <- exp(dt[t][h] * A[h]) * state[p][n] + dt[t][h] * x[t][h][p] * B[t][g][n]
 *     y[t][h][p]   = sum_n state[p][n] * C[t][g][n] + D[h] * x[t][h][p]
 *
 * y reads the state AFTER the token's update.  A and D are per-head fp32
 * scalars, dt is the final per-(token, head) step size in fp32 (already passed
 * through any bias / softplus / clamp), and B, C are shared by the heads of a
 * group.  The recurrent state is always fp32 (the walk-through's section on
 * why the SSM cache defaults to float32).
 *
 * Layouts (row-major, contiguous, no padding between rows):
 *   x, y          [T][nheads][head_dim]
 *   dt            [T][nheads]               fp32
 *   A, D          [nheads]                  fp32
 *   B, C          [T][ngroups][d_state]
 *   state         [nseq or batch][nheads][head_dim][d_state]   fp32
 * where T is the number of tokens (for decode, T = batch).
 *
 * Ownership: the caller allocates every buffer and owns it.  No entry point
 * allocates device memory, synchronises the device or the stream, or keeps
 * state between calls; all work is enqueued on the given stream.  Pointers
 * marked "device" must be device-accessible (cudaMalloc'd or managed).
 *
 * Errors: shapes, dtypes, null pointers and alignment are checked on the host
 * BEFORE anything is launched; on any error nothing is launched and the call
 * returns the status.  A launch failure returns SSM_ERR_CUDA (from
 * cudaGetLastError, no synchronisation).  Problems only the device can see
 * (inconsistent cu_seqlens) are reported through the optional status word.
 */
#ifndef LIBSSM_SSM_H
#define LIBSSM_SSM_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define SSM_API __attribute__((visibility("default")))
#else
#define SSM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SSM_OK = 0,
    SSM_ERR_INVALID_ARG = 1,   /* bad shape, null pointer, aliasing, range */
    SSM_ERR_UNSUPPORTED = 2,   /* valid request this build does not handle */
    SSM_ERR_MISALIGNED = 3,    /* a pointer is not 16-byte aligned */
    SSM_ERR_CUDA = 4,          /* the CUDA runtime reported a launch error */
    SSM_ERR_TIMEOUT = 5,       /* written to status_dev: a bounded device wait expired */
    SSM_ERR_DEVICE_INPUT = 6,  /* written to status_dev: bad cu_seqlens or slot index */
    SSM_ERR_RANGE = 7,         /* written to status_dev: a value beyond the fp16 range of the
                                  tensor-core operands made y non-finite (see ssd_chunk_scan) */
    SSM_ERR_INTERNAL = 8,      /* written to status_dev: a launch broke a kernel's own layout
                                  rule (e.g. shared-memory alignment); nothing was computed */
    SSM_ERR_SCRATCH_LIMIT = 9  /* ssd_chunk_scan_noalloc: the shapes need more workspace than
                                  the library's built-in scratch holds; nothing launched */
} ssm_status;

typedef enum {
    SSM_F32 = 0,
    SSM_BF16 = 1,
    SSM_F16 = 2    /* state pools only (the *_slots entry points) */
} ssm_dtype;

/*
 * Optional transform of dt inside the kernels that read it, so that the raw
 * dt of the input projection can be passed (the dt_bias input of the
 * TensorRT MambaPlugin, deep-research note section "TensorRT Plugin 做
 * selective state update"; softplus and the time-step clamp of the Mamba-2
 * mixer).  Per (token, head h):
 *     v = dt + dt_bias[h]          (dt_bias: device fp32 [nheads], or NULL)
 *     v = log(1 + e^v)             (if softplus; v itself above 20)
 *     v = min(max(v, dt_min), dt_max)   (if clamp; dt_min <= dt_max)
 * A NULL ssm_dt_params pointer means dt is already final.
 */
typedef struct {
    const float *dt_bias;
    int softplus;
    int clamp;
    float dt_min, dt_max;
} ssm_dt_params;

/*
 * Stochastic rounding of an fp16 state pool (the float16 SSM cache with
 * stochastic rounding and Philox rounds of the deployment flags listed in the
 * modeling_nemotron_h.py walk-through, section "部署时如何调这些缓存").  The
 * state is computed in fp32 and rounded to fp16 when it is written: a value
 * moves to its fp16 neighbour away from zero iff u < frac, frac being its
 * distance from the neighbour toward zero in units of the fp16 spacing there
 * and u = r16 / 2^16 for 16 random bits r16; magnitudes beyond 65504
 * saturate.  The 16 bits of state element e (its index in the pool) are half
 * e % 2 (0 = the low half) of 32-bit word (e % 8) / 2 of one Philox-4x32
 * output with philox_rounds rounds (10 = the published Philox-4x32-10),
 * key = seed (low word first), counter = (e / 8 as 64 bits, offset as 64
 * bits; low words first), so one generator call serves 8 adjacent elements.
 * Callers pass a fresh offset per call (e.g. the decode step).  A NULL
 * ssm_rounding pointer means round to nearest even.
 */
typedef struct {
    uint64_t seed;
    uint64_t offset;
    int philox_rounds;   /* 1 .. 16 */
} ssm_rounding;

/* Human-readable name of a status code (static string, never NULL). */
SSM_API const char *ssm_status_string(int status);

/* Library version as major*10000 + minor*100 + patch (200 = 0.2.0). */
SSM_API int ssm_version(void);

/*
 * ssd_chunk_scan -- prefill: the recurrence over whole sequences, computed as
 * a chunked SSD (structured state-space duality) scan.  Chunks of chunk_size
 * tokens restart at every sequence start; inside a chunk the token-to-token
 * interactions form a decay-masked C.B^T product on the tensor cores, and the
 * state is carried from chunk to chunk on chip.  This is the
 * mamba_chunk_scan_combined(..., return_final_states=True) step of the
 * walk-through's section "Prefill 阶段" (128-token chunks), and the in-place
 * initial/final state of the MAX mamba2_ssd_chunk_scan_varlen_fwd_inplace
 * kernel (MAX nemotron_h article, section 5.4 item 3).
 *
 * Sequences:
 *   cu_seqlens == NULL: nseq sequences of seqlen tokens each, T = nseq*seqlen.
 *   cu_seqlens != NULL: device int32 [nseq+1], packed varlen; cu[0] = 0,
 *     non-decreasing, cu[nseq] = seqlen = T (seqlen is then the total).  A
 *     device-side inconsistency (cu[0] != 0, a decreasing offset, cu[nseq] !=
 *     seqlen) skips the affected sequences and writes SSM_ERR_DEVICE_INPUT to
 *     *status_dev when status_dev is given.
 *
 * Shapes: nheads % ngroups == 0; head_dim in {16, 32, 64, 128};
 *   d_state in {16, 32, 64, 128}; chunk_size in {64, 128}; seqlen >= 0.
 * in_dtype: storage type of x, B and C (SSM_BF16 or SSM_F32).  dt, A, D are
 *   always fp32.  Accumulation is fp32; bf16 operands of the tensor-core
 *   products are carried as fp16 (exact for |v| < 65504) so that derived
 *   operands (decay-masked C.B^T, decay-weighted x, the carried state) keep
 *   11 significant bits.
 * Range of the tensor-core path (bf16 x/B/C, head_dim 64, d_state 128,
 *   chunk 128, an even number of heads per group): x, B, C, every
 *   decay-masked C.B^T entry dt_j exp(cs_i - cs_j) C_i.B_j and every carried
 *   state entry must stay below 65504 in magnitude.  Beyond it an fp16
 *   operand becomes infinite, y of the affected chunks is not valid, and the
 *   kernel writes SSM_ERR_RANGE to *status_dev (the final state, computed
 *   from x, B and the decay weights only, stays valid unless x or B is out of
 *   range).  Values below 2^-14 keep an absolute precision of 2^-25.  Every
 *   other shape and fp32 inputs run in fp32 on the CUDA cores, without this
 *   limit.
 * D: device [nheads] or NULL (no skip term).
 * initial_state: device fp32 [nseq][nheads][head_dim][d_state] or NULL (zero).
 *   It may be the same pointer as final_state (in-place update of a state
 *   slot); any other overlap with an output is rejected.
 * y: device [T][nheads][head_dim], y_dtype (SSM_F32 or SSM_BF16, round to
 *   nearest even).  Must not overlap any input.
 * final_state: device fp32 [nseq][nheads][head_dim][d_state] or NULL.
 * workspace / workspace_bytes: optional device scratch of at least
 *   ssd_chunk_scan_workspace_size(...) bytes (16-byte aligned, not overlapping
 *   any argument), or NULL / 0.  With it, fixed-length batches on the
 *   tensor-core path run a balanced schedule: the (sequence, head pair)
 *   chains laid end to end are cut into one run per SM, and the carried state
 *   crosses each cut through the workspace (one fp32 [2][head_dim][d_state]
 *   slot and one flag per run; the flags are zeroed on `stream` before the
 *   launch).  Without it, or for packed varlen input, each chain runs in one
 *   CTA.  The results are identical either way (the same chunk arithmetic in
 *   the same order).  Calls that share a workspace must not overlap on the
 *   GPU.
 * status_dev: device int32 or NULL; the kernels only ever write a nonzero
 *   status into it (the caller zeroes it).
 * stream: the CUDA stream to enqueue on (0 = legacy default stream).
 * All device pointers must be 16-byte aligned (SSM_ERR_MISALIGNED).
 */
SSM_API int ssd_chunk_scan(int nseq, int seqlen, const int32_t *cu_seqlens,
                   int nheads, int head_dim, int d_state, int ngroups,
                   int chunk_size, int in_dtype,
                   const void *x, const float *dt, const float *A,
                   const void *B, const void *C, const float *D,
                   const float *initial_state,
                   int y_dtype, void *y, float *final_state,
                   void *workspace, size_t workspace_bytes,
                   int *status_dev, cudaStream_t stream);

/* Workspace bytes ssd_chunk_scan can use for these shapes on the current
 * device.  0 when no workspace helps: other shapes; no more chains than SMs
 * (one wave, where every chain is already its own critical path); or chains
 * that fill their last wave of SMs to nine tenths or more. */
SSM_API size_t ssd_chunk_scan_workspace_size(int nseq, int seqlen, int nheads,
                                     int head_dim, int d_state, int ngroups,
                                     int chunk_size);

/* Size of the scratch built into the library for ssd_chunk_scan_noalloc
 * (one static device array per device the library runs on). */
#define SSM_NOALLOC_SCRATCH_BYTES ((size_t)10 << 20)

/*
 * ssd_chunk_scan_noalloc -- ssd_chunk_scan whose workspace comes from scratch
 * memory built into the library rather than from the caller.  The method has
 * no counterpart to this: it is a convenience of the library.
 *
 * It exists for callers that cannot provide device memory: C or C++ hosts
 * that have no device allocator of their own, and serving processes whose
 * device memory is already reserved by another framework's pool, where a
 * cudaMalloc would take memory outside that pool and a cudaFree would
 * synchronise the device.  Nothing in this call allocates.  The balanced
 * schedule's hand-off slots and flags (ssd_chunk_scan_workspace_size bytes)
 * live in a static device array of SSM_NOALLOC_SCRATCH_BYTES.
 *
 * Arguments, layouts, results and statuses are those of ssd_chunk_scan with
 * that scratch as the workspace; the results are identical.  Shapes that
 * need no workspace run as ssd_chunk_scan does without one.  Shapes whose
 * workspace would exceed the scratch return SSM_ERR_SCRATCH_LIMIT and
 * launch nothing.
 *
 * Setup: the first call on each device, made with that device current,
 * looks up the scratch's device address with cudaGetSymbolAddress (which
 * loads the library's device code on that device if it is not loaded yet)
 * and keeps it for later calls; a failed lookup returns SSM_ERR_CUDA.  Make
 * that first call before any stream capture begins.  Each call zeroes the
 * hand-off flags on `stream` with a memset before its launch; the slots need
 * no clearing.
 *
 * There is one scratch per device: calls whose work overlaps on the GPU
 * (launched on different streams, or from different host threads, without
 * ordering between them) race on it, so the caller must order them.
 */
SSM_API int ssd_chunk_scan_noalloc(int nseq, int seqlen, const int32_t *cu_seqlens,
                           int nheads, int head_dim, int d_state, int ngroups,
                           int chunk_size, int in_dtype,
                           const void *x, const float *dt, const float *A,
                           const void *B, const void *C, const float *D,
                           const float *initial_state,
                           int y_dtype, void *y, float *final_state,
                           int *status_dev, cudaStream_t stream);

/*
 * ssm_state_update -- decode: one token per batch element, applied in place
 * to the fp32 state (the selective_state_update step of the walk-through's
 * section "Decode 阶段"; the TensorRT MambaPlugin update_ssm_state of the
 * deep-research note, section "TensorRT Plugin 做 selective state update",
 * without its copy-to-output since the update here is in place).
 *
 *   state  device fp32 [batch][nheads][head_dim][d_state], read and written
 *   x      device [batch][nheads][head_dim], in_dtype
 *   dt     device fp32 [batch][nheads]
 *   A      device fp32 [nheads]
 *   B, C   device [batch][ngroups][d_state], in_dtype
 *   D      device fp32 [nheads] or NULL
 *   y      device [batch][nheads][head_dim], y_dtype; must not overlap state
 *          or any input
 * Shapes: nheads % ngroups == 0; head_dim >= 1 and <= 256;
 *   d_state in {16, 32, 64, 128, 256}; batch >= 0 (0 is a no-op).
 * The kernel reads and writes each state element exactly once.
 */
SSM_API int ssm_state_update(int batch, int nheads, int head_dim, int d_state,
                     int ngroups, int in_dtype, float *state,
                     const void *x, const float *dt, const float *A,
                     const void *B, const void *C, const float *D,
                     int y_dtype, void *y, cudaStream_t stream);

/*
 * Slot-indexed state pools.  A serving engine keeps every live request's
 * recurrent state in one pool [max_slots][nheads][head_dim][d_state] (fp32)
 * and hands each call the pool slot of each sequence or batch row, so that no
 * gather/scatter of states around the call is needed: the kernels read and
 * write the slots in place.  This is the slot_idx -> ssm_pool design of the
 * MAX nemotron_h article, section 8 (state pools and request lifecycle), with
 * its has_initial_state flag (section 5.5).
 */

/*
 * ssd_chunk_scan_slots -- ssd_chunk_scan whose initial and final states are
 * rows of a state pool.
 *   state_pool         device [max_slots][nheads][head_dim][d_state], read and
 *                      written in place (only the rows named in slot_idx)
 *   state_dtype        SSM_F32, or SSM_F16 (computed in fp32, rounded on write
 *                      with `rounding`: see ssm_rounding; NULL = nearest even)
 *   max_slots          number of rows of the pool (> 0)
 *   slot_idx           device int32 [nseq]: pool row of sequence s.  Rows must
 *                      be distinct; an index outside [0, max_slots) skips that
 *                      sequence (no output written) and sets
 *                      SSM_ERR_DEVICE_INPUT in *status_dev.
 *                      NULL: sequence s uses row s (max_slots >= nseq).
 *   has_initial_state  device int32 [nseq] or NULL (all true): 0 starts the
 *                      sequence from a zero state (a freshly claimed slot)
 *                      instead of the slot's contents.
 *   dt_params          optional dt transform (see ssm_dt_params), or NULL.
 * Every other argument is as for ssd_chunk_scan.  A zero-length sequence
 * leaves its slot unchanged, or zeroes it when it has no initial state.  The
 * pool must not overlap any input or y.
 */
SSM_API int ssd_chunk_scan_slots(int nseq, int seqlen, const int32_t *cu_seqlens,
                                 int nheads, int head_dim, int d_state, int ngroups,
                                 int chunk_size, int in_dtype,
                                 const void *x, const float *dt, const float *A,
                                 const void *B, const void *C, const float *D,
                                 const ssm_dt_params *dt_params,
                                 void *state_pool, int state_dtype,
                                 const ssm_rounding *rounding, int max_slots,
                                 const int32_t *slot_idx,
                                 const int32_t *has_initial_state,
                                 int y_dtype, void *y, int *status_dev, cudaStream_t stream);

/*
 * ssm_state_update_slots -- ssm_state_update on pool rows: batch row b updates
 * state_pool[slot_idx[b]] in place.  A negative slot index marks a padding row
 * (no state update, y not written); an index >= max_slots skips the row and
 * sets SSM_ERR_DEVICE_INPUT in *status_dev (status_dev may be NULL).  Slot
 * indices of non-padding rows must be distinct; slot_idx NULL means row b
 * (max_slots >= batch).  dt_params: optional dt transform, or NULL.
 * state_dtype / rounding: as for ssd_chunk_scan_slots (fp16 pools are read as
 * fp16, updated in fp32 and rounded back).  Other arguments as for
 * ssm_state_update.
 */
SSM_API int ssm_state_update_slots(int batch, int nheads, int head_dim, int d_state,
                                   int ngroups, int in_dtype, void *state_pool, int state_dtype,
                                   const ssm_rounding *rounding, int max_slots,
                                   const int32_t *slot_idx,
                                   const void *x, const float *dt, const float *A,
                                   const void *B, const void *C, const float *D,
                                   const ssm_dt_params *dt_params,
                                   int y_dtype, void *y, int *status_dev, cudaStream_t stream);

/*
 * Causal depthwise conv1d, the short convolution in front of the scan that
 * mixes each channel of the concatenated (x, B, C) projection over the last
 * `width` tokens ("Depthwise SiLU 卷积" of the MAX nemotron_h article,
 * section 5.4 item 2; causal_conv1d_fn for prefill and causal_conv1d_update
 * for decode in the modeling_nemotron_h.py walk-through, sections
 * "Prefill 阶段" and "Decode 阶段").  For channel c and token t of a sequence:
 *
 *     y[t][c] = act(bias[c] + sum_{k<width} weight[c][k] * in[t-(width-1)+k][c])
 *
 * where the inputs before the sequence start are its conv state (its
 * width-1 most recent earlier inputs, oldest first) or zero.  Afterwards the
 * conv state holds the width-1 most recent inputs of the sequence (for a
 * sequence shorter than width-1, the newest old entries shift down).
 *
 * Layouts (channels-last, row-major, contiguous):
 *   x, y        [T][dim]              (in_dtype / y_dtype)
 *   weight      [dim][width]          fp32
 *   bias        [dim]                 fp32 or NULL
 *   conv_state  [rows][dim][width-1]  in_dtype (the inputs' own type)
 * activation: 0 = identity, 1 = SiLU (v * sigmoid(v)).  width in [1, 8].
 * Accumulation is fp32; y rounds to nearest even when bf16, the conv state
 * holds inputs verbatim.  All device pointers must be 16-byte aligned; y must
 * not overlap x, the state or any other input.
 */
enum { SSM_ACT_NONE = 0, SSM_ACT_SILU = 1 };

/*
 * causal_conv1d_fwd -- prefill over whole sequences.
 *   nseq, seqlen, cu_seqlens   as for ssd_chunk_scan (cu_seqlens device int32
 *                              [nseq+1] for packed sequences, or NULL)
 *   conv_state   device [rows][dim][width-1] or NULL (zero history; no state
 *                written).  rows = nseq when slot_idx is NULL, else max_slots.
 *   slot_idx     device int32 [nseq] or NULL: conv-state row of each sequence;
 *                an index outside [0, max_slots) skips that sequence (no y,
 *                no state written) and sets SSM_ERR_DEVICE_INPUT.
 *   has_initial_state  device int32 [nseq] or NULL: 0 = zero history for that
 *                sequence (its state row is still written).
 * Two launches (the convolution, then the state roll) on `stream`.
 */
SSM_API int causal_conv1d_fwd(int nseq, int seqlen, const int32_t *cu_seqlens, int dim,
                              int width, int in_dtype, const void *x, const float *weight,
                              const float *bias, int activation, void *conv_state,
                              int max_slots, const int32_t *slot_idx,
                              const int32_t *has_initial_state, int y_dtype, void *y,
                              int *status_dev, cudaStream_t stream);

/*
 * causal_conv1d_update -- decode: one token per batch row; the window is
 * [conv_state row, x] and the state row rolls by one in place.
 *   x, y         device [batch][dim]
 *   conv_state   device [rows][dim][width-1] (rows = batch without slot_idx,
 *                else max_slots); may be NULL only when width == 1.
 *   slot_idx     device int32 [batch] or NULL: a negative index marks a
 *                padding row (y and state untouched); an index >= max_slots
 *                skips the row and sets SSM_ERR_DEVICE_INPUT.  Indices of
 *                non-padding rows must be distinct.
 */
SSM_API int causal_conv1d_update(int batch, int dim, int width, int in_dtype, const void *x,
                                 const float *weight, const float *bias, int activation,
                                 void *conv_state, int max_slots, const int32_t *slot_idx,
                                 int y_dtype, void *y, int *status_dev, cudaStream_t stream);

/*
 * Speculative (multi-token) decode.  A draft proposes ntok candidate tokens
 * per batch row; the model verifies them in one call, each candidate
 * producing an intermediate state, and the number accepted decides which
 * intermediate state (recurrent and conv) becomes the row's state (the
 * "MTP / speculative decoding" item of the deep-research note; multi-token
 * prediction with a draft model in "How NVIDIA's new Nemotron model works",
 * section "训练流程与推理加速").  Two flows are supported:
 *   1. verify with inter_states, then ssm_state_commit scatters
 *      inter_states[b][accept_len[b]-1] into the row (state read once,
 *      ntok states written);
 *   2. verify without inter_states, then call ssm_state_update_multi again
 *      on the same draft inputs with accept_len and y = NULL, which rewrites
 *      the row in place (state read twice, written once: the cheaper flow on
 *      HBM for ntok >= 2).
 */

/*
 * ssm_state_update_multi -- ntok tokens per batch row, in order, from the
 * row's fp32 state (state[b], or state[slot_idx[b]] of a pool).
 *   x  [batch][ntok][nheads][head_dim]     dt [batch][ntok][nheads] fp32
 *   B, C [batch][ntok][ngroups][d_state]   A, D as for ssm_state_update
 *   y  [batch][ntok][nheads][head_dim] or NULL
 *   inter_states  fp32 [batch][ntok][nheads][head_dim][d_state] or NULL: the
 *                 state after each draft token
 *   accept_len    device int32 [batch] or NULL.  When given, the row is
 *                 rewritten with the state after accept_len[b] tokens
 *                 (0 leaves it unchanged); a value outside [0, ntok] skips
 *                 the row and sets SSM_ERR_DEVICE_INPUT.  When NULL the
 *                 state is only read.
 *   slot_idx / max_slots  as for ssm_state_update_slots (negative = padding);
 *                 NULL / 0 when the state has one row per batch row.
 *   dt_params     optional dt transform (see ssm_dt_params), or NULL.
 * At least one of y, inter_states, accept_len must be given.  No output may
 * overlap an input or another output.
 */
SSM_API int ssm_state_update_multi(int batch, int ntok, int nheads, int head_dim, int d_state,
                                   int ngroups, int in_dtype, float *state, int max_slots,
                                   const int32_t *slot_idx, const void *x, const float *dt,
                                   const float *A, const void *B, const void *C,
                                   const float *D, const ssm_dt_params *dt_params,
                                   const int32_t *accept_len,
                                   float *inter_states, int y_dtype, void *y,
                                   int *status_dev, cudaStream_t stream);

/*
 * ssm_state_commit -- state row of b <- inter_states[b][accept_len[b] - 1]
 * (unchanged where accept_len[b] == 0; outside [0, ntok]: skipped and
 * SSM_ERR_DEVICE_INPUT).  Layouts as for ssm_state_update_multi.
 */
SSM_API int ssm_state_commit(int batch, int ntok, int nheads, int head_dim, int d_state,
                             const float *inter_states, const int32_t *accept_len,
                             float *state, int max_slots, const int32_t *slot_idx,
                             int *status_dev, cudaStream_t stream);

/*
 * causal_conv1d_update_multi -- ntok tokens per batch row through the
 * causal conv1d from the row's conv state.  x, y [batch][ntok][dim] (y may
 * be NULL when accept_len is given).  accept_len as for
 * ssm_state_update_multi: the conv state row is rewritten with its window
 * after accept_len[b] tokens, or left alone when accept_len is NULL.  The
 * intermediate conv states are not materialised: the commit call recomputes
 * the window from the draft inputs, which costs (width-1) values per channel.
 */
SSM_API int causal_conv1d_update_multi(int batch, int ntok, int dim, int width, int in_dtype,
                                       const void *x, const float *weight, const float *bias,
                                       int activation, void *conv_state, int max_slots,
                                       const int32_t *slot_idx, const int32_t *accept_len,
                                       int y_dtype, void *y, int *status_dev,
                                       cudaStream_t stream);

/*
 * ssm_gated_rmsnorm -- the gated group RMSNorm after the scan, gate first
 * (norm_before_gate = False: the _gated_group_rmsnorm kernel of the MAX
 * nemotron_h article, section 5.4 item 4).  For each row and each group of
 * group_size consecutive channels:
 *     g = y * silu(z),   out = g / sqrt(mean over the group of g^2 + eps) * weight
 * computed in fp32.
 *   y    [rows][dim], y_dtype (the scan output viewed as [T][nheads*head_dim])
 *   z    [rows][dim], z_dtype (the gate from the input projection)
 *   weight  device fp32 [dim];  eps >= 0
 *   out  [rows][dim], out_dtype; may be y itself (same dtype), must not
 *        overlap z or weight otherwise
 * dim must be a multiple of group_size; group_size a multiple of 256, at most
 * 8192 (SSM_ERR_UNSUPPORTED otherwise).  One launch on `stream`.
 */
SSM_API int ssm_gated_rmsnorm(int rows, int dim, int group_size, int y_dtype, const void *y,
                              int z_dtype, const void *z, const float *weight, float eps,
                              int out_dtype, void *out, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* LIBSSM_SSM_H */
