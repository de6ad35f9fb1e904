// abi.cu -- the extern "C" entry points of libssm: host-side validation of
// every argument, then one kernel launch on the caller's stream.  Nothing
// here allocates, synchronises or keeps state between calls.
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ssm.h"
#include "../../include/ssm_testing.h"
#include "ssm_internal.h"

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Range {
    uintptr_t lo, hi;   // [lo, hi)
};

Range range_of(const void *p, size_t bytes)
{
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    return Range{a, a + bytes};
}

bool overlap(Range a, Range b)
{
    if (a.lo == a.hi || b.lo == b.hi || a.lo == 0 || b.lo == 0) return false;
    return a.lo < b.hi && b.lo < a.hi;
}

size_t dtype_size(int dt) { return dt == SSM_BF16 ? 2 : 4; }

bool valid_dtype(int dt) { return dt == SSM_F32 || dt == SSM_BF16; }

bool pow2_in(int v, int lo, int hi)
{
    return v >= lo && v <= hi && (v & (v - 1)) == 0;
}

// Device-side form of the optional dt transform.  Returns SSM_OK, or the
// status for a malformed one (misaligned bias, dt_min > dt_max, NaN bounds).
int read_dt_params(const ssm_dt_params *p, ssm::DtParams &out)
{
    out = ssm::DtParams{};
    if (!p) return SSM_OK;
    if (p->dt_bias && !aligned16(p->dt_bias)) return SSM_ERR_MISALIGNED;
    if (p->clamp && !(p->dt_min <= p->dt_max)) return SSM_ERR_INVALID_ARG;
    out.bias = p->dt_bias;
    out.softplus = p->softplus != 0;
    out.clamp = p->clamp != 0;
    out.lo = p->dt_min;
    out.hi = p->dt_max;
    return SSM_OK;
}

// Storage of a state pool: fp32, or fp16 with round-to-nearest (rounding
// NULL) or stochastic rounding.
int read_state_format(int state_dtype, const ssm_rounding *r, ssm::RoundParams &out)
{
    out = ssm::RoundParams{};
    if (state_dtype == SSM_F32) return SSM_OK;
    if (state_dtype != SSM_F16) return SSM_ERR_INVALID_ARG;
    out.f16 = 1;
    if (r) {
        if (r->philox_rounds < 1 || r->philox_rounds > 16) return SSM_ERR_INVALID_ARG;
        out.stochastic = 1;
        out.key0 = (uint32_t)r->seed;
        out.key1 = (uint32_t)(r->seed >> 32);
        out.off0 = (uint32_t)r->offset;
        out.off1 = (uint32_t)(r->offset >> 32);
        out.rounds = r->philox_rounds;
    }
    return SSM_OK;
}

}  // namespace

extern "C" {

const char *ssm_status_string(int status)
{
    switch (status) {
    case SSM_OK: return "SSM_OK";
    case SSM_ERR_INVALID_ARG: return "SSM_ERR_INVALID_ARG: invalid argument";
    case SSM_ERR_UNSUPPORTED: return "SSM_ERR_UNSUPPORTED: shape or dtype not supported";
    case SSM_ERR_MISALIGNED: return "SSM_ERR_MISALIGNED: pointer not 16-byte aligned";
    case SSM_ERR_CUDA: return "SSM_ERR_CUDA: CUDA launch error";
    case SSM_ERR_TIMEOUT: return "SSM_ERR_TIMEOUT: bounded device wait expired";
    case SSM_ERR_DEVICE_INPUT: return "SSM_ERR_DEVICE_INPUT: inconsistent cu_seqlens or slot index";
    case SSM_ERR_RANGE: return "SSM_ERR_RANGE: a value beyond the fp16 range of the tensor-core operands";
    case SSM_ERR_INTERNAL: return "SSM_ERR_INTERNAL: launch configuration broke a kernel layout rule";
    case SSM_ERR_SCRATCH_LIMIT: return "SSM_ERR_SCRATCH_LIMIT: workspace needed exceeds the built-in scratch";
    default: return "unknown ssm status";
    }
}

int ssm_version(void) { return 200; }

size_t ssd_chunk_scan_workspace_size(int nseq, int seqlen, int nheads, int head_dim, int d_state,
                                     int ngroups, int chunk_size)
{
    if (nseq <= 0 || seqlen <= 0 || !ssm::scan_tc_shape(head_dim, d_state, chunk_size, nheads, ngroups))
        return 0;
    const int runs = ssm::scan_tc_balanced_runs(nseq, seqlen, nheads);
    return runs ? ssm::scan_tc_handoff_bytes(runs) : 0;
}

int ssd_chunk_scan(int nseq, int seqlen, const int32_t *cu_seqlens,
                   int nheads, int head_dim, int d_state, int ngroups,
                   int chunk_size, int in_dtype,
                   const void *x, const float *dt, const float *A,
                   const void *B, const void *C, const float *D,
                   const float *initial_state,
                   int y_dtype, void *y, float *final_state,
                   void *workspace, size_t workspace_bytes,
                   int *status_dev, cudaStream_t stream)
{
    if (nseq < 0 || seqlen < 0 || nheads <= 0 || ngroups <= 0 || nheads % ngroups)
        return SSM_ERR_INVALID_ARG;
    if (!valid_dtype(in_dtype) || !valid_dtype(y_dtype)) return SSM_ERR_INVALID_ARG;
    if (!pow2_in(head_dim, 16, 128) || !pow2_in(d_state, 16, 128)) return SSM_ERR_UNSUPPORTED;
    if (chunk_size != 64 && chunk_size != 128) return SSM_ERR_UNSUPPORTED;
    if (nseq == 0) return SSM_OK;
    const long long T = cu_seqlens ? (long long)seqlen : (long long)nseq * seqlen;
    if (T > 0x7fffffffLL) return SSM_ERR_UNSUPPORTED;
    if (T == 0 && !cu_seqlens) {
        // every sequence is empty: final = initial
        if (final_state && final_state != initial_state) {
            const size_t bytes = (size_t)nseq * nheads * head_dim * d_state * sizeof(float);
            cudaError_t e = initial_state
                ? cudaMemcpyAsync(final_state, initial_state, bytes, cudaMemcpyDeviceToDevice, stream)
                : cudaMemsetAsync(final_state, 0, bytes, stream);
            return e == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
        }
        return SSM_OK;
    }
    if (!A) return SSM_ERR_INVALID_ARG;
    if (T > 0 && (!x || !dt || !B || !C || !y)) return SSM_ERR_INVALID_ARG;
    const void *ptrs[] = {cu_seqlens, x, dt, A, B, C, D, initial_state, y, final_state, status_dev};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return SSM_ERR_MISALIGNED;

    const size_t es = dtype_size(in_dtype);
    const size_t state_bytes = (size_t)nseq * nheads * head_dim * d_state * sizeof(float);
    const Range rx = range_of(x, (size_t)T * nheads * head_dim * es);
    const Range rdt = range_of(dt, (size_t)T * nheads * sizeof(float));
    const Range rA = range_of(A, (size_t)nheads * sizeof(float));
    const Range rB = range_of(B, (size_t)T * ngroups * d_state * es);
    const Range rC = range_of(C, (size_t)T * ngroups * d_state * es);
    const Range rD = range_of(D, D ? (size_t)nheads * sizeof(float) : 0);
    const Range rh0 = range_of(initial_state, initial_state ? state_bytes : 0);
    const Range ry = range_of(y, (size_t)T * nheads * head_dim * dtype_size(y_dtype));
    const Range rhT = range_of(final_state, final_state ? state_bytes : 0);
    const Range rcu = range_of(cu_seqlens, cu_seqlens ? (size_t)(nseq + 1) * sizeof(int32_t) : 0);
    const Range ins[] = {rx, rdt, rA, rB, rC, rD, rh0, rcu};
    for (const Range &r : ins) {
        if (overlap(ry, r)) return SSM_ERR_INVALID_ARG;
        if (&r != &ins[6] && overlap(rhT, r)) return SSM_ERR_INVALID_ARG;
    }
    if (overlap(ry, rhT)) return SSM_ERR_INVALID_ARG;
    if (initial_state && final_state && initial_state != final_state && overlap(rh0, rhT))
        return SSM_ERR_INVALID_ARG;

    ssm::ScanArgs a{};
    a.nseq = nseq; a.seqlen = seqlen; a.cu_seqlens = cu_seqlens;
    a.nheads = nheads; a.head_dim = head_dim; a.d_state = d_state;
    a.ngroups = ngroups; a.chunk_size = chunk_size;
    a.in_dtype = in_dtype; a.y_dtype = y_dtype;
    a.x = x; a.dt = dt; a.A = A; a.B = B; a.C = C; a.D = D;
    a.initial_state = initial_state; a.y = y; a.final_state = final_state;
    a.status_dev = status_dev;
    a.slot_idx = nullptr; a.has_initial = nullptr; a.max_slots = 0;
    const bool tc = ssm::scan_tc_supports(a);
    if (tc && !cu_seqlens && workspace && workspace_bytes) {
        // balanced schedule: the carried state crosses the cuts through the workspace
        const int runs = ssm::scan_tc_balanced_runs(nseq, seqlen, nheads);
        const size_t need = runs ? ssm::scan_tc_handoff_bytes(runs) : 0;
        if (runs && workspace_bytes >= need) {
            if (!aligned16(workspace)) return SSM_ERR_MISALIGNED;
            const Range rw = range_of(workspace, need);
            const Range outs[] = {ry, rhT};
            for (const Range &r : ins)
                if (overlap(rw, r)) return SSM_ERR_INVALID_ARG;
            for (const Range &r : outs)
                if (overlap(rw, r)) return SSM_ERR_INVALID_ARG;
            a.runs = runs;
            a.handoff = static_cast<float *>(workspace);
            a.handoff_flags = reinterpret_cast<int *>(static_cast<char *>(workspace) + (need - runs * sizeof(int)));
        }
    }
    const cudaError_t e = tc ? ssm::launch_scan_tc(a, stream) : ssm::launch_scan_simt(a, stream);
    return e == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

int ssd_chunk_scan_slots(int nseq, int seqlen, const int32_t *cu_seqlens,
                         int nheads, int head_dim, int d_state, int ngroups,
                         int chunk_size, int in_dtype,
                         const void *x, const float *dt, const float *A,
                         const void *B, const void *C, const float *D,
                         const ssm_dt_params *dt_params,
                         void *state_pool, int state_dtype, const ssm_rounding *rounding,
                         int max_slots, const int32_t *slot_idx,
                         const int32_t *has_initial_state,
                         int y_dtype, void *y, int *status_dev, cudaStream_t stream)
{
    if (nseq < 0 || seqlen < 0 || nheads <= 0 || ngroups <= 0 || nheads % ngroups)
        return SSM_ERR_INVALID_ARG;
    if (!valid_dtype(in_dtype) || !valid_dtype(y_dtype)) return SSM_ERR_INVALID_ARG;
    if (!pow2_in(head_dim, 16, 128) || !pow2_in(d_state, 16, 128)) return SSM_ERR_UNSUPPORTED;
    if (chunk_size != 64 && chunk_size != 128) return SSM_ERR_UNSUPPORTED;
    if (nseq == 0) return SSM_OK;
    if (max_slots <= 0 || !state_pool || !A) return SSM_ERR_INVALID_ARG;
    if (!slot_idx && max_slots < nseq) return SSM_ERR_INVALID_ARG;   // row s per sequence
    ssm::DtParams dtp;
    if (const int st = read_dt_params(dt_params, dtp)) return st;
    ssm::RoundParams rp;
    if (const int st = read_state_format(state_dtype, rounding, rp)) return st;
    const size_t sz_state = rp.f16 ? 2 : 4;
    const long long T = cu_seqlens ? (long long)seqlen : (long long)nseq * seqlen;
    if (T > 0x7fffffffLL) return SSM_ERR_UNSUPPORTED;
    if (T > 0 && (!x || !dt || !B || !C || !y)) return SSM_ERR_INVALID_ARG;
    const void *ptrs[] = {cu_seqlens, x, dt, A, B, C, D, state_pool, slot_idx, has_initial_state,
                          y, status_dev};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return SSM_ERR_MISALIGNED;
    const size_t es = dtype_size(in_dtype);
    const Range rpool = range_of(state_pool, (size_t)max_slots * nheads * head_dim * d_state * sz_state);
    const Range ry = range_of(y, (size_t)T * nheads * head_dim * dtype_size(y_dtype));
    const Range ins[] = {range_of(x, (size_t)T * nheads * head_dim * es),
                         range_of(dt, (size_t)T * nheads * sizeof(float)),
                         range_of(A, (size_t)nheads * sizeof(float)),
                         range_of(B, (size_t)T * ngroups * d_state * es),
                         range_of(C, (size_t)T * ngroups * d_state * es),
                         range_of(D, D ? (size_t)nheads * sizeof(float) : 0),
                         range_of(slot_idx, slot_idx ? (size_t)nseq * sizeof(int32_t) : 0),
                         range_of(has_initial_state, has_initial_state ? (size_t)nseq * sizeof(int32_t) : 0),
                         range_of(dtp.bias, dtp.bias ? (size_t)nheads * sizeof(float) : 0),
                         range_of(cu_seqlens, cu_seqlens ? (size_t)(nseq + 1) * sizeof(int32_t) : 0)};
    for (const Range &r : ins)
        if (overlap(ry, r) || overlap(rpool, r)) return SSM_ERR_INVALID_ARG;
    if (overlap(ry, rpool)) return SSM_ERR_INVALID_ARG;

    ssm::ScanArgs a{};
    a.nseq = nseq; a.seqlen = seqlen; a.cu_seqlens = cu_seqlens;
    a.nheads = nheads; a.head_dim = head_dim; a.d_state = d_state;
    a.ngroups = ngroups; a.chunk_size = chunk_size;
    a.in_dtype = in_dtype; a.y_dtype = y_dtype;
    a.x = x; a.dt = dt; a.A = A; a.B = B; a.C = C; a.D = D;
    a.initial_state = state_pool; a.y = y; a.final_state = state_pool;
    a.status_dev = status_dev;
    a.slot_idx = slot_idx; a.has_initial = has_initial_state; a.max_slots = max_slots;
    a.dtp = dtp;
    a.rp = rp;
    // empty sequences still run: a slot without an initial state is reset to zero
    const cudaError_t e = ssm::scan_tc_supports(a) ? ssm::launch_scan_tc(a, stream)
                                                   : ssm::launch_scan_simt(a, stream);
    return e == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

int ssm_state_update(int batch, int nheads, int head_dim, int d_state,
                     int ngroups, int in_dtype, float *state,
                     const void *x, const float *dt, const float *A,
                     const void *B, const void *C, const float *D,
                     int y_dtype, void *y, cudaStream_t stream)
{
    if (batch < 0 || nheads <= 0 || ngroups <= 0 || nheads % ngroups || head_dim <= 0)
        return SSM_ERR_INVALID_ARG;
    if (!valid_dtype(in_dtype) || !valid_dtype(y_dtype)) return SSM_ERR_INVALID_ARG;
    if (head_dim > 256 || !pow2_in(d_state, 16, 256)) return SSM_ERR_UNSUPPORTED;
    if ((long long)batch * nheads > 0x7fffffffLL) return SSM_ERR_UNSUPPORTED;
    if (batch == 0) return SSM_OK;
    if (!state || !x || !dt || !A || !B || !C || !y) return SSM_ERR_INVALID_ARG;
    const void *ptrs[] = {state, x, dt, A, B, C, D, y};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return SSM_ERR_MISALIGNED;

    const size_t es = dtype_size(in_dtype);
    const Range rs = range_of(state, (size_t)batch * nheads * head_dim * d_state * sizeof(float));
    const Range rx = range_of(x, (size_t)batch * nheads * head_dim * es);
    const Range rdt = range_of(dt, (size_t)batch * nheads * sizeof(float));
    const Range rA = range_of(A, (size_t)nheads * sizeof(float));
    const Range rB = range_of(B, (size_t)batch * ngroups * d_state * es);
    const Range rC = range_of(C, (size_t)batch * ngroups * d_state * es);
    const Range rD = range_of(D, D ? (size_t)nheads * sizeof(float) : 0);
    const Range ry = range_of(y, (size_t)batch * nheads * head_dim * dtype_size(y_dtype));
    const Range ins[] = {rx, rdt, rA, rB, rC, rD};
    for (const Range &r : ins)
        if (overlap(ry, r) || overlap(rs, r)) return SSM_ERR_INVALID_ARG;
    if (overlap(ry, rs)) return SSM_ERR_INVALID_ARG;

    ssm::StateUpdateArgs a{};
    a.batch = batch; a.nheads = nheads; a.head_dim = head_dim; a.d_state = d_state;
    a.ngroups = ngroups; a.in_dtype = in_dtype; a.y_dtype = y_dtype;
    a.state = state; a.x = x; a.dt = dt; a.A = A; a.B = B; a.C = C; a.D = D; a.y = y;
    a.slot_idx = nullptr; a.max_slots = 0; a.status_dev = nullptr;
    return ssm::launch_state_update(a, stream) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

int ssm_state_update_slots(int batch, int nheads, int head_dim, int d_state,
                           int ngroups, int in_dtype, void *state_pool, int state_dtype,
                           const ssm_rounding *rounding, int max_slots,
                           const int32_t *slot_idx,
                           const void *x, const float *dt, const float *A,
                           const void *B, const void *C, const float *D,
                           const ssm_dt_params *dt_params,
                           int y_dtype, void *y, int *status_dev, cudaStream_t stream)
{
    if (batch < 0 || nheads <= 0 || ngroups <= 0 || nheads % ngroups || head_dim <= 0)
        return SSM_ERR_INVALID_ARG;
    if (!valid_dtype(in_dtype) || !valid_dtype(y_dtype)) return SSM_ERR_INVALID_ARG;
    if (head_dim > 256 || !pow2_in(d_state, 16, 256)) return SSM_ERR_UNSUPPORTED;
    if ((long long)batch * nheads > 0x7fffffffLL) return SSM_ERR_UNSUPPORTED;
    if (batch == 0) return SSM_OK;
    if (max_slots <= 0 || !state_pool || !x || !dt || !A || !B || !C || !y)
        return SSM_ERR_INVALID_ARG;
    if (!slot_idx && max_slots < batch) return SSM_ERR_INVALID_ARG;   // row b per batch row
    ssm::DtParams dtp;
    if (const int st = read_dt_params(dt_params, dtp)) return st;
    ssm::RoundParams rp;
    if (const int st = read_state_format(state_dtype, rounding, rp)) return st;
    const void *ptrs[] = {state_pool, slot_idx, x, dt, A, B, C, D, y, status_dev};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return SSM_ERR_MISALIGNED;
    const size_t es = dtype_size(in_dtype);
    const Range rs = range_of(state_pool, (size_t)max_slots * nheads * head_dim * d_state * (rp.f16 ? 2 : 4));
    const Range ry = range_of(y, (size_t)batch * nheads * head_dim * dtype_size(y_dtype));
    const Range ins[] = {range_of(x, (size_t)batch * nheads * head_dim * es),
                         range_of(dt, (size_t)batch * nheads * sizeof(float)),
                         range_of(A, (size_t)nheads * sizeof(float)),
                         range_of(B, (size_t)batch * ngroups * d_state * es),
                         range_of(C, (size_t)batch * ngroups * d_state * es),
                         range_of(D, D ? (size_t)nheads * sizeof(float) : 0),
                         range_of(slot_idx, slot_idx ? (size_t)batch * sizeof(int32_t) : 0),
                         range_of(dtp.bias, dtp.bias ? (size_t)nheads * sizeof(float) : 0)};
    for (const Range &r : ins)
        if (overlap(ry, r) || overlap(rs, r)) return SSM_ERR_INVALID_ARG;
    if (overlap(ry, rs)) return SSM_ERR_INVALID_ARG;

    ssm::StateUpdateArgs a{};
    a.batch = batch; a.nheads = nheads; a.head_dim = head_dim; a.d_state = d_state;
    a.ngroups = ngroups; a.in_dtype = in_dtype; a.y_dtype = y_dtype;
    a.state = state_pool; a.x = x; a.dt = dt; a.A = A; a.B = B; a.C = C; a.D = D; a.y = y;
    a.slot_idx = slot_idx; a.max_slots = max_slots; a.status_dev = status_dev;
    a.dtp = dtp;
    a.rp = rp;
    return ssm::launch_state_update(a, stream) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

int causal_conv1d_fwd(int nseq, int seqlen, const int32_t *cu_seqlens, int dim, int width,
                      int in_dtype, const void *x, const float *weight, const float *bias,
                      int activation, void *conv_state, int max_slots, const int32_t *slot_idx,
                      const int32_t *has_initial_state, int y_dtype, void *y, int *status_dev,
                      cudaStream_t stream)
{
    if (nseq < 0 || seqlen < 0 || dim <= 0) return SSM_ERR_INVALID_ARG;
    if (!valid_dtype(in_dtype) || !valid_dtype(y_dtype)) return SSM_ERR_INVALID_ARG;
    if (activation != 0 && activation != 1) return SSM_ERR_INVALID_ARG;
    if (width < 1) return SSM_ERR_INVALID_ARG;
    if (width > 8 || nseq > 0x7fffffff / 2) return SSM_ERR_UNSUPPORTED;
    if (cu_seqlens && nseq == 0 && seqlen != 0) return SSM_ERR_INVALID_ARG;
    const long long T = cu_seqlens ? (long long)seqlen : (long long)nseq * seqlen;
    if (nseq == 0 || (T == 0 && !conv_state)) return SSM_OK;
    if (!weight || (T > 0 && (!x || !y))) return SSM_ERR_INVALID_ARG;
    if (slot_idx && (!conv_state || max_slots <= 0)) return SSM_ERR_INVALID_ARG;
    const void *ptrs[] = {cu_seqlens, x, weight, bias, conv_state, slot_idx, has_initial_state,
                          y, status_dev};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return SSM_ERR_MISALIGNED;
    const size_t es = dtype_size(in_dtype);
    const long long rows = slot_idx ? max_slots : nseq;
    const Range rs = range_of(conv_state, conv_state ? (size_t)rows * dim * (width - 1) * es : 0);
    const Range ry = range_of(y, (size_t)T * dim * dtype_size(y_dtype));
    const Range ins[] = {range_of(x, (size_t)T * dim * es),
                         range_of(weight, (size_t)dim * width * sizeof(float)),
                         range_of(bias, bias ? (size_t)dim * sizeof(float) : 0),
                         range_of(cu_seqlens, cu_seqlens ? (size_t)(nseq + 1) * sizeof(int32_t) : 0),
                         range_of(slot_idx, slot_idx ? (size_t)nseq * sizeof(int32_t) : 0),
                         range_of(has_initial_state,
                                  has_initial_state ? (size_t)nseq * sizeof(int32_t) : 0)};
    for (const Range &r : ins)
        if (overlap(ry, r) || overlap(rs, r)) return SSM_ERR_INVALID_ARG;
    if (overlap(ry, rs)) return SSM_ERR_INVALID_ARG;

    ssm::ConvArgs a{};
    a.update = 0; a.nseq = nseq; a.seqlen = seqlen; a.cu_seqlens = cu_seqlens;
    a.dim = dim; a.width = width; a.activation = activation;
    a.in_dtype = in_dtype; a.y_dtype = y_dtype;
    a.x = x; a.weight = weight; a.bias = bias; a.state = conv_state;
    a.slot_idx = slot_idx; a.has_initial = has_initial_state; a.max_slots = max_slots;
    a.y = y; a.status_dev = status_dev;
    return ssm::launch_conv1d(a, stream) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

int causal_conv1d_update(int batch, int dim, int width, int in_dtype, const void *x,
                         const float *weight, const float *bias, int activation,
                         void *conv_state, int max_slots, const int32_t *slot_idx,
                         int y_dtype, void *y, int *status_dev, cudaStream_t stream)
{
    if (batch < 0 || dim <= 0) return SSM_ERR_INVALID_ARG;
    if (!valid_dtype(in_dtype) || !valid_dtype(y_dtype)) return SSM_ERR_INVALID_ARG;
    if (activation != 0 && activation != 1) return SSM_ERR_INVALID_ARG;
    if (width < 1) return SSM_ERR_INVALID_ARG;
    if (width > 8) return SSM_ERR_UNSUPPORTED;
    if (batch == 0) return SSM_OK;
    if (!x || !weight || !y || (width > 1 && !conv_state)) return SSM_ERR_INVALID_ARG;
    if (slot_idx && max_slots <= 0) return SSM_ERR_INVALID_ARG;
    const void *ptrs[] = {x, weight, bias, conv_state, slot_idx, y, status_dev};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return SSM_ERR_MISALIGNED;
    const size_t es = dtype_size(in_dtype);
    const long long rows = slot_idx ? max_slots : batch;
    const Range rs = range_of(conv_state, conv_state ? (size_t)rows * dim * (width - 1) * es : 0);
    const Range ry = range_of(y, (size_t)batch * dim * dtype_size(y_dtype));
    const Range ins[] = {range_of(x, (size_t)batch * dim * es),
                         range_of(weight, (size_t)dim * width * sizeof(float)),
                         range_of(bias, bias ? (size_t)dim * sizeof(float) : 0),
                         range_of(slot_idx, slot_idx ? (size_t)batch * sizeof(int32_t) : 0)};
    for (const Range &r : ins)
        if (overlap(ry, r) || overlap(rs, r)) return SSM_ERR_INVALID_ARG;
    if (overlap(ry, rs)) return SSM_ERR_INVALID_ARG;

    ssm::ConvArgs a{};
    a.update = 1; a.nseq = batch; a.seqlen = 1; a.ntok = 1; a.commit_all = 1;
    a.dim = dim; a.width = width; a.activation = activation;
    a.in_dtype = in_dtype; a.y_dtype = y_dtype;
    a.x = x; a.weight = weight; a.bias = bias; a.state = conv_state;
    a.slot_idx = slot_idx; a.max_slots = max_slots;
    a.y = y; a.status_dev = status_dev;
    return ssm::launch_conv1d(a, stream) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

int causal_conv1d_update_multi(int batch, int ntok, int dim, int width, int in_dtype,
                               const void *x, const float *weight, const float *bias,
                               int activation, void *conv_state, int max_slots,
                               const int32_t *slot_idx, const int32_t *accept_len, int y_dtype,
                               void *y, int *status_dev, cudaStream_t stream)
{
    if (batch < 0 || ntok < 0 || dim <= 0) return SSM_ERR_INVALID_ARG;
    if (!valid_dtype(in_dtype) || !valid_dtype(y_dtype)) return SSM_ERR_INVALID_ARG;
    if (activation != 0 && activation != 1) return SSM_ERR_INVALID_ARG;
    if (width < 1) return SSM_ERR_INVALID_ARG;
    if (width > 8) return SSM_ERR_UNSUPPORTED;
    if (batch == 0 || ntok == 0) return SSM_OK;
    if (!x || !weight || (width > 1 && !conv_state)) return SSM_ERR_INVALID_ARG;
    if (!y && !accept_len) return SSM_ERR_INVALID_ARG;        // nothing would be produced
    if (slot_idx && max_slots <= 0) return SSM_ERR_INVALID_ARG;
    if ((long long)batch * ntok > 0x7fffffffLL) return SSM_ERR_UNSUPPORTED;
    const void *ptrs[] = {x, weight, bias, conv_state, slot_idx, accept_len, y, status_dev};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return SSM_ERR_MISALIGNED;
    const size_t es = dtype_size(in_dtype);
    const long long rows = slot_idx ? max_slots : batch;
    const Range rs = range_of(conv_state, conv_state ? (size_t)rows * dim * (width - 1) * es : 0);
    const Range ry = range_of(y, y ? (size_t)batch * ntok * dim * dtype_size(y_dtype) : 0);
    const Range ins[] = {range_of(x, (size_t)batch * ntok * dim * es),
                         range_of(weight, (size_t)dim * width * sizeof(float)),
                         range_of(bias, bias ? (size_t)dim * sizeof(float) : 0),
                         range_of(slot_idx, slot_idx ? (size_t)batch * sizeof(int32_t) : 0),
                         range_of(accept_len, accept_len ? (size_t)batch * sizeof(int32_t) : 0)};
    for (const Range &r : ins)
        if (overlap(ry, r) || overlap(rs, r)) return SSM_ERR_INVALID_ARG;
    if (overlap(ry, rs)) return SSM_ERR_INVALID_ARG;

    ssm::ConvArgs a{};
    a.update = 1; a.nseq = batch; a.seqlen = 1; a.ntok = ntok; a.commit_all = 0;
    a.accept_len = accept_len;
    a.dim = dim; a.width = width; a.activation = activation;
    a.in_dtype = in_dtype; a.y_dtype = y_dtype;
    a.x = x; a.weight = weight; a.bias = bias; a.state = conv_state;
    a.slot_idx = slot_idx; a.max_slots = max_slots;
    a.y = y; a.status_dev = status_dev;
    return ssm::launch_conv1d(a, stream) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

int ssm_state_update_multi(int batch, int ntok, int nheads, int head_dim, int d_state,
                           int ngroups, int in_dtype, float *state, int max_slots,
                           const int32_t *slot_idx, const void *x, const float *dt,
                           const float *A, const void *B, const void *C, const float *D,
                           const ssm_dt_params *dt_params,
                           const int32_t *accept_len, float *inter_states, int y_dtype, void *y,
                           int *status_dev, cudaStream_t stream)
{
    if (batch < 0 || ntok < 0 || nheads <= 0 || ngroups <= 0 || nheads % ngroups ||
        head_dim <= 0)
        return SSM_ERR_INVALID_ARG;
    if (!valid_dtype(in_dtype) || !valid_dtype(y_dtype)) return SSM_ERR_INVALID_ARG;
    if (head_dim > 256 || !pow2_in(d_state, 16, 256)) return SSM_ERR_UNSUPPORTED;
    if ((long long)batch * nheads > 0x7fffffffLL) return SSM_ERR_UNSUPPORTED;
    if (batch == 0 || ntok == 0) return SSM_OK;
    if (!state || !x || !dt || !A || !B || !C) return SSM_ERR_INVALID_ARG;
    if (!y && !inter_states && !accept_len) return SSM_ERR_INVALID_ARG;
    if (slot_idx && max_slots <= 0) return SSM_ERR_INVALID_ARG;
    ssm::DtParams dtp;
    if (const int st = read_dt_params(dt_params, dtp)) return st;
    const void *ptrs[] = {state, slot_idx, x, dt, A, B, C, D, accept_len, inter_states, y,
                          status_dev};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return SSM_ERR_MISALIGNED;
    const size_t es = dtype_size(in_dtype);
    const size_t bt = (size_t)batch * ntok;
    const size_t rows = slot_idx ? (size_t)max_slots : (size_t)batch;
    const size_t slice = (size_t)nheads * head_dim * d_state * sizeof(float);
    const Range rs = range_of(state, rows * slice);
    const Range ri = range_of(inter_states, inter_states ? bt * slice : 0);
    const Range ry = range_of(y, y ? bt * nheads * head_dim * dtype_size(y_dtype) : 0);
    const Range ins[] = {range_of(x, bt * nheads * head_dim * es),
                         range_of(dt, bt * nheads * sizeof(float)),
                         range_of(A, (size_t)nheads * sizeof(float)),
                         range_of(B, bt * ngroups * d_state * es),
                         range_of(C, bt * ngroups * d_state * es),
                         range_of(D, D ? (size_t)nheads * sizeof(float) : 0),
                         range_of(slot_idx, slot_idx ? (size_t)batch * sizeof(int32_t) : 0),
                         range_of(accept_len, accept_len ? (size_t)batch * sizeof(int32_t) : 0),
                         range_of(dtp.bias, dtp.bias ? (size_t)nheads * sizeof(float) : 0)};
    for (const Range &r : ins)
        if (overlap(ry, r) || overlap(rs, r) || overlap(ri, r)) return SSM_ERR_INVALID_ARG;
    if (overlap(ry, rs) || overlap(ri, rs) || overlap(ri, ry)) return SSM_ERR_INVALID_ARG;

    ssm::MultiUpdateArgs a{};
    a.batch = batch; a.ntok = ntok; a.nheads = nheads; a.head_dim = head_dim;
    a.d_state = d_state; a.ngroups = ngroups; a.in_dtype = in_dtype; a.y_dtype = y_dtype;
    a.state = state; a.slot_idx = slot_idx; a.max_slots = max_slots;
    a.x = x; a.dt = dt; a.A = A; a.B = B; a.C = C; a.D = D;
    a.accept_len = accept_len; a.inter = inter_states; a.y = y; a.status_dev = status_dev;
    a.dtp = dtp;
    return ssm::launch_state_update_multi(a, stream) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

int ssm_state_commit(int batch, int ntok, int nheads, int head_dim, int d_state,
                     const float *inter_states, const int32_t *accept_len, float *state,
                     int max_slots, const int32_t *slot_idx, int *status_dev,
                     cudaStream_t stream)
{
    if (batch < 0 || ntok < 0 || nheads <= 0 || head_dim <= 0) return SSM_ERR_INVALID_ARG;
    if (head_dim > 256 || !pow2_in(d_state, 16, 256)) return SSM_ERR_UNSUPPORTED;
    if ((long long)batch * nheads > 0x7fffffffLL) return SSM_ERR_UNSUPPORTED;
    if (batch == 0 || ntok == 0) return SSM_OK;
    if (!inter_states || !accept_len || !state) return SSM_ERR_INVALID_ARG;
    if (slot_idx && max_slots <= 0) return SSM_ERR_INVALID_ARG;
    const void *ptrs[] = {inter_states, accept_len, state, slot_idx, status_dev};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return SSM_ERR_MISALIGNED;
    const size_t slice = (size_t)nheads * head_dim * d_state * sizeof(float);
    const size_t rows = slot_idx ? (size_t)max_slots : (size_t)batch;
    const Range rs = range_of(state, rows * slice);
    const Range ins[] = {range_of(inter_states, (size_t)batch * ntok * slice),
                         range_of(accept_len, (size_t)batch * sizeof(int32_t)),
                         range_of(slot_idx, slot_idx ? (size_t)batch * sizeof(int32_t) : 0)};
    for (const Range &r : ins)
        if (overlap(rs, r)) return SSM_ERR_INVALID_ARG;

    ssm::CommitArgs a{};
    a.batch = batch; a.ntok = ntok; a.nheads = nheads; a.head_dim = head_dim;
    a.d_state = d_state; a.inter = inter_states; a.accept_len = accept_len; a.state = state;
    a.slot_idx = slot_idx; a.max_slots = max_slots; a.status_dev = status_dev;
    return ssm::launch_state_commit(a, stream) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

int ssm_gated_rmsnorm(int rows, int dim, int group_size, int y_dtype, const void *y,
                      int z_dtype, const void *z, const float *weight, float eps,
                      int out_dtype, void *out, cudaStream_t stream)
{
    if (rows < 0 || dim <= 0 || group_size <= 0) return SSM_ERR_INVALID_ARG;
    if (!valid_dtype(y_dtype) || !valid_dtype(z_dtype) || !valid_dtype(out_dtype))
        return SSM_ERR_INVALID_ARG;
    if (dim % group_size || !(eps >= 0.f)) return SSM_ERR_INVALID_ARG;
    if (group_size % 256 || group_size > 8192) return SSM_ERR_UNSUPPORTED;   // whole warps
    if ((long long)rows * (dim / group_size) > 0x7fffffffLL) return SSM_ERR_UNSUPPORTED;
    if (rows == 0) return SSM_OK;
    if (!y || !z || !weight || !out) return SSM_ERR_INVALID_ARG;
    const void *ptrs[] = {y, z, weight, out};
    for (const void *p : ptrs)
        if (!aligned16(p)) return SSM_ERR_MISALIGNED;
    const size_t n = (size_t)rows * dim;
    const Range ro = range_of(out, n * dtype_size(out_dtype));
    const Range ryr = range_of(y, n * dtype_size(y_dtype));
    // out may be y itself (same dtype: each element is read before it is written)
    const bool in_place = out == y && out_dtype == y_dtype;
    if (!in_place && overlap(ro, ryr)) return SSM_ERR_INVALID_ARG;
    if (overlap(ro, range_of(z, n * dtype_size(z_dtype))) ||
        overlap(ro, range_of(weight, (size_t)dim * sizeof(float))))
        return SSM_ERR_INVALID_ARG;

    ssm::GatedNormArgs a{};
    a.rows = rows; a.dim = dim; a.group_size = group_size;
    a.y_dtype = y_dtype; a.z_dtype = z_dtype; a.out_dtype = out_dtype;
    a.y = y; a.z = z; a.weight = weight; a.eps = eps; a.out = out;
    return ssm::launch_gated_rmsnorm(a, stream) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}


// ---------------------------------------------------------------- testing hooks
int ssm_testing_balanced_runs(int nseq, int seqlen, int nheads, int sms)
{
    if (nseq <= 0 || seqlen <= 0 || nheads <= 0 || sms <= 0) return 0;
    return ssm::scan_tc_balanced_runs_for(nseq, seqlen, nheads, sms);
}

int ssm_testing_scan_stalled(int nseq, int seqlen, int nheads, int ngroups,
                             const void *x, const float *dt, const float *A,
                             const void *B, const void *C, void *y,
                             unsigned long long wait_ns, int *status_dev, cudaStream_t stream)
{
    if (nseq <= 0 || seqlen <= 0 || nheads <= 0 || ngroups <= 0 || nheads % ngroups)
        return SSM_ERR_INVALID_ARG;
    if (!x || !dt || !A || !B || !C || !y || !status_dev) return SSM_ERR_INVALID_ARG;
    if (wait_ns < 1000ull || wait_ns > 10000000000ull) return SSM_ERR_INVALID_ARG;
    const void *ptrs[] = {x, dt, A, B, C, y, status_dev};
    for (const void *p : ptrs)
        if (!aligned16(p)) return SSM_ERR_MISALIGNED;
    if ((long long)nseq * seqlen > 0x7fffffffLL) return SSM_ERR_UNSUPPORTED;
    ssm::ScanArgs a{};
    a.nseq = nseq; a.seqlen = seqlen; a.cu_seqlens = nullptr;
    a.nheads = nheads; a.head_dim = 64; a.d_state = 128; a.ngroups = ngroups; a.chunk_size = 128;
    a.in_dtype = SSM_BF16; a.y_dtype = SSM_BF16;
    a.x = x; a.dt = dt; a.A = A; a.B = B; a.C = C; a.D = nullptr;
    a.y = y; a.status_dev = status_dev;
    a.wait_ns = wait_ns; a.stall_producer = 1;
    if (!ssm::scan_tc_supports(a)) return SSM_ERR_UNSUPPORTED;
    return ssm::launch_scan_tc(a, stream) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

int ssm_testing_conv1d_stalled(int nseq, int seqlen, int dim, int width, const void *x,
                               const float *weight, void *y, unsigned long long wait_ns,
                               int *status_dev, cudaStream_t stream)
{
    if (nseq <= 0 || seqlen <= 0 || dim <= 0 || dim % 8 || width < 1 || width > 8)
        return SSM_ERR_INVALID_ARG;
    if (!x || !weight || !y || !status_dev) return SSM_ERR_INVALID_ARG;
    if (wait_ns < 1000ull || wait_ns > 10000000000ull) return SSM_ERR_INVALID_ARG;
    const void *ptrs[] = {x, weight, y, status_dev};
    for (const void *p : ptrs)
        if (!aligned16(p)) return SSM_ERR_MISALIGNED;
    if ((long long)nseq * seqlen > 0x7fffffffLL) return SSM_ERR_UNSUPPORTED;
    ssm::ConvArgs a{};
    a.update = 0; a.nseq = nseq; a.seqlen = seqlen;
    a.dim = dim; a.width = width; a.activation = 0;
    a.in_dtype = SSM_BF16; a.y_dtype = SSM_BF16;
    a.x = x; a.weight = weight; a.y = y; a.status_dev = status_dev;
    a.wait_ns = wait_ns; a.stall_producer = 1;
    return ssm::launch_conv1d(a, stream) == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

}  // extern "C"
