// state_update.cu -- decode: one-token selective state update, in place on the
// fp32 state.
//
// Per (batch b, head h) with group g = h / heads_per_group:
//   decay = exp(dt[b,h] * A[h])
//   s[p,n] <- decay * s[p,n] + (dt[b,h] * x[b,h,p]) * B[b,g,n]
//   y[b,h,p] = sum_n s[p,n] * C[b,g,n] + D[h] * x[b,h,p]
// (the decode form of the selective-SSM recurrence, "Decode 阶段" of the
// modeling_nemotron_h.py walk-through).
//
// The kernel is bound by HBM: every state element is read once and written
// once (streaming, evict-first), and everything else is tiny.  A CTA owns one
// (b, h) slice of head_dim x d_state floats.  Each state row (one p, d_state
// floats) is covered by d_state/4 lanes, each holding one float4 (two for
// d_state = 256); a warp issues all of its rows' loads before any arithmetic
// so that 32 KB per CTA are in flight.  The row sum for y is a shuffle
// reduction inside the lanes of a row.
#include "common.cuh"
#include "ssm_internal.h"

namespace ssm {

constexpr int kDecodeWarps = 8;
constexpr int kDecodeUnroll = 8;

template <int N, typename TIn, typename TOut>
__global__ void __launch_bounds__(kDecodeWarps * 32)
state_update_kernel(int nheads, int head_dim, int heads_per_group, int ngroups,
                    float *__restrict__ state, const TIn *__restrict__ x,
                    const float *__restrict__ dt, const float *__restrict__ A,
                    const TIn *__restrict__ B, const TIn *__restrict__ C,
                    const float *__restrict__ D, TOut *__restrict__ y,
                    const int32_t *__restrict__ slot_idx, int max_slots, int *status,
                    DtParams dtp)
{
    constexpr int LPR = (N / 4 < 32) ? N / 4 : 32;   // lanes per state row
    constexpr int VEC = N / (4 * LPR);               // float4s per lane
    constexpr int RPW = 32 / LPR;                    // rows per warp step
    constexpr int ROWS_PER_PASS = kDecodeWarps * RPW * kDecodeUnroll;

    const int bh = blockIdx.x;
    const int b = bh / nheads;
    const int h = bh - b * nheads;
    const int g = h / heads_per_group;
    size_t srow = (size_t)b;   // state row of this batch row
    if (slot_idx) {
        const int slot = __ldg(slot_idx + b);
        if (slot < 0) return;                        // padding row: nothing to do
        if (slot >= max_slots) {
            if (threadIdx.x == 0) report_status(status, 6);
            return;
        }
        srow = (size_t)slot;
    }
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int li = lane % LPR;
    const int ri = lane / LPR;

    const float dtv = dt_apply(dtp, __ldg(dt + bh), h);
    const float decay = expf(dtv * __ldg(A + h));
    const float Dh = D ? __ldg(D + h) : 0.f;

    float4 bv[VEC], cv[VEC];
    const TIn *Bp = B + ((size_t)b * ngroups + g) * N;
    const TIn *Cp = C + ((size_t)b * ngroups + g) * N;
#pragma unroll
    for (int v = 0; v < VEC; ++v) {
        const int n0 = (v * LPR + li) * 4;
        bv[v] = load4(Bp + n0);
        cv[v] = load4(Cp + n0);
    }

    float *st = state + (srow * nheads + h) * (size_t)head_dim * N;
    const TIn *xp = x + (size_t)bh * head_dim;
    TOut *yp = y + (size_t)bh * head_dim;

    for (int base = 0; base < head_dim; base += ROWS_PER_PASS) {
        float4 s[kDecodeUnroll][VEC];
#pragma unroll
        for (int k = 0; k < kDecodeUnroll; ++k) {
            const int r = base + (k * kDecodeWarps + warp) * RPW + ri;
#pragma unroll
            for (int v = 0; v < VEC; ++v) {
                if (r < head_dim)
                    s[k][v] = __ldcs(reinterpret_cast<const float4 *>(
                        st + (size_t)r * N + (v * LPR + li) * 4));
                else
                    s[k][v] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
#pragma unroll
        for (int k = 0; k < kDecodeUnroll; ++k) {
            const int r = base + (k * kDecodeWarps + warp) * RPW + ri;
            const float xr = (r < head_dim) ? load_f32(xp + r) : 0.f;
            const float dtx = dtv * xr;
            float acc = 0.f;
#pragma unroll
            for (int v = 0; v < VEC; ++v) {
                float4 q = s[k][v];
                q.x = fmaf(q.x, decay, dtx * bv[v].x);
                q.y = fmaf(q.y, decay, dtx * bv[v].y);
                q.z = fmaf(q.z, decay, dtx * bv[v].z);
                q.w = fmaf(q.w, decay, dtx * bv[v].w);
                acc = fmaf(q.x, cv[v].x, acc);
                acc = fmaf(q.y, cv[v].y, acc);
                acc = fmaf(q.z, cv[v].z, acc);
                acc = fmaf(q.w, cv[v].w, acc);
                if (r < head_dim)
                    __stcs(reinterpret_cast<float4 *>(
                               st + (size_t)r * N + (v * LPR + li) * 4), q);
            }
#pragma unroll
            for (int o = LPR / 2; o > 0; o >>= 1)
                acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (li == 0 && r < head_dim) store_out(yp + r, fmaf(Dh, xr, acc));
        }
    }
}

// fp16 state pool: the state is read as fp16, updated in fp32 and rounded
// back (nearest even, or stochastically with 16 Philox bits per element).
// Each lane owns 8 adjacent d_state elements of a row (one 16-byte load and
// store, one Philox call), so a warp covers 32 / (d_state / 8) rows per step
// and a CTA has its whole 64 x 128 fp16 slice (16 KB) in flight at once.
constexpr int kF16Unroll = 4;

template <int N, typename TIn, typename TOut>
__global__ void __launch_bounds__(kDecodeWarps * 32)
state_update_f16_kernel(int nheads, int head_dim, int heads_per_group, int ngroups,
                        __half *__restrict__ state, const TIn *__restrict__ x,
                        const float *__restrict__ dt, const float *__restrict__ A,
                        const TIn *__restrict__ B, const TIn *__restrict__ C,
                        const float *__restrict__ D, TOut *__restrict__ y,
                        const int32_t *__restrict__ slot_idx, int max_slots, int *status,
                        DtParams dtp, RoundParams rp)
{
    constexpr int LPR = (N / 8 < 32) ? N / 8 : 32;   // lanes per state row
    constexpr int RPW = 32 / LPR;                    // rows per warp step
    constexpr int ROWS_PER_PASS = kDecodeWarps * RPW * kF16Unroll;
    static_assert(N == 8 * LPR, "one 8-element vector per lane");

    const int bh = blockIdx.x;
    const int b = bh / nheads;
    const int h = bh - b * nheads;
    const int g = h / heads_per_group;
    size_t srow = (size_t)b;
    if (slot_idx) {
        const int slot = __ldg(slot_idx + b);
        if (slot < 0) return;
        if (slot >= max_slots) {
            if (threadIdx.x == 0) report_status(status, 6);
            return;
        }
        srow = (size_t)slot;
    }
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int li = lane % LPR;
    const int ri = lane / LPR;
    const float dtv = dt_apply(dtp, __ldg(dt + bh), h);
    const float decay = expf(dtv * __ldg(A + h));
    const float Dh = D ? __ldg(D + h) : 0.f;
    float bv[8], cv[8];
    {
        const float4 b0 = load4(B + ((size_t)b * ngroups + g) * N + li * 8);
        const float4 b1 = load4(B + ((size_t)b * ngroups + g) * N + li * 8 + 4);
        const float4 c0 = load4(C + ((size_t)b * ngroups + g) * N + li * 8);
        const float4 c1 = load4(C + ((size_t)b * ngroups + g) * N + li * 8 + 4);
        const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
        const float cc[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) { bv[j] = bb[j]; cv[j] = cc[j]; }
    }
    const size_t st0 = (srow * nheads + h) * (size_t)head_dim * N;   // element index of the slice
    __half *st = state + st0;
    const TIn *xp = x + (size_t)bh * head_dim;
    TOut *yp = y + (size_t)bh * head_dim;

    for (int base = 0; base < head_dim; base += ROWS_PER_PASS) {
        uint4 raw[kF16Unroll];
#pragma unroll
        for (int k = 0; k < kF16Unroll; ++k) {
            const int r = base + (k * kDecodeWarps + warp) * RPW + ri;
            raw[k] = (r < head_dim) ? __ldcs(reinterpret_cast<const uint4 *>(st + (size_t)r * N + li * 8))
                                    : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int k = 0; k < kF16Unroll; ++k) {
            const int r = base + (k * kDecodeWarps + warp) * RPW + ri;
            const float xr = (r < head_dim) ? load_f32(xp + r) : 0.f;
            const float dtx = dtv * xr;
            const __half2 *hv = reinterpret_cast<const __half2 *>(&raw[k]);
            float q[8];
            float acc = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 f = __half22float2(hv[j]);
                q[2 * j] = fmaf(f.x, decay, dtx * bv[2 * j]);
                q[2 * j + 1] = fmaf(f.y, decay, dtx * bv[2 * j + 1]);
                acc = fmaf(q[2 * j], cv[2 * j], acc);
                acc = fmaf(q[2 * j + 1], cv[2 * j + 1], acc);
            }
            if (r < head_dim) {
                const size_t off = (size_t)r * N + li * 8;
                uint32_t w[4] = {0u, 0u, 0u, 0u};
                if (rp.stochastic) {
                    const uint4 rnd = state_random8(rp, st0 + off);
                    w[0] = rnd.x; w[1] = rnd.y; w[2] = rnd.z; w[3] = rnd.w;
                }
                uint32_t packed[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const __half2 hh = __halves2half2(state_to_half(rp, q[2 * j], w[j] & 0xFFFFu),
                                                      state_to_half(rp, q[2 * j + 1], w[j] >> 16));
                    packed[j] = *reinterpret_cast<const uint32_t *>(&hh);
                }
                __stcs(reinterpret_cast<uint4 *>(st + off),
                       make_uint4(packed[0], packed[1], packed[2], packed[3]));
            }
#pragma unroll
            for (int o = LPR / 2; o > 0; o >>= 1)
                acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (li == 0 && r < head_dim) store_out(yp + r, fmaf(Dh, xr, acc));
        }
    }
}

template <int N, typename TIn, typename TOut>
static cudaError_t launch_state_update_t(const StateUpdateArgs &a, cudaStream_t stream)
{
    dim3 grid((unsigned)((size_t)a.batch * a.nheads));
    if (a.rp.f16) {
        state_update_f16_kernel<N, TIn, TOut><<<grid, kDecodeWarps * 32, 0, stream>>>(
            a.nheads, a.head_dim, a.nheads / a.ngroups, a.ngroups, static_cast<__half *>(a.state),
            static_cast<const TIn *>(a.x), a.dt, a.A, static_cast<const TIn *>(a.B),
            static_cast<const TIn *>(a.C), a.D, static_cast<TOut *>(a.y), a.slot_idx,
            a.max_slots, a.status_dev, a.dtp, a.rp);
        return cudaGetLastError();
    }
    state_update_kernel<N, TIn, TOut><<<grid, kDecodeWarps * 32, 0, stream>>>(
        a.nheads, a.head_dim, a.nheads / a.ngroups, a.ngroups, static_cast<float *>(a.state),
        static_cast<const TIn *>(a.x), a.dt, a.A, static_cast<const TIn *>(a.B),
        static_cast<const TIn *>(a.C), a.D, static_cast<TOut *>(a.y), a.slot_idx, a.max_slots,
        a.status_dev, a.dtp);
    return cudaGetLastError();
}

template <int N>
static cudaError_t launch_state_update_n(const StateUpdateArgs &a, cudaStream_t stream)
{
    const bool in_bf16 = a.in_dtype == 1, out_bf16 = a.y_dtype == 1;
    if (in_bf16 && out_bf16) return launch_state_update_t<N, __nv_bfloat16, __nv_bfloat16>(a, stream);
    if (in_bf16) return launch_state_update_t<N, __nv_bfloat16, float>(a, stream);
    if (out_bf16) return launch_state_update_t<N, float, __nv_bfloat16>(a, stream);
    return launch_state_update_t<N, float, float>(a, stream);
}

cudaError_t launch_state_update(const StateUpdateArgs &a, cudaStream_t stream)
{
    switch (a.d_state) {
    case 16: return launch_state_update_n<16>(a, stream);
    case 32: return launch_state_update_n<32>(a, stream);
    case 64: return launch_state_update_n<64>(a, stream);
    case 128: return launch_state_update_n<128>(a, stream);
    case 256: return launch_state_update_n<256>(a, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace ssm
