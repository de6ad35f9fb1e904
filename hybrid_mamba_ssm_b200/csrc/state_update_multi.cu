// state_update_multi.cu -- speculative (multi-token) decode.
//
// Candidate tokens of a draft produce intermediate states; how many of them
// are accepted decides which intermediate state becomes the row's state (the
// "MTP / speculative decoding" item of the deep-research note).  Per batch
// row b and head h, the row's ntok draft tokens run in order through the
// decode recurrence
//   s[p,n] <- exp(dt A_h) s[p,n] + dt x[p] B[g,n],   y[p] = s[p,:] . C[g,:] + D_h x[p]
// from the row's state, producing y for every token and, on request, the
// state after every token (the intermediate states, for a later scatter) and
// an in-place update of the row with the state after accept_len[b] tokens.
//
// Layout and memory pattern follow the one-token kernel: a CTA owns one
// (b, h) slice; each state row (one p) is spread over d_state/4 lanes with
// one float4 each (two at d_state = 256).  A pass of rows is loaded once and
// then carried through all ntok tokens in registers, so the state is read
// once, and written once per requested output (intermediate, commit).  The
// draft tokens' B, C, x and decay are staged in shared memory, 8 tokens at a
// time, with one round of loads, so the token loop waits on no global load.
#include "common.cuh"
#include "ssm_internal.h"

namespace ssm {

constexpr int kMultiWarps = 8;
constexpr int kMultiUnroll = 8;
constexpr int kTokBlock = 8;        // draft tokens staged in shared memory at a time
constexpr int kMaxHeadDim = 256;

template <int N, typename TIn, typename TOut>
__global__ void __launch_bounds__(kMultiWarps * 32, (N >= 256 ? 2 : 3))
state_update_multi_kernel(MultiUpdateArgs a)
{
    constexpr int LPR = (N / 4 < 32) ? N / 4 : 32;   // lanes per state row
    constexpr int VEC = N / (4 * LPR);               // float4s per lane
    constexpr int RPW = 32 / LPR;                    // rows per warp step
    constexpr int ROWS_PER_PASS = kMultiWarps * RPW * kMultiUnroll;
    // per draft token of the current block, staged in shared memory as fp32:
    // B[N], C[N] of the head's group, x[head_dim] of the head, and the decay
    __shared__ __align__(16) float sB[kTokBlock][N], sC[kTokBlock][N];
    __shared__ float sX[kTokBlock][kMaxHeadDim], sDt[kTokBlock], sDecay[kTokBlock];

    const int H = a.nheads, P = a.head_dim;
    const int bh = blockIdx.x;
    const int b = bh / H;
    const int h = bh - b * H;
    const int g = h / (H / a.ngroups);
    size_t srow = (size_t)b;
    if (a.slot_idx) {
        const int slot = __ldg(a.slot_idx + b);
        if (slot < 0) return;                        // padding row
        if (slot >= a.max_slots) {
            if (threadIdx.x == 0) report_status(a.status_dev, 6);
            return;
        }
        srow = (size_t)slot;
    }
    int commit = 0;                                  // tokens after which the row is written
    if (a.accept_len) {
        commit = __ldg(a.accept_len + b);
        if (commit < 0 || commit > a.ntok) {
            if (threadIdx.x == 0) report_status(a.status_dev, 6);
            return;
        }
    }
    // without y or intermediate states only the committed tokens matter
    const int nsteps = (!a.y && !a.inter) ? commit : a.ntok;
    if (nsteps == 0) return;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int li = lane % LPR;
    const int ri = lane / LPR;
    const float Ah = __ldg(a.A + h);
    const float Dh = a.D ? __ldg(a.D + h) : 0.f;
    const TIn *x = static_cast<const TIn *>(a.x);
    const TIn *Bm = static_cast<const TIn *>(a.B);
    const TIn *Cm = static_cast<const TIn *>(a.C);
    TOut *y = static_cast<TOut *>(a.y);
    float *st = a.state + (srow * H + h) * (size_t)P * N;

    for (int base = 0; base < P; base += ROWS_PER_PASS) {
        float4 s[kMultiUnroll][VEC];
#pragma unroll
        for (int k = 0; k < kMultiUnroll; ++k) {
            const int r = base + (k * kMultiWarps + warp) * RPW + ri;
#pragma unroll
            for (int v = 0; v < VEC; ++v)
                s[k][v] = (r < P) ? __ldcs(reinterpret_cast<const float4 *>(
                                        st + (size_t)r * N + (v * LPR + li) * 4))
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        for (int t0 = 0; t0 < nsteps; t0 += kTokBlock) {
            const int nt = min(kTokBlock, nsteps - t0);
            // stage the block's per-token inputs (issued while the state loads fly)
            for (int i = threadIdx.x; i < nt * N; i += blockDim.x) {
                const int t = i / N, n = i - t * N;
                const size_t bt = (size_t)b * a.ntok + t0 + t;
                sB[t][n] = load_f32(Bm + (bt * a.ngroups + g) * N + n);
                sC[t][n] = load_f32(Cm + (bt * a.ngroups + g) * N + n);
            }
            for (int i = threadIdx.x; i < nt * P; i += blockDim.x) {
                const int t = i / P, p = i - t * P;
                sX[t][p] = load_f32(x + (((size_t)b * a.ntok + t0 + t) * H + h) * P + p);
            }
            if (threadIdx.x < nt) {
                const float d = dt_apply(a.dtp, __ldg(a.dt + ((size_t)b * a.ntok + t0 + threadIdx.x) * H + h), h);
                sDt[threadIdx.x] = d;
                sDecay[threadIdx.x] = expf(d * Ah);
            }
            __syncthreads();
            for (int tt = 0; tt < nt; ++tt) {
                const int t = t0 + tt;
                const size_t bt = (size_t)b * a.ntok + t;
                const float dtv = sDt[tt], decay = sDecay[tt];
                float4 bv[VEC], cv[VEC];
#pragma unroll
                for (int v = 0; v < VEC; ++v) {
                    bv[v] = *reinterpret_cast<const float4 *>(&sB[tt][(v * LPR + li) * 4]);
                    cv[v] = *reinterpret_cast<const float4 *>(&sC[tt][(v * LPR + li) * 4]);
                }
                const size_t xrow = (bt * H + h) * (size_t)P;
                float *ip = a.inter ? a.inter + (bt * H + h) * (size_t)P * N : nullptr;
                float part[kMultiUnroll];   // this lane's share of each row's y
#pragma unroll
                for (int k = 0; k < kMultiUnroll; ++k) {
                    const int r = base + (k * kMultiWarps + warp) * RPW + ri;
                    const float xr = (r < P) ? sX[tt][r] : 0.f;
                    const float2 dec2 = make_float2(decay, decay);
                    const float2 dtx2 = make_float2(dtv * xr, dtv * xr);
                    float2 acc2 = make_float2(0.f, 0.f);
#pragma unroll
                    for (int v = 0; v < VEC; ++v) {
                        // s <- decay s + (dt x) B ;  acc += s C   (fp32x2 lanes)
                        float2 lo = make_float2(s[k][v].x, s[k][v].y);
                        float2 hi = make_float2(s[k][v].z, s[k][v].w);
                        lo = __ffma2_rn(lo, dec2, __fmul2_rn(dtx2, make_float2(bv[v].x, bv[v].y)));
                        hi = __ffma2_rn(hi, dec2, __fmul2_rn(dtx2, make_float2(bv[v].z, bv[v].w)));
                        acc2 = __ffma2_rn(lo, make_float2(cv[v].x, cv[v].y), acc2);
                        acc2 = __ffma2_rn(hi, make_float2(cv[v].z, cv[v].w), acc2);
                        const float4 q = make_float4(lo.x, lo.y, hi.x, hi.y);
                        s[k][v] = q;
                        if (r < P) {
                            const size_t off = (size_t)r * N + (v * LPR + li) * 4;
                            if (ip) __stcs(reinterpret_cast<float4 *>(ip + off), q);
                            if (t + 1 == commit) __stcs(reinterpret_cast<float4 *>(st + off), q);
                        }
                    }
                    part[k] = acc2.x + acc2.y;
                }
                if (y) {
                    if constexpr (LPR == 32 && kMultiUnroll == 8) {
                        // transpose-reduce: halve the rows held per lane at
                        // offsets 16, 8, 4 (4 + 2 + 1 shuffles), then finish
                        // with offsets 2, 1: lane bits 4..2 name the row.
#pragma unroll
                        for (int lvl = 0; lvl < 3; ++lvl) {
                            const int half = 4 >> lvl, off = 16 >> lvl;
                            const bool upper = lane & off;
#pragma unroll
                            for (int i = 0; i < half; ++i) {
                                const float send = upper ? part[i] : part[i + half];
                                const float keep = upper ? part[i + half] : part[i];
                                part[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                            }
                        }
                        float acc = part[0];
                        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                        const int k = ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1);
                        const int r = base + (k * kMultiWarps + warp) * RPW;
                        if ((lane & 3) == 0 && r < P) {
                            const float xr = sX[tt][r];
                            store_out(y + xrow + r, fmaf(Dh, xr, acc));
                        }
                    } else {
#pragma unroll
                        for (int k = 0; k < kMultiUnroll; ++k) {
                            const int r = base + (k * kMultiWarps + warp) * RPW + ri;
                            float acc = part[k];
#pragma unroll
                            for (int o = LPR / 2; o > 0; o >>= 1)
                                acc += __shfl_xor_sync(0xffffffffu, acc, o);
                            if (li == 0 && r < P) store_out(y + xrow + r, fmaf(Dh, sX[tt][r], acc));
                        }
                    }
                }
            }
            __syncthreads();   // the next block overwrites the staged inputs
        }
    }
}

// Verify pass without intermediate states or a commit (y only), d_state 128,
// head_dim <= 64, at most 8 draft tokens: the outputs follow from the
// starting state without stepping it.  With cs_t = sum_{k<=t} dt_k A_h,
//   y_t[p] = exp(cs_t) (s0[p,:] . C_t) + sum_{k<=t} L[t][k] x_k[p] + D_h x_t[p],
//   L[t][k] = exp(cs_t - cs_k) dt_k (C_t . B_k),
// the chunked (state-space-duality) form of the same recurrence over the
// draft.  Per token a thread does one 4-wide dot product per state row it
// holds, instead of updating the state, so the state is read once and the
// arithmetic per state element drops from ~3 operations per token to 1.
constexpr int kVerifyMaxTok = 8;

// Tokens padded to a power of two, for the joint reduction of y.
constexpr int verify_pad(int nt) { return nt <= 1 ? 1 : nt <= 2 ? 2 : nt <= 4 ? 4 : 8; }

template <typename TIn, typename TOut, int NT>
__global__ void __launch_bounds__(kMultiWarps * 32, (NT <= 2 ? 4 : NT <= 4 ? 3 : 2))
state_verify_kernel(MultiUpdateArgs a)
{
    constexpr int N = 128;
    __shared__ __align__(16) float sB[kVerifyMaxTok][N], sC[kVerifyMaxTok][N];
    __shared__ float sX[kVerifyMaxTok][64], sDt[kVerifyMaxTok], sCs[kVerifyMaxTok];
    __shared__ float sL[kVerifyMaxTok][kVerifyMaxTok];

    constexpr int nt = NT;   // draft tokens (a.ntok)
    const int H = a.nheads, P = a.head_dim;
    const int bh = blockIdx.x;
    const int b = bh / H;
    const int h = bh - b * H;
    const int g = h / (H / a.ngroups);
    size_t srow = (size_t)b;
    if (a.slot_idx) {
        const int slot = __ldg(a.slot_idx + b);
        if (slot < 0) return;
        if (slot >= a.max_slots) {
            if (threadIdx.x == 0) report_status(a.status_dev, 6);
            return;
        }
        srow = (size_t)slot;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float Ah = __ldg(a.A + h);
    const float Dh = a.D ? __ldg(a.D + h) : 0.f;
    const TIn *x = static_cast<const TIn *>(a.x);
    const TIn *Bm = static_cast<const TIn *>(a.B);
    const TIn *Cm = static_cast<const TIn *>(a.C);
    TOut *y = static_cast<TOut *>(a.y);
    const float *st = a.state + (srow * H + h) * (size_t)P * N;

    // the starting state: rows warp + 8 k, columns 4 lane .. 4 lane + 3
    float4 s[kMultiUnroll];
#pragma unroll
    for (int k = 0; k < kMultiUnroll; ++k) {
        const int r = k * kMultiWarps + warp;
        s[k] = (r < P) ? __ldcs(reinterpret_cast<const float4 *>(st + (size_t)r * N + lane * 4))
                       : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    // the draft's inputs, staged as fp32
    for (int i = threadIdx.x; i < nt * N; i += blockDim.x) {
        const int t = i >> 7, n = i & (N - 1);
        const size_t bt = (size_t)b * nt + t;
        sB[t][n] = load_f32(Bm + (bt * a.ngroups + g) * N + n);
        sC[t][n] = load_f32(Cm + (bt * a.ngroups + g) * N + n);
    }
    for (int i = threadIdx.x; i < nt * P; i += blockDim.x) {
        const int t = i / P, p = i - t * P;
        sX[t][p] = load_f32(x + (((size_t)b * nt + t) * H + h) * P + p);
    }
    if (threadIdx.x < nt)
        sDt[threadIdx.x] = dt_apply(a.dtp, __ldg(a.dt + ((size_t)b * nt + threadIdx.x) * H + h), h);
    __syncthreads();
    if (threadIdx.x == 0) {
        float c = 0.f;
        for (int t = 0; t < nt; ++t) {
            c += sDt[t] * Ah;
            sCs[t] = c;
        }
    }
    __syncthreads();
    // L[t][k]: one warp per (t, k) pair, a 128-long dot product over the lanes
    for (int pr = warp; pr < nt * nt; pr += kMultiWarps) {
        const int t = pr / nt, k = pr - t * nt;
        float d = 0.f;
        if (k <= t) {
            const float4 c4 = *reinterpret_cast<const float4 *>(&sC[t][lane * 4]);
            const float4 b4 = *reinterpret_cast<const float4 *>(&sB[k][lane * 4]);
            d = c4.x * b4.x + c4.y * b4.y + c4.z * b4.z + c4.w * b4.w;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
            d *= expf(sCs[t] - sCs[k]) * sDt[k];
        }
        if (lane == 0) sL[t][k] = d;
    }
    __syncthreads();

    // y of every token at once: this lane's partial dot products of its 8
    // rows with each C_t (index k NP + t), then one transpose-reduction over
    // all (row, token) pairs: each level keeps half of the values (the upper
    // half in the lanes whose bit `off` is set) and adds the partner's other
    // half, so the tokens share 5 dependent shuffle rounds instead of 5 each.
    constexpr int NP = verify_pad(NT);
    constexpr int M = kMultiUnroll * NP;                       // values per lane
    constexpr int LEVELS = M >= 32 ? 5 : (M == 16 ? 4 : 3);    // lane bits folded with halving
    float part[M];
#pragma unroll
    for (int t = 0; t < NP; ++t) {
        const float4 c4 = t < NT ? *reinterpret_cast<const float4 *>(&sC[t][lane * 4])
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int k = 0; k < kMultiUnroll; ++k) {
            const float2 d2 = __ffma2_rn(make_float2(s[k].x, s[k].y), make_float2(c4.x, c4.y),
                                         __fmul2_rn(make_float2(s[k].z, s[k].w), make_float2(c4.z, c4.w)));
            part[k * NP + t] = d2.x + d2.y;
        }
    }
#pragma unroll
    for (int lvl = 0; lvl < LEVELS; ++lvl) {
        const int half = M >> (lvl + 1), off = 16 >> lvl;
        const bool upper = lane & off;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float send = upper ? part[i] : part[i + half];
            const float keep = upper ? part[i + half] : part[i];
            part[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    // the lane bits not folded: a plain butterfly over the one value left
#pragma unroll
    for (int off = (1 << (5 - LEVELS)) >> 1; off > 0; off >>= 1)
        part[0] += __shfl_xor_sync(0xffffffffu, part[0], off);
    // Lane L now holds the values of index (L >> (5 - LEVELS)) * V + j,
    // j < V = M >> LEVELS (its folded lane bits name the halves it kept);
    // lanes that share those bits hold the same values, and the first writes.
    constexpr int V = M >> LEVELS;
    if ((lane & ((1 << (5 - LEVELS)) - 1)) == 0) {
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const int idx = (lane >> (5 - LEVELS)) * V + j;
            const int k = idx / NP, t = idx - k * NP;
            const int r = k * kMultiWarps + warp;
            if (t < NT && r < P) {
                float v = expf(sCs[t]) * part[j] + Dh * sX[t][r];
                for (int q = 0; q <= t; ++q) v = fmaf(sL[t][q], sX[q][r], v);
                store_out(y + (((size_t)b * nt + t) * H + h) * P + r, v);
            }
        }
    }
}

// state row <- inter[b][accept_len[b] - 1] (unchanged where accept_len is 0).
__global__ void __launch_bounds__(256)
state_commit_kernel(CommitArgs a)
{
    const int H = a.nheads;
    const int bh = blockIdx.x;
    const int b = bh / H;
    const int h = bh - b * H;
    const int acc = __ldg(a.accept_len + b);
    if (acc < 0 || acc > a.ntok) {
        if (threadIdx.x == 0) report_status(a.status_dev, 6);
        return;
    }
    if (acc == 0) return;
    size_t srow = (size_t)b;
    if (a.slot_idx) {
        const int slot = __ldg(a.slot_idx + b);
        if (slot < 0) return;
        if (slot >= a.max_slots) {
            if (threadIdx.x == 0) report_status(a.status_dev, 6);
            return;
        }
        srow = (size_t)slot;
    }
    const size_t elems = (size_t)a.head_dim * a.d_state;   // multiple of 16
    const float4 *src = reinterpret_cast<const float4 *>(
        a.inter + (((size_t)b * a.ntok + (acc - 1)) * H + h) * elems);
    float4 *dst = reinterpret_cast<float4 *>(a.state + (srow * H + h) * elems);
    for (size_t i = threadIdx.x; i < elems / 4; i += blockDim.x) __stcs(dst + i, __ldcs(src + i));
}

template <int N, typename TIn, typename TOut>
static cudaError_t launch_multi_t(const MultiUpdateArgs &a, cudaStream_t stream)
{
    const unsigned grid = (unsigned)((size_t)a.batch * a.nheads);
    if (N == 128 && a.head_dim <= 64 && a.ntok >= 1 && a.ntok <= kVerifyMaxTok && !a.inter &&
        !a.accept_len && a.y) {
        switch (a.ntok) {
        case 1: state_verify_kernel<TIn, TOut, 1><<<grid, kMultiWarps * 32, 0, stream>>>(a); break;
        case 2: state_verify_kernel<TIn, TOut, 2><<<grid, kMultiWarps * 32, 0, stream>>>(a); break;
        case 3: state_verify_kernel<TIn, TOut, 3><<<grid, kMultiWarps * 32, 0, stream>>>(a); break;
        case 4: state_verify_kernel<TIn, TOut, 4><<<grid, kMultiWarps * 32, 0, stream>>>(a); break;
        case 5: state_verify_kernel<TIn, TOut, 5><<<grid, kMultiWarps * 32, 0, stream>>>(a); break;
        case 6: state_verify_kernel<TIn, TOut, 6><<<grid, kMultiWarps * 32, 0, stream>>>(a); break;
        case 7: state_verify_kernel<TIn, TOut, 7><<<grid, kMultiWarps * 32, 0, stream>>>(a); break;
        default: state_verify_kernel<TIn, TOut, 8><<<grid, kMultiWarps * 32, 0, stream>>>(a); break;
        }
        return cudaGetLastError();
    }
    state_update_multi_kernel<N, TIn, TOut><<<grid, kMultiWarps * 32, 0, stream>>>(a);
    return cudaGetLastError();
}

template <int N>
static cudaError_t launch_multi_n(const MultiUpdateArgs &a, cudaStream_t stream)
{
    const bool in_bf16 = a.in_dtype == 1, out_bf16 = a.y_dtype == 1;
    if (in_bf16 && out_bf16) return launch_multi_t<N, __nv_bfloat16, __nv_bfloat16>(a, stream);
    if (in_bf16) return launch_multi_t<N, __nv_bfloat16, float>(a, stream);
    if (out_bf16) return launch_multi_t<N, float, __nv_bfloat16>(a, stream);
    return launch_multi_t<N, float, float>(a, stream);
}

cudaError_t launch_state_update_multi(const MultiUpdateArgs &a, cudaStream_t stream)
{
    switch (a.d_state) {
    case 16: return launch_multi_n<16>(a, stream);
    case 32: return launch_multi_n<32>(a, stream);
    case 64: return launch_multi_n<64>(a, stream);
    case 128: return launch_multi_n<128>(a, stream);
    case 256: return launch_multi_n<256>(a, stream);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_state_commit(const CommitArgs &a, cudaStream_t stream)
{
    state_commit_kernel<<<(unsigned)((size_t)a.batch * a.nheads), 256, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace ssm
