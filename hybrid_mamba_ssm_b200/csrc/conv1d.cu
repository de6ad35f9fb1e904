// conv1d.cu -- causal depthwise conv1d (+ optional SiLU) in the channels-last
// layout, the short convolution that produces the scan's x, B and C
// ("Depthwise SiLU 卷积" of the MAX nemotron_h article, section 5.4 item 2;
// causal_conv1d_fn / causal_conv1d_update of the modeling_nemotron_h.py
// walk-through).  For channel c, width K and token t of a sequence:
//
//   y[t][c] = act(bias[c] + sum_{k<K} w[c][k] * in[t - (K-1) + k][c])
//
// where the inputs before the sequence start come from its conv state (the
// K-1 most recent earlier inputs, oldest first) or are zero.  Afterwards the
// state holds the sequence's K-1 most recent inputs.
//
// Prefill runs as two launches: the convolution over 64-token tiles of the
// packed stream (several tiles of one sequence read its old state
// concurrently), then one pass per (sequence, channel) that rolls the state.
// Decode is one launch per token batch; the window rolls in place.
// All three are bound by HBM: each input and output is touched once.
#include "common.cuh"
#include "ssm_internal.h"
#include "tc_ptx.cuh"

namespace ssm {

constexpr int kConvThreads = 256;   // channels per CTA
constexpr int kConvTile = 64;       // tokens per CTA
constexpr int kMaxWidth = 8;

// SiLU as v * (1 / (1 + e^-v)) with the hardware approximate reciprocal
// (rcp of +inf is 0, so large negative v gives -0 as the limit does).
__device__ __forceinline__ float conv_act(float v, int act) {
    return act ? v * rcp_approx(1.f + __expf(-v)) : v;
}

__device__ __forceinline__ float ld_in(const float *p) { return *p; }
__device__ __forceinline__ float ld_in(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st_in(float *p, float v) { *p = v; }
__device__ __forceinline__ void st_in(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }

// Prefill state row of sequence s: >= 0 a row of the state (or pool), -1 no
// state given, -2 a slot index outside [0, max_slots) (reported; the sequence
// is skipped, as the scan does).
__device__ __forceinline__ long conv_state_row(const ConvArgs &a, int s, bool &load_init) {
    load_init = a.state != nullptr;
    if (!a.state) return -1;
    if (a.has_initial && a.has_initial[s] == 0) load_init = false;
    if (!a.slot_idx) return s;
    const int slot = a.slot_idx[s];
    if (slot < 0 || slot >= a.max_slots) {
        report_status(a.status_dev, 6);
        return -2;
    }
    return slot;
}

template <typename TIn, typename TOut>
__global__ void __launch_bounds__(kConvThreads)
conv1d_fwd_kernel(ConvArgs a)
{
    const int c = blockIdx.y * kConvThreads + threadIdx.x;
    const long tok0 = (long)blockIdx.x * kConvTile;
    const long T = a.cu_seqlens ? (long)a.seqlen : (long)a.nseq * a.seqlen;
    if (tok0 >= T) return;
    const long tok1 = min(tok0 + kConvTile, T);
    const int K = a.width, dim = a.dim;
    const TIn *x = static_cast<const TIn *>(a.x);
    const TIn *st = static_cast<const TIn *>(a.state);
    TOut *y = static_cast<TOut *>(a.y);

    // sequence holding tok0 (last s with start <= tok0 and end > tok0)
    __shared__ int s_seq;
    if (threadIdx.x == 0) {
        int s;
        if (a.cu_seqlens) {
            int lo = 0, hi = a.nseq - 1;
            while (lo < hi) {   // largest s with cu[s] <= tok0
                const int mid = (lo + hi + 1) >> 1;
                if (a.cu_seqlens[mid] <= tok0) lo = mid; else hi = mid - 1;
            }
            s = lo;
            while (s + 1 < a.nseq && a.cu_seqlens[s + 1] <= tok0) ++s;
        } else {
            s = (int)(tok0 / a.seqlen);
        }
        s_seq = s;
    }
    __syncthreads();
    if (c >= dim) return;

    float w[kMaxWidth];
#pragma unroll
    for (int k = 0; k < kMaxWidth; ++k) w[k] = (k < K) ? a.weight[(size_t)c * K + k] : 0.f;
    const float bias = a.bias ? a.bias[c] : 0.f;

    int s = s_seq;
    auto seq_start = [&](int q) -> long { return a.cu_seqlens ? (long)a.cu_seqlens[q] : (long)q * a.seqlen; };
    auto seq_end = [&](int q) -> long { return a.cu_seqlens ? (long)a.cu_seqlens[q + 1] : (long)(q + 1) * a.seqlen; };

    // window: win[K-2] is the input just before the current token
    float win[kMaxWidth - 1];
    bool skip = false;
    auto load_window = [&](long t) {
        const long ts = seq_start(s);
        bool load_init;
        const long row = conv_state_row(a, s, load_init);
        skip = row == -2;
#pragma unroll
        for (int j = 0; j < kMaxWidth - 1; ++j) {
            float v = 0.f;
            if (j < K - 1) {
                const long src = t - (K - 1) + j;   // absolute token of window slot j
                if (src >= ts && src >= 0) v = ld_in(x + (size_t)src * dim + c);
                else if (row >= 0 && load_init && src - ts >= -(K - 1))
                    v = ld_in(st + ((size_t)row * dim + c) * (K - 1) + (K - 1) + (src - ts));
            }
            win[j] = v;
        }
    };
    load_window(tok0);
    long te = seq_end(s);
    for (long t = tok0; t < tok1; ++t) {
        if (t >= te) {   // next sequence (skipping empty ones)
            do { ++s; } while (s + 1 < a.nseq && seq_end(s) <= t);
            if (s >= a.nseq) {   // offsets end before T: reported by the state pass
                report_status(a.status_dev, 6);
                return;
            }
            te = seq_end(s);
            load_window(t);
        }
        const float cur = ld_in(x + (size_t)t * dim + c);
        float acc = bias;
#pragma unroll
        for (int j = 0; j < kMaxWidth - 1; ++j)
            if (j < K - 1) acc = fmaf(w[j], win[j], acc);
        acc = fmaf(w[K - 1], cur, acc);
        if (!skip) store_out(y + (size_t)t * dim + c, conv_act(acc, a.activation));
#pragma unroll
        for (int j = 0; j < kMaxWidth - 1; ++j) {
            if (j < K - 2) win[j] = win[j + 1];
            else if (j == K - 2) win[j] = cur;
        }
    }
}

// Vectorised form for dim % V == 0: each thread owns V adjacent channels
// (one 16-byte load per token row: 8 bf16 or 4 fp32), the width is a
// template constant, and tiles whose whole window lies inside one sequence
// (all but the tiles at a sequence start) issue 8 row loads before using
// any, so every warp keeps 4 KB of loads in flight.
template <typename T> struct ConvVec;
template <> struct ConvVec<__nv_bfloat16> { static constexpr int V = 8; using Raw = uint4; };
template <> struct ConvVec<float> { static constexpr int V = 4; using Raw = float4; };

constexpr int kVecThreads = 128;

__device__ __forceinline__ void unpack_row(const uint4 &r, float (&f)[8]) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 v = __bfloat1622float2(h[i]);
        f[2 * i] = v.x;
        f[2 * i + 1] = v.y;
    }
}
__device__ __forceinline__ void unpack_row(const float4 &r, float (&f)[4]) {
    f[0] = r.x; f[1] = r.y; f[2] = r.z; f[3] = r.w;
}

template <int V>
__device__ __forceinline__ void store_row(float *p, const float (&v)[V]) {
#pragma unroll
    for (int i = 0; i < V / 4; ++i)
        reinterpret_cast<float4 *>(p)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}
template <int V>
__device__ __forceinline__ void store_row(__nv_bfloat16 *p, const float (&v)[V]) {
    uint32_t w[V / 2];
#pragma unroll
    for (int i = 0; i < V / 2; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t *>(&h);
    }
    if constexpr (V == 8) *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    else *reinterpret_cast<uint2 *>(p) = make_uint2(w[0], w[1]);
}

// The same rows as channel pairs (fp32x2 lanes).
__device__ __forceinline__ void unpack_row2(const uint4 &r, float2 (&f)[4]) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) f[i] = __bfloat1622float2(h[i]);
}
__device__ __forceinline__ void unpack_row2(const float4 &r, float2 (&f)[2]) {
    f[0] = make_float2(r.x, r.y);
    f[1] = make_float2(r.z, r.w);
}
template <int P2>
__device__ __forceinline__ void store_row2(float *p, const float2 (&v)[P2]) {
#pragma unroll
    for (int i = 0; i < P2 / 2; ++i)
        reinterpret_cast<float4 *>(p)[i] = make_float4(v[2 * i].x, v[2 * i].y, v[2 * i + 1].x, v[2 * i + 1].y);
}
template <int P2>
__device__ __forceinline__ void store_row2(__nv_bfloat16 *p, const float2 (&v)[P2]) {
    uint32_t w[P2];
#pragma unroll
    for (int i = 0; i < P2; ++i) {
        const __nv_bfloat162 h = __float22bfloat162_rn(v[i]);
        w[i] = *reinterpret_cast<const uint32_t *>(&h);
    }
    if constexpr (P2 == 4) *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    else *reinterpret_cast<uint2 *>(p) = make_uint2(w[0], w[1]);
}

// SiLU of two lanes: v / (1 + 2^(-v log2 e)), the exponential and the
// reciprocal on the special-function unit, the rest as fp32x2 arithmetic.
__device__ __forceinline__ float2 silu2(float2 v) {
    constexpr float kNegLog2e = -1.4426950408889634f;
    const float2 e = __fmul2_rn(v, make_float2(kNegLog2e, kNegLog2e));
    float2 d = make_float2(ex2_approx(e.x), ex2_approx(e.y));
    d = __fadd2_rn(d, make_float2(1.f, 1.f));
    return __fmul2_rn(v, make_float2(rcp_approx(d.x), rcp_approx(d.y)));
}

template <typename TIn>
__device__ __forceinline__ typename ConvVec<TIn>::Raw load_row(const TIn *p) {
    return __ldg(reinterpret_cast<const typename ConvVec<TIn>::Raw *>(p));
}

// Pipelined prefill for dim % V == 0.  A CTA owns one strip of
// kPipeThreads*V channels (2 KB of a token row) and a contiguous range of
// tokens; one thread streams the strip's rows into a ring of shared-memory
// stages with bulk copies (kPipeRows rows per stage, completion on an
// mbarrier) while all threads convolve the stage before.  The window carries
// across rows in registers; at the range start and at every sequence start
// inside the range it is reloaded from x, the conv state or zeros.
constexpr int kPipeRows = 8;
constexpr int kPipeStages = 3;
constexpr int kPipeRowBytes = kVecThreads * 16;
constexpr int kPipeSmem = kPipeStages * kPipeRows * kPipeRowBytes + kPipeStages * 8;
// Resident pipelined CTAs per SM: shared memory allows 4; the register cap
// that keeps 4 (128) only fits the narrow windows of 8-channel threads.
__host__ __device__ constexpr int pipe_ctas(int V, int K) {
    return V * K <= 32 ? 4 : (V * K <= 48 ? 3 : 2);
}

template <typename TIn, typename TOut, int K, bool ACT>
__global__ void __launch_bounds__(kVecThreads, pipe_ctas(ConvVec<TIn>::V, K))
conv1d_fwd_pipe_kernel(ConvArgs a, int ncta)
{
    constexpr int V = ConvVec<TIn>::V;
    constexpr int W = K > 1 ? K - 1 : 1;
    using Raw = typename ConvVec<TIn>::Raw;
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ int s_seq;
    __shared__ int s_abort;   // set when a stage's wait expires
    const uint32_t ring = tc::smem_u32(smem);
    const uint32_t bar0 = ring + kPipeStages * kPipeRows * kPipeRowBytes;
    const int tid = threadIdx.x, dim = a.dim;
    const int c_base = blockIdx.y * kVecThreads * V;
    const uint32_t strip_bytes = (uint32_t)min(kVecThreads * V, dim - c_base) * sizeof(TIn);
    const int c0 = c_base + tid * V;
    const bool active = c0 < dim;
    const long T = a.cu_seqlens ? (long)a.seqlen : (long)a.nseq * a.seqlen;
    const long t_begin = T * blockIdx.x / ncta, t_end = T * (blockIdx.x + 1) / ncta;
    if (t_begin >= t_end) return;                       // uniform over the CTA
    const int groups = (int)((t_end - t_begin + kPipeRows - 1) / kPipeRows);
    const TIn *x = static_cast<const TIn *>(a.x);
    TOut *y = static_cast<TOut *>(a.y);

    const bool produce = a.stall_producer == 0;
    int issued = 0;   // stages armed so far (thread 0), for the drain after an abort
    auto issue = [&](int g) {
        if (!produce) return;
        issued = g + 1;
        const int slot = g % kPipeStages;
        const long r0 = t_begin + (long)g * kPipeRows;
        const int n = (int)min((long)kPipeRows, t_end - r0);
        const uint32_t bar = bar0 + 8 * slot;
        tc::mbar_arrive_expect_tx(bar, n * strip_bytes);
        for (int r = 0; r < n; ++r)
            tc::bulk_load_1d(ring + (slot * kPipeRows + r) * kPipeRowBytes,
                             x + (size_t)(r0 + r) * dim + c_base, strip_bytes, bar);
    };
    if (tid == 0) {
        for (int i = 0; i < kPipeStages; ++i) tc::mbar_init(bar0 + 8 * i, 1);
        s_abort = 0;
        tc::fence_mbar_init();
        for (int g = 0; g < min(kPipeStages, groups); ++g) issue(g);
        int s = 0;
        if (a.cu_seqlens) {
            int lo = 0, hi = a.nseq - 1;
            while (lo < hi) {   // last sequence starting at or before t_begin
                const int mid = (lo + hi + 1) >> 1;
                if (a.cu_seqlens[mid] <= t_begin) lo = mid; else hi = mid - 1;
            }
            s = lo;
        } else {
            s = (int)(t_begin / a.seqlen);
        }
        s_seq = s;
    }
    __syncthreads();

    // channels in pairs: the products and the SiLU run on packed fp32x2
    constexpr int P2 = V / 2;
    float2 w2[K][P2], b2[P2];
    if (active) {
        float wv[V * K];
#pragma unroll
        for (int i = 0; i < V * K / 4; ++i) {
            const float4 q = __ldg(reinterpret_cast<const float4 *>(a.weight + (size_t)c0 * K) + i);
            wv[4 * i] = q.x; wv[4 * i + 1] = q.y; wv[4 * i + 2] = q.z; wv[4 * i + 3] = q.w;
        }
#pragma unroll
        for (int k = 0; k < K; ++k)
#pragma unroll
            for (int p = 0; p < P2; ++p) w2[k][p] = make_float2(wv[(2 * p) * K + k], wv[(2 * p + 1) * K + k]);
#pragma unroll
        for (int p = 0; p < P2; ++p)
            b2[p] = a.bias ? make_float2(__ldg(a.bias + c0 + 2 * p), __ldg(a.bias + c0 + 2 * p + 1))
                           : make_float2(0.f, 0.f);
    }

    int s = s_seq;
    auto seq_start = [&](int q) -> long { return a.cu_seqlens ? (long)a.cu_seqlens[q] : (long)q * a.seqlen; };
    auto seq_end = [&](int q) -> long { return a.cu_seqlens ? (long)a.cu_seqlens[q + 1] : (long)(q + 1) * a.seqlen; };
    long ts = seq_start(s), te = seq_end(s);
    const TIn *st = static_cast<const TIn *>(a.state);
    bool skip = false, dead = false;
    float2 win[W][P2];   // win[j] = inputs of token t-(K-1)+j
    auto load_window = [&](long t) {
        bool load_init;
        const long row = conv_state_row(a, s, load_init);
        skip = row == -2;
#pragma unroll
        for (int j = 0; j < K - 1; ++j) {
            const long src = t - (K - 1) + j;
            if (src >= ts && src >= 0) {
                unpack_row2(load_row(x + (size_t)src * dim + c0), win[j]);
            } else {
                auto sv = [&](int c) {
                    return (row >= 0 && load_init)
                        ? ld_in(st + ((size_t)row * dim + c) * (K - 1) + (K - 1) + (src - ts)) : 0.f;
                };
#pragma unroll
                for (int p = 0; p < P2; ++p) win[j][p] = make_float2(sv(c0 + 2 * p), sv(c0 + 2 * p + 1));
            }
        }
    };
    if (active) load_window(t_begin);

    // one token: y row from the window and the staged row, then roll the window
    auto token = [&](long t, const uint8_t *rowp, bool write) {
        float2 cur[P2], out[P2];
        unpack_row2(*reinterpret_cast<const Raw *>(rowp), cur);
#pragma unroll
        for (int p = 0; p < P2; ++p) {
            float2 acc = b2[p];
#pragma unroll
            for (int j = 0; j < K - 1; ++j) acc = __ffma2_rn(w2[j][p], win[j][p], acc);
            acc = __ffma2_rn(w2[K - 1][p], cur[p], acc);
            out[p] = ACT ? silu2(acc) : acc;
        }
        if (write) store_row2<P2>(y + (size_t)t * dim + c0, out);
#pragma unroll
        for (int j = 0; j < K - 2; ++j)
#pragma unroll
            for (int p = 0; p < P2; ++p) win[j][p] = win[j + 1][p];
        if (K > 1)
#pragma unroll
            for (int p = 0; p < P2; ++p) win[W - 1][p] = cur[p];
    };

    const uint64_t limit_ns = a.wait_ns ? a.wait_ns : kDefaultWaitNs;
    bool ok = true;
    int g = 0;
    for (; g < groups; ++g) {
        const int slot = g % kPipeStages;
        // A stage that does not land in time raises the CTA-wide abort flag;
        // every thread sees it after this iteration's barrier and leaves the
        // loop, and thread 0 then drains the copies still in flight.
        if (!tc::mbar_wait_bounded(bar0 + 8 * slot, (uint32_t)((g / kPipeStages) & 1), ok, limit_ns))
            *reinterpret_cast<volatile int *>(&s_abort) = 1;
        const long r0 = t_begin + (long)g * kPipeRows;
        const int n = (int)min((long)kPipeRows, t_end - r0);
        const uint8_t *base = smem + slot * kPipeRows * kPipeRowBytes + tid * 16;
        if (ok && active && !dead) {
            if (n == kPipeRows && r0 + kPipeRows <= te) {
                // whole stage inside the current sequence
#pragma unroll
                for (int r = 0; r < kPipeRows; ++r) token(r0 + r, base + r * kPipeRowBytes, !skip);
            } else {
                for (int r = 0; r < n; ++r) {
                    const long t = r0 + r;
                    if (t >= te) {   // next sequence (skipping empty ones)
                        do { ++s; } while (s + 1 < a.nseq && seq_end(s) <= t);
                        if (s >= a.nseq) {   // offsets end before T
                            report_status(a.status_dev, 6);
                            dead = true;
                            break;
                        }
                        ts = seq_start(s);
                        te = seq_end(s);
                        load_window(t);
                    }
                    token(t, base + r * kPipeRowBytes, !skip);
                }
            }
        }
        __syncthreads();                 // every thread is done with this slot
        if (*reinterpret_cast<volatile int *>(&s_abort)) break;   // uniform after the barrier
        if (tid == 0 && g + kPipeStages < groups) {
            tc::fence_proxy_async_smem();
            issue(g + kPipeStages);
        }
    }
    if (g < groups && tid == 0) {
        // Aborted at stage g: wait (bounded) for the last phase armed on each
        // ring slot, so that no bulk copy lands after the CTA has exited.
        for (int q = max(g, issued - kPipeStages); q < issued; ++q) {
            bool dok = true;
            tc::mbar_wait_bounded(bar0 + 8 * (q % kPipeStages), (uint32_t)((q / kPipeStages) & 1), dok,
                                  limit_ns);
        }
        report_status(a.status_dev, kStatusTimeout);
    }
}

// New conv state of each sequence: its K-1 most recent inputs, with older
// state entries (or zeros) shifting in when the sequence is shorter.
template <typename TIn>
__global__ void __launch_bounds__(kConvThreads)
conv1d_state_kernel(ConvArgs a)
{
    const int c = blockIdx.y * kConvThreads + threadIdx.x;
    const int s = blockIdx.x;
    if (c >= a.dim) return;
    const int K = a.width, dim = a.dim;
    long t0, t1;
    if (a.cu_seqlens) {
        t0 = a.cu_seqlens[s]; t1 = a.cu_seqlens[s + 1];
        if (a.cu_seqlens[0] != 0 || t1 < t0 || t0 < 0 || t1 > a.seqlen ||
            a.cu_seqlens[a.nseq] != a.seqlen) {
            if (c == 0) report_status(a.status_dev, 6);
            return;
        }
    } else {
        t0 = (long)s * a.seqlen; t1 = t0 + a.seqlen;
    }
    bool load_init;
    const long row = conv_state_row(a, s, load_init);
    if (row < 0) return;
    const TIn *x = static_cast<const TIn *>(a.x);
    TIn *st = static_cast<TIn *>(a.state) + ((size_t)row * dim + c) * (K - 1);
    float nw[kMaxWidth - 1];
    const long L = t1 - t0;
#pragma unroll
    for (int k = 0; k < kMaxWidth - 1; ++k) {
        if (k >= K - 1) break;
        const long src = L - (K - 1) + k;
        nw[k] = src >= 0 ? ld_in(x + (size_t)(t0 + src) * dim + c)
                         : (load_init ? ld_in(st + (K - 1) + src) : 0.f);
    }
#pragma unroll
    for (int k = 0; k < kMaxWidth - 1; ++k)
        if (k < K - 1) st_in(st + k, nw[k]);
}

// Tokens after which decode row b writes its state back: all ntok for the
// plain update, accept_len[b] for a speculative commit, none otherwise; -1
// for a bad row (reported).
__device__ __forceinline__ int conv_commit_count(const ConvArgs &a, int b) {
    if (a.accept_len) {
        const int n = a.accept_len[b];
        if (n < 0 || n > a.ntok) {
            report_status(a.status_dev, 6);
            return -1;
        }
        return n;
    }
    return a.commit_all ? a.ntok : 0;
}

// Decode: ntok tokens per batch row (x, y [batch][ntok][dim]) from the row's
// window; the state row is rewritten after the committed tokens.
template <typename TIn, typename TOut>
__global__ void __launch_bounds__(kConvThreads)
conv1d_update_kernel(ConvArgs a)
{
    const int c = blockIdx.y * kConvThreads + threadIdx.x;
    const int b = blockIdx.x;
    if (c >= a.dim) return;
    const int K = a.width, dim = a.dim;
    long row = b;
    if (a.slot_idx) {
        const int slot = a.slot_idx[b];
        if (slot < 0) return;                   // padding row
        if (slot >= a.max_slots) {
            if (c == 0) report_status(a.status_dev, 6);
            return;
        }
        row = slot;
    }
    const int commit = conv_commit_count(a, b);
    if (commit < 0) return;
    TIn *st = static_cast<TIn *>(a.state) + ((size_t)row * dim + c) * (K - 1);
    float win[kMaxWidth - 1];
#pragma unroll
    for (int j = 0; j < kMaxWidth - 1; ++j) win[j] = (j < K - 1) ? ld_in(st + j) : 0.f;
    const float bias = a.bias ? a.bias[c] : 0.f;
    for (int t = 0; t < a.ntok; ++t) {
        const size_t xi = ((size_t)b * a.ntok + t) * dim + c;
        const float cur = ld_in(static_cast<const TIn *>(a.x) + xi);
        float acc = bias;
#pragma unroll
        for (int j = 0; j < kMaxWidth - 1; ++j)
            if (j < K - 1) acc = fmaf(a.weight[(size_t)c * K + j], win[j], acc);
        acc = fmaf(a.weight[(size_t)c * K + K - 1], cur, acc);
        if (a.y) store_out(static_cast<TOut *>(a.y) + xi, conv_act(acc, a.activation));
#pragma unroll
        for (int j = 0; j < kMaxWidth - 1; ++j) {
            if (j < K - 2) win[j] = win[j + 1];
            else if (j == K - 2) win[j] = cur;
        }
        if (t + 1 == commit) {
#pragma unroll
            for (int j = 0; j < kMaxWidth - 1; ++j)
                if (j < K - 1) st_in(st + j, win[j]);
        }
    }
}

// Vectorised decode for dim % V == 0: V adjacent channels per thread, whose
// state windows are (K-1) consecutive 16-byte vectors of the state row.  A
// thread serves kUpdateRows batch rows of its channels: the loads of all of
// them go out first, and the weights and bias (the same for every row) are
// loaded once for them.
constexpr int kUpdateRows = 2;

template <typename TIn, typename TOut, int K>
__global__ void __launch_bounds__(kVecThreads)
conv1d_update_vec_kernel(ConvArgs a)
{
    constexpr int V = ConvVec<TIn>::V;
    constexpr int W = K > 1 ? K - 1 : 1;
    using Raw = typename ConvVec<TIn>::Raw;
    const int c0 = (blockIdx.y * kVecThreads + threadIdx.x) * V;
    const int dim = a.dim;
    if (c0 >= dim) return;
    const TIn *x = static_cast<const TIn *>(a.x);
    // the rows' state rows (-1: nothing to do), commit counts, state windows
    // and first tokens, all requested before any arithmetic
    long rows[kUpdateRows];
    int commits[kUpdateRows];
    Raw raw[kUpdateRows][W], x0[kUpdateRows];
#pragma unroll
    for (int j = 0; j < kUpdateRows; ++j) {
        const int b = blockIdx.x * kUpdateRows + j;
        rows[j] = -1;
        commits[j] = 0;
        if (b >= a.nseq) continue;
        long row = b;
        if (a.slot_idx) {
            const int slot = __ldg(a.slot_idx + b);
            if (slot < 0) continue;                 // padding row
            if (slot >= a.max_slots) {
                if (c0 == 0) report_status(a.status_dev, 6);
                continue;
            }
            row = slot;
        }
        const int commit = conv_commit_count(a, b);
        if (commit < 0) continue;
        rows[j] = row;
        commits[j] = commit;
        const TIn *st = static_cast<const TIn *>(a.state) + ((size_t)row * dim + c0) * (K - 1);
#pragma unroll
        for (int i = 0; i < K - 1; ++i) raw[j][i] = *reinterpret_cast<const Raw *>(st + (size_t)i * V);
        if (a.ntok > 0) x0[j] = load_row(x + (size_t)b * a.ntok * dim + c0);
    }
    float w[V * K], bias[V];
#pragma unroll
    for (int i = 0; i < V * K / 4; ++i) {
        const float4 q = __ldg(reinterpret_cast<const float4 *>(a.weight + (size_t)c0 * K) + i);
        w[4 * i] = q.x; w[4 * i + 1] = q.y; w[4 * i + 2] = q.z; w[4 * i + 3] = q.w;
    }
#pragma unroll
    for (int v = 0; v < V; ++v) bias[v] = a.bias ? __ldg(a.bias + c0 + v) : 0.f;
#pragma unroll
    for (int j = 0; j < kUpdateRows; ++j) {
        if (rows[j] < 0) continue;
        const int b = blockIdx.x * kUpdateRows + j;
        const int commit = commits[j];
        // state of channels c0..c0+V-1: V*(K-1) values, channel-major
        TIn *st = static_cast<TIn *>(a.state) + ((size_t)rows[j] * dim + c0) * (K - 1);
        float win[W][V];   // win[i][v]: channel c0+v, window slot i (oldest first)
#pragma unroll
        for (int i = 0; i < K - 1; ++i) {
            float f[V];
            unpack_row(raw[j][i], f);
#pragma unroll
            for (int e = 0; e < V; ++e) win[(i * V + e) % W][(i * V + e) / W] = f[e];
        }
        for (int t = 0; t < a.ntok; ++t) {
            const size_t xi = ((size_t)b * a.ntok + t) * dim + c0;
            float cur[V], out[V];
            unpack_row(t == 0 ? x0[j] : load_row(x + xi), cur);
#pragma unroll
            for (int v = 0; v < V; ++v) {
                float acc = bias[v];
#pragma unroll
                for (int i = 0; i < K - 1; ++i) acc = fmaf(w[v * K + i], win[i][v], acc);
                acc = fmaf(w[v * K + K - 1], cur[v], acc);
                out[v] = conv_act(acc, a.activation);
            }
            if (a.y) store_row<V>(static_cast<TOut *>(a.y) + xi, out);
#pragma unroll
            for (int i = 0; i < K - 2; ++i)
#pragma unroll
                for (int v = 0; v < V; ++v) win[i][v] = win[i + 1][v];
            if (K > 1)
#pragma unroll
                for (int v = 0; v < V; ++v) win[W - 1][v] = cur[v];
            if (t + 1 == commit) {
#pragma unroll
                for (int i = 0; i < K - 1; ++i) {
                    float f[V];
#pragma unroll
                    for (int e = 0; e < V; ++e) f[e] = win[(i * V + e) % W][(i * V + e) / W];
                    store_row<V>(st + (size_t)i * V, f);
                }
            }
        }
    }
}

static int sm_count() {
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

template <typename TIn, typename TOut, int K, bool ACT>
static cudaError_t launch_pipe_k(const ConvArgs &a, dim3 grid, int ncta, cudaStream_t stream) {
    auto kern = conv1d_fwd_pipe_kernel<TIn, TOut, K, ACT>;
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kPipeSmem);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    kern<<<grid, kVecThreads, kPipeSmem, stream>>>(a, ncta);
    return cudaGetLastError();
}

template <typename TIn, typename TOut, bool ACT>
static cudaError_t launch_pipe(const ConvArgs &a, dim3 grid, int ncta, cudaStream_t stream) {
    switch (a.width) {
    case 1: return launch_pipe_k<TIn, TOut, 1, ACT>(a, grid, ncta, stream);
    case 2: return launch_pipe_k<TIn, TOut, 2, ACT>(a, grid, ncta, stream);
    case 3: return launch_pipe_k<TIn, TOut, 3, ACT>(a, grid, ncta, stream);
    case 4: return launch_pipe_k<TIn, TOut, 4, ACT>(a, grid, ncta, stream);
    case 5: return launch_pipe_k<TIn, TOut, 5, ACT>(a, grid, ncta, stream);
    case 6: return launch_pipe_k<TIn, TOut, 6, ACT>(a, grid, ncta, stream);
    case 7: return launch_pipe_k<TIn, TOut, 7, ACT>(a, grid, ncta, stream);
    default: return launch_pipe_k<TIn, TOut, 8, ACT>(a, grid, ncta, stream);
    }
}

template <typename TIn, typename TOut>
static cudaError_t launch_conv_t(const ConvArgs &a, cudaStream_t stream)
{
    const unsigned cblocks = (unsigned)((a.dim + kConvThreads - 1) / kConvThreads);
    constexpr int V = ConvVec<TIn>::V;
    if (a.update) {
        if (a.dim % V == 0) {
            const dim3 grid((unsigned)((a.nseq + kUpdateRows - 1) / kUpdateRows),
                            (unsigned)((a.dim / V + kVecThreads - 1) / kVecThreads));
            switch (a.width) {
            case 1: conv1d_update_vec_kernel<TIn, TOut, 1><<<grid, kVecThreads, 0, stream>>>(a); break;
            case 2: conv1d_update_vec_kernel<TIn, TOut, 2><<<grid, kVecThreads, 0, stream>>>(a); break;
            case 3: conv1d_update_vec_kernel<TIn, TOut, 3><<<grid, kVecThreads, 0, stream>>>(a); break;
            case 4: conv1d_update_vec_kernel<TIn, TOut, 4><<<grid, kVecThreads, 0, stream>>>(a); break;
            case 5: conv1d_update_vec_kernel<TIn, TOut, 5><<<grid, kVecThreads, 0, stream>>>(a); break;
            case 6: conv1d_update_vec_kernel<TIn, TOut, 6><<<grid, kVecThreads, 0, stream>>>(a); break;
            case 7: conv1d_update_vec_kernel<TIn, TOut, 7><<<grid, kVecThreads, 0, stream>>>(a); break;
            default: conv1d_update_vec_kernel<TIn, TOut, 8><<<grid, kVecThreads, 0, stream>>>(a); break;
            }
        } else {
            conv1d_update_kernel<TIn, TOut><<<dim3((unsigned)a.nseq, cblocks), kConvThreads, 0, stream>>>(a);
        }
        return cudaGetLastError();
    }
    const long T = a.cu_seqlens ? (long)a.seqlen : (long)a.nseq * a.seqlen;
    if (T > 0 && a.dim % V == 0) {
        const int strips = (a.dim / V + kVecThreads - 1) / kVecThreads;
        // enough CTAs to fill the GPU once, each with at least 4 stages of rows
        const long fill = (long)pipe_ctas(V, a.width) * sm_count() / strips;
        const long by_rows = (T + 4 * kPipeRows - 1) / (4 * kPipeRows);
        const int ncta = (int)(fill < by_rows ? (fill > 0 ? fill : 1) : by_rows);
        const dim3 grid((unsigned)ncta, (unsigned)strips);
        cudaError_t e = a.activation ? launch_pipe<TIn, TOut, true>(a, grid, ncta, stream)
                                     : launch_pipe<TIn, TOut, false>(a, grid, ncta, stream);
        if (e != cudaSuccess) return e;
    } else if (T > 0) {
        const unsigned tiles = (unsigned)((T + kConvTile - 1) / kConvTile);
        conv1d_fwd_kernel<TIn, TOut><<<dim3(tiles, cblocks), kConvThreads, 0, stream>>>(a);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (a.state && a.width > 1) {
        conv1d_state_kernel<TIn><<<dim3((unsigned)a.nseq, cblocks), kConvThreads, 0, stream>>>(a);
        return cudaGetLastError();
    }
    return cudaSuccess;
}

cudaError_t launch_conv1d(const ConvArgs &a, cudaStream_t stream)
{
    const bool in_bf16 = a.in_dtype == 1, out_bf16 = a.y_dtype == 1;
    if (in_bf16 && out_bf16) return launch_conv_t<__nv_bfloat16, __nv_bfloat16>(a, stream);
    if (in_bf16) return launch_conv_t<__nv_bfloat16, float>(a, stream);
    if (out_bf16) return launch_conv_t<float, __nv_bfloat16>(a, stream);
    return launch_conv_t<float, float>(a, stream);
}

}  // namespace ssm
