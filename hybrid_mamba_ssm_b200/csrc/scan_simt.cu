// scan_simt.cu -- chunked SSD scan on the CUDA cores (fp32 arithmetic).
//
// This kernel covers every shape and dtype the ABI accepts, including fp32
// inputs and small head_dim / d_state / chunk sizes below the tensor-core
// tile minimums.  The bf16 workloads with head_dim 64 and d_state 128 run on
// the tensor-core kernel (scan_tc.cu) instead.
//
// Chunked form of the recurrence (Mamba-2's structured semiseparable view,
// "2. Mamba block 的常见路径" of the deep-research note): inside a chunk of L
// tokens with cs[i] = sum_{k<=i} dt_k * A (inclusive, from the chunk start),
//   y[i]   = sum_{j<=i} (C_i . B_j) exp(cs_i - cs_j) dt_j x_j      (intra-chunk)
//          + exp(cs_i) * (C_i . H_prev)                           (carried state)
//          + D * x_i
//   H_next = exp(cs_{L-1}) H_prev + sum_j exp(cs_{L-1} - cs_j) dt_j x_j (outer) B_j
// which equals the token-by-token recurrence in exact arithmetic.  Decay
// factors are always exp of a non-positive difference (never a ratio of two
// exponentials), so nothing overflows for A <= 0, dt >= 0.
//
// One CTA per (sequence, head); chunks in order; the state H stays in shared
// memory in fp32 for the whole sequence.
#include "common.cuh"
#include "ssm_internal.h"

namespace ssm {

constexpr int kSimtThreads = 256;
constexpr int kSimtRowBlock = 16;

struct SimtSmem {
    int N1, Q, P, N;
    size_t Bs, Cb, Xs, Hs, Ms, cs, ex, w, dts, total;   // float offsets
};

__host__ __device__ inline SimtSmem simt_smem(int Q, int P, int N)
{
    SimtSmem s;
    s.N1 = N + 1; s.Q = Q; s.P = P; s.N = N;
    size_t o = 0;
    s.Bs = o; o += (size_t)Q * s.N1;
    s.Cb = o; o += (size_t)kSimtRowBlock * s.N1;
    s.Xs = o; o += (size_t)Q * P;
    s.Hs = o; o += (size_t)P * s.N1;
    s.Ms = o; o += (size_t)kSimtRowBlock * Q;
    s.cs = o; o += Q;
    s.ex = o; o += Q;
    s.w = o; o += Q;
    s.dts = o; o += Q;
    s.total = o;
    return s;
}

constexpr int kSimtLongestFirstSeqs = 64;   // packed batches up to this many sequences run longest first

template <typename TIn, typename TOut>
__global__ void __launch_bounds__(kSimtThreads)
scan_simt_kernel(ScanArgs a)
{
    extern __shared__ float smem[];
    const int H = a.nheads, P = a.head_dim, N = a.d_state, G = a.ngroups;
    const int Q = a.chunk_size;
    const SimtSmem L = simt_smem(Q, P, N);
    const int N1 = L.N1;
    float *Bs = smem + L.Bs, *Cb = smem + L.Cb, *Xs = smem + L.Xs;
    float *Hs = smem + L.Hs, *Ms = smem + L.Ms;
    float *cs = smem + L.cs, *ex = smem + L.ex, *w = smem + L.w, *dts = smem + L.dts;

    const int tid = threadIdx.x;
    int s = blockIdx.x / H;
    const int h = blockIdx.x - s * H;
    const int g = h / (H / G);
    if (a.cu_seqlens && a.nseq <= kSimtLongestFirstSeqs) {
        // Packed sequences of mixed lengths run longest first (ties by
        // index): CTAs [r H, (r + 1) H) take the sequence of length rank r.
        __shared__ int s_seq;
        if (tid < a.nseq) {
            const int len = __ldg(a.cu_seqlens + tid + 1) - __ldg(a.cu_seqlens + tid);
            int rank = 0;
            for (int q = 0; q < a.nseq; ++q) {
                const int lq = __ldg(a.cu_seqlens + q + 1) - __ldg(a.cu_seqlens + q);
                rank += (lq > len) || (lq == len && q < tid);
            }
            if (rank == s) s_seq = tid;
        }
        __syncthreads();
        s = s_seq;
    }

    long t0, t1;
    if (a.cu_seqlens) {
        const int c0 = a.cu_seqlens[0], cs0 = a.cu_seqlens[s], cs1 = a.cu_seqlens[s + 1];
        const int cend = a.cu_seqlens[a.nseq];
        if (c0 != 0 || cs1 < cs0 || cs0 < 0 || cend != a.seqlen || cs1 > a.seqlen) {
            if (tid == 0) report_status(a.status_dev, 6);
            return;
        }
        t0 = cs0; t1 = cs1;
    } else {
        t0 = (long)s * a.seqlen; t1 = t0 + a.seqlen;
    }

    const TIn *x = static_cast<const TIn *>(a.x);
    const TIn *Bg = static_cast<const TIn *>(a.B);
    const TIn *Cg = static_cast<const TIn *>(a.C);
    TOut *y = static_cast<TOut *>(a.y);
    const float Ah = a.A[h];
    const float Dh = a.D ? a.D[h] : 0.f;
    size_t srow = (size_t)s;   // state row of this sequence
    bool load_init = a.initial_state != nullptr;
    if (a.slot_idx) {
        const int slot = a.slot_idx[s];
        if (slot < 0 || slot >= a.max_slots) {
            if (tid == 0) report_status(a.status_dev, 6);
            return;
        }
        srow = (size_t)slot;
        if (a.has_initial && a.has_initial[s] == 0) load_init = false;
    }
    const size_t state_off = (srow * H + h) * (size_t)P * N;

    for (int i = tid; i < P * N; i += kSimtThreads) {
        const int p = i / N, n = i - p * N;
        Hs[p * N1 + n] = load_init ? state_load1(a.initial_state, state_off + i, a.rp) : 0.f;
    }

    for (long c0 = t0; c0 < t1; c0 += Q) {
        const int Lc = (int)min((long)Q, t1 - c0);
        __syncthreads();
        for (int i = tid; i < Q; i += kSimtThreads)
            dts[i] = (i < Lc) ? dt_apply(a.dtp, a.dt[(size_t)(c0 + i) * H + h], h) : 0.f;
        for (int i = tid; i < Q * N; i += kSimtThreads) {
            const int j = i / N, n = i - j * N;
            Bs[j * N1 + n] = (j < Lc) ? load_f32(Bg + ((size_t)(c0 + j) * G + g) * N + n) : 0.f;
        }
        for (int i = tid; i < Q * P; i += kSimtThreads) {
            const int j = i / P, p = i - j * P;
            Xs[i] = (j < Lc) ? load_f32(x + ((size_t)(c0 + j) * H + h) * P + p) : 0.f;
        }
        __syncthreads();
        if (tid < 32) {   // inclusive cumulative sum of dt*A over the chunk
            float carry = 0.f;
            for (int base = 0; base < Q; base += 32) {
                float v = dts[base + tid] * Ah;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float u = __shfl_up_sync(0xffffffffu, v, o);
                    if (tid >= o) v += u;
                }
                v += carry;
                cs[base + tid] = v;
                carry = __shfl_sync(0xffffffffu, v, 31);
            }
        }
        __syncthreads();
        const float cs_last = cs[Lc - 1];
        for (int i = tid; i < Q; i += kSimtThreads) {
            ex[i] = expf(cs[i]);
            w[i] = (i < Lc) ? expf(cs_last - cs[i]) * dts[i] : 0.f;
        }

        for (int rb = 0; rb < Lc; rb += kSimtRowBlock) {
            __syncthreads();
            for (int i = tid; i < kSimtRowBlock * N; i += kSimtThreads) {
                const int r = i / N, n = i - r * N;
                const int row = rb + r;
                Cb[r * N1 + n] = (row < Lc) ? load_f32(Cg + ((size_t)(c0 + row) * G + g) * N + n) : 0.f;
            }
            __syncthreads();
            for (int i = tid; i < kSimtRowBlock * Q; i += kSimtThreads) {
                const int r = i / Q, j = i - r * Q;
                const int row = rb + r;
                float m = 0.f;
                if (row < Lc && j <= row) {
                    const float *cr = Cb + r * N1, *br = Bs + j * N1;
                    float dot = 0.f;
                    for (int n = 0; n < N; ++n) dot = fmaf(cr[n], br[n], dot);
                    m = dot * expf(cs[row] - cs[j]) * dts[j];
                }
                Ms[i] = m;
            }
            __syncthreads();
            for (int i = tid; i < kSimtRowBlock * P; i += kSimtThreads) {
                const int r = i / P, p = i - r * P;
                const int row = rb + r;
                if (row >= Lc) continue;
                const float *mr = Ms + r * Q;
                float acc = 0.f;
                for (int j = 0; j <= row; ++j) acc = fmaf(mr[j], Xs[j * P + p], acc);
                const float *cr = Cb + r * N1, *hr = Hs + p * N1;
                float off = 0.f;
                for (int n = 0; n < N; ++n) off = fmaf(cr[n], hr[n], off);
                const float xv = Xs[row * P + p];
                store_out(y + ((size_t)(c0 + row) * H + h) * P + p,
                          acc + ex[row] * off + Dh * xv);
            }
        }
        __syncthreads();
        const float a_last = expf(cs_last);
        for (int i = tid; i < P * N; i += kSimtThreads) {
            const int p = i / N, n = i - p * N;
            float acc = 0.f;
            for (int j = 0; j < Lc; ++j) acc = fmaf(w[j] * Xs[j * P + p], Bs[j * N1 + n], acc);
            Hs[p * N1 + n] = fmaf(a_last, Hs[p * N1 + n], acc);
        }
    }
    __syncthreads();
    if (a.final_state) {
        for (int i = tid; i < P * N; i += kSimtThreads) {
            const int p = i / N, n = i - p * N;
            state_store1(a.final_state, state_off + i, Hs[p * N1 + n], a.rp);
        }
    }
}

template <typename TIn, typename TOut>
static cudaError_t launch_simt_t(const ScanArgs &a, cudaStream_t stream)
{
    const SimtSmem L = simt_smem(a.chunk_size, a.head_dim, a.d_state);
    const size_t bytes = L.total * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(scan_simt_kernel<TIn, TOut>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)bytes);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((size_t)a.nseq * a.nheads));
    scan_simt_kernel<TIn, TOut><<<grid, kSimtThreads, bytes, stream>>>(a);
    return cudaGetLastError();
}

size_t scan_simt_smem_bytes(int Q, int P, int N)
{
    return simt_smem(Q, P, N).total * sizeof(float);
}

cudaError_t launch_scan_simt(const ScanArgs &a, cudaStream_t stream)
{
    const bool in_bf16 = a.in_dtype == 1, out_bf16 = a.y_dtype == 1;
    if (in_bf16 && out_bf16) return launch_simt_t<__nv_bfloat16, __nv_bfloat16>(a, stream);
    if (in_bf16) return launch_simt_t<__nv_bfloat16, float>(a, stream);
    if (out_bf16) return launch_simt_t<float, __nv_bfloat16>(a, stream);
    return launch_simt_t<float, float>(a, stream);
}

}  // namespace ssm
