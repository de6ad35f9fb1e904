// scan_tc.cu -- chunked SSD scan on the 5th-generation tensor cores
// (tcgen05 MMAs with TMEM accumulators, operands staged by TMA).
//
// Covers bf16 x/B/C with head_dim 64, d_state 128 and 128-token chunks (the
// Nemotron-H / Nemotron-3 Mamba-layer shape); other shapes run on the CUDA-core
// kernel in scan_simt.cu.
//
// Per chunk of L <= 128 tokens of one (sequence, head), with group g, the
// inclusive cumulative decay cs[i] = sum_{k<=i} dt_k A and the carried state H
// ([head_dim, d_state], fp32), the chunked (state-space-duality) form of the
// recurrence is four contractions and an elementwise state pass:
//   G    = C B^T                          (128 x 128, K = d_state)     MMA
//   M    = G o exp(cs_i - cs_j) dt_j [j<=i] (decay mask, fp16)          CUDA cores
//   Y    = M X                            (128 x 64,  K = chunk)       MMA
//   S^T  = B^T (w o X), w_j = exp(cs_L - cs_j) dt_j  (128 x 64, K = chunk)  MMA
//   Yoff = C H^T                          (128 x 64,  K = d_state)     MMA
//   y    = Y + exp(cs_i) Yoff + D x                                    epilogue
//   H   <- exp(cs_L) H + S                                             epilogue
// The diagonal j = i is part of M because the output reads the updated state.
//
// One CTA of 128 threads per (sequence, head); thread i owns TMEM lane i, i.e.
// row i of G / Y / Yoff and d_state index i of S^T and of the carried state,
// which stays in registers (fp32) for the whole sequence.  B, C and x arrive
// by TMA in 128-byte-swizzled tiles; bf16 operands are converted in place to
// fp16 so that the derived operands (M, w o X, H) keep 11 significant bits and
// every MMA is fp16 x fp16 -> fp32.
#include <cuda.h>

#include "common.cuh"
#include "ssm_internal.h"
#include "tc_ptx.cuh"

namespace ssm {
namespace {

constexpr int kQ = 128;       // chunk length
constexpr int kP = 64;        // head_dim
constexpr int kN = 128;       // d_state
constexpr int kThreads = 128;

// Shared memory (bytes from a 1024-aligned base).  16-bit tiles are stored in
// the 128B-swizzled layout TMA writes and the MMA descriptors expect: rows of
// 64 elements (128 bytes), 8-row groups of 1024 bytes, the 16-byte chunk c of
// row r at position c ^ (r % 8).  Tiles 128 elements wide are two such
// 64-column halves, 16 KB apart.
constexpr uint32_t OFF_C = 0;          // C   [128 token i][128 n]
constexpr uint32_t OFF_B = 32768;      // B   [128 token j][128 n]
constexpr uint32_t OFF_X = 65536;      // X   [128 token j][64 p]
constexpr uint32_t OFF_W = 81920;      // w o X [128 token j][64 p]
constexpr uint32_t OFF_M = 98304;      // M   [128 i][128 j]
constexpr uint32_t OFF_H = 131072;     // H^T [128 n][64 p]
constexpr uint32_t OFF_CS = 147456;    // float[128] cumulative dt*A
constexpr uint32_t OFF_DT = OFF_CS + 512;
constexpr uint32_t OFF_WS = OFF_DT + 512;   // float[4] warp partial sums
constexpr uint32_t OFF_BAR = OFF_WS + 64;   // two mbarriers
constexpr uint32_t OFF_TM = OFF_BAR + 16;   // TMEM base address
constexpr uint32_t SMEM_USED = OFF_TM + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;   // + alignment slack
constexpr uint32_t HALF = 16384;
constexpr uint32_t TMA_BYTES = 2 * 2 * HALF + HALF;  // C, B (two halves each), X

// TMEM columns (fp32 accumulators, lane = row).
constexpr uint32_t TM_G = 0, TM_S = 128, TM_YO = 192, TM_Y = 256;
constexpr uint32_t TM_COLS = 512;

constexpr uint32_t IDESC_G = tc::idesc_f16_f32(128, 128, 0, 0);   // C (K-major) x B (K-major)
constexpr uint32_t IDESC_S = tc::idesc_f16_f32(128, 64, 1, 1);    // B^T (MN-major) x wX (MN-major)
constexpr uint32_t IDESC_YO = tc::idesc_f16_f32(128, 64, 0, 1);   // C (K-major) x H^T (MN-major)
constexpr uint32_t IDESC_Y = tc::idesc_f16_f32(128, 64, 0, 1);    // M (K-major) x X (MN-major)

__device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t chunk) {
    return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

__device__ __forceinline__ uint32_t bf2_to_h2(uint32_t v, float scale) {
    const float lo = __uint_as_float(v << 16) * scale;
    const float hi = __uint_as_float(v & 0xffff0000u) * scale;
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ uint32_t f2_to_h2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ float2 h2_to_f2(uint32_t v) {
    return __half22float2(*reinterpret_cast<__half2 *>(&v));
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};"
                 ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

__device__ __forceinline__ void store_row(float *dst, const float (&v)[32]) {
#pragma unroll
    for (int q = 0; q < 8; ++q)
        reinterpret_cast<float4 *>(dst)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

__device__ __forceinline__ void store_row(__nv_bfloat16 *dst, const float (&v)[32]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint4 u;
        __nv_bfloat162 b0 = __floats2bfloat162_rn(v[8 * q + 0], v[8 * q + 1]);
        __nv_bfloat162 b1 = __floats2bfloat162_rn(v[8 * q + 2], v[8 * q + 3]);
        __nv_bfloat162 b2 = __floats2bfloat162_rn(v[8 * q + 4], v[8 * q + 5]);
        __nv_bfloat162 b3 = __floats2bfloat162_rn(v[8 * q + 6], v[8 * q + 7]);
        u.x = *reinterpret_cast<uint32_t *>(&b0);
        u.y = *reinterpret_cast<uint32_t *>(&b1);
        u.z = *reinterpret_cast<uint32_t *>(&b2);
        u.w = *reinterpret_cast<uint32_t *>(&b3);
        reinterpret_cast<uint4 *>(dst)[q] = u;
    }
}

// Write the carried state (this thread's d_state row, 64 values) as fp16 into
// the H^T tile.
__device__ __forceinline__ void write_state_tile(uint32_t sH, uint32_t n, const float (&Hs)[kP]) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        uint4 u;
        u.x = f2_to_h2(Hs[8 * k + 0], Hs[8 * k + 1]);
        u.y = f2_to_h2(Hs[8 * k + 2], Hs[8 * k + 3]);
        u.z = f2_to_h2(Hs[8 * k + 4], Hs[8 * k + 5]);
        u.w = f2_to_h2(Hs[8 * k + 6], Hs[8 * k + 7]);
        sts128(sH + sw128(n, k), u);
    }
}

template <typename TOut>
__global__ void __launch_bounds__(kThreads, 1)
scan_tc_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_b,
               const __grid_constant__ CUtensorMap map_c, const ScanArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = tc::smem_u32(smem);
    float *sCS = reinterpret_cast<float *>(smem + OFF_CS);
    float *sDT = reinterpret_cast<float *>(smem + OFF_DT);
    float *sWS = reinterpret_cast<float *>(smem + OFF_WS);
    const uint32_t bar_tma = sbase + OFF_BAR, bar_mma = sbase + OFF_BAR + 8;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = a.nheads, G = a.ngroups;
    const int s = blockIdx.x / H;
    const int h = blockIdx.x - s * H;
    const int g = h / (H / G);

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

    if (warp == 0) {
        tc::tmem_alloc(sbase + OFF_TM, TM_COLS);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        tc::mbar_init(bar_tma, 1);
        tc::mbar_init(bar_mma, 1);
        tc::fence_mbar_init();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + OFF_TM);
    const uint32_t tlane = (uint32_t)(warp * 32) << 16;

    const size_t state_off = ((size_t)s * H + h) * (size_t)(kP * kN);
    float Hs[kP];
#pragma unroll
    for (int p = 0; p < kP; ++p)
        Hs[p] = a.initial_state ? a.initial_state[state_off + (size_t)p * kN + tid] : 0.f;
    write_state_tile(sbase + OFF_H, tid, Hs);
    tc::fence_proxy_async_smem();
    __syncthreads();

    const float Ah = a.A[h];
    const float Dh = a.D ? a.D[h] : 0.f;
    TOut *y = static_cast<TOut *>(a.y);
    bool ok = true;
    uint32_t ph_tma = 0, ph_mma = 0;

    for (long c0 = t0; c0 < t1; c0 += kQ) {
        const int Lc = (int)min((long)kQ, t1 - c0);
        if (tid == 0) {
            tc::mbar_arrive_expect_tx(bar_tma, TMA_BYTES);
            tc::tma_load_3d(sbase + OFF_C, &map_c, bar_tma, 0, g, (int)c0);
            tc::tma_load_3d(sbase + OFF_C + HALF, &map_c, bar_tma, 64, g, (int)c0);
            tc::tma_load_3d(sbase + OFF_B, &map_b, bar_tma, 0, g, (int)c0);
            tc::tma_load_3d(sbase + OFF_B + HALF, &map_b, bar_tma, 64, g, (int)c0);
            tc::tma_load_3d(sbase + OFF_X, &map_x, bar_tma, 0, h, (int)c0);
        }

        // ---- decay: inclusive cumulative sum of dt*A over the chunk ----
        const bool live = tid < Lc;
        const float dtv = live ? a.dt[(size_t)(c0 + tid) * H + h] : 0.f;
        float v = dtv * Ah;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float u = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += u;
        }
        if (lane == 31) sWS[warp] = v;
        __syncthreads();
        float pre = 0.f;
        for (int w = 0; w < warp; ++w) pre += sWS[w];
        const float cs_i = v + pre;
        sCS[tid] = cs_i;
        sDT[tid] = dtv;
        __syncthreads();
        const float cs_last = sCS[Lc - 1];
        const float w_i = live ? expf(cs_last - cs_i) * dtv : 0.f;

        // ---- operands: bf16 -> fp16 in place, w o X, rows past the end zeroed ----
        tc::mbar_wait_bounded(bar_tma, ph_tma, ok);
        ph_tma ^= 1;
        {
            const float keep = live ? 1.f : 0.f;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t off = half * HALF + sw128(tid, k);
                    uint4 c = lds128(sbase + OFF_C + off);
                    uint4 b = lds128(sbase + OFF_B + off);
                    c = make_uint4(bf2_to_h2(c.x, keep), bf2_to_h2(c.y, keep),
                                   bf2_to_h2(c.z, keep), bf2_to_h2(c.w, keep));
                    b = make_uint4(bf2_to_h2(b.x, keep), bf2_to_h2(b.y, keep),
                                   bf2_to_h2(b.z, keep), bf2_to_h2(b.w, keep));
                    sts128(sbase + OFF_C + off, c);
                    sts128(sbase + OFF_B + off, b);
                }
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t off = sw128(tid, k);
                const uint4 xr = lds128(sbase + OFF_X + off);
                const uint4 xh = make_uint4(bf2_to_h2(xr.x, keep), bf2_to_h2(xr.y, keep),
                                            bf2_to_h2(xr.z, keep), bf2_to_h2(xr.w, keep));
                const uint4 wx = make_uint4(bf2_to_h2(xr.x, w_i), bf2_to_h2(xr.y, w_i),
                                            bf2_to_h2(xr.z, w_i), bf2_to_h2(xr.w, w_i));
                sts128(sbase + OFF_X + off, xh);
                sts128(sbase + OFF_W + off, wx);
            }
        }
        tc::fence_proxy_async_smem();
        __syncthreads();

        // ---- G = C B^T,  S^T = B^T (w o X),  Yoff = C H^T ----
        if (tid == 0) {
            tc::tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t koff = (kk >> 2) * HALF + (kk & 3) * 32;
                tc::mma_f16_ss(tmem + TM_G, tc::sdesc_sw128(sbase + OFF_C + koff, 16, 1024),
                               tc::sdesc_sw128(sbase + OFF_B + koff, 16, 1024), IDESC_G, kk > 0);
            }
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                tc::mma_f16_ss(tmem + TM_S, tc::sdesc_sw128(sbase + OFF_B + kk * 2048, HALF, 1024),
                               tc::sdesc_sw128(sbase + OFF_W + kk * 2048, HALF, 1024), IDESC_S, kk > 0);
            }
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t koff = (kk >> 2) * HALF + (kk & 3) * 32;
                tc::mma_f16_ss(tmem + TM_YO, tc::sdesc_sw128(sbase + OFF_C + koff, 16, 1024),
                               tc::sdesc_sw128(sbase + OFF_H + kk * 2048, HALF, 1024), IDESC_YO, kk > 0);
            }
            tc::mma_commit(bar_mma);
        }
        __syncwarp();
        tc::mbar_wait_bounded(bar_mma, ph_mma, ok);
        ph_mma ^= 1;
        tc::tc_fence_after();

        // ---- M = G o exp(cs_i - cs_j) dt_j for j <= i (row i = tid) ----
#pragma unroll
        for (int jc = 0; jc < 4; ++jc) {
            const uint32_t mrow = sbase + OFF_M + (jc >> 1) * HALF;
            if (jc <= warp) {
                uint32_t r[32];
                tc::tmem_ld32(tmem + tlane + TM_G + jc * 32, r);
                tc::tmem_ld_wait();
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float m[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = jc * 32 + q * 8 + e;
                        m[e] = (j <= tid) ? __uint_as_float(r[q * 8 + e]) * expf(cs_i - sCS[j]) * sDT[j]
                                          : 0.f;
                    }
                    const uint4 u = make_uint4(f2_to_h2(m[0], m[1]), f2_to_h2(m[2], m[3]),
                                               f2_to_h2(m[4], m[5]), f2_to_h2(m[6], m[7]));
                    sts128(mrow + sw128(tid, (jc & 1) * 4 + q), u);
                }
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    sts128(mrow + sw128(tid, (jc & 1) * 4 + q), make_uint4(0, 0, 0, 0));
            }
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();

        // ---- Y = M X ----
        if (tid == 0) {
            tc::tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t koff = (kk >> 2) * HALF + (kk & 3) * 32;
                tc::mma_f16_ss(tmem + TM_Y, tc::sdesc_sw128(sbase + OFF_M + koff, 16, 1024),
                               tc::sdesc_sw128(sbase + OFF_X + kk * 2048, HALF, 1024), IDESC_Y, kk > 0);
            }
            tc::mma_commit(bar_mma);
        }
        __syncwarp();

        // ---- carried state: H <- exp(cs_L) H + S  (this thread: d_state row tid) ----
        {
            const float a_last = expf(cs_last);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t r[32];
                tc::tmem_ld32(tmem + tlane + TM_S + half * 32, r);
                tc::tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    Hs[half * 32 + e] = fmaf(a_last, Hs[half * 32 + e], __uint_as_float(r[e]));
            }
            write_state_tile(sbase + OFF_H, tid, Hs);
        }

        tc::mbar_wait_bounded(bar_mma, ph_mma, ok);
        ph_mma ^= 1;
        tc::tc_fence_after();

        // ---- y = Y + exp(cs_i) Yoff + D x  (row i = tid) ----
        {
            const float e_i = expf(cs_i);
            TOut *yrow = y + ((size_t)(c0 + tid) * H + h) * kP;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t ry[32], ro[32];
                tc::tmem_ld32(tmem + tlane + TM_Y + half * 32, ry);
                tc::tmem_ld32(tmem + tlane + TM_YO + half * 32, ro);
                tc::tmem_ld_wait();
                float out[32];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint4 xr = lds128(sbase + OFF_X + sw128(tid, half * 4 + q));
                    const float2 x01 = h2_to_f2(xr.x), x23 = h2_to_f2(xr.y);
                    const float2 x45 = h2_to_f2(xr.z), x67 = h2_to_f2(xr.w);
                    const float xv[8] = {x01.x, x01.y, x23.x, x23.y, x45.x, x45.y, x67.x, x67.y};
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int c = q * 8 + e;
                        out[c] = fmaf(Dh, xv[e], fmaf(e_i, __uint_as_float(ro[c]), __uint_as_float(ry[c])));
                    }
                }
                if (live) store_row(yrow + half * 32, out);
            }
        }
        tc::tc_fence_before();
        tc::fence_proxy_async_smem();
        __syncthreads();
    }

    if (a.final_state) {
#pragma unroll
        for (int p = 0; p < kP; ++p)
            a.final_state[state_off + (size_t)p * kN + tid] = Hs[p];
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, TM_COLS);
    }
    if (!ok && tid == 0) report_status(a.status_dev, 5);
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 3-D bf16 map over [d2][d1][d0] (d0 contiguous) with a {64, 1, 128} box and
// 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
    const cuuint32_t box[3] = {64, 1, 128};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename TOut>
cudaError_t launch_tc_t(const ScanArgs &a, cudaStream_t stream)
{
    const uint64_t T = a.cu_seqlens ? (uint64_t)a.seqlen : (uint64_t)a.nseq * a.seqlen;
    CUtensorMap mx, mb, mc;
    if (!make_map(&mx, a.x, kP, a.nheads, T) || !make_map(&mb, a.B, kN, a.ngroups, T) ||
        !make_map(&mc, a.C, kN, a.ngroups, T))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(scan_tc_kernel<TOut>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((size_t)a.nseq * a.nheads));
    scan_tc_kernel<TOut><<<grid, kThreads, SMEM_BYTES, stream>>>(mx, mb, mc, a);
    return cudaGetLastError();
}

}  // namespace

bool scan_tc_supports(const ScanArgs &a)
{
    const long long T = a.cu_seqlens ? (long long)a.seqlen : (long long)a.nseq * a.seqlen;
    return a.in_dtype == 1 && a.head_dim == kP && a.d_state == kN && a.chunk_size == kQ &&
           T > 0 && encode_fn() != nullptr;
}

cudaError_t launch_scan_tc(const ScanArgs &a, cudaStream_t stream)
{
    return a.y_dtype == 1 ? launch_tc_t<__nv_bfloat16>(a, stream) : launch_tc_t<float>(a, stream);
}

}  // namespace ssm
