// scan_tc.cu -- chunked SSD scan on the 5th-generation tensor cores
// (tcgen05 MMAs with TMEM accumulators, operands staged by TMA).
//
// Covers bf16 x/B/C with head_dim 64, d_state 128, 128-token chunks and an
// even number of heads per group (the Nemotron-H / Nemotron-3 Mamba-layer
// shapes); other shapes run on the CUDA-core kernel in scan_simt.cu.
//
// Chunked (state-space-duality) form of the recurrence.  For one chunk of
// L <= 128 tokens of one (sequence, head) with group g, cumulative decay
// cs[i] = sum_{k<=i} dt_k A (inclusive, from the chunk start) and carried
// state H ([head_dim, d_state], fp32):
//   G    = C B^T                                   (shared by the group's heads)
//   M    = G o exp(cs_i - cs_j) dt_j [j <= i]  + D I (decay mask; skip term on
//                                                     the diagonal)
//   Y    = M X
//   S^T  = B^T (w o X),  w_j = exp(cs_{L-1} - cs_j) dt_j
//   Yoff = C H^T
//   y    = Y + exp(cs_i) Yoff,   H <- exp(cs_{L-1}) H + S
// The diagonal j = i belongs to M because the output reads the updated state.
//
// Work decomposition: a CTA sweeps the chunks of (sequence, pair of heads of
// one group) chains in order: one chain per CTA, or (with the caller's
// workspace, for fixed-length batches with more chains than SMs) one run per
// SM of the chains laid end to end, the carried state crossing each cut
// through the workspace.  544 threads: four compute
// warpgroups and one issuing warp.  Compute warpgroup wg works on head
// 2k + (wg & 1) and on half (wg >> 1) of the columns: thread i of it owns TMEM
// lane i (row i of G, M, Y, Yoff; d_state index i of S^T and of the carried
// state, 32 of whose 64 head_dim entries it keeps in fp32 registers for the
// whole sequence).  Lane 0 of the issuing warp issues TMA and the MMAs; the
// products shared by both heads (C.B^T, and B^T or C against the two heads'
// operands side by side) are single N = 128 MMAs.
//
// Pipeline per chunk (single-buffered tiles, with prefetch where a buffer
// frees early):
//   wait TMA(x), TMA(B, C) -> convert bf16 -> fp16 (C into TMEM and B in
//   place, a quarter of d_state per warpgroup; x per head)
//   -> issue TMA(x of next chunk) into the raw x buffers
//   -> MMA S^T (2 heads), G  [commit] , Yoff (2 heads) [commit]
//   -> the next chunk's cumulative decay (while the MMAs run)
//   -> issue TMA(B, C of next chunk) once S^T and G are done
//   -> state update from S^T, decay mask M per head (overlap the Yoff MMAs)
//   -> MMA Y (2 heads) [commit]; meanwhile w o x of the next chunk, whose
//      raw x has landed -> epilogue y.
//
// Precision: bf16 inputs are converted to fp16 (exact for |v| < 65504) so the
// derived operands M, w o x and H (rounded to fp16, 11 significant bits) keep
// the result within ~3e-4 of the fp64 recurrence; accumulation is fp32.
//
// Decay factors are never ratios of exponentials.  With block ends r_K =
// 32K+31, exp(cs_i - cs_j) = exp(cs_i - cs_{r_I}) exp(cs_{r_I} - cs_{r_J})
// exp(cs_{r_J} - cs_j) for i in block I >= J >= j's block: the last two
// factors are <= 1, the first is >= 1 but bounded by the decay over one
// 32-token block; if that exceeds e^80 the block uses exp(cs_i - cs_j) per
// element instead.
#include <cuda.h>

#include "common.cuh"
#include "ssm_internal.h"
#include "tc_ptx.cuh"

namespace ssm {
namespace {

constexpr int kQ = 128;       // chunk length
constexpr int kP = 64;        // head_dim
constexpr int kN = 128;       // d_state
constexpr int kThreads = 544;   // 16 compute warps + 1 issuing warp

// Shared memory (bytes from the 1024-aligned dynamic base).  16-bit tiles use
// the 128B-swizzled layout TMA writes and the MMA descriptors read: rows of 64
// elements (128 B), 8-row groups of 1024 B, 16-byte chunk c of row r stored at
// c ^ (r % 8).  128-wide tiles are two 64-column halves 16 KB apart.
constexpr uint32_t HALF = 16384;
constexpr uint32_t OFF_C = 0;            // C [128 i][128 n]  bf16 (TMA target; fp16 copy in TMEM)
constexpr uint32_t OFF_B = 32768;        // B [128 j][128 n]  (bf16 -> fp16 in place)
constexpr uint32_t OFF_XR = 65536;       // raw x, 2 heads x [128 j][64 p] bf16 (TMA target)
constexpr uint32_t OFF_XH = 98304;       // x as fp16, 2 heads
constexpr uint32_t OFF_WM = 131072;      // w o x, 2 heads x [128 j][64 p]
constexpr uint32_t OFF_MB = 163840;      // y staging, 2 heads x [128 t][64 p] bf16
constexpr uint32_t OFF_H = 196608;       // H^T fp16, 2 heads x [128 n][64 p]
constexpr uint32_t OFF_MISC = 229376;
constexpr uint32_t OFF_VD = OFF_MISC;              // float[2 buffers][2 heads][128]: column factors vd
constexpr uint32_t OFF_CSBT = OFF_VD + 2048;       // float[2 buffers][2 heads][8]: block-end cs, cs_last
constexpr uint32_t OFF_CSB = OFF_CSBT + 128;       // float[4][8]: scan scratch per warpgroup
constexpr uint32_t OFF_PART = OFF_CSB + 128;       // float[4][4] warp partial sums
constexpr uint32_t OFF_BAR = OFF_PART + 64;        // 6 mbarriers
constexpr uint32_t OFF_TM = OFF_BAR + 48;          // TMEM base address (4 B)
constexpr uint32_t OFF_ABORT = OFF_TM + 4;         // CTA-wide abort flag (int)
constexpr uint32_t OFF_RANGE = OFF_TM + 8;         // set when an output is not finite (int)
constexpr uint32_t OFF_SEQ = OFF_TM + 12;          // sequence this CTA sweeps (packed varlen)
constexpr uint32_t OFF_NXP = OFF_TM + 16;          // balanced: first chunk of the next piece (3 ints)
constexpr uint32_t SMEM_BYTES = OFF_TM + 32;

// TMEM columns (fp32 accumulators, lane = row).
// G and Y share columns: the y MMAs write Y only after the mask has read G,
// and the next chunk's G is issued only after the epilogue has read Y.  C
// (fp16, two values per column) is the TMEM A operand of C.B^T and C.H^T.
constexpr uint32_t TM_G = 0, TM_Y = 0, TM_S = 128, TM_YO = 256, TM_C = 384;
constexpr uint32_t TM_COLS = 512;

constexpr uint32_t IDESC_G = tc::idesc_f16_f32(128, 128, 0, 0);   // C (K-major) x B (K-major)
constexpr uint32_t IDESC_S2 = tc::idesc_f16_f32(128, 128, 1, 1);  // B^T (MN-major) x [wX_a|wX_b] (MN-major)
constexpr uint32_t IDESC_YO2 = tc::idesc_f16_f32(128, 128, 0, 1); // C (K-major) x [H_a^T|H_b^T] (MN-major)
constexpr uint32_t IDESC_Y = tc::idesc_f16_f32(128, 64, 0, 1);    // M (TMEM) x X (MN-major)

constexpr float kSafeBlockDecay = 80.f;   // max exp argument taken by the factorised path
constexpr int kLongestFirstSeqs = 64;     // packed batches up to this many sequences run longest first

__device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t chunk) {
    return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

// bf16 pair (low half first) -> two floats, exactly: a mixed-precision add of
// -0 to each bf16 half, which runs on the FMA pipes and needs no unpacking
// shifts or masks on the ALU (the compute warps' busiest pipe).
__device__ __forceinline__ float2 bf2_to_f2(uint32_t v) {
    float lo, hi;
    asm("{\n\t.reg .b16 l, h;\n\t"
        "mov.b32 {l, h}, %2;\n\t"
        "add.rn.f32.bf16 %0, l, 0f80000000;\n\t"
        "add.rn.f32.bf16 %1, h, 0f80000000;\n\t}"
        : "=f"(lo), "=f"(hi) : "r"(v));
    return make_float2(lo, hi);
}

__device__ __forceinline__ uint32_t bf2_to_h2(uint32_t v, float scale) {
    const float2 p = __fmul2_rn(bf2_to_f2(v), make_float2(scale, scale));
    __half2 h = __floats2half2_rn(p.x, p.y);
    return *reinterpret_cast<uint32_t *>(&h);
}

// exp(v) as 2^(v log2 e) with the hardware base-2 exponential (ex2.approx,
// relative error ~2^-22).  The decay arguments here are cumulative sums of
// dt A differences (|v| up to a few hundred), so the rounding of v log2 e
// adds a relative error of about |v| 2^-24, far below the fp16 operands'.
__device__ __forceinline__ float exp_dec(float v) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v * 1.4426950408889634f));
    return r;
}

__device__ __forceinline__ uint32_t f2_to_h2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
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

__device__ __forceinline__ void wg_sync(int wg) {
    asm volatile("bar.sync %0, 128;" ::"r"(wg + 1) : "memory");
}

// Bounded mbarrier wait that, when it expires, raises the CTA-wide abort
// flag: the issuing warp stops issuing TMA loads and MMAs, and every other
// thread skips its remaining waits (it reads the flag after the next named
// barrier).  The kernel then drains what is in flight and exits, reporting
// SSM_ERR_TIMEOUT.
extern __shared__ __align__(1024) uint8_t smem[];

__device__ __forceinline__ int flag_get(uint32_t off) {
    int v;
    asm volatile("ld.volatile.shared.u32 %0, [%1];" : "=r"(v) : "r"(tc::smem_u32(smem) + off) : "memory");
    return v;
}
__device__ __forceinline__ void flag_set(uint32_t off, int v) {
    asm volatile("st.volatile.shared.u32 [%0], %1;" ::"r"(tc::smem_u32(smem) + off), "r"(v) : "memory");
}
__device__ __forceinline__ uint64_t wait_limit(unsigned long long wait_ns) {
    return wait_ns ? wait_ns : kDefaultWaitNs;
}

__device__ __forceinline__ void wait_or_abort(uint32_t bar, uint32_t parity, bool &ok,
                                              unsigned long long wait_ns) {
    if (ok && !tc::mbar_wait_bounded(bar, parity, ok, wait_limit(wait_ns))) flag_set(OFF_ABORT, 1);
}

__device__ __forceinline__ void store16(float *dst, const float (&v)[16]) {
#pragma unroll
    for (int q = 0; q < 4; ++q)
        reinterpret_cast<float4 *>(dst)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

__device__ __forceinline__ void store16(__nv_bfloat16 *dst, const float (&v)[16]) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        __nv_bfloat162 b0 = __floats2bfloat162_rn(v[8 * q + 0], v[8 * q + 1]);
        __nv_bfloat162 b1 = __floats2bfloat162_rn(v[8 * q + 2], v[8 * q + 3]);
        __nv_bfloat162 b2 = __floats2bfloat162_rn(v[8 * q + 4], v[8 * q + 5]);
        __nv_bfloat162 b3 = __floats2bfloat162_rn(v[8 * q + 6], v[8 * q + 7]);
        reinterpret_cast<uint4 *>(dst)[q] =
            make_uint4(*reinterpret_cast<uint32_t *>(&b0), *reinterpret_cast<uint32_t *>(&b1),
                       *reinterpret_cast<uint32_t *>(&b2), *reinterpret_cast<uint32_t *>(&b3));
    }
}

// bf16 pair -> fp16 pair (exact for |v| < 65504).
__device__ __forceinline__ uint32_t bf2h(uint32_t v) {
    const float2 f = bf2_to_f2(v);
    return f2_to_h2(f.x, f.y);
}

__device__ __forceinline__ uint4 cvt_chunk(uint4 r) {
    return make_uint4(bf2h(r.x), bf2h(r.y), bf2h(r.z), bf2h(r.w));
}

__device__ __forceinline__ uint4 cvt_chunk_scaled(uint4 r, float w) {
    return make_uint4(bf2_to_h2(r.x, w), bf2_to_h2(r.y, w), bf2_to_h2(r.z, w), bf2_to_h2(r.w, w));
}

// 32 of this thread's d_state row of the carried state (p in [32 ch, 32 ch + 32))
// as fp16 into the H^T tile (MN-major operand: row n, p contiguous).
__device__ __forceinline__ void write_state_half(uint32_t sH, uint32_t n, int ch, const float (&Hs)[32]) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        uint4 u;
        u.x = f2_to_h2(Hs[8 * k + 0], Hs[8 * k + 1]);
        u.y = f2_to_h2(Hs[8 * k + 2], Hs[8 * k + 3]);
        u.z = f2_to_h2(Hs[8 * k + 4], Hs[8 * k + 5]);
        u.w = f2_to_h2(Hs[8 * k + 6], Hs[8 * k + 7]);
        sts128(sH + sw128(n, 4 * ch + k), u);
    }
}

// Diagonal block jc of row i when the block's own decay is beyond the
// factorised path's bound: one exp per element.  It only runs for extreme
// decays, so it is kept out of line, out of the instruction stream of the
// chunk loop.
__device__ __noinline__ void mask_block_exact(uint32_t g_taddr, uint32_t m_taddr, int jc, int lane,
                                              float cs, float dtv, float Dh)
{
    uint32_t pk[16];
#pragma unroll
    for (int qq = 0; qq < 2; ++qq) {   // 16 columns at a time
        uint32_t r[16];
        tc::tmem_ld16(g_taddr + jc * 32 + qq * 16, r);
        tc::tmem_ld_wait();
        float m[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int jl = qq * 16 + e;   // column within the block = lane of its row
            const float csj = __shfl_sync(0xffffffffu, cs, jl);
            const float dtj = __shfl_sync(0xffffffffu, dtv, jl);
            const float mv = (jl <= lane) ? __uint_as_float(r[e]) * expf(cs - csj) * dtj : 0.f;
            m[e] = (jl == lane) ? mv + Dh : mv;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) pk[qq * 8 + e] = f2_to_h2(m[2 * e], m[2 * e + 1]);
    }
    tc::tmem_st16(m_taddr + jc * 16, pk);
}

// One 32-column block jc of row i of the decay mask M, as fp16 pairs into
// TMEM (lane i, columns m_taddr + 16 jc ..  + 16: the A operand of the y MMA):
//   off-diagonal (jc < wq):  G[i][j] * exp(cs_i - cs_{r_jc}) * vd[j]
//   diagonal (jc == wq):     j <= i only, plus D on j == i
//   above (jc > wq):         zeros
// with vd[j] = exp(cs_{r_J} - cs_j) dt_j (J = j's block) from shared memory.
__device__ __forceinline__ float lds_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ float4 lds_f32x4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
    return v;
}
__device__ __forceinline__ void sts_f32(uint32_t addr, float v) {
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ void mask_block(uint32_t g_taddr, uint32_t m_taddr, uint32_t sVD,
                                           int jc, int wq, int lane, float ua,
                                           bool block_safe, float cs, float dtv, float Dh)
{
    uint32_t pk[16];
    if (jc > wq) {
#pragma unroll
        for (int q = 0; q < 16; ++q) pk[q] = 0u;
        tc::tmem_st16(m_taddr + jc * 16, pk);
        return;
    }
    if (jc == wq && !block_safe) {
        mask_block_exact(g_taddr, m_taddr, jc, lane, cs, dtv, Dh);
        return;
    }
    const uint32_t vd4 = sVD + jc * 128;
#pragma unroll
    for (int qq = 0; qq < 2; ++qq) {   // 16 columns at a time
        uint32_t r[16];
        tc::tmem_ld16(g_taddr + jc * 32 + qq * 16, r);
        tc::tmem_ld_wait();
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
            const int q = qq * 2 + q2;   // 8-column chunk within the block
            const float4 v0 = lds_f32x4(vd4 + 32 * q), v1 = lds_f32x4(vd4 + 32 * q + 16);
            const float vd[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            float m[8];
            if (jc < wq) {
                // (G ua) vd on fp32x2 lanes
                const float2 ua2 = make_float2(ua, ua);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 g2 = make_float2(__uint_as_float(r[q2 * 8 + 2 * e]),
                                                  __uint_as_float(r[q2 * 8 + 2 * e + 1]));
                    const float2 m2 = __fmul2_rn(__fmul2_rn(g2, ua2), make_float2(vd[2 * e], vd[2 * e + 1]));
                    m[2 * e] = m2.x;
                    m[2 * e + 1] = m2.y;
                }
            } else {   // diagonal block, factorised
                const float2 ua2 = make_float2(ua, ua);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 g2 = make_float2(__uint_as_float(r[q2 * 8 + 2 * e]),
                                                  __uint_as_float(r[q2 * 8 + 2 * e + 1]));
                    const float2 m2 = __fmul2_rn(__fmul2_rn(g2, ua2), make_float2(vd[2 * e], vd[2 * e + 1]));
                    const int j0 = q * 8 + 2 * e;
                    const float a0 = (j0 <= lane) ? m2.x : 0.f, a1 = (j0 + 1 <= lane) ? m2.y : 0.f;
                    m[2 * e] = (j0 == lane) ? a0 + Dh : a0;
                    m[2 * e + 1] = (j0 + 1 == lane) ? a1 + Dh : a1;
                }
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) pk[q * 4 + e] = f2_to_h2(m[2 * e], m[2 * e + 1]);
        }
    }
    tc::tmem_st16(m_taddr + jc * 16, pk);
}

// 16 bf16 outputs of row i (two 16-byte chunks starting at chunk c) into the
// y staging tile [128][64] (128B-swizzled, the box the y tensor map stores).
__device__ __forceinline__ void stage16_bf16(uint32_t stage, int i, int c, const float (&v)[16]) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        __nv_bfloat162 b0 = __floats2bfloat162_rn(v[8 * q + 0], v[8 * q + 1]);
        __nv_bfloat162 b1 = __floats2bfloat162_rn(v[8 * q + 2], v[8 * q + 3]);
        __nv_bfloat162 b2 = __floats2bfloat162_rn(v[8 * q + 4], v[8 * q + 5]);
        __nv_bfloat162 b3 = __floats2bfloat162_rn(v[8 * q + 6], v[8 * q + 7]);
        sts128(stage + sw128(i, c + q),
               make_uint4(*reinterpret_cast<uint32_t *>(&b0), *reinterpret_cast<uint32_t *>(&b1),
                          *reinterpret_cast<uint32_t *>(&b2), *reinterpret_cast<uint32_t *>(&b3)));
    }
}

// Per-chunk decay quantities of one head for this thread's row i.
struct ChunkDecay {
    float cs;        // inclusive cumulative dt*A at row i
    float dtv;       // dt of row i (0 past the chunk end)
    float uaA, uaB;  // exp(cs_i - cs_{r_K}) for this thread's two column blocks
    float w;         // exp(cs_last - cs_i) dt_i   (weights of the chunk state)
    float e;         // exp(cs_i)                  (decay of the carried state to row i)
    float a_last;    // exp(cs_last)               (decay over the whole chunk)
    bool safe;       // the row block's own decay fits the factorised path
};

// Raw dt of row i of the chunk starting at c0 (0 past the sequence end t1),
// loaded ahead of use: the compute loop keeps two chunks of it in flight.
__device__ __forceinline__ float load_dt(const ScanArgs &a, int H, int hh, long c0, long t1, int i) {
    return (c0 + i < t1) ? __ldg(a.dt + (size_t)(c0 + i) * H + hh) : 0.f;
}

// Cumulative decay of head hh over a chunk of Lc tokens whose raw dt for row
// i is dt_raw (warpgroup-wide).  Returns row i's (cs_i, dt_i, w_i) with the
// chunk-state weight w_i = exp(cs_last - cs_i) dt_i.  The warpgroup with
// ch == 0 also publishes the chunk's tables for decay_derive and the mask:
//   vd[j]  = exp(cs_{r_J} - cs_j) dt_j, J = j's 32-row block (column factors)
//   csb[J] = cs_{r_J} (J < 4), csb[4] = cs_last
__device__ __forceinline__ float3 decay_scan(const ScanArgs &a, int hh, float Ah, float dt_raw,
                                             int Lc, int i, int wq, int lane, int wg, int ch,
                                             uint32_t sPART, uint32_t sCSB, uint32_t vd_out,
                                             uint32_t csb_out)
{
    const float dtv = (i < Lc) ? dt_apply(a.dtp, dt_raw, hh) : 0.f;
    float v = dtv * Ah;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    if (lane == 31) sts_f32(sPART + 4 * wq, v);
    wg_sync(wg);
    float pre = 0.f;
    for (int w = 0; w < wq; ++w) pre += lds_f32(sPART + 4 * w);
    const float cs = v + pre;
    if (lane == 31) sts_f32(sCSB + 4 * wq, cs);
    if (i == Lc - 1) sts_f32(sCSB + 16, cs);
    wg_sync(wg);
    const float cs_last = lds_f32(sCSB + 16);
    if (ch == 0) {
        sts_f32(vd_out + 4 * i, exp_dec(lds_f32(sCSB + 4 * wq) - cs) * dtv);   // <= dt
        if (i < 5) sts_f32(csb_out + 4 * i, lds_f32(sCSB + 4 * i));
    }
    return make_float3(cs, dtv, (i < Lc) ? exp_dec(cs_last - cs) * dtv : 0.f);
}

// The per-row decay quantities of ChunkDecay from row i's (cs, dt, w) and
// the chunk's published block ends csb.
__device__ __forceinline__ ChunkDecay decay_derive(float3 csdtw, uint32_t csb, int wq, int ch) {
    ChunkDecay d;
    d.cs = csdtw.x;
    d.dtv = csdtw.y;
    d.w = csdtw.z;
    const int kA = ch == 0 ? 0 : 1, kB = ch == 0 ? 3 : 2;
    d.uaA = (kA <= wq) ? exp_dec(d.cs - lds_f32(csb + 4 * kA)) : 0.f;
    d.uaB = (kB <= wq) ? exp_dec(d.cs - lds_f32(csb + 4 * kB)) : 0.f;
    d.safe = (__shfl_sync(0xffffffffu, d.cs, 0) - lds_f32(csb + 4 * wq)) <= kSafeBlockDecay;
    d.e = exp_dec(d.cs);
    d.a_last = exp_dec(lds_f32(csb + 16));
    return d;
}

// Named barriers: 1..4 per-warpgroup; the compute warps signal the issuing
// warp with bar.arrive on 5 (operands ready), 6 (decay mask ready) and 7 (y
// staged); 8 is compute-warps-only.
constexpr uint32_t BAR_OPERANDS = 5, BAR_MASK = 6, BAR_YSTAGED = 7, BAR_COMPUTE = 8;
constexpr uint32_t kCompute = 512;

// The chunks one CTA sweeps.  Chains are (sequence, pair of heads): chain c
// = sequence c / pairs, heads 2 (c % pairs) and 2 (c % pairs) + 1.
//   * one CTA per chain (runs == 0): chain blockIdx.x, all of its chunks;
//   * balanced (runs > 0, fixed-length sequences of nch chunks): the chains
//     laid end to end are cut into `runs` runs of equal chunk counts, and run
//     r covers global chunks [lo, hi).  It sweeps the head of its last chain
//     cl (chunks [0, kl), ending at a cut: its carried state is handed on
//     through slot r), then its whole chains, then the tail of its first
//     chain cf (chunks [kf, nch), starting at a cut: its state comes from slot
//     r - 1).  A tail is swept last and a head first, so a hand-off has long
//     been written when it is read; a run inside one chain (cf == cl) reads
//     at its start a state that the previous run wrote first, after a head of
//     fewer chunks than one run.
struct Sweep {
    int nch;          // chunks per chain (balanced) or of this CTA's chain
    int cf, kf;       // first chain and its first chunk
    int cl, kl;       // last chain and the end (exclusive) of its chunks
    int total;        // chunks swept
};

// Piece p of a sweep: chain and its chunk range [k0, k1).  Pieces are the
// head of the last chain, the whole chains between, and the tail of the
// first chain (one piece when the run lies in one chain).
__device__ __forceinline__ void sweep_piece(const Sweep &w, int p, int &chain, int &k0, int &k1) {
    if (w.cf == w.cl) { chain = w.cf; k0 = w.kf; k1 = w.kl; }
    else if (p == 0) { chain = w.cl; k0 = 0; k1 = w.kl; }
    else if (p < w.cl - w.cf) { chain = w.cf + p; k0 = 0; k1 = w.nch; }
    else { chain = w.cf; k0 = w.kf; k1 = w.nch; }
}

// Position of a sweep: piece p, chunk k of its chain, and the chunk's token
// rows.  step() moves to the next chunk; it divides (chain -> sequence) only
// when it enters a new piece.
struct Item {
    int p, k, k1;   // piece, chunk, end (exclusive) of the piece's chunks
    int s, pair;    // sequence and head pair of the chunk's chain
    int t1, c0;     // end of the sequence's tokens; first token of the chunk
};
// Where a chain's tokens lie: [t0, t1) of the packed token axis.
__device__ __forceinline__ void chain_span(const ScanArgs &a, int s, long &t0, long &t1) {
    if (a.cu_seqlens) {
        t0 = a.cu_seqlens[s];
        t1 = a.cu_seqlens[s + 1];
    } else {
        t0 = (long)s * a.seqlen;
        t1 = t0 + a.seqlen;
    }
}

// The first chunk of piece p.
__device__ __forceinline__ Item piece_item(const ScanArgs &a, const Sweep &w, int p, int pairs) {
    Item it;
    int chain, k0;
    it.p = p;
    sweep_piece(w, p, chain, k0, it.k1);
    it.k = k0;
    it.s = chain / pairs;
    it.pair = chain - it.s * pairs;
    long t0, t1;
    chain_span(a, it.s, t0, t1);
    it.t1 = (int)t1;
    it.c0 = (int)(t0 + (long)k0 * kQ);
    return it;
}

// The next chunk of the sweep.
__device__ __forceinline__ void step(const ScanArgs &a, const Sweep &w, Item &it, int pairs) {
    if (it.k + 1 < it.k1) {
        ++it.k;
        it.c0 += kQ;
    } else {
        it = piece_item(a, w, it.p + 1, pairs);
    }
}

// Bounded acquire-spin on a hand-off flag written by another CTA.
__device__ __forceinline__ bool wait_flag(const int *flag, unsigned long long wait_ns) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    if (v) return true;
    const uint64_t t0 = tc::globaltimer_ns(), lim = wait_limit(wait_ns);
    for (;;) {
        __nanosleep(256);
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
        if (v) return true;
        if (tc::globaltimer_ns() - t0 > lim) return false;
    }
}

// kPieces = false: one CTA per (sequence, head pair) chain, sweeping its
// chunks in order.  kPieces = true (fixed-length batches, no slot pools): CTA
// r sweeps run r of the chains laid end to end, cut into one run per CTA, and
// hands the carried state across each cut through the caller's workspace.
// Both instantiations share the per-chunk phases below; only the walk over
// chunks differs.
template <typename TOut, bool kPieces>
__global__ void __launch_bounds__(kThreads, 1)
scan_tc_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_b,
               const __grid_constant__ CUtensorMap map_c, const __grid_constant__ CUtensorMap map_y,
               const ScanArgs a)
{
    // bf16 y of full chunks is staged in shared memory (the M tile of head 1,
    // free between the y MMAs and the next chunk's mask) and written by TMA;
    // fp32 y and partial chunks are stored row by row.
    constexpr bool kStoreByTma = sizeof(TOut) == 2;
    const uint32_t sbase = tc::smem_u32(smem);
    const int tid = threadIdx.x;
    const bool issuer = tid >= (int)kCompute;  // warp 16: TMA and MMA issue
    const int wg = (tid >> 7) & 3;       // compute warpgroup 0..3
    const int hd = wg & 1;               // head slot of the pair
    const int ch = wg >> 1;              // column half
    const int i = tid & 127;             // row / TMEM lane / d_state index
    const int wq = i >> 5;               // warp within the warpgroup = 32-row block
    const int lane = tid & 31;

    const int H = a.nheads, G = a.ngroups;
    const int hpg = H / G;
    const int pairs = H >> 1;

    if (sbase & 1023u || (kPieces && (a.cu_seqlens || a.slot_idx || a.runs <= 0))) {
        // the swizzled layouts need 1024-B alignment; runs cover fixed-length
        // batches without slot pools only
        if (tid == 0) report_status(a.status_dev, kStatusInternal);
        return;
    }

    // ---- what this CTA sweeps ----
    Sweep sw{};                 // kPieces: run r of the chains laid end to end
    int s = 0, h0 = 0;          // otherwise: sequence s, heads h0, h0 + 1 ...
    long t0 = 0, t1 = 0;        // ... over tokens [t0, t1)
    size_t srow = 0;            // ... with state row srow
    bool load_init = a.initial_state != nullptr;
    if constexpr (kPieces) {
        const int r = blockIdx.x;
        sw.nch = (a.seqlen + kQ - 1) / kQ;
        const long ctot = (long)a.nseq * pairs * sw.nch;
        const long lo = ctot * r / a.runs, hi = ctot * (r + 1) / a.runs;
        sw.cf = (int)(lo / sw.nch);
        sw.kf = (int)(lo - (long)sw.cf * sw.nch);
        sw.cl = (int)((hi - 1) / sw.nch);
        sw.kl = (int)(hi - (long)sw.cl * sw.nch);
        sw.total = (int)(hi - lo);
        if (sw.total <= 0) {   // the host cuts at most one run per chunk
            if (tid == 0) report_status(a.status_dev, kStatusInternal);
            return;
        }
    } else {
        s = blockIdx.x / pairs;
        h0 = (blockIdx.x - s * pairs) * 2;
        if (a.cu_seqlens && a.nseq <= kLongestFirstSeqs) {
            // Packed sequences of mixed lengths: the CTAs take the sequences
            // longest first (ties by index), so the long chains start in the
            // first wave and the short ones fill in behind them.  Rank r of
            // the order goes to CTAs [r pairs, (r + 1) pairs).
            if (tid < a.nseq) {
                const int len = __ldg(a.cu_seqlens + tid + 1) - __ldg(a.cu_seqlens + tid);
                int rank = 0;
                for (int q = 0; q < a.nseq; ++q) {
                    const int lq = __ldg(a.cu_seqlens + q + 1) - __ldg(a.cu_seqlens + q);
                    rank += (lq > len) || (lq == len && q < tid);
                }
                if (rank == s) flag_set(OFF_SEQ, tid);
            }
            __syncthreads();
            s = flag_get(OFF_SEQ);
        }
        if (a.cu_seqlens) {
            const int c0 = a.cu_seqlens[0], cs0 = a.cu_seqlens[s], cs1 = a.cu_seqlens[s + 1];
            const int cend = a.cu_seqlens[a.nseq];
            if (c0 != 0 || cs1 < cs0 || cs0 < 0 || cend != a.seqlen || cs1 > a.seqlen) {
                if (tid == 0) report_status(a.status_dev, kStatusDeviceInput);
                return;
            }
        }
        chain_span(a, s, t0, t1);
        srow = (size_t)s;
        if (a.slot_idx) {
            const int slot = a.slot_idx[s];
            if (slot < 0 || slot >= a.max_slots) {
                if (tid == 0) report_status(a.status_dev, kStatusDeviceInput);
                return;
            }
            srow = (size_t)slot;
            if (a.has_initial && a.has_initial[s] == 0) load_init = false;
        }
    }

    const uint32_t sCSB = sbase + OFF_CSB + wg * 32;
    const uint32_t sPART = sbase + OFF_PART + wg * 16;
    const uint32_t bar_x = sbase + OFF_BAR, bar_cb = bar_x + 8, bar_sg = bar_x + 16;
    const uint32_t bar_yo = bar_x + 24, bar_y = bar_x + 32, bar_drain = bar_x + 40;

    if (tid < 32) {
        tc::tmem_alloc(sbase + OFF_TM, TM_COLS);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        tc::mbar_init(bar_x, 1);
        tc::mbar_init(bar_cb, 1);
        tc::mbar_init(bar_sg, 1);
        tc::mbar_init(bar_yo, 1);
        tc::mbar_init(bar_y, 1);
        tc::mbar_init(bar_drain, 1);
        flag_set(OFF_ABORT, 0);
        flag_set(OFF_RANGE, 0);
        tc::fence_mbar_init();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + OFF_TM);
    bool ok = true;

    if (issuer) {
        // ================= TMA / MMA issuing warp =================
        const bool leader = lane == 0;
        // descriptors (start-address field advanced by offset >> 4 per K step)
        const uint64_t dBmn = tc::sdesc_sw128(sbase + OFF_B, HALF, 1024);   // B^T, MN-major
        const uint64_t dW = tc::sdesc_sw128(sbase + OFF_WM, HALF, 1024);    // [wX_a | wX_b]
        const uint64_t dBk = tc::sdesc_sw128(sbase + OFF_B, 16, 1024);      // B, K-major
        const uint64_t dH = tc::sdesc_sw128(sbase + OFF_H, HALF, 1024);     // [H_a^T | H_b^T]
        const uint64_t dXa = tc::sdesc_sw128(sbase + OFF_XH, HALF, 1024);
        const uint64_t dXb = dXa + (HALF >> 4);
        // Work in flight, for the drain after an abort: phases armed on the
        // two load barriers, and whether any MMA was issued.
        uint32_t nx_armed = 0, ncb_armed = 0;
        bool mma_issued = false;
        const bool produce = a.stall_producer == 0;
        // x and y are touched once (evict-first in L2); B and C are read by
        // every head pair of their group, and keep the default policy.
        const uint64_t once = tc::l2_evict_first_policy();
        // x of heads hp, hp + 1 and C, B of group gg for the chunk at token row
        auto load_x = [&](int hp, int row) {
            tc::mbar_arrive_expect_tx(bar_x, 2 * HALF);
            tc::tma_load_3d_hint(sbase + OFF_XR, &map_x, bar_x, 0, hp, row, once);
            tc::tma_load_3d_hint(sbase + OFF_XR + HALF, &map_x, bar_x, 0, hp + 1, row, once);
            ++nx_armed;
        };
        auto load_cb = [&](int gg, int row) {
            tc::mbar_arrive_expect_tx(bar_cb, 4 * HALF);
            tc::tma_load_3d(sbase + OFF_C, &map_c, bar_cb, 0, gg, row);
            tc::tma_load_3d(sbase + OFF_C + HALF, &map_c, bar_cb, 64, gg, row);
            tc::tma_load_3d(sbase + OFF_B, &map_b, bar_cb, 0, gg, row);
            tc::tma_load_3d(sbase + OFF_B + HALF, &map_b, bar_cb, 64, gg, row);
            ++ncb_armed;
        };
        // One chunk: S^T and G, then Yoff, once the operands are ready (the
        // next chunk's x and C, B loads go out as their buffers free); Y once
        // the decay mask is in TMEM; the y tiles once staged.
        auto issue_chunk = [&](uint32_t phase, bool has_next, int hp_n, int row_n, int hp, int row,
                               bool full) {
            tc::named_sync(BAR_OPERANDS, kCompute + 32);
            if (flag_get(OFF_ABORT)) ok = false;   // a compute warp's wait expired: issue nothing more
            if (leader && ok && produce) {
                tc::bulk_wait_read();   // previous y staging (in the M tiles) was read
                if (has_next) load_x(hp_n, row_n);
                tc::tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_f16_ss(tmem + TM_S, dBmn + kk * 128, dW + kk * 128, IDESC_S2, kk > 0);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t ko = (kk >> 2) * (HALF >> 4) + (kk & 3) * 2;
                    tc::mma_f16_ts(tmem + TM_G, tmem + TM_C + kk * 8, dBk + ko, IDESC_G, kk > 0);
                }
                tc::mma_commit(bar_sg);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_f16_ts(tmem + TM_YO, tmem + TM_C + kk * 8, dH + kk * 128, IDESC_YO2, kk > 0);
                tc::mma_commit(bar_yo);
                mma_issued = true;
                // The compute warps read C from shared memory before the operand
                // barrier; B is read by the S and G MMAs only: both tiles are free
                // once those complete.
                wait_or_abort(bar_sg, phase, ok, a.wait_ns);
                if (has_next && ok) load_cb(hp_n / hpg, row_n);
            }
            __syncwarp();
            tc::named_sync(BAR_MASK, kCompute + 32);
            if (flag_get(OFF_ABORT)) ok = false;
            if (leader && ok && produce) {
                tc::tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_f16_ts(tmem + TM_Y, tmem + TM_S + kk * 8, dXa + kk * 128, IDESC_Y, kk > 0);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_f16_ts(tmem + TM_Y + 64, tmem + TM_S + 64 + kk * 8, dXb + kk * 128, IDESC_Y, kk > 0);
                tc::mma_commit(bar_y);
            }
            __syncwarp();
            tc::named_sync(BAR_YSTAGED, kCompute + 32);
            if (flag_get(OFF_ABORT)) ok = false;
            if (kStoreByTma && leader && ok && produce && full) {
                // full chunk: both heads' y tiles by TMA
                tc::tma_store_3d_hint(&map_y, sbase + OFF_MB, 0, hp, row, once);
                tc::tma_store_3d_hint(&map_y, sbase + OFF_MB + HALF, 0, hp + 1, row, once);
                tc::bulk_commit();
            }
            __syncwarp();
        };
        if constexpr (kPieces) {
            Item itq = piece_item(a, sw, 0, pairs);   // the chunk being computed
            if (leader && sw.total > 0 && produce) {
                load_x(2 * itq.pair, itq.c0);
                load_cb(2 * itq.pair / hpg, itq.c0);
            }
            uint32_t phase = 0;
            for (int q = 0; q < sw.total; ++q, phase ^= 1u) {
                const bool has_next = q + 1 < sw.total;
                Item itn = itq;
                if (has_next) step(a, sw, itn, pairs);
                issue_chunk(phase, has_next, 2 * itn.pair, itn.c0, 2 * itq.pair, itq.c0,
                            itq.c0 + kQ <= itq.t1);
                itq = itn;
            }
        } else {
            if (leader && t1 > t0 && produce) {
                load_x(h0, (int)t0);
                load_cb(h0 / hpg, (int)t0);
            }
            uint32_t phase = 0;
            for (long c0 = t0; c0 < t1; c0 += kQ, phase ^= 1u) {
                const long c1 = c0 + kQ;
                issue_chunk(phase, c1 < t1, h0, (int)c1, h0, (int)c0, c1 <= t1);
            }
        }
        if (leader) {
            if (!ok) {
                // Aborted: wait (bounded) for every MMA issued and for the last
                // phase armed on each load barrier, so that nothing writes TMEM
                // or shared memory after they are released.
                bool dok = true;
                if (mma_issued) {
                    tc::mma_commit(bar_drain);
                    tc::mbar_wait_bounded(bar_drain, 0, dok, wait_limit(a.wait_ns));
                }
                bool xok = true, cbok = true;
                if (nx_armed) tc::mbar_wait_bounded(bar_x, (nx_armed - 1) & 1u, xok, wait_limit(a.wait_ns));
                if (ncb_armed) tc::mbar_wait_bounded(bar_cb, (ncb_armed - 1) & 1u, cbok, wait_limit(a.wait_ns));
            }
            tc::bulk_wait_all();
        }
        __syncwarp();
    } else {
        // ================= compute warpgroups =================
        const uint32_t tlane = (uint32_t)(wq * 32) << 16;
        const uint32_t vd_tab = sbase + OFF_VD;     // float [2 buffers][2 heads][128]
        const uint32_t csb_tab = sbase + OFF_CSBT;  // float [2 buffers][2 heads][8]
        TOut *y = static_cast<TOut *>(a.y);
        float Hs[32];   // carried state: d_state row i, head_dim entries 32 ch ..

        // ---- operands to fp16 (rows past the chunk end zeroed) ----
        // (w o x already written when wm_ready: see convert_wm)
        auto convert = [&](uint32_t phase, bool live, float w, bool wm_ready) {
            wait_or_abort(bar_x, phase, ok, a.wait_ns);
            wait_or_abort(bar_cb, phase, ok, a.wait_ns);
            // warpgroup wg takes d_state columns n in [32 wg, 32 wg + 32) of row i:
            // C as fp16 pairs into TMEM (lane i, columns 16 wg ..), B in place
            const uint32_t ctile = sbase + OFF_C + (wg >> 1) * HALF;
            const uint32_t btile = sbase + OFF_B + (wg >> 1) * HALF;
            uint32_t pc[16];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 v = live ? cvt_chunk(lds128(ctile + sw128(i, 4 * (wg & 1) + q)))
                                     : make_uint4(0, 0, 0, 0);
                pc[4 * q] = v.x;
                pc[4 * q + 1] = v.y;
                pc[4 * q + 2] = v.z;
                pc[4 * q + 3] = v.w;
            }
            tc::tmem_st16(tmem + tlane + TM_C + 16 * wg, pc);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t addr = btile + sw128(i, 4 * (wg & 1) + q);
                sts128(addr, live ? cvt_chunk(lds128(addr)) : make_uint4(0, 0, 0, 0));
            }
#pragma unroll
            for (int k = 4 * ch; k < 4 * ch + 4; ++k) {
                const uint32_t off = hd * HALF + sw128(i, k);
                if (live) {
                    const uint4 r = lds128(sbase + OFF_XR + off);
                    sts128(sbase + OFF_XH + off, cvt_chunk(r));
                    if (!wm_ready) sts128(sbase + OFF_WM + off, cvt_chunk_scaled(r, w));
                } else {
                    sts128(sbase + OFF_XH + off, make_uint4(0, 0, 0, 0));
                    if (!wm_ready) sts128(sbase + OFF_WM + off, make_uint4(0, 0, 0, 0));
                }
            }
            tc::tmem_st_wait();
            tc::fence_proxy_async_smem();
            tc::tc_fence_before();
            tc::named_arrive(BAR_OPERANDS, kCompute + 32);
        };
        // ---- w o x of the next chunk while this chunk's Y MMAs run: its raw x
        // has landed by then (requested at this chunk's operand barrier), and
        // the S MMA that read this chunk's w o x has completed ----
        auto convert_wm = [&](uint32_t phase_n, bool live_n, float w_n) {
            wait_or_abort(bar_x, phase_n, ok, a.wait_ns);
#pragma unroll
            for (int k = 4 * ch; k < 4 * ch + 4; ++k) {
                const uint32_t off = hd * HALF + sw128(i, k);
                sts128(sbase + OFF_WM + off, live_n ? cvt_chunk_scaled(lds128(sbase + OFF_XR + off), w_n)
                                                    : make_uint4(0, 0, 0, 0));
            }
        };
        // ---- carried state: H <- exp(cs_L) H + S (d_state row i, p half ch) ----
        auto update_state = [&](uint32_t phase, float a_last) {
            wait_or_abort(bar_sg, phase, ok, a.wait_ns);
            tc::tc_fence_after();
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                uint32_t r[16];
                tc::tmem_ld16(tmem + tlane + TM_S + hd * 64 + ch * 32 + q * 16, r);
                tc::tmem_ld_wait();
                const float2 al2 = make_float2(a_last, a_last);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float2 h2 = __ffma2_rn(al2, make_float2(Hs[q * 16 + 2 * e], Hs[q * 16 + 2 * e + 1]),
                                                 make_float2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1])));
                    Hs[q * 16 + 2 * e] = h2.x;
                    Hs[q * 16 + 2 * e + 1] = h2.y;
                }
            }
            tc::tc_fence_before();
            tc::named_sync(BAR_COMPUTE, kCompute);   // every S column read: M may overwrite them
            tc::tc_fence_after();
            if (flag_get(OFF_ABORT)) ok = false;
        };
        // ---- decay mask M of head hd into TMEM (over S of this head) ----
        auto build_mask = [&](const ChunkDecay &cur, uint32_t vb, float Dh) {
            const uint32_t vd = vd_tab + vb * 1024 + hd * 512;
            const int kA = ch == 0 ? 0 : 1, kB = ch == 0 ? 3 : 2;
            const uint32_t m_taddr = tmem + tlane + TM_S + hd * 64;
            mask_block(tmem + tlane + TM_G, m_taddr, vd, kA, wq, lane, cur.uaA, cur.safe, cur.cs, cur.dtv, Dh);
            mask_block(tmem + tlane + TM_G, m_taddr, vd, kB, wq, lane, cur.uaB, cur.safe, cur.cs, cur.dtv, Dh);
            tc::tmem_st_wait();
            tc::tc_fence_before();
            tc::named_arrive(BAR_MASK, kCompute + 32);
        };
        // ---- y = Y + exp(cs_i) Yoff (row i, p half ch; D x is inside Y) ----
        // An fp16 operand out of range (a bf16 input, a decay-masked C.B^T
        // entry or a carried-state entry beyond 65504) turns some output into
        // inf or NaN; each group of 16 outputs is summed and the range flag
        // raised when a sum is not finite.
        auto epilogue = [&](uint32_t phase, float e, bool full, bool live, TOut *yrow) {
            wait_or_abort(bar_y, phase, ok, a.wait_ns);
            tc::tc_fence_after();
#pragma unroll
            for (int q = 0; q < 2; ++q) {   // 16 columns at a time
                uint32_t ry[16], ro[16];
                tc::tmem_ld16(tmem + tlane + TM_Y + hd * 64 + ch * 32 + q * 16, ry);
                tc::tmem_ld16(tmem + tlane + TM_YO + hd * 64 + ch * 32 + q * 16, ro);
                tc::tmem_ld_wait();
                float out[16];
                const float2 e2 = make_float2(e, e);
                float2 ysum = make_float2(0.f, 0.f);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const float2 o2 = __ffma2_rn(e2, make_float2(__uint_as_float(ro[2 * c]), __uint_as_float(ro[2 * c + 1])),
                                                 make_float2(__uint_as_float(ry[2 * c]), __uint_as_float(ry[2 * c + 1])));
                    out[2 * c] = o2.x;
                    out[2 * c + 1] = o2.y;
                    ysum = __fadd2_rn(ysum, o2);
                }
                if (!isfinite(ysum.x + ysum.y)) flag_set(OFF_RANGE, 1);
                if (kStoreByTma && full) {
                    stage16_bf16(sbase + OFF_MB + hd * HALF, i, 4 * ch + 2 * q, out);
                } else if (live) {
                    store16(yrow + 32 * ch + 16 * q, out);
                }
            }
            tc::fence_proxy_async_smem();
            tc::tc_fence_before();
            tc::named_arrive(BAR_YSTAGED, kCompute + 32);
        };

        if constexpr (!kPieces) {
            const int hh = h0 + hd;
            const size_t state_off = (srow * H + hh) * (size_t)(kP * kN) + (size_t)(32 * ch) * kN + i;
#pragma unroll
            for (int p = 0; p < 32; ++p)
                Hs[p] = load_init ? state_load1(a.initial_state, state_off + (size_t)p * kN, a.rp) : 0.f;
            write_state_half(sbase + OFF_H + hd * HALF, i, ch, Hs);

            const float Ah = a.A[hh];
            const float Dh = a.D ? a.D[hh] : 0.f;
            float3 dcur = make_float3(0.f, 0.f, 0.f);   // (cs_i, dt_i, w_i) of the current chunk
            if (t1 > t0)
                dcur = decay_scan(a, hh, Ah, load_dt(a, H, hh, t0, t1, i), (int)min((long)kQ, t1 - t0),
                                  i, wq, lane, wg, ch, sPART, sCSB, vd_tab + hd * 512, csb_tab + hd * 32);
            float dt_n1 = load_dt(a, H, hh, t0 + kQ, t1, i);   // raw dt of the next chunk
            tc::named_sync(BAR_COMPUTE, kCompute);
            uint32_t phase = 0, vb = 0;
            for (long c0 = t0; c0 < t1; c0 += kQ, phase ^= 1u, vb ^= 1u) {
                const int Lc = (int)min((long)kQ, t1 - c0);
                const long c1 = c0 + kQ;
                const bool has_next = c1 < t1;
                const bool live = i < Lc;
                const ChunkDecay cur = decay_derive(dcur, csb_tab + vb * 64 + hd * 32, wq, ch);

                // dt two chunks ahead, so its load has a whole chunk to land
                const float dt_n2 = load_dt(a, H, hh, c0 + 2 * kQ, t1, i);

                convert(phase, live, cur.w, c0 != t0);

                // ---- next chunk's decay while the MMAs run ----
                float3 dnxt = make_float3(0.f, 0.f, 0.f);
                if (has_next)
                    dnxt = decay_scan(a, hh, Ah, dt_n1, (int)min((long)kQ, t1 - c1), i, wq, lane, wg, ch,
                                      sPART, sCSB, vd_tab + (vb ^ 1u) * 1024 + hd * 512,
                                      csb_tab + (vb ^ 1u) * 64 + hd * 32);

                update_state(phase, cur.a_last);
                build_mask(cur, vb, Dh);

                // ---- new H^T tile for the next chunk (Yoff of this chunk read the old one) ----
                wait_or_abort(bar_yo, phase, ok, a.wait_ns);
                write_state_half(sbase + OFF_H + hd * HALF, i, ch, Hs);
                if (has_next) convert_wm(phase ^ 1u, c1 + i < t1, dnxt.z);

                epilogue(phase, cur.e, Lc == kQ, live, y + ((size_t)(c0 + i) * H + hh) * kP);
                dcur = dnxt;
                dt_n1 = dt_n2;
            }
            if (a.final_state) {
#pragma unroll
                for (int p = 0; p < 32; ++p) state_store1(a.final_state, state_off + (size_t)p * kN, Hs[p], a.rp);
            }
        } else {
            const int r = blockIdx.x;
            // This thread's 32 values of the state row of sequence sq, head hh.
            auto state_at = [&](int sq, int hh) {
                return ((size_t)sq * H + hh) * (size_t)(kP * kN) + (size_t)(32 * ch) * kN + i;
            };
            // Hand-off slot of cut rr: [2 heads][64 p][128 n] fp32; this thread's
            // 32 values sit at (hd * 64 + 32 ch + p) * 128 + i.
            auto slot_at = [&](int rr) {
                return a.handoff + (size_t)rr * (2 * kP * kN) + (size_t)(hd * kP + 32 * ch) * kN + i;
            };
            // Carried state at the start of a piece: the initial state (or zero)
            // at a chain start, else the state handed over through slot r - 1.
            auto load_piece_state = [&](const Item &it) {
                if (it.k == 0) {
                    const size_t off = state_at(it.s, 2 * it.pair + hd);
#pragma unroll
                    for (int p = 0; p < 32; ++p)
                        Hs[p] = load_init ? state_load1(a.initial_state, off + (size_t)p * kN, a.rp) : 0.f;
                } else {
                    if (tid == 0 && ok && !wait_flag(a.handoff_flags + (r - 1), a.wait_ns)) flag_set(OFF_ABORT, 1);
                    tc::named_sync(BAR_COMPUTE, kCompute);
                    const float *src = slot_at(r - 1);
#pragma unroll
                    for (int p = 0; p < 32; ++p) Hs[p] = __ldcg(src + (size_t)p * kN);
                }
            };
            // Carried state at the end of a piece: the final state at a chain end,
            // else handed on through slot r (written, fenced, then flagged).
            auto store_piece_state = [&](const Item &it) {
                if (it.c0 + kQ >= it.t1) {
                    if (a.final_state) {
                        const size_t off = state_at(it.s, 2 * it.pair + hd);
#pragma unroll
                        for (int p = 0; p < 32; ++p) state_store1(a.final_state, off + (size_t)p * kN, Hs[p], a.rp);
                    }
                } else {
                    float *dst = slot_at(r);
#pragma unroll
                    for (int p = 0; p < 32; ++p) __stcg(dst + (size_t)p * kN, Hs[p]);
                    __threadfence();
                    tc::named_sync(BAR_COMPUTE, kCompute);
                    if (tid == 0)
                        asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(a.handoff_flags + r), "r"(1) : "memory");
                }
            };

            Item it = piece_item(a, sw, 0, pairs);
            int hh = 2 * it.pair + hd;
            float Ah = a.A[hh];
            float Dh = a.D ? a.D[hh] : 0.f;
            load_piece_state(it);
            write_state_half(sbase + OFF_H + hd * HALF, i, ch, Hs);
            float3 dcur = decay_scan(a, hh, Ah, load_dt(a, H, hh, it.c0, it.t1, i), min(kQ, it.t1 - it.c0),
                                     i, wq, lane, wg, ch, sPART, sCSB, vd_tab + hd * 512, csb_tab + hd * 32);
            // The first chunk of the next piece (needed only at a piece's last
            // chunk) is kept in shared memory, not in registers across the chunk
            // loop: its first head, first token and sequence end.
            const int npieces = sw.cf == sw.cl ? 1 : sw.cl - sw.cf + 1;
            auto publish_next = [&](int p) {
                if (tid == 0) {
                    const Item n = piece_item(a, sw, p, pairs);
                    flag_set(OFF_NXP, 2 * n.pair);
                    flag_set(OFF_NXP + 4, n.c0);
                    flag_set(OFF_NXP + 8, n.t1);
                }
            };
            if (npieces > 1) publish_next(1);
            tc::named_sync(BAR_COMPUTE, kCompute);
            uint32_t phase = 0, vb = 0;
            int q = 0;
            // Outer loop over pieces (the carried state is stored, handed on and
            // loaded between them); the inner loop over a piece's chunks keeps the
            // next chunk's operands and decay in flight across piece boundaries.
            for (int pc_ = 0; pc_ < npieces; ++pc_) {
                for (; it.k < it.k1; ++it.k, it.c0 += kQ, ++q, phase ^= 1u, vb ^= 1u) {
                    const int c0 = it.c0;
                    const int Lc = min(kQ, it.t1 - c0);
                    const bool has_next = q + 1 < sw.total;
                    const bool live = i < Lc;
                    const ChunkDecay cur = decay_derive(dcur, csb_tab + vb * 64 + hd * 32, wq, ch);
                    // the next chunk: in this piece, or the first of the next piece
                    const bool same = it.k + 1 < it.k1;
                    int hh_n = hh, c0_n = c0 + kQ, t1_n = it.t1;
                    float Ah_n = Ah;
                    if (!same && has_next) {
                        hh_n = flag_get(OFF_NXP) + hd;
                        c0_n = flag_get(OFF_NXP + 4);
                        t1_n = flag_get(OFF_NXP + 8);
                        Ah_n = a.A[hh_n];
                    }
                    // its raw dt, a whole conversion ahead of its decay
                    const float dt_n1 = has_next ? load_dt(a, H, hh_n, c0_n, t1_n, i) : 0.f;

                    convert(phase, live, cur.w, q > 0);

                    // ---- next chunk's decay while the MMAs run ----
                    float3 dnxt = make_float3(0.f, 0.f, 0.f);
                    if (has_next)
                        dnxt = decay_scan(a, hh_n, Ah_n, dt_n1, min(kQ, t1_n - c0_n), i, wq, lane, wg, ch,
                                          sPART, sCSB, vd_tab + (vb ^ 1u) * 1024 + hd * 512,
                                          csb_tab + (vb ^ 1u) * 64 + hd * 32);

                    update_state(phase, cur.a_last);
                    build_mask(cur, vb, Dh);

                    // ---- new H^T tile for the next chunk (Yoff of this chunk read the old one) ----
                    wait_or_abort(bar_yo, phase, ok, a.wait_ns);
                    write_state_half(sbase + OFF_H + hd * HALF, i, ch, Hs);
                    if (has_next) convert_wm(phase ^ 1u, c0_n + i < t1_n, dnxt.z);

                    epilogue(phase, cur.e, Lc == kQ, live, y + ((size_t)(c0 + i) * H + hh) * kP);
                    dcur = dnxt;
                }
                // ---- piece boundary: store or hand on the state, start the next piece
                // (its H^T tile replaces the one the last chunk wrote before the next
                // chunk's operands are released to the MMAs) ----
                it.k = it.k1 - 1;
                it.c0 -= kQ;
                store_piece_state(it);
                if (pc_ + 1 < npieces) {
                    it = piece_item(a, sw, pc_ + 1, pairs);
                    hh = 2 * it.pair + hd;
                    Ah = a.A[hh];
                    Dh = a.D ? a.D[hh] : 0.f;
                    load_piece_state(it);
                    write_state_half(sbase + OFF_H + hd * HALF, i, ch, Hs);
                    if (pc_ + 2 < npieces) publish_next(pc_ + 2);
                    // (every thread has read the previous value: the last chunk's
                    // state-update barrier lies between; this one publishes the new)
                    tc::named_sync(BAR_COMPUTE, kCompute);
                }
            }
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (tid < 32) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, TM_COLS);
    }
    if (flag_get(OFF_ABORT)) {
        if (tid == 0) report_status(a.status_dev, kStatusTimeout);
    } else if (tid == 0 && flag_get(OFF_RANGE)) {
        report_status(a.status_dev, kStatusRange);
    }
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

// 3-D map over [d2][d1][d0] (d0 contiguous) of 16-bit elements with a
// {64, 1, 128} box (one 128-token tile of one head or group, 64 elements
// wide) and 128-byte swizzle.
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
    CUtensorMap mx, mb, mc, my;
    if (!make_map(&mx, a.x, kP, a.nheads, T) || !make_map(&mb, a.B, kN, a.ngroups, T) ||
        !make_map(&mc, a.C, kN, a.ngroups, T))
        return cudaErrorInvalidValue;
    if (sizeof(TOut) == 2) {
        if (!make_map(&my, a.y, kP, a.nheads, T)) return cudaErrorInvalidValue;
    } else {
        my = mx;   // unused: fp32 y is stored row by row
    }
    cudaError_t e = cudaFuncSetAttribute(scan_tc_kernel<TOut, false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (a.runs > 0) {
        e = cudaFuncSetAttribute(scan_tc_kernel<TOut, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 SMEM_BYTES);
        if (e != cudaSuccess) return e;
        // Balanced: every run must be resident at once (a run may wait for a
        // state another run hands over), which a cooperative launch
        // guarantees or refuses; the hand-off flags start at zero.
        e = cudaMemsetAsync(a.handoff_flags, 0, (size_t)a.runs * sizeof(int), stream);
        if (e != cudaSuccess) return e;
        ScanArgs ac = a;
        void *args[] = {&mx, &mb, &mc, &my, &ac};
        e = cudaLaunchCooperativeKernel((const void *)scan_tc_kernel<TOut, true>, dim3((unsigned)a.runs),
                                        dim3(kThreads), args, SMEM_BYTES, stream);
        if (e == cudaSuccess) return cudaSuccess;
        (void)cudaGetLastError();   // not resident all at once: one CTA per chain instead
    }
    ScanArgs a1 = a;
    a1.runs = 0;
    const dim3 grid((unsigned)((size_t)a.nseq * (a.nheads / 2)));
    scan_tc_kernel<TOut, false><<<grid, kThreads, SMEM_BYTES, stream>>>(mx, mb, mc, my, a1);
    return cudaGetLastError();
}

int sm_count()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

}  // namespace

bool scan_tc_shape(int head_dim, int d_state, int chunk_size, int nheads, int ngroups)
{
    return head_dim == kP && d_state == kN && chunk_size == kQ && ngroups > 0 &&
           nheads % ngroups == 0 && (nheads / ngroups) % 2 == 0;
}

bool scan_tc_supports(const ScanArgs &a)
{
    const long long T = a.cu_seqlens ? (long long)a.seqlen : (long long)a.nseq * a.seqlen;
    return a.in_dtype == 1 && scan_tc_shape(a.head_dim, a.d_state, a.chunk_size, a.nheads, a.ngroups) &&
           T > 0 && encode_fn() != nullptr;
}

int scan_tc_balanced_runs(int nseq, int seqlen, int nheads)
{
    return scan_tc_balanced_runs_for(nseq, seqlen, nheads, sm_count());
}

int scan_tc_balanced_runs_for(int nseq, int seqlen, int nheads, int sms)
{
    // One CTA per (sequence, head pair) chain leaves SMs idle when the chains
    // do not fill whole waves; cutting the chains into one run per SM fills
    // them.  A chain's chunks stay a sequential recurrence whichever runs
    // sweep them, so with no more chains than SMs (one wave, each chain its
    // own critical path) the cut gains nothing and is not used.
    const long long chains = (long long)nseq * (nheads / 2);
    const long long nch = ((long long)seqlen + kQ - 1) / kQ;
    if (sms <= 0 || chains <= sms || nch <= 0) return 0;
    // A run's chunks cost about a tenth more than one chain's (the hand-offs,
    // and a compute loop that also walks pieces): cut only when the last wave
    // leaves more than a tenth of the SM slots idle.
    const long long waves = (chains + sms - 1) / sms;
    if (chains * 10 >= waves * sms * 9) return 0;
    return sms;
}

size_t scan_tc_handoff_bytes(int runs)
{
    return (size_t)runs * (2 * kP * kN * sizeof(float)) + (size_t)runs * sizeof(int);
}

cudaError_t launch_scan_tc(const ScanArgs &a, cudaStream_t stream)
{
    return a.y_dtype == 1 ? launch_tc_t<__nv_bfloat16>(a, stream) : launch_tc_t<float>(a, stream);
}

}  // namespace ssm
