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
// Work decomposition: one CTA per (sequence, pair of heads of one group),
// sweeping the sequence's chunks in order, with three warp roles that work on
// different chunks at the same time (640 threads, 20 warps):
//   * compute warpgroups (warps 4-19): head 2k + (wg & 1), column half wg >> 1;
//     thread i owns TMEM lane i (row i of G, M, Y, Yoff; d_state index i of
//     S^T and of the carried state, 32 of whose 64 head_dim entries it keeps
//     in fp32 registers for the whole sequence).  Per chunk: the next chunk's
//     cumulative decay (published for the converters), state update, decay
//     mask, new H^T tile, the next chunk's C converted into TMEM (the A
//     operand of C.B^T and C.H^T, double-buffered), output epilogue;
//   * converter warps (warps 0-2): one chunk ahead of the compute warps, they
//     convert the chunk's bf16 B and x tiles to fp16 in place in shared
//     memory and form the decay-weighted x (w o x) from the published decay;
//   * issuing warp (warp 3): lane 0 issues the TMA loads and stores and the
//     MMAs as their operands become ready.
// Every hand-off between roles is an mbarrier with a bounded wait (no named
// barrier spans two roles), so a wait that never completes cannot hang the
// kernel: it raises a CTA-wide abort flag instead.  20 warps keep 5 warps on
// each SM sub-partition, so every thread gets 96 registers.
//
// Per chunk k, the issuing thread runs
//   S_k = B^T [wX_a|wX_b]  (once Y_{k-1} has read M_{k-1}, whose TMEM S reuses)
//   G_k = C B^T            (once the epilogue of k-1 has read Y_{k-1})
//   Yoff_k = C [H_a^T|H_b^T] (once H_{k-1}^T is in shared memory)
//   Y_k = M_k X_k          (once the mask of chunk k is in TMEM)
// while the compute warps work through chunk k and the converters prepare
// chunk k+1.
//
// Precision: bf16 inputs are converted to fp16 (exact for |v| < 65504) so the
// derived operands M, w o x and H (rounded to fp16, 11 significant bits) keep
// the result within ~3e-4 of the fp64 recurrence; accumulation is fp32.  An
// operand beyond the fp16 range makes some output non-finite; the epilogue
// detects that and the kernel reports SSM_ERR_RANGE.
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
constexpr int kConvThreads = 96;       // converter warps 0-2 (lane-free work)
constexpr int kIssuerBase = 96;        // warp 3
constexpr int kComputeBase = 128;      // compute warpgroups: warps 4-19
constexpr int kCompute = 512;
constexpr int kThreads = kComputeBase + kCompute;      // 640

// Shared memory (bytes from the 1024-aligned dynamic base).  16-bit tiles use
// the 128B-swizzled layout TMA writes and the MMA descriptors read: rows of 64
// elements (128 B), 8-row groups of 1024 B, 16-byte chunk c of row r stored at
// c ^ (r % 8).  128-wide tiles are two 64-column halves 16 KB apart.
constexpr uint32_t HALF = 16384;
constexpr uint32_t OFF_C = 0;            // C [128 i][128 n] bf16 (TMA target; fp16 copy in TMEM)
constexpr uint32_t OFF_B = 32768;        // B buffer 0 [128 j][128 n] (bf16 -> fp16 in place)
constexpr uint32_t OFF_X = 65536;        // x, 2 buffers x 2 heads x [128 j][64 p] (bf16 -> fp16 in
                                         // place; after Y_k, the staging of y_k for its TMA store)
constexpr uint32_t XBUF = 32768;
constexpr uint32_t OFF_W = 131072;       // w o x, 2 heads x [128 j][64 p] fp16
constexpr uint32_t OFF_H = 163840;       // H^T fp16, 2 heads x [128 n][64 p]
constexpr uint32_t OFF_B1 = 196608;      // B buffer 1
constexpr uint32_t OFF_MISC = 229376;
constexpr uint32_t OFF_VD = OFF_MISC;              // float[2 buffers][2 heads][128]: column factors vd
constexpr uint32_t OFF_WF = OFF_VD + 2048;         // float[2 buffers][2 heads][4]: exp(cs_last - cs_{r_J})
constexpr uint32_t OFF_CSBT = OFF_WF + 64;         // float[2 buffers][2 heads][8]: block-end cs, cs_last
constexpr uint32_t OFF_CSB = OFF_CSBT + 128;       // float[4][8]: scan scratch per compute warpgroup
constexpr uint32_t OFF_PART = OFF_CSB + 128;       // float[4][4]: compute warp partial sums
constexpr uint32_t OFF_BAR = OFF_PART + 64;        // mbarriers (8 B each)
constexpr uint32_t NBAR = 18;
constexpr uint32_t OFF_TM = OFF_BAR + 8 * NBAR;    // TMEM base address (4 B)
constexpr uint32_t OFF_ABORT = OFF_TM + 4;         // CTA-wide abort flag (int)
constexpr uint32_t OFF_RANGE = OFF_TM + 8;         // set when an output is not finite (int)
constexpr uint32_t SMEM_BYTES = OFF_TM + 16;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// mbarrier indices (address OFF_BAR + 8 * index).  A barrier that serves
// alternate chunks (x buffers, converter hand-off, decay tables) comes in a
// pair indexed by chunk parity, so that no waiter can ever be two phases
// behind the barrier it waits on.
enum : uint32_t {
    BAR_X0 = 0, BAR_X1 = 1,   // x tiles of buffer 0 / 1 landed (TMA)
    BAR_CT = 2,               // C tile landed (TMA)
    BAR_BT0 = 3, BAR_BT1 = 4, // B tile of buffer 0 / 1 landed (TMA)
    BAR_CRAW = 5,             // compute warps have read the C tile (16 warp arrivals)
    BAR_CV0 = 6, BAR_CV1 = 7, // converters done with a chunk of parity 0 / 1 (3 warp arrivals)
    BAR_DC0 = 8, BAR_DC1 = 9, // decay tables of a chunk of parity 0 / 1 published (8 warp arrivals)
    BAR_S = 10,               // S MMAs of a chunk done (commit): w o x may be rewritten
    BAR_SG = 11,              // S and G MMAs of a chunk done (commit)
    BAR_YO = 12,              // Yoff MMAs done (commit)
    BAR_Y = 13,               // Y MMAs done (commit)
    BAR_MASK = 14,            // decay mask written (16 compute-warp arrivals)
    BAR_STATE = 15,           // H^T tile written (16 compute-warp arrivals)
    BAR_EPI = 16,             // epilogue done and next C in TMEM (16 compute-warp arrivals)
    BAR_DRAIN = 17            // abort path: every issued MMA done (commit)
};

// TMEM columns (fp32 accumulators, lane = row).
// G and Y share columns: the y MMAs write Y only after the mask has read G,
// and the next chunk's G is issued only after the epilogue has read Y.  C
// (fp16, two values per column, double-buffered) is the TMEM A operand of
// C.B^T and C.H^T.
constexpr uint32_t TM_G = 0, TM_Y = 0, TM_S = 128, TM_YO = 256, TM_C = 384;
constexpr uint32_t TM_COLS = 512;

constexpr uint32_t IDESC_G = tc::idesc_f16_f32(128, 128, 0, 0);   // C (K-major) x B (K-major)
constexpr uint32_t IDESC_S2 = tc::idesc_f16_f32(128, 128, 1, 1);  // B^T (MN-major) x [wX_a|wX_b] (MN-major)
constexpr uint32_t IDESC_YO2 = tc::idesc_f16_f32(128, 128, 0, 1); // C (K-major) x [H_a^T|H_b^T] (MN-major)
constexpr uint32_t IDESC_Y = tc::idesc_f16_f32(128, 64, 0, 1);    // M (TMEM) x X (MN-major)

constexpr float kSafeBlockDecay = 80.f;   // max exp argument taken by the factorised path

// Named barriers (never shared between roles): 1..4 per compute warpgroup,
// 5 all compute warps.
constexpr uint32_t NB_COMPUTE = 5;

extern __shared__ __align__(1024) uint8_t smem[];

__device__ __forceinline__ volatile int &abort_flag() {
    return *reinterpret_cast<volatile int *>(smem + OFF_ABORT);
}
__device__ __forceinline__ volatile int &range_flag() {
    return *reinterpret_cast<volatile int *>(smem + OFF_RANGE);
}
__device__ __forceinline__ uint64_t wait_limit(unsigned long long wait_ns) {
    return wait_ns ? wait_ns : kDefaultWaitNs;
}

// Bounded mbarrier wait: when it expires (or the abort flag is already up)
// `ok` turns false, the CTA-wide abort flag goes up, and every later wait of
// this thread returns at once.  The roles then run to the end of their loops
// without waiting, the issuing thread drains what it has in flight, and the
// kernel reports SSM_ERR_TIMEOUT.
__device__ __forceinline__ void wait_or_abort(uint32_t bar, uint32_t parity, bool &ok,
                                              unsigned long long wait_ns) {
    if (ok && abort_flag()) ok = false;
    if (ok && !tc::mbar_wait_bounded(bar, parity, ok, wait_limit(wait_ns))) abort_flag() = 1;
}

// One arrival per warp on an mbarrier, after every lane's prior writes.
__device__ __forceinline__ void warp_arrive(uint32_t bar, int lane) {
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(bar);
}

__device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t chunk) {
    return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

__device__ __forceinline__ uint32_t bf2_to_h2(uint32_t v, float scale) {
    const float2 p = __fmul2_rn(make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u)),
                                make_float2(scale, scale));
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
    return f2_to_h2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
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
__device__ __forceinline__ void mask_block(uint32_t g_taddr, uint32_t m_taddr, const float *sVD,
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
    const float4 *vd4 = reinterpret_cast<const float4 *>(sVD + jc * 32);
#pragma unroll
    for (int qq = 0; qq < 2; ++qq) {   // 16 columns at a time
        uint32_t r[16];
        tc::tmem_ld16(g_taddr + jc * 32 + qq * 16, r);
        tc::tmem_ld_wait();
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
            const int q = qq * 2 + q2;   // 8-column chunk within the block
            const float4 v0 = vd4[2 * q], v1 = vd4[2 * q + 1];
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
    float e;         // exp(cs_i)                  (decay of the carried state to row i)
    float a_last;    // exp(cs_last)               (decay over the whole chunk)
    bool safe;       // the row block's own decay fits the factorised path
};

// Raw dt of row i of the chunk starting at c0 (0 past the sequence end t1),
// loaded ahead of use: the compute and converter loops keep two chunks of it
// in flight.
__device__ __forceinline__ float load_dt(const ScanArgs &a, int H, int hh, long c0, long t1, int i) {
    return (c0 + i < t1) ? __ldg(a.dt + (size_t)(c0 + i) * H + hh) : 0.f;
}

// Cumulative decay of head hh over a chunk of Lc tokens whose raw dt for row
// i is dt_raw (warpgroup-wide); returns (cs_i, dt_i).  The warpgroup with
// ch == 0 publishes the chunk's tables, read later by the compute warps
// (decay_derive, the mask) and by the converters (w o x):
//   vd[j]   = exp(cs_{r_J} - cs_j) dt_j, J = j's 32-row block (column factors)
//   wf[J]   = exp(cs_last - cs_{r_J})      (so the chunk-state weight is
//                                          w_j = wf[J] vd_j: two factors <= 1)
//   csb[J]  = cs_{r_J} (J < 4), csb[4] = cs_last
__device__ __forceinline__ float2 decay_scan(const ScanArgs &a, int hh, float Ah, float dt_raw,
                                             int Lc, int i, int wq, int lane, int wg, int ch,
                                             float *sPART, float *sCSB, float *vd_out,
                                             float *wf_out, float *csb_out)
{
    const float dtv = (i < Lc) ? dt_apply(a.dtp, dt_raw, hh) : 0.f;
    float v = dtv * Ah;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    if (lane == 31) sPART[wq] = v;
    wg_sync(wg);
    float pre = 0.f;
    for (int w = 0; w < wq; ++w) pre += sPART[w];
    const float cs = v + pre;
    if (lane == 31) sCSB[wq] = cs;
    if (i == Lc - 1) sCSB[4] = cs;
    wg_sync(wg);
    if (ch == 0) {
        const float cs_last = sCSB[4];
        vd_out[i] = exp_dec(sCSB[wq] - cs) * dtv;   // <= dt
        if (i < 4) wf_out[i] = exp_dec(cs_last - sCSB[i]);
        if (i < 5) csb_out[i] = sCSB[i];
    }
    return make_float2(cs, dtv);
}

// The per-row decay quantities of ChunkDecay from row i's (cs, dt) and the
// chunk's published block ends csb.
__device__ __forceinline__ ChunkDecay decay_derive(float2 csdt, const float *csb, int wq, int ch) {
    ChunkDecay d;
    d.cs = csdt.x;
    d.dtv = csdt.y;
    const int kA = ch == 0 ? 0 : 1, kB = ch == 0 ? 3 : 2;
    d.uaA = (kA <= wq) ? exp_dec(d.cs - csb[kA]) : 0.f;
    d.uaB = (kB <= wq) ? exp_dec(d.cs - csb[kB]) : 0.f;
    d.safe = (__shfl_sync(0xffffffffu, d.cs, 0) - csb[wq]) <= kSafeBlockDecay;
    d.e = exp_dec(d.cs);
    d.a_last = exp_dec(csb[4]);
    return d;
}

template <typename TOut>
__global__ void __launch_bounds__(kThreads, 1)
scan_tc_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_b,
               const __grid_constant__ CUtensorMap map_c, const __grid_constant__ CUtensorMap map_y,
               const ScanArgs a)
{
    // bf16 y of full chunks is staged in shared memory and written by TMA;
    // fp32 y and partial chunks are stored row by row.
    constexpr bool kStoreByTma = sizeof(TOut) == 2;
    const uint32_t sbase = tc::smem_u32(smem);
    const int tid = threadIdx.x;
    const int lane = tid & 31;

    const int H = a.nheads, G = a.ngroups;
    const int hpg = H / G;
    const int pairs = H >> 1;
    const int s = blockIdx.x / pairs;
    const int h0 = (blockIdx.x - s * pairs) * 2;
    const int g = h0 / hpg;

    if (sbase & 1023u) {                 // the swizzled layouts need 1024-B alignment
        if (tid == 0) report_status(a.status_dev, kStatusInternal);
        return;
    }

    long t0, t1;
    if (a.cu_seqlens) {
        const int c0 = a.cu_seqlens[0], cs0 = a.cu_seqlens[s], cs1 = a.cu_seqlens[s + 1];
        const int cend = a.cu_seqlens[a.nseq];
        if (c0 != 0 || cs1 < cs0 || cs0 < 0 || cend != a.seqlen || cs1 > a.seqlen) {
            if (tid == 0) report_status(a.status_dev, kStatusDeviceInput);
            return;
        }
        t0 = cs0; t1 = cs1;
    } else {
        t0 = (long)s * a.seqlen; t1 = t0 + a.seqlen;
    }
    const int nch = (int)((t1 - t0 + kQ - 1) / kQ);   // chunks of this sequence

    size_t srow = (size_t)s;   // state row of this sequence
    bool load_init = a.initial_state != nullptr;
    if (a.slot_idx) {
        const int slot = a.slot_idx[s];
        if (slot < 0 || slot >= a.max_slots) {
            if (tid == 0) report_status(a.status_dev, kStatusDeviceInput);
            return;
        }
        srow = (size_t)slot;
        if (a.has_initial && a.has_initial[s] == 0) load_init = false;
    }

    const uint32_t bar0 = sbase + OFF_BAR;
    auto bar = [&](uint32_t idx) { return bar0 + 8u * idx; };

    if (tid < 32) {
        tc::tmem_alloc(sbase + OFF_TM, TM_COLS);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        tc::mbar_init(bar(BAR_X0), 1);
        tc::mbar_init(bar(BAR_X1), 1);
        tc::mbar_init(bar(BAR_CT), 1);
        tc::mbar_init(bar(BAR_BT0), 1);
        tc::mbar_init(bar(BAR_BT1), 1);
        tc::mbar_init(bar(BAR_S), 1);
        tc::mbar_init(bar(BAR_CRAW), 16);
        tc::mbar_init(bar(BAR_CV0), 3);
        tc::mbar_init(bar(BAR_CV1), 3);
        tc::mbar_init(bar(BAR_DC0), 8);
        tc::mbar_init(bar(BAR_DC1), 8);
        tc::mbar_init(bar(BAR_SG), 1);
        tc::mbar_init(bar(BAR_YO), 1);
        tc::mbar_init(bar(BAR_Y), 1);
        tc::mbar_init(bar(BAR_MASK), 16);
        tc::mbar_init(bar(BAR_STATE), 16);
        tc::mbar_init(bar(BAR_EPI), 16);
        tc::mbar_init(bar(BAR_DRAIN), 1);
        abort_flag() = 0;
        range_flag() = 0;
        tc::fence_mbar_init();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + OFF_TM);
    bool ok = true;
    float *vd_tab = reinterpret_cast<float *>(smem + OFF_VD);   // [2 buffers][2 heads][128]
    float *wf_tab = reinterpret_cast<float *>(smem + OFF_WF);   // [2 buffers][2 heads][4]

    if (tid >= kIssuerBase && tid < kComputeBase) {
        // ================= TMA / MMA issuing thread =================
        if (lane == 0) {
            const bool produce = a.stall_producer == 0;
            // Work in flight, for the drain after an abort: phases armed on the
            // TMA barriers, and whether any MMA was issued.
            uint32_t armed_x[2] = {0, 0}, armed_b[2] = {0, 0}, armed_c = 0;
            bool mma_issued = false;
            auto tile_row = [&](int k) { return (int)(t0 + (long)k * kQ); };
            auto load_x = [&](int k) {
                const uint32_t b = (uint32_t)k & 1u;
                tc::mbar_arrive_expect_tx(bar(BAR_X0 + b), 2 * HALF);
                tc::tma_load_3d(sbase + OFF_X + b * XBUF, &map_x, bar(BAR_X0 + b), 0, h0, tile_row(k));
                tc::tma_load_3d(sbase + OFF_X + b * XBUF + HALF, &map_x, bar(BAR_X0 + b), 0, h0 + 1, tile_row(k));
                ++armed_x[b];
            };
            auto load_c = [&](int k) {
                tc::mbar_arrive_expect_tx(bar(BAR_CT), 2 * HALF);
                tc::tma_load_3d(sbase + OFF_C, &map_c, bar(BAR_CT), 0, g, tile_row(k));
                tc::tma_load_3d(sbase + OFF_C + HALF, &map_c, bar(BAR_CT), 64, g, tile_row(k));
                ++armed_c;
            };
            auto load_b = [&](int k) {
                const uint32_t b = (uint32_t)k & 1u;
                const uint32_t dst = b ? sbase + OFF_B1 : sbase + OFF_B;
                tc::mbar_arrive_expect_tx(bar(BAR_BT0 + b), 2 * HALF);
                tc::tma_load_3d(dst, &map_b, bar(BAR_BT0 + b), 0, g, tile_row(k));
                tc::tma_load_3d(dst + HALF, &map_b, bar(BAR_BT0 + b), 64, g, tile_row(k));
                ++armed_b[b];
            };
            auto store_y = [&](int k) {   // y tiles of full chunk k, staged in its x buffer
                const uint32_t src = sbase + OFF_X + ((uint32_t)k & 1u) * XBUF;
                tc::tma_store_3d(&map_y, src, 0, h0, tile_row(k));
                tc::tma_store_3d(&map_y, src + HALF, 0, h0 + 1, tile_row(k));
                tc::bulk_commit();
            };
            if (produce && nch > 0) {
                load_c(0);
                load_x(0);
                load_b(0);
                if (nch > 1) {
                    load_x(1);
                    load_b(1);
                }
                wait_or_abort(bar(BAR_CRAW), 0, ok, a.wait_ns);   // compute warps read C_0
                if (ok && nch > 1) load_c(1);
            }
            for (int k = 0; k < nch && produce && ok; ++k) {
                const uint32_t b = (uint32_t)k & 1u;
                const uint32_t ph = (uint32_t)k & 1u;
                // chunk k converted (B and x in fp16, w o x)
                wait_or_abort(bar(BAR_CV0 + b), ((uint32_t)k >> 1) & 1u, ok, a.wait_ns);
                // S_k overwrites TMEM that held M_{k-1}: Y_{k-1} must be done
                if (k > 0) wait_or_abort(bar(BAR_Y), ph ^ 1u, ok, a.wait_ns);
                if (!ok) break;
                tc::tc_fence_after();
                const uint32_t sB = b ? sbase + OFF_B1 : sbase + OFF_B;
                {
                    const uint64_t dBmn = tc::sdesc_sw128(sB, HALF, 1024);               // B^T, MN-major
                    const uint64_t dW = tc::sdesc_sw128(sbase + OFF_W, HALF, 1024);    // [wX_a | wX_b]
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_f16_ss(tmem + TM_S, dBmn + kk * 128, dW + kk * 128, IDESC_S2, kk > 0);
                }
                tc::mma_commit(bar(BAR_S));
                mma_issued = true;
                // G_k overwrites Y_{k-1}, Yoff_k overwrites Yoff_{k-1}, and G_k needs C_k
                // in TMEM: the epilogue of k-1 (which converts C_k) must be done
                wait_or_abort(bar(BAR_EPI), ph, ok, a.wait_ns);
                if (!ok) break;
                if (k > 0 && kStoreByTma) store_y(k - 1);   // chunk k-1 is full (chunk k follows it)
                tc::tc_fence_after();
                const uint32_t tC = tmem + TM_C + 64u * b;
                {
                    const uint64_t dBk = tc::sdesc_sw128(sB, 16, 1024);                  // B, K-major
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t ko = (kk >> 2) * (HALF >> 4) + (kk & 3) * 2;
                        tc::mma_f16_ts(tmem + TM_G, tC + kk * 8, dBk + ko, IDESC_G, kk > 0);
                    }
                }
                tc::mma_commit(bar(BAR_SG));
                // x of chunk k+1 into the buffer of chunk k-1, once Y_{k-1} has read
                // x_{k-1} and the store of y_{k-1} (staged there) has read it
                if (k > 0 && k + 1 < nch) {
                    tc::bulk_wait_read();
                    load_x(k + 1);
                }
                // Yoff_k reads H_{k-1}^T (the initial state's for k = 0)
                wait_or_abort(bar(BAR_STATE), ph, ok, a.wait_ns);
                if (!ok) break;
                tc::tc_fence_after();
                {
                    const uint64_t dH = tc::sdesc_sw128(sbase + OFF_H, HALF, 1024);     // [H_a^T | H_b^T]
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_f16_ts(tmem + TM_YO, tC + kk * 8, dH + kk * 128, IDESC_YO2, kk > 0);
                }
                tc::mma_commit(bar(BAR_YO));
                // B of chunk k+2 into this buffer once S_k and G_k have read B_k
                wait_or_abort(bar(BAR_SG), ph, ok, a.wait_ns);
                if (!ok) break;
                if (k + 2 < nch) load_b(k + 2);
                // Y_k needs the mask
                wait_or_abort(bar(BAR_MASK), ph, ok, a.wait_ns);
                if (!ok) break;
                tc::tc_fence_after();
                {
                    const uint64_t dX = tc::sdesc_sw128(sbase + OFF_X + b * XBUF, HALF, 1024);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_f16_ts(tmem + TM_Y, tmem + TM_S + kk * 8, dX + kk * 128, IDESC_Y, kk > 0);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_f16_ts(tmem + TM_Y + 64, tmem + TM_S + 64 + kk * 8,
                                       dX + (HALF >> 4) + kk * 128, IDESC_Y, kk > 0);
                }
                tc::mma_commit(bar(BAR_Y));
                // C of chunk k+2 once the compute warps have read C_{k+1}
                if (k + 2 < nch) {
                    wait_or_abort(bar(BAR_CRAW), ((uint32_t)k + 1u) & 1u, ok, a.wait_ns);
                    if (!ok) break;
                    load_c(k + 2);
                }
            }
            // y of the last chunk
            if (ok && produce && nch > 0) {
                wait_or_abort(bar(BAR_EPI), (uint32_t)nch & 1u, ok, a.wait_ns);
                if (ok && kStoreByTma && t0 + (long)nch * kQ <= t1) store_y(nch - 1);
            }
            if (!ok) {
                // Aborted: wait (bounded) for every MMA issued and for the last
                // phase armed on each load barrier, so that nothing writes TMEM
                // or shared memory after they are released.
                const uint64_t lim = wait_limit(a.wait_ns);
                bool dok = true;
                if (mma_issued) {
                    tc::mma_commit(bar(BAR_DRAIN));
                    tc::mbar_wait_bounded(bar(BAR_DRAIN), 0, dok, lim);
                }
                for (int b = 0; b < 2; ++b) {
                    bool xok = true;
                    if (armed_x[b]) tc::mbar_wait_bounded(bar(BAR_X0 + b), (armed_x[b] - 1) & 1u, xok, lim);
                }
                for (int b = 0; b < 2; ++b) {
                    bool bok = true;
                    if (armed_b[b]) tc::mbar_wait_bounded(bar(BAR_BT0 + b), (armed_b[b] - 1) & 1u, bok, lim);
                }
                bool cok = true;
                if (armed_c) tc::mbar_wait_bounded(bar(BAR_CT), (armed_c - 1) & 1u, cok, lim);
            }
            tc::bulk_wait_all();
        }
        __syncwarp();
    } else if (tid < kConvThreads) {
        // ================= converter warps: one chunk ahead =================
        // 4096 jobs of one 16-byte chunk (8 values) per tile row: jobs 0..2047
        // are x (head, row, chunk): x -> fp16 in place and w o x; jobs
        // 2048..4095 are B (half, row, chunk) -> fp16 in place.  Thread t takes
        // jobs t, t + 96, ...; a warp's 32 consecutive jobs cover 4 whole rows,
        // so its 16-byte accesses hit every bank once per 128 bytes.
        for (int k = 0; k < nch; ++k) {
            const uint32_t b = (uint32_t)k & 1u;
            const long c0 = t0 + (long)k * kQ;
            const int Lc = (int)min((long)kQ, t1 - c0);
            const uint32_t xt = sbase + OFF_X + b * XBUF;
            wait_or_abort(bar(BAR_X0 + b), ((uint32_t)k >> 1) & 1u, ok, a.wait_ns);
            wait_or_abort(bar(BAR_DC0 + b), ((uint32_t)k >> 1) & 1u, ok, a.wait_ns);
            // w o x overwrites the tile S_{k-1} read
            if (k >= 1) wait_or_abort(bar(BAR_S), ((uint32_t)k - 1u) & 1u, ok, a.wait_ns);
            const float *vd = vd_tab + b * 256;
            const float *wf = wf_tab + b * 8;
#pragma unroll 4
            for (int j = tid; j < 2048; j += kConvThreads) {
                const int hd = j >> 10, row = (j >> 3) & 127, q = j & 7;
                const uint32_t off = hd * HALF + sw128(row, q);
                if (row < Lc) {
                    const float w = wf[hd * 4 + (row >> 5)] * vd[hd * 128 + row];
                    const uint4 v = lds128(xt + off);
                    sts128(xt + off, cvt_chunk(v));
                    sts128(sbase + OFF_W + off, cvt_chunk_scaled(v, w));
                } else {
                    sts128(xt + off, make_uint4(0, 0, 0, 0));
                    sts128(sbase + OFF_W + off, make_uint4(0, 0, 0, 0));
                }
            }
            wait_or_abort(bar(BAR_BT0 + b), ((uint32_t)k >> 1) & 1u, ok, a.wait_ns);
            const uint32_t bt = b ? sbase + OFF_B1 : sbase + OFF_B;
#pragma unroll 4
            for (int j = tid; j < 2048; j += kConvThreads) {
                const int hf = j >> 10, row = (j >> 3) & 127, q = j & 7;
                const uint32_t addr = bt + hf * HALF + sw128(row, q);
                sts128(addr, row < Lc ? cvt_chunk(lds128(addr)) : make_uint4(0, 0, 0, 0));
            }
            tc::fence_proxy_async_smem();
            warp_arrive(bar(BAR_CV0 + b), lane);
        }
    } else if (tid >= kComputeBase) {
        // ================= compute warpgroups =================
        const int ctid = tid - kComputeBase;
        const int wg = ctid >> 7;            // compute warpgroup 0..3
        const int hd = wg & 1;               // head slot of the pair
        const int ch = wg >> 1;              // column half
        const int i = ctid & 127;            // row / TMEM lane / d_state index
        const int wq = i >> 5;               // warp within the warpgroup = 32-row block
        const int hh = h0 + hd;
        const uint32_t tlane = (uint32_t)(wq * 32) << 16;
        float *sCSB = reinterpret_cast<float *>(smem + OFF_CSB) + wg * 8;
        float *sPART = reinterpret_cast<float *>(smem + OFF_PART) + wg * 4;
        const size_t state_off = (srow * H + hh) * (size_t)(kP * kN) + (size_t)(32 * ch) * kN + i;

        // Row i's quarter wg of C_k (d_state n in [32 wg, 32 wg + 32)) as fp16
        // pairs into TMEM C[k & 1] (lane i, columns 16 wg ..): the A operand
        // of C.B^T and C.H^T.  Rows past the chunk end are zero.
        auto convert_c = [&](int k) {
            const long ck = t0 + (long)k * kQ;
            const bool live_c = i < (int)min((long)kQ, t1 - ck);
            wait_or_abort(bar(BAR_CT), (uint32_t)k & 1u, ok, a.wait_ns);
            const uint32_t ctile = sbase + OFF_C + (wg >> 1) * HALF;
            uint4 v[4];
#pragma unroll
            for (int q = 0; q < 4; ++q)
                v[q] = live_c ? lds128(ctile + sw128(i, 4 * (wg & 1) + q)) : make_uint4(0, 0, 0, 0);
            warp_arrive(bar(BAR_CRAW), lane);   // the C tile may be reloaded
            uint32_t pc[16];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 u = cvt_chunk(v[q]);
                pc[4 * q] = u.x; pc[4 * q + 1] = u.y; pc[4 * q + 2] = u.z; pc[4 * q + 3] = u.w;
            }
            tc::tmem_st16(tmem + tlane + TM_C + 64u * ((uint32_t)k & 1u) + 16 * wg, pc);
            tc::tmem_st_wait();
        };

        float Hs[32];
#pragma unroll
        for (int p = 0; p < 32; ++p)
            Hs[p] = load_init ? state_load1(a.initial_state, state_off + (size_t)p * kN, a.rp) : 0.f;
        write_state_half(sbase + OFF_H + hd * HALF, i, ch, Hs);
        tc::fence_proxy_async_smem();
        warp_arrive(bar(BAR_STATE), lane);     // H_{-1}^T ready for Yoff_0

        const float Ah = a.A[hh];
        const float Dh = a.D ? a.D[hh] : 0.f;
        TOut *y = static_cast<TOut *>(a.y);
        float *csb_tab = reinterpret_cast<float *>(smem + OFF_CSBT);   // [2 buffers][2 heads][8]
        float2 cs_cur = make_float2(0.f, 0.f);   // (cs_i, dt_i) of the current chunk
        if (nch > 0) {
            convert_c(0);
            tc::tc_fence_before();
            warp_arrive(bar(BAR_EPI), lane);   // C_0 in TMEM for G_0
            cs_cur = decay_scan(a, hh, Ah, load_dt(a, H, hh, t0, t1, i), (int)min((long)kQ, t1 - t0),
                                i, wq, lane, wg, ch, sPART, sCSB, vd_tab + hd * 128, wf_tab + hd * 4,
                                csb_tab + hd * 8);
            if (ch == 0) warp_arrive(bar(BAR_DC0), lane);
        }
        tc::named_sync(NB_COMPUTE, kCompute);   // chunk 0's tables visible to every compute warp
        float dt_n1 = load_dt(a, H, hh, t0 + kQ, t1, i);   // raw dt of the next chunk
        for (int k = 0; k < nch; ++k) {
            const uint32_t ph = (uint32_t)k & 1u, vb = (uint32_t)k & 1u;
            const long c0 = t0 + (long)k * kQ;
            const int Lc = (int)min((long)kQ, t1 - c0);
            const long c1 = c0 + kQ;
            const bool has_next = c1 < t1;
            const bool live = i < Lc;
            // dt two chunks ahead, so its load has a whole chunk to land
            const float dt_n2 = load_dt(a, H, hh, c0 + 2 * kQ, t1, i);

            const ChunkDecay cur = decay_derive(cs_cur, csb_tab + vb * 16 + hd * 8, wq, ch);
            // ---- next chunk's decay, published for the converters (while S_k, G_k run) ----
            float2 cs_nxt = make_float2(0.f, 0.f);
            if (has_next) {
                cs_nxt = decay_scan(a, hh, Ah, dt_n1, (int)min((long)kQ, t1 - c1), i, wq, lane, wg, ch,
                                    sPART, sCSB, vd_tab + (vb ^ 1u) * 256 + hd * 128,
                                    wf_tab + (vb ^ 1u) * 8 + hd * 4, csb_tab + (vb ^ 1u) * 16 + hd * 8);
                if (ch == 0) warp_arrive(bar(BAR_DC0 + (vb ^ 1u)), lane);
            }

            // ---- carried state: H <- exp(cs_L) H + S (d_state row i, p half ch) ----
            wait_or_abort(bar(BAR_SG), ph, ok, a.wait_ns);
            tc::tc_fence_after();
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                uint32_t rr[16];
                tc::tmem_ld16(tmem + tlane + TM_S + hd * 64 + ch * 32 + q * 16, rr);
                tc::tmem_ld_wait();
                const float2 al2 = make_float2(cur.a_last, cur.a_last);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float2 h2 = __ffma2_rn(al2, make_float2(Hs[q * 16 + 2 * e], Hs[q * 16 + 2 * e + 1]),
                                                 make_float2(__uint_as_float(rr[2 * e]), __uint_as_float(rr[2 * e + 1])));
                    Hs[q * 16 + 2 * e] = h2.x;
                    Hs[q * 16 + 2 * e + 1] = h2.y;
                }
            }
            tc::tc_fence_before();
            tc::named_sync(NB_COMPUTE, kCompute);   // every S column read: M may overwrite them
            tc::tc_fence_after();

            // ---- decay mask M of head hd into TMEM (over S of this head) ----
            {
                const float *vd = vd_tab + vb * 256 + hd * 128;
                const int kA = ch == 0 ? 0 : 1, kB = ch == 0 ? 3 : 2;
                const uint32_t m_taddr = tmem + tlane + TM_S + hd * 64;
                mask_block(tmem + tlane + TM_G, m_taddr, vd, kA, wq, lane, cur.uaA, cur.safe, cur.cs, cur.dtv, Dh);
                mask_block(tmem + tlane + TM_G, m_taddr, vd, kB, wq, lane, cur.uaB, cur.safe, cur.cs, cur.dtv, Dh);
                tc::tmem_st_wait();
            }
            tc::tc_fence_before();
            warp_arrive(bar(BAR_MASK), lane);

            // ---- new H^T tile for the next chunk (Yoff_k read the old one) ----
            wait_or_abort(bar(BAR_YO), ph, ok, a.wait_ns);
            write_state_half(sbase + OFF_H + hd * HALF, i, ch, Hs);
            tc::fence_proxy_async_smem();
            warp_arrive(bar(BAR_STATE), lane);

            // ---- C of the next chunk into TMEM (while the y MMAs run) ----
            if (has_next) convert_c(k + 1);

            // ---- y = Y + exp(cs_i) Yoff (row i, p half ch; D x is inside Y) ----
            wait_or_abort(bar(BAR_Y), ph, ok, a.wait_ns);
            tc::tc_fence_after();
#pragma unroll
            for (int q = 0; q < 2; ++q) {   // 16 columns at a time
                uint32_t ry[16], ro[16];
                tc::tmem_ld16(tmem + tlane + TM_Y + hd * 64 + ch * 32 + q * 16, ry);
                tc::tmem_ld16(tmem + tlane + TM_YO + hd * 64 + ch * 32 + q * 16, ro);
                tc::tmem_ld_wait();
                float out[16];
                const float2 e2 = make_float2(cur.e, cur.e);
                float2 ysum = make_float2(0.f, 0.f);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const float2 o2 = __ffma2_rn(e2, make_float2(__uint_as_float(ro[2 * c]), __uint_as_float(ro[2 * c + 1])),
                                                 make_float2(__uint_as_float(ry[2 * c]), __uint_as_float(ry[2 * c + 1])));
                    out[2 * c] = o2.x;
                    out[2 * c + 1] = o2.y;
                    ysum = __fadd2_rn(ysum, o2);
                }
                if (!isfinite(ysum.x + ysum.y)) range_flag() = 1;
                if (kStoreByTma && Lc == kQ) {   // into x_k's buffer: Y_k has read it
                    stage16_bf16(sbase + OFF_X + vb * XBUF + hd * HALF, i, 4 * ch + 2 * q, out);
                } else if (live) {
                    store16(y + ((size_t)(c0 + i) * H + hh) * kP + 32 * ch + 16 * q, out);
                }
            }
            tc::fence_proxy_async_smem();
            tc::tc_fence_before();
            warp_arrive(bar(BAR_EPI), lane);
            cs_cur = cs_nxt;
            dt_n1 = dt_n2;
        }
        if (a.final_state) {
#pragma unroll
            for (int p = 0; p < 32; ++p) state_store1(a.final_state, state_off + (size_t)p * kN, Hs[p], a.rp);
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (tid < 32) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, TM_COLS);
    }
    if (abort_flag()) {
        if (tid == 0) report_status(a.status_dev, kStatusTimeout);
    } else if (tid == 0 && range_flag()) {
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
    cudaError_t e = cudaFuncSetAttribute(scan_tc_kernel<TOut>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)((size_t)a.nseq * (a.nheads / 2)));
    scan_tc_kernel<TOut><<<grid, kThreads, SMEM_BYTES, stream>>>(mx, mb, mc, my, a);
    return cudaGetLastError();
}

}  // namespace

bool scan_tc_supports(const ScanArgs &a)
{
    const long long T = a.cu_seqlens ? (long long)a.seqlen : (long long)a.nseq * a.seqlen;
    return a.in_dtype == 1 && a.head_dim == kP && a.d_state == kN && a.chunk_size == kQ &&
           (a.nheads / a.ngroups) % 2 == 0 && T > 0 && encode_fn() != nullptr;
}

cudaError_t launch_scan_tc(const ScanArgs &a, cudaStream_t stream)
{
    return a.y_dtype == 1 ? launch_tc_t<__nv_bfloat16>(a, stream) : launch_tc_t<float>(a, stream);
}

}  // namespace ssm
