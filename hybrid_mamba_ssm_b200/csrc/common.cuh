// common.cuh -- small device helpers shared by the libssm kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssm {

// Storage types of x / B / C and y.
struct bf16_t { uint16_t bits; };

__device__ __forceinline__ float load_f32(const float *p) { return __ldg(p); }
__device__ __forceinline__ float load_f32(const __nv_bfloat16 *p) {
    return __bfloat162float(__ldg(p));
}

// Four consecutive values starting at p (p 8-byte aligned for bf16, 16-byte
// aligned for fp32).
__device__ __forceinline__ float4 load4(const float *p) {
    return __ldg(reinterpret_cast<const float4 *>(p));
}
__device__ __forceinline__ float4 load4(const __nv_bfloat16 *p) {
    uint2 u = __ldg(reinterpret_cast<const uint2 *>(p));
    __nv_bfloat162 lo = *reinterpret_cast<__nv_bfloat162 *>(&u.x);
    __nv_bfloat162 hi = *reinterpret_cast<__nv_bfloat162 *>(&u.y);
    float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
    return make_float4(a.x, a.y, b.x, b.y);
}

__device__ __forceinline__ void store_out(float *p, float v) { *p = v; }
__device__ __forceinline__ void store_out(__nv_bfloat16 *p, float v) {
    *p = __float2bfloat16_rn(v);
}

// Step-size transform applied where a kernel reads dt (the raw projection
// output): v = dt + bias[h]; v = log(1 + e^v) if softplus (v itself above
// 20, where the two agree to fp32); clamp to [lo, hi] if clamp.  All off is
// the identity.
struct DtParams {
    const float *bias;   // [nheads] or nullptr
    int softplus, clamp;
    float lo, hi;
};

__device__ __forceinline__ float dt_apply(const DtParams &p, float v, int h) {
    if (p.bias) v += __ldg(p.bias + h);
    if (p.softplus) v = v > 20.f ? v : log1pf(__expf(v));
    if (p.clamp) v = fminf(fmaxf(v, p.lo), p.hi);
    return v;
}

// Hardware approximate reciprocal and base-2 exponential (one special-
// function-unit operation each; rcp(+inf) = 0, ex2 of a large negative
// argument = 0).
__device__ __forceinline__ float rcp_approx(float v) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}
__device__ __forceinline__ float ex2_approx(float v) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}

// SiLU v * sigmoid(v) = v / (1 + 2^(-v log2 e)); -0 for large negative v.
__device__ __forceinline__ float silu_approx(float v) {
    return v * rcp_approx(1.f + ex2_approx(v * -1.4426950408889634f));
}

// ---------------------------------------------------------------------------
// fp16 state storage with stochastic rounding.
//
// Random bits: Philox-4x32 (Salmon, Moraes, Dror, Shaw, "Parallel random
// numbers: as easy as 1, 2, 3", SC'11), a counter-based generator: each round
// multiplies two of the four 32-bit counter words by fixed odd constants,
// swaps and xors the high halves with the other words and the key, and the
// key is bumped by two Weyl constants between rounds.  State element e (its
// index in the state buffer) draws 16 bits: half (e % 2, low half first) of
// word (e % 8) / 2 of Philox(counter = (e / 8 as 64 bits, offset as 64 bits),
// key = seed), so one Philox call serves 8 adjacent elements.
struct RoundParams {
    int f16;             // state stored as fp16 (else fp32)
    int stochastic;      // fp16 rounding: stochastic (else round to nearest even)
    uint32_t key0, key1; // seed
    uint32_t off0, off1; // per-call offset (e.g. the decode step)
    int rounds;          // Philox rounds (10 = Philox-4x32-10)
};

__device__ __forceinline__ uint4 philox4x32(uint4 c, uint32_t k0, uint32_t k1, int rounds) {
    for (int r = 0; r < rounds; ++r) {
        const uint32_t lo0 = c.x * 0xD2511F53u, hi0 = __umulhi(c.x, 0xD2511F53u);
        const uint32_t lo1 = c.z * 0xCD9E8D57u, hi1 = __umulhi(c.z, 0xCD9E8D57u);
        c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    return c;
}

// The four random words for state elements e .. e+7 (e a multiple of 8).
__device__ __forceinline__ uint4 state_random8(const RoundParams &p, size_t e) {
    const size_t q = e >> 3;
    return philox4x32(make_uint4((uint32_t)q, (uint32_t)(q >> 32), p.off0, p.off1),
                      p.key0, p.key1, p.rounds);
}

// fp32 -> fp16 with stochastic rounding: v moves to the fp16 neighbour away
// from zero iff u < frac, where frac is v's distance from the neighbour
// toward zero in units of the fp16 spacing there, and u = r / 2^16 for the
// element's 16 random bits r.  Magnitudes beyond 65504 saturate; NaN stays NaN.
__device__ __forceinline__ __half sr_to_half(float v, uint32_t r) {
    const float a = fabsf(v);
    if (!(a < 65504.f)) return __float2half_rn(a == a ? copysignf(65504.f, v) : v);
    float m;
    if (a >= 6.103515625e-05f) {        // fp16 normal range: 13 mantissa bits dropped
        const uint32_t b = __float_as_uint(a);
        const uint32_t low = b & 0x1FFFu;
        m = __uint_as_float((b & ~0x1FFFu) + (((r >> 3) < low) ? 0x2000u : 0u));
    } else {                            // fp16 subnormals: spacing 2^-24
        const float x = a * 16777216.f;
        const float fl = floorf(x);
        m = (fl + (((float)r < (x - fl) * 65536.f) ? 1.f : 0.f)) * 5.9604644775390625e-08f;
    }
    m = fminf(m, 65504.f);
    return __float2half_rn(copysignf(m, v));
}

__device__ __forceinline__ __half state_to_half(const RoundParams &p, float v, uint32_t r) {
    return p.stochastic ? sr_to_half(v, r) : __float2half_rn(v);
}

// One state element e of a state buffer in either storage type.
__device__ __forceinline__ float state_load1(const void *base, size_t e, const RoundParams &p) {
    return p.f16 ? __half2float(static_cast<const __half *>(base)[e])
                 : static_cast<const float *>(base)[e];
}
__device__ __forceinline__ void state_store1(void *base, size_t e, float v, const RoundParams &p) {
    if (!p.f16) {
        __stcs(static_cast<float *>(base) + e, v);   // written once: streaming (evict-first)
        return;
    }
    uint32_t r = 0;
    if (p.stochastic) {
        const uint4 q = state_random8(p, e & ~(size_t)7);
        const uint32_t w = (uint32_t)((e & 7) >> 1);
        const uint32_t word = w == 0 ? q.x : (w == 1 ? q.y : (w == 2 ? q.z : q.w));
        r = (word >> (16 * (uint32_t)(e & 1))) & 0xFFFFu;
    }
    static_cast<__half *>(base)[e] = state_to_half(p, v, r);
}

// Status word written by kernels (only ever set to a nonzero code).
// Codes a kernel writes to the caller's status word (the ssm_status values of
// include/ssm.h).
constexpr int kStatusTimeout = 5;      // a bounded wait expired
constexpr int kStatusDeviceInput = 6;  // inconsistent cu_seqlens or slot index
constexpr int kStatusRange = 7;        // a tensor-core operand beyond the fp16 range
constexpr int kStatusInternal = 8;     // a launch that breaks the kernel's own layout rule

// Default limit of a bounded wait (wall time, via %globaltimer).
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;

__device__ __forceinline__ void report_status(int *status, int code) {
    if (status) atomicCAS(status, 0, code);
}

}  // namespace ssm
