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

// Status word written by kernels (only ever set to a nonzero code).
__device__ __forceinline__ void report_status(int *status, int code) {
    if (status) atomicCAS(status, 0, code);
}

}  // namespace ssm
