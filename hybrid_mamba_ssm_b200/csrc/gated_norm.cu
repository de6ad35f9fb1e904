// gated_norm.cu -- gated group RMSNorm after the scan, gate first (the
// _gated_group_rmsnorm kernel of the MAX nemotron_h article, section 5.4
// item 4, with norm_before_gate = False): for each row and each group of
// group_size channels,
//
//   g   = y * silu(z)
//   out = g / sqrt(mean_group(g^2) + eps) * weight
//
// all in fp32.  A group spans several heads (1024 or 2048 channels at the
// Nemotron-H shapes), i.e. several scan CTAs, so it is its own kernel rather
// than the scan's epilogue.  One CTA per (row, group): each thread owns 8
// adjacent channels (one 16-byte load of bf16 y and z), keeps g in registers
// and takes part in one block reduction of the sum of squares.  Bound by HBM:
// y, z read once, out written once.
#include "common.cuh"
#include "ssm_internal.h"

namespace ssm {

__device__ __forceinline__ void load8(const float *p, float (&v)[8]) {
    const float4 a = __ldcs(reinterpret_cast<const float4 *>(p));
    const float4 b = __ldcs(reinterpret_cast<const float4 *>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&v)[8]) {
    const uint4 r = __ldcs(reinterpret_cast<const uint4 *>(p));
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}
__device__ __forceinline__ void store8(float *p, const float (&v)[8]) {
    reinterpret_cast<float4 *>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4 *>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void store8(__nv_bfloat16 *p, const float (&v)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t *>(&h);
    }
    *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

template <typename TY, typename TZ, typename TO>
__global__ void __launch_bounds__(1024)
gated_rmsnorm_kernel(GatedNormArgs a)
{
    __shared__ float red[32];
    const int G = a.dim / a.group_size;
    const size_t rg = blockIdx.x;
    const size_t row = rg / G;
    const int grp = (int)(rg - row * G);
    const int c0 = grp * a.group_size + threadIdx.x * 8;
    const size_t off = row * (size_t)a.dim + c0;

    float yv[8], zv[8], g[8];
    load8(static_cast<const TY *>(a.y) + off, yv);
    load8(static_cast<const TZ *>(a.z) + off, zv);
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        g[i] = yv[i] * silu_approx(zv[i]);
        ss = fmaf(g[i], g[i], ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    if (warp == 0) {
        float v = (lane < (int)(blockDim.x >> 5)) ? red[lane] : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red[0] = v;
    }
    __syncthreads();
    const float r = rsqrtf(red[0] / (float)a.group_size + a.eps);
    const float4 w0 = __ldg(reinterpret_cast<const float4 *>(a.weight + c0));
    const float4 w1 = __ldg(reinterpret_cast<const float4 *>(a.weight + c0) + 1);
    const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    float o8[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) o8[i] = g[i] * r * wv[i];
    store8(static_cast<TO *>(a.out) + off, o8);
}

template <typename TY, typename TZ>
static cudaError_t launch_norm_yz(const GatedNormArgs &a, cudaStream_t stream)
{
    const unsigned blocks = (unsigned)((size_t)a.rows * (a.dim / a.group_size));
    const unsigned threads = (unsigned)(a.group_size / 8);
    if (a.out_dtype == 1)
        gated_rmsnorm_kernel<TY, TZ, __nv_bfloat16><<<blocks, threads, 0, stream>>>(a);
    else
        gated_rmsnorm_kernel<TY, TZ, float><<<blocks, threads, 0, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_gated_rmsnorm(const GatedNormArgs &a, cudaStream_t stream)
{
    const bool yb = a.y_dtype == 1, zb = a.z_dtype == 1;
    if (yb && zb) return launch_norm_yz<__nv_bfloat16, __nv_bfloat16>(a, stream);
    if (yb) return launch_norm_yz<__nv_bfloat16, float>(a, stream);
    if (zb) return launch_norm_yz<float, __nv_bfloat16>(a, stream);
    return launch_norm_yz<float, float>(a, stream);
}

}  // namespace ssm
