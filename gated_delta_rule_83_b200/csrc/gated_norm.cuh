// gated_norm.cuh -- the output gate of a KDA layer: y = o / sqrt(mean_g(o^2) + eps) * weight * act(z).
//
// The attention review's GDN/KDA pseudo-code (lanjinlin.com.cn, entry on Qwen3-Next GDN, step
// "门控归一化") normalises the attention output with an RMS norm and multiplies it by the output gate
// z.  The Ring-linear notes of the same review describe two refinements used here: the RMS norm is
// taken over groups of channels, each group on its own ("Grouped RMSNorm"), and the norm, the
// sigmoid of the gate and the product run as one fused kernel so that the output is read and
// written once.  One streaming pass: every thread owns 8 consecutive channels of one row (16-byte
// bf16 or 32-byte fp32 vectors), the group's sum of squares is reduced with shuffles inside the
// aligned lane group that holds it, and o, z are read and y written exactly once.
#pragma once

#include "common.cuh"
#include "profile.cuh"

namespace kda {

constexpr int kNormThreads = 256;

template <typename T> struct Vec8;
template <> struct Vec8<__nv_bfloat16> {
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float* f)
    {
        const uint4 r = __ldcs(reinterpret_cast<const uint4*>(p));
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float2 t = __bfloat1622float2(h[m]);
            f[2 * m] = t.x;
            f[2 * m + 1] = t.y;
        }
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float* f)
    {
        uint4 r;
        __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&r);
#pragma unroll
        for (int m = 0; m < 4; ++m) h[m] = __floats2bfloat162_rn(f[2 * m], f[2 * m + 1]);
        __stcs(reinterpret_cast<uint4*>(p), r);
    }
};
template <> struct Vec8<float> {
    static __device__ __forceinline__ void load(const float* p, float* f)
    {
        const float4 a = __ldcs(reinterpret_cast<const float4*>(p)), b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    }
    static __device__ __forceinline__ void store(float* p, const float* f)
    {
        __stcs(reinterpret_cast<float4*>(p), make_float4(f[0], f[1], f[2], f[3]));
        __stcs(reinterpret_cast<float4*>(p) + 1, make_float4(f[4], f[5], f[6], f[7]));
    }
};

// sigmoid through the hardware's base-2 exponential (ex2.approx, relative error ~2^-22)
__device__ __forceinline__ float sigmoid_fast(float x)
{
    float e;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(-x * 1.4426950408889634f));
    return 1.f / (1.f + e);
}

// LG = log2(lanes per group) = log2(group / 8); d = channels per row (64 or 128).  One 8-channel
// chunk per thread at 32 registers, so eight CTAs (2,048 threads) per SM keep loads in flight.
template <typename T, int LG>
__global__ void __launch_bounds__(kNormThreads, 8)
gated_rmsnorm_kernel(const T* __restrict__ o, const T* __restrict__ z, const float* __restrict__ weight, T* y,
                     long long chunks, int d, float inv_group, float eps, int sigmoid_gate)
{
    const long long t = (long long)blockIdx.x * kNormThreads + threadIdx.x;
    const bool live = t < chunks;                  // every lane joins the shuffles below
    const long long e0 = (live ? t : 0) * 8;       // first element of this thread's 8 channels
    float x[8], g[8];
    Vec8<T>::load(o + e0, x);
    Vec8<T>::load(z + e0, g);
    float ss = 0.f;
#pragma unroll
    for (int m = 0; m < 8; ++m) ss = fmaf(x[m], x[m], ss);
#pragma unroll
    for (int s = 0; s < LG; ++s) ss += __shfl_xor_sync(0xffffffffu, ss, 1 << s);
    const float r = rsqrtf(ss * inv_group + eps);
    const int c0 = 8 * (int)(t & (d / 8 - 1));     // first channel within the row (d / 8 is 8 or 16)
    float w[8];
    if (weight) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(weight + c0));
        const float4 b = __ldg(reinterpret_cast<const float4*>(weight + c0) + 1);
        w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    } else {
#pragma unroll
        for (int m = 0; m < 8; ++m) w[m] = 1.f;
    }
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const float gate = sigmoid_gate ? sigmoid_fast(g[m]) : g[m];
        x[m] = x[m] * r * w[m] * gate;
    }
    if (live) Vec8<T>::store(y + e0, x);
}

template <typename T>
cudaError_t launch_gated_rmsnorm(const void* o, const void* z, const float* weight, void* y, long long rows, int d,
                                 int group, float eps, int sigmoid_gate, cudaStream_t stream)
{
    const long long chunks = rows * (d / 8);
    if (chunks == 0) return cudaSuccess;
    const long long blocks = (chunks + kNormThreads - 1) / kNormThreads;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    const T *oo = (const T*)o, *zz = (const T*)z;
    T* yy = (T*)y;
    const float ig = 1.f / (float)group;
    LaunchScope ls("gated_rmsnorm", stream);
    switch (group) {  // lanes per group: 1, 2, 4, 8 or 16
        case 8: gated_rmsnorm_kernel<T, 0><<<(unsigned)blocks, kNormThreads, 0, stream>>>(oo, zz, weight, yy, chunks, d, ig, eps, sigmoid_gate); break;
        case 16: gated_rmsnorm_kernel<T, 1><<<(unsigned)blocks, kNormThreads, 0, stream>>>(oo, zz, weight, yy, chunks, d, ig, eps, sigmoid_gate); break;
        case 32: gated_rmsnorm_kernel<T, 2><<<(unsigned)blocks, kNormThreads, 0, stream>>>(oo, zz, weight, yy, chunks, d, ig, eps, sigmoid_gate); break;
        case 64: gated_rmsnorm_kernel<T, 3><<<(unsigned)blocks, kNormThreads, 0, stream>>>(oo, zz, weight, yy, chunks, d, ig, eps, sigmoid_gate); break;
        default: gated_rmsnorm_kernel<T, 4><<<(unsigned)blocks, kNormThreads, 0, stream>>>(oo, zz, weight, yy, chunks, d, ig, eps, sigmoid_gate); break;
    }
    return cudaGetLastError();
}

}  // namespace kda
