// common.cuh -- small device helpers shared by the KDA kernels (one translation unit: kda_lib.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kda.h"

namespace kda {

// Device error word.  Kernels record the first error they detect (a malformed cu_seqlens, a
// bounded wait that gave up) with set_error(); kda_check() reads and clears it.
__device__ int g_error_word;

__device__ __forceinline__ void set_error(int code) { atomicCAS(&g_error_word, 0, code); }

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Chunk length used by every prefill path.
constexpr int kChunk = 64;

// Input prologue (kda_options.prologue): activations of raw projections, in fp32.
constexpr float kQkNormEps = 1e-6f;  // x / sqrt(sum x^2 + eps) for the q/k L2 normalisation
__device__ __forceinline__ float sigmoid_f(float x) { return 1.f / (1.f + expf(-x)); }
// log sigmoid(x) = min(x, 0) - log(1 + e^{-|x|}), written so that neither branch overflows
__device__ __forceinline__ float log_sigmoid_f(float x) { return fminf(x, 0.f) - log1pf(expf(-fabsf(x))); }

// Workspace header written by the chunk-table kernel (first 256 bytes of every workspace).
struct WsHeader {
    int total_chunks;   // sum over sequences of ceil(len / 64)
    int bad;            // nonzero: cu_seqlens malformed, nothing is computed
    int next_unit;      // work counter of the persistent intra-chunk kernel (zeroed with the table)
    int pad[61];
};

// Map a global chunk index j (0 <= j < total) to (sequence n, first token t0, length L), with
// off[n] = number of chunks of sequences < n.  cu == nullptr means regular batches of Tseq tokens.
__device__ __forceinline__ void locate_chunk(int j, const int* __restrict__ off, const int32_t* __restrict__ cu,
                                             int Tseq, int N, int& n, long long& t0, int& L)
{
    int lo = 0, hi = N - 1;
    while (lo < hi) {  // largest n with off[n] <= j
        const int mid = (lo + hi + 1) >> 1;
        if (off[mid] <= j) lo = mid; else hi = mid - 1;
    }
    n = lo;
    const long long s0 = cu ? (long long)cu[n] : (long long)n * Tseq;
    const long long s1 = cu ? (long long)cu[n + 1] : (long long)(n + 1) * Tseq;
    t0 = s0 + (long long)(j - off[n]) * kChunk;
    const long long rem = s1 - t0;
    L = rem < kChunk ? (int)rem : kChunk;
}

__device__ __forceinline__ void seq_bounds(int n, const int32_t* __restrict__ cu, int Tseq, long long& s0, long long& s1)
{
    s0 = cu ? (long long)cu[n] : (long long)n * Tseq;
    s1 = cu ? (long long)cu[n + 1] : (long long)(n + 1) * Tseq;
}

}  // namespace kda
