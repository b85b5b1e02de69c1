// backward_simt.cuh -- the chunked KDA backward pass (training) on CUDA cores in fp32.
//
// The pages name a custom backward only in passing; this is the reverse-mode derivative of the
// chunk form that the forward uses (the "Kimi Linear" explainer, section "硬件效率的深度优化":
// chunk-parallel inside a chunk, recurrent between chunks, WY representation, UT transform).
// For a loss with cotangents dO (per token) and dS_final, the derivative splits the same way:
//
// per chunk, with start state S and chunk-local quantities from the forward's phase A
// (W = T Kt, Uv = T V, Qg = q e^g, Kd = k e^{g_last - g}, gam = e^{g_last}, P = lower(Qf Kb^T)):
//     U    = Uv - W S,   O = Qg S + P U,   S_next = Diag(gam) S + Kd^T U
//
//   1. forward recompute: the CUDA-core phase A, then its phase B storing every chunk's start
//      state S_c and its corrected values U.
//   2. reverse chain over chunks (one CTA per (sequence, head, 32 state columns), chunks last to
//      first), carrying D = dL/dS_next, with E = P^T dO and F = Qg^T dO computed chunk-parallel
//      beforehand (they do not depend on D):
//          dU = E + Kd D
//          D <- Diag(gam) D + F - W^T dU                 (= dL/dS at the chunk start)
//      storing every chunk's end cotangent D_c and dU; D after the first chunk is dL/dS0.
//   3. chunk-parallel, state side (one CTA per (chunk, head)): with S_c, D_c, U and dU,
//          dQg = dO S_c^T,  dW = -dU S_c^T,  dKd = U D_c^T,  dP = lower_incl(dO U^T),
//          dgam_c = sum_j D_c[c][j] S_c[c][j]
//   4. chunk-parallel, input side (one CTA per (chunk, head)): through the UT transform,
//          T = N Diag(beta), N = (I + Diag(beta) At)^{-1}, At = strict_lower(Kf Kb^T):
//          dT = dW Kt^T + dU V^T (lower incl),  dV = T^T dU,  dKt = T^T dW,
//          dN = dT Diag(beta),  dbeta_i += sum_r dT[r][i] N[r][i],
//          dM = -N^T dN N^T (strict lower),  dbeta_r += sum_i dM[r][i] At[r][i],  dAt = Diag(beta) dM,
//      then through the gated products (P = Qf Kb^T, At = Kf Kb^T with the per-channel factors
//      e^{g_r - g_i}) and the gating itself to dq, dk and dg; dlog_alpha is the reverse cumulative
//      sum of dg inside the chunk (g restarts every chunk).
//
// Steps 3 and 4 work on tiles of the key dimension, so each CTA holds a few 64 x 64 matrices plus
// tiles; their products are register-tiled (each thread owns a 4 x 4, 4 x 2 or 8 x 2 block of
// rows tr + 16 i and columns tc + 16 j, so the shared-memory reads of a warp hit distinct banks).  The per-channel factors use the same centre-of-range reference as the
// forward; a tile whose in-chunk gate spread exceeds kFactorSpread takes the exact per-element
// factor e^{g_r - g_i} (never above 1) instead.  Padding rows of a partial chunk are identity
// steps with zero inputs and zero cotangents, so they contribute nothing.
#pragma once

#include "common.cuh"
#include "prefill_simt.cuh"
#include "profile.cuh"

namespace kda {

constexpr int kBwdCT = 32;        // key channels per tile
constexpr int kBwdLT = kBwdCT + 1; // padded tile row stride
constexpr int kBwdL64 = kChunk + 1;

// fp32 scratch of one (chunk, head), written by steps 1-3 and read by steps 3-4:
//   U [64 x dv] | dU [64 x dv] | dQg [64 x dk] | dW [64 x dk] | dKd [64 x dk] | dP [64 x 64] | dgam [dk]
__host__ __device__ inline size_t bwd_scr_floats(int dk, int dv)
{
    return 2 * (size_t)kChunk * dv + 3 * (size_t)kChunk * dk + (size_t)kChunk * kChunk + dk;
}

// 16-byte asynchronous global -> shared copies (zero-filled past src_bytes), in commit groups
__device__ __forceinline__ void bwd_cp16(float* dst, const void* src, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void bwd_cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bwd_cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// n floats (a multiple of 4), contiguous, by all threads
__device__ __forceinline__ void bwd_cp_block(float* dst, const float* src, int n)
{
    for (int e = 4 * threadIdx.x; e < n; e += 4 * kSimtThreads) bwd_cp16(dst + e, src + e, 16);
}

// chunk j of sequence n (global chunk index) -> first token and length
__device__ __forceinline__ void bwd_chunk_span(int j, int n, const int* __restrict__ off, long long s0, long long s1,
                                               long long& t0, int& L)
{
    t0 = s0 + (long long)(j - off[n]) * kChunk;
    L = (s1 - t0) < kChunk ? (int)(s1 - t0) : kChunk;
}

// ------------------------------------------------------------------------------------------------
// Step 1b: forward chain keeping each chunk's start state and its U (one CTA per (sequence, head,
// 32 state columns)).  Chunk c's W and Uv, and its Kd and gam, are copied in two cp.async groups
// while the previous chunk's other half computes.
// ------------------------------------------------------------------------------------------------
template <int DK>
__global__ void __launch_bounds__(kSimtThreads)
bwd_fwd_chain_kernel(const float* __restrict__ S0, const WsHeader* __restrict__ hdr, const int* __restrict__ off,
                     const int32_t* __restrict__ cu, int Tseq, int N, int H, int dv, const float* __restrict__ slots,
                     float* __restrict__ S_chunks, float* __restrict__ scr)
{
    extern __shared__ __align__(16) float smem[];
    const int n = blockIdx.x, h = blockIdx.y, v0 = blockIdx.z * kSimtNV, tid = threadIdx.x;
    if (hdr->bad) return;
    constexpr int NV = kSimtNV, TMD = DK / 16;
    float* sS = smem;                 // [DK][NV]
    float* sW = sS + DK * NV;         // [64][DK]
    float* sKd = sW + kChunk * DK;    // [64][DK]
    float* sUv = sKd + kChunk * DK;   // [64][NV]
    float* sU = sUv + kChunk * NV;    // [64][NV]
    float* sG = sU + kChunk * NV;     // [DK]
    const int tr = tid >> 4, tc = tid & 15;
    const size_t slot_f = simt_slot_floats(DK, dv), scr_f = bwd_scr_floats(DK, dv);
    const size_t sidx = ((size_t)n * H + h) * DK * dv;
    for (int e = tid; e < DK * NV; e += kSimtThreads)
        sS[e] = S0 ? S0[sidx + (size_t)(e / NV) * dv + v0 + (e % NV)] : 0.f;
    const int j0 = off[n], j1 = off[n + 1];
    auto issue_w = [&](int j) {  // W and the Uv columns of chunk j
        const float* slot = slots + ((size_t)j * H + h) * slot_f;
        bwd_cp_block(sW, slot, kChunk * DK);
        const float* gUv = slot + (size_t)kChunk * (3 * DK + kChunk);
        for (int e = 4 * tid; e < kChunk * NV; e += 4 * kSimtThreads)
            bwd_cp16(sUv + e, gUv + (size_t)(e / NV) * dv + v0 + (e % NV), 16);
        bwd_cp_commit();
    };
    auto issue_k = [&](int j) {  // Kd and gam of chunk j
        const float* slot = slots + ((size_t)j * H + h) * slot_f;
        bwd_cp_block(sKd, slot + 2 * (size_t)kChunk * DK, kChunk * DK);
        bwd_cp_block(sG, slot + (size_t)kChunk * (3 * DK + kChunk + dv), DK);
        bwd_cp_commit();
    };
    if (j0 < j1) {
        issue_w(j0);
        issue_k(j0);
    }
    for (int j = j0; j < j1; ++j) {
        const size_t u = (size_t)j * H + h;
        bwd_cp_wait<1>();  // W, Uv of chunk j landed (Kd may still be in flight)
        __syncthreads();
        float* dst = S_chunks + u * DK * dv + v0;
        for (int e = tid; e < DK * NV; e += kSimtThreads) dst[(size_t)(e / NV) * dv + (e % NV)] = sS[e];
        {  // U = Uv - W S
            float x[4][2] = {};
            mm_acc<4, 2>(x, sW, DK, 1, sS, NV, 1, DK, tr, tc);
            float* gU = scr + u * scr_f + v0;
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 2; ++b) {
                    const int r = tr + 16 * a, jj = tc + 16 * b;
                    const float uu = sUv[r * NV + jj] - x[a][b];
                    sU[r * NV + jj] = uu;
                    gU[(size_t)r * dv + jj] = uu;
                }
        }
        __syncthreads();
        if (j + 1 < j1) issue_w(j + 1);
        else bwd_cp_commit();  // keep one group per step
        bwd_cp_wait<1>();      // Kd, gam of chunk j
        __syncthreads();
        {  // S <- Diag(gam) S + Kd^T U
            float acc[TMD][2];
#pragma unroll
            for (int a = 0; a < TMD; ++a)
#pragma unroll
                for (int b = 0; b < 2; ++b) acc[a][b] = sG[tr + 16 * a] * sS[(tr + 16 * a) * NV + tc + 16 * b];
            mm_acc<TMD, 2>(acc, sKd, 1, DK, sU, NV, 1, kChunk, tr, tc);
            __syncthreads();  // every thread has read the old S
#pragma unroll
            for (int a = 0; a < TMD; ++a)
#pragma unroll
                for (int b = 0; b < 2; ++b) sS[(tr + 16 * a) * NV + tc + 16 * b] = acc[a][b];
        }
        __syncthreads();
        if (j + 1 < j1) issue_k(j + 1);
        else bwd_cp_commit();
    }
    bwd_cp_wait<0>();
}

// ------------------------------------------------------------------------------------------------
// Step 2a: the dO terms of the reverse chain, chunk-parallel (one CTA per (chunk, head)):
//     E = P^T dO  (64 x dv, into the unit's dU scratch),   F = Qg^T dO  (dk x dv)
// Neither depends on the carried cotangent, so the chain itself only does the D-dependent half.
// ------------------------------------------------------------------------------------------------
template <typename TIn, int DK, int DV>
__global__ void __launch_bounds__(kSimtThreads, 2)
bwd_do_terms_kernel(const TIn* __restrict__ dout, const WsHeader* __restrict__ hdr, const int* __restrict__ off,
                    const int32_t* __restrict__ cu, int Tseq, int N, int H, const float* __restrict__ slots,
                    float* __restrict__ scr, float* __restrict__ F_chunks)
{
    extern __shared__ __align__(16) float smem[];
    const int j = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    if (hdr->bad || j >= hdr->total_chunks) return;
    int n, L;
    long long t0;
    locate_chunk(j, off, cu, Tseq, N, n, t0, L);
    constexpr int L64 = kChunk + 1, LK = DK + 1, LV = DV + 1;
    float* sP = smem;                 // [64][65]
    float* sQ = sP + kChunk * L64;    // [64][DK+1]  Qg
    float* sO = sQ + kChunk * LK;     // [64][DV+1]  dO (rows past the end zero)
    const size_t u = (size_t)j * H + h;
    const float* slot = slots + u * simt_slot_floats(DK, DV);
    const float* gQ = slot + (size_t)kChunk * DK;
    const float* gP = slot + 3 * (size_t)kChunk * DK;
    for (int e = tid; e < kChunk * kChunk / 8; e += kSimtThreads) {
        float f[8];
        load8(gP + 8 * e, f);
#pragma unroll
        for (int m = 0; m < 8; ++m) sP[((8 * e) / kChunk) * L64 + (8 * e) % kChunk + m] = f[m];
    }
    for (int e = tid; e < kChunk * DK / 8; e += kSimtThreads) {
        float f[8];
        load8(gQ + 8 * e, f);
#pragma unroll
        for (int m = 0; m < 8; ++m) sQ[((8 * e) / DK) * LK + (8 * e) % DK + m] = f[m];
    }
    for (int e = tid; e < kChunk * DV / 8; e += kSimtThreads) {
        const int r = e / (DV / 8), jj = 8 * (e % (DV / 8));
        float f[8] = {};
        if (r < L) load8(dout + ((size_t)(t0 + r) * H + h) * DV + jj, f);
#pragma unroll
        for (int m = 0; m < 8; ++m) sO[r * LV + jj + m] = f[m];
    }
    __syncthreads();
    const int tr = tid >> 4, tc = tid & 15;
    {   // E = P^T dO
        float acc[4][DV / 16] = {};
        mm_acc<4, DV / 16>(acc, sP, 1, L64, sO, LV, 1, kChunk, tr, tc);
        float* gE = scr + u * bwd_scr_floats(DK, DV) + (size_t)kChunk * DV;
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < DV / 16; ++b) gE[(size_t)(tr + 16 * a) * DV + tc + 16 * b] = acc[a][b];
    }
    float* gF = F_chunks + u * DK * DV;
#pragma unroll 1
    for (int c0 = 0; c0 < DK; c0 += kChunk) {  // F = Qg^T dO, 64 rows at a time
        float acc[4][DV / 16] = {};
        mm_acc<4, DV / 16>(acc, sQ + c0, 1, LK, sO, LV, 1, kChunk, tr, tc);
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < DV / 16; ++b) gF[(size_t)(c0 + tr + 16 * a) * DV + tc + 16 * b] = acc[a][b];
    }
}

// ------------------------------------------------------------------------------------------------
// Step 2b: reverse chain of the state cotangent (chunks last to first):
//     dU = E + Kd D,   D <- Diag(gam) D + F - W^T dU
// {Kd, E} and {W, F, gam} of the next chunk are copied while the current chunk's other half runs.
// ------------------------------------------------------------------------------------------------
template <int DK>
__global__ void __launch_bounds__(kSimtThreads)
bwd_dstate_kernel(const float* __restrict__ dS_final, float* __restrict__ dS0, const WsHeader* __restrict__ hdr,
                  const int* __restrict__ off, int N, int H, int dv, const float* __restrict__ slots,
                  float* __restrict__ dSn_chunks, float* __restrict__ scr, const float* __restrict__ F_chunks)
{
    extern __shared__ __align__(16) float smem[];
    const int n = blockIdx.x, h = blockIdx.y, v0 = blockIdx.z * kSimtNV, tid = threadIdx.x;
    if (hdr->bad) return;
    constexpr int NV = kSimtNV, TMD = DK / 16;
    float* sD = smem;                 // [DK][NV]   D = dL/dS
    float* sW = sD + DK * NV;         // [64][DK]
    float* sKd = sW + kChunk * DK;    // [64][DK]
    float* sE = sKd + kChunk * DK;    // [64][NV]   E
    float* sU = sE + kChunk * NV;     // [64][NV]   dU
    float* sF = sU + kChunk * NV;     // [DK][NV]
    float* sG = sF + DK * NV;         // [DK]
    const int tr = tid >> 4, tc = tid & 15;
    const size_t slot_f = simt_slot_floats(DK, dv), scr_f = bwd_scr_floats(DK, dv);
    const size_t sidx = ((size_t)n * H + h) * DK * dv;
    for (int e = tid; e < DK * NV; e += kSimtThreads)
        sD[e] = dS_final ? dS_final[sidx + (size_t)(e / NV) * dv + v0 + (e % NV)] : 0.f;
    const int j0 = off[n], j1 = off[n + 1];
    auto issue_k = [&](int j) {  // Kd and the E columns of chunk j
        const size_t u = (size_t)j * H + h;
        bwd_cp_block(sKd, slots + u * slot_f + 2 * (size_t)kChunk * DK, kChunk * DK);
        const float* gE = scr + u * scr_f + (size_t)kChunk * dv + v0;
        for (int e = 4 * tid; e < kChunk * NV; e += 4 * kSimtThreads)
            bwd_cp16(sE + e, gE + (size_t)(e / NV) * dv + (e % NV), 16);
        bwd_cp_commit();
    };
    auto issue_w = [&](int j) {  // W, the F columns and gam of chunk j
        const size_t u = (size_t)j * H + h;
        const float* slot = slots + u * slot_f;
        bwd_cp_block(sW, slot, kChunk * DK);
        const float* gF = F_chunks + u * DK * dv + v0;
        for (int e = 4 * tid; e < DK * NV; e += 4 * kSimtThreads)
            bwd_cp16(sF + e, gF + (size_t)(e / NV) * dv + (e % NV), 16);
        bwd_cp_block(sG, slot + (size_t)kChunk * (3 * DK + kChunk + dv), DK);
        bwd_cp_commit();
    };
    if (j0 < j1) {
        issue_k(j1 - 1);
        issue_w(j1 - 1);
    }
    for (int j = j1 - 1; j >= j0; --j) {
        const size_t u = (size_t)j * H + h;
        bwd_cp_wait<1>();  // Kd, E of chunk j
        __syncthreads();   // ... visible to all, and the previous step is done with D
        float* dst = dSn_chunks + u * DK * dv + v0;
        for (int e = tid; e < DK * NV; e += kSimtThreads) dst[(size_t)(e / NV) * dv + (e % NV)] = sD[e];
        {  // dU = E + Kd D
            float x[4][2];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 2; ++b) x[a][b] = sE[(tr + 16 * a) * NV + tc + 16 * b];
            mm_acc<4, 2>(x, sKd, DK, 1, sD, NV, 1, DK, tr, tc);
            float* gdU = scr + u * scr_f + (size_t)kChunk * dv + v0;
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 2; ++b) {
                    const int i = tr + 16 * a, jj = tc + 16 * b;
                    sU[i * NV + jj] = x[a][b];
                    gdU[(size_t)i * dv + jj] = x[a][b];
                }
        }
        __syncthreads();  // dU complete; Kd and E are free for the next chunk
        if (j > j0) issue_k(j - 1);
        else bwd_cp_commit();
        bwd_cp_wait<1>();  // W, F, gam of chunk j
        __syncthreads();
        {  // D <- Diag(gam) D + F - W^T dU
            float acc[TMD][2], neg[TMD][2] = {};
#pragma unroll
            for (int a = 0; a < TMD; ++a)
#pragma unroll
                for (int b = 0; b < 2; ++b) {
                    const int c = tr + 16 * a, jj = tc + 16 * b;
                    acc[a][b] = fmaf(sG[c], sD[c * NV + jj], sF[c * NV + jj]);
                }
            mm_acc<TMD, 2>(neg, sW, 1, DK, sU, NV, 1, kChunk, tr, tc);
            __syncthreads();  // every thread has read the old D, W, F
#pragma unroll
            for (int a = 0; a < TMD; ++a)
#pragma unroll
                for (int b = 0; b < 2; ++b) sD[(tr + 16 * a) * NV + tc + 16 * b] = acc[a][b] - neg[a][b];
        }
        if (j > j0) issue_w(j - 1);
        else bwd_cp_commit();
    }
    bwd_cp_wait<0>();
    __syncthreads();
    if (dS0)
        for (int e = tid; e < DK * NV; e += kSimtThreads)
            dS0[sidx + (size_t)(e / NV) * dv + v0 + (e % NV)] = sD[e];
}

// ------------------------------------------------------------------------------------------------
// Step 3: per-chunk gradients on the state side
// ------------------------------------------------------------------------------------------------
template <typename TIn>
__global__ void __launch_bounds__(kSimtThreads)
bwd_state_side_kernel(const TIn* __restrict__ dout, const WsHeader* __restrict__ hdr, const int* __restrict__ off,
                      const int32_t* __restrict__ cu, int Tseq, int N, int H, int dk, int dv,
                      const float* __restrict__ S_chunks, const float* __restrict__ dSn_chunks,
                      float* __restrict__ scr)
{
    extern __shared__ __align__(16) float smem[];
    const int j = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    if (hdr->bad || j >= hdr->total_chunks) return;
    int n, L;
    long long t0;
    locate_chunk(j, off, cu, Tseq, N, n, t0, L);
    const int LDV = dv + 1;
    float* sO = smem;               // [64][dv+1]  dO
    float* sU = sO + kChunk * LDV;  // [64][dv+1]  U
    float* sdU = sU + kChunk * LDV; // [64][dv+1]  dU
    float* sS = sdU + kChunk * LDV; // [64][dv+1]  64 channels (rows) of S_c
    float* sD = sS + kChunk * LDV;  // [64][dv+1]  ... and of D_c

    const size_t u = (size_t)j * H + h;
    const float* Sc = S_chunks + u * dk * dv;
    const float* Dc = dSn_chunks + u * dk * dv;
    float* o = scr + u * bwd_scr_floats(dk, dv);
    const float* oU = o;
    const float* odU = oU + (size_t)kChunk * dv;
    float* oQg = o + 2 * (size_t)kChunk * dv;
    float* oW = oQg + (size_t)kChunk * dk;
    float* oKd = oW + (size_t)kChunk * dk;
    float* oP = oKd + (size_t)kChunk * dk;
    float* oGam = oP + (size_t)kChunk * kChunk;

    for (int e = tid; e < kChunk * dv / 8; e += kSimtThreads) {
        const int r = e / (dv / 8), jj = 8 * (e % (dv / 8));
        float fo[8] = {}, fu[8], fd[8];
        if (r < L) load8(dout + ((size_t)(t0 + r) * H + h) * dv + jj, fo);
        load8(oU + (size_t)r * dv + jj, fu);
        load8(odU + (size_t)r * dv + jj, fd);
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            sO[r * LDV + jj + m] = fo[m];
            sU[r * LDV + jj + m] = fu[m];
            sdU[r * LDV + jj + m] = fd[m];
        }
    }
    __syncthreads();
    const int tr = tid >> 4, tc = tid & 15;
    {  // dP = lower_incl(dO U^T)
        float acc[4][4] = {};
        mm_acc<4, 4>(acc, sO, LDV, 1, sU, 1, LDV, dv, tr, tc);
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int r = tr + 16 * a, i = tc + 16 * b;
                oP[r * kChunk + i] = (i <= r) ? acc[a][b] : 0.f;
            }
    }
    // dQg = dO S_c^T, dW = -dU S_c^T, dKd = U D_c^T, dgam = rowsum(D_c * S_c), 64 channels at a time
    for (int c0 = 0; c0 < dk; c0 += kChunk) {
        __syncthreads();
        for (int e = tid; e < kChunk * dv / 8; e += kSimtThreads) {
            const int cc = e / (dv / 8), jj = 8 * (e % (dv / 8));
            float fs[8], fd[8];
            load8(Sc + (size_t)(c0 + cc) * dv + jj, fs);
            load8(Dc + (size_t)(c0 + cc) * dv + jj, fd);
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                sS[cc * LDV + jj + m] = fs[m];
                sD[cc * LDV + jj + m] = fd[m];
            }
        }
        __syncthreads();
        float aq[4][4] = {}, aw[4][4] = {}, ak[4][4] = {};
#pragma unroll 2
        for (int jj = 0; jj < dv; ++jj) {
            float x0[4], x1[4], x2[4], bs[4], bd[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                x0[a] = sO[(tr + 16 * a) * LDV + jj];
                x1[a] = sdU[(tr + 16 * a) * LDV + jj];
                x2[a] = sU[(tr + 16 * a) * LDV + jj];
                bs[a] = sS[(tc + 16 * a) * LDV + jj];
                bd[a] = sD[(tc + 16 * a) * LDV + jj];
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    aq[a][b] = fmaf(x0[a], bs[b], aq[a][b]);
                    aw[a][b] = fmaf(x1[a], bs[b], aw[a][b]);
                    ak[a][b] = fmaf(x2[a], bd[b], ak[a][b]);
                }
        }
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const size_t oi = (size_t)(tr + 16 * a) * dk + c0 + tc + 16 * b;
                oQg[oi] = aq[a][b];
                oW[oi] = -aw[a][b];
                oKd[oi] = ak[a][b];
            }
        if (tid < kChunk) {
            float g = 0.f;
            for (int jj = 0; jj < dv; ++jj) g = fmaf(sD[tid * LDV + jj], sS[tid * LDV + jj], g);
            oGam[c0 + tid] = g;
        }
    }
}

// ------------------------------------------------------------------------------------------------
// Step 4: per-chunk gradients on the input side
// ------------------------------------------------------------------------------------------------
// cumulative gate of one 32-channel tile (rows past the chunk's end add nothing), its reference
// point and whether the factorised form is safe for it
// (tg must hold no live data: it is filled with the gates, then scanned in place)
__device__ __forceinline__ void bwd_gate_tile(const void* __restrict__ log_alpha, bool la16, long long t0, int L,
                                              int H, int h, int dk, int c0, float* tg, float* tref, int* s_wide)
{
    const int tid = threadIdx.x;
    for (int e = tid; e < kChunk * kBwdCT / 8; e += kSimtThreads) {
        const int r = e / (kBwdCT / 8), cc = 8 * (e % (kBwdCT / 8));
        float x[8] = {};
        if (r < L) {
            const size_t ia = ((size_t)(t0 + r) * H + h) * dk + c0 + cc;
            if (la16) load8(reinterpret_cast<const __nv_bfloat16*>(log_alpha) + ia, x);
            else load8(reinterpret_cast<const float*>(log_alpha) + ia, x);
        }
#pragma unroll
        for (int m = 0; m < 8; ++m) tg[r * kBwdLT + cc + m] = x[m];
    }
    __syncthreads();
    if (tid < kBwdCT) {
        float acc = 0.f, lo = 0.f, hi = 0.f;
        for (int r = 0; r < kChunk; ++r) {
            acc += tg[r * kBwdLT + tid];  // rows past the chunk's end hold 0
            tg[r * kBwdLT + tid] = acc;
            lo = fminf(lo, acc);
            hi = fmaxf(hi, acc);
        }
        tref[tid] = 0.5f * (lo + hi);
        if (!(hi - lo <= kFactorSpread)) atomicOr(s_wide, 1);
    }
}

template <typename TIn>
__device__ __forceinline__ void bwd_load_tile(const TIn* __restrict__ x, long long t0, int L, int H, int h, int d,
                                              int c0, float* t)
{
    for (int e = threadIdx.x; e < kChunk * kBwdCT / 8; e += kSimtThreads) {
        const int r = e / (kBwdCT / 8), cc = 8 * (e % (kBwdCT / 8));
        float f[8] = {};
        if (r < L) load8(x + ((size_t)(t0 + r) * H + h) * d + c0 + cc, f);
#pragma unroll
        for (int m = 0; m < 8; ++m) t[r * kBwdLT + cc + m] = f[m];
    }
}

__device__ __forceinline__ void bwd_load_scr_tile(const float* __restrict__ x, int ld, int c0, float* t)
{
    for (int e = threadIdx.x; e < kChunk * kBwdCT / 8; e += kSimtThreads) {
        const int r = e / (kBwdCT / 8), cc = 8 * (e % (kBwdCT / 8));
        float f[8];
        load8(x + (size_t)r * ld + c0 + cc, f);
#pragma unroll
        for (int m = 0; m < 8; ++m) t[r * kBwdLT + cc + m] = f[m];
    }
}

// Step 4a on the tensor cores (backward_tc.cuh; bf16 inputs, dk = dv = 128): At (strictly lower,
// factorised tiles only) and dT (lower, inclusive) into sAt and sM, with the exact products of the
// wide tiles added into accA at the thread's (tr, tc) elements; scratch = the kernel's shared memory
// below sb
__device__ void bwd_ut_y_dm_tc(const float* sN, float* sM, float* tiles);
__device__ void bwd_ut_dv_tc(const float* sN, const float* sb, const float* __restrict__ gdU, __nv_bfloat16* dv_out,
                             long long t0, int L, int H, int h, float* tiles);
__device__ void bwd_ut_step4a_tc(const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                                 const void* __restrict__ log_alpha, bool la16, long long t0, int L, int H, int Hk,
                                 int h, const float* __restrict__ gdW, const float* __restrict__ gdU, float* smem,
                                 float* sAt, float* sM, float (&accA)[4][4]);

// Step 4, first half (one CTA per (chunk, head)): At and dT over all channel and value tiles, the
// UT transform backwards (N, dbeta, dM -> dAt) and dV.  N and dAt go to the unit's scratch (over U
// and dU, both dead by then) for the second half.
template <typename TIn, bool TC>
__global__ void __launch_bounds__(kSimtThreads, 2)
bwd_ut_kernel(const TIn* __restrict__ k, const TIn* __restrict__ v, const void* __restrict__ log_alpha,
              const float* __restrict__ beta, const WsHeader* __restrict__ hdr, const int* __restrict__ off,
              const int32_t* __restrict__ cu, int Tseq, int N, int H, int Hk, unsigned pro, int dk, int dv,
              float* __restrict__ scr, TIn* __restrict__ dv_out, float* __restrict__ dbeta)
{
    extern __shared__ __align__(16) float smem[];
    const int j = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    if (hdr->bad || j >= hdr->total_chunks) return;
    int n, L;
    long long t0;
    locate_chunk(j, off, cu, Tseq, N, n, t0, L);
    const bool la16 = (pro & KDA_PROLOGUE_GATE_BF16) != 0;
    constexpr int M64 = kChunk * kBwdL64;
    constexpr int MT = kChunk * kBwdLT;
    constexpr int L64 = kBwdL64, LT = kBwdLT;
    float* sAt = smem;            // [64][65] At = strict_lower(Kf Kb^T) (without beta)
    float* sN = sAt + M64;        // [64][65] N = (I + Diag(beta) At)^{-1}
    float* sM = sN + M64;         // [64][65] dT -> dN -> dM -> dAt
    float* tk = sM + M64;         // tiles [64][33]: k (or v), g and four temporaries
    float* tg = tk + MT;
    float* tA = tg + MT;
    float* tB = tA + MT;
    float* tC = tB + MT;
    float* tD = tC + MT;
    float* sY = tA;               // [64][65] dN N^T, over tA..tB (the tiles are idle in the UT step)
    float* sb = tD + MT;          // [64] beta
    float* sdb = sb + kChunk;     // [64] dbeta
    float* tref = sdb + kChunk;   // [32]
    __shared__ int s_wide;

    const size_t u = (size_t)j * H + h;
    float* o = scr + u * bwd_scr_floats(dk, dv);
    const float* gdU = o + (size_t)kChunk * dv;
    const float* gdW = gdU + (size_t)kChunk * dv + (size_t)kChunk * dk;
    const int tr = tid >> 4, tc = tid & 15;

    for (int r = tid; r < kChunk; r += kSimtThreads) sb[r] = (r < L) ? beta[(size_t)(t0 + r) * H + h] : 0.f;

    // ---- step 4a: At and dT = dW Kt^T + dU V^T, accumulated in registers over tiles
    float accA[4][4] = {}, accT[4][4] = {};
    if constexpr (TC) {
        bwd_ut_step4a_tc(reinterpret_cast<const __nv_bfloat16*>(k), reinterpret_cast<const __nv_bfloat16*>(v),
                         log_alpha, la16, t0, L, H, Hk, h, gdW, gdU, smem, sAt, sM, accA);
    } else {
        for (int c0 = 0; c0 < dk; c0 += kBwdCT) {
            __syncthreads();
            if (tid == 0) s_wide = 0;
            __syncthreads();
            bwd_load_tile(k, t0, L, Hk, h / (H / Hk), dk, c0, tk);  // the q/k head of value head h
            bwd_gate_tile(log_alpha, la16, t0, L, H, h, dk, c0, tg, tref, &s_wide);
            bwd_load_scr_tile(gdW, dk, c0, tD);
            __syncthreads();
            const bool wide = s_wide != 0;
            for (int e = tid; e < kChunk * kBwdCT; e += kSimtThreads) {
                const int r = e / kBwdCT, cc = e % kBwdCT;
                const float g = tg[r * LT + cc], x = g - tref[cc], kv = tk[r * LT + cc];
                tA[r * LT + cc] = wide ? 0.f : kv * fast_exp(x);   // Kf
                tB[r * LT + cc] = wide ? 0.f : kv * fast_exp(-x);  // Kb
                tC[r * LT + cc] = kv * fast_exp(g);                // Kt
            }
            __syncthreads();
            if (!wide) {
                mm_acc<4, 4>(accA, tA, LT, 1, tB, 1, LT, kBwdCT, tr, tc);
            } else {
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int b = 0; b < 4; ++b) {
                        const int r = tr + 16 * a, i = tc + 16 * b;
                        if (i >= r) continue;
                        float x = 0.f;
                        for (int cc = 0; cc < kBwdCT; ++cc)
                            x = fmaf(tk[r * LT + cc] * tk[i * LT + cc], fast_exp(tg[r * LT + cc] - tg[i * LT + cc]), x);
                        accA[a][b] += x;
                    }
            }
            mm_acc<4, 4>(accT, tD, LT, 1, tC, 1, LT, kBwdCT, tr, tc);
        }
        for (int c0 = 0; c0 < dv; c0 += kBwdCT) {
            __syncthreads();
            bwd_load_tile(v, t0, L, H, h, dv, c0, tk);
            bwd_load_scr_tile(gdU, dv, c0, tD);
            __syncthreads();
            mm_acc<4, 4>(accT, tD, LT, 1, tk, 1, LT, kBwdCT, tr, tc);
        }
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int r = tr + 16 * a, i = tc + 16 * b;
                sAt[r * L64 + i] = (i < r) ? accA[a][b] : 0.f;
                sM[r * L64 + i] = (i <= r) ? accT[a][b] : 0.f;
            }
        __syncthreads();
    }

    // ---- step 4b: the UT transform backwards
    // N = (I + Diag(beta) At)^{-1}: Diag(beta) At copied into N, then inverted in place (the tiles
    // tC..tD are idle here and serve as scratch)
    for (int e = tid; e < kChunk * kChunk; e += kSimtThreads) {
        const int r = e / kChunk, i = e % kChunk;
        sN[r * L64 + i] = sb[r] * sAt[r * L64 + i];
    }
    __syncthreads();
    simt_unit_lower_inverse(sN, tC);
    if (tid < kChunk) {  // dbeta_i = sum_r dT[r][i] N[r][i]   (T = N Diag(beta))
        float x = 0.f;
        for (int r = tid; r < kChunk; ++r) x = fmaf(sM[r * L64 + tid], sN[r * L64 + tid], x);
        sdb[tid] = x;
    }
    __syncthreads();
    for (int e = tid; e < kChunk * kChunk; e += kSimtThreads) {  // dN = dT Diag(beta)
        const int r = e / kChunk, i = e % kChunk;
        sM[r * L64 + i] *= sb[i];
    }
    __syncthreads();
    if constexpr (TC) {
        bwd_ut_y_dm_tc(sN, sM, tk);
    } else {
        {  // Y = dN N^T
            float acc[4][4] = {};
            mm_acc<4, 4>(acc, sM, L64, 1, sN, 1, L64, kChunk, tr, tc);
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) sY[(tr + 16 * a) * L64 + tc + 16 * b] = acc[a][b];
        }
        __syncthreads();
        {  // dM = -N^T Y, strictly lower (dN is no longer needed: overwritten in place)
            float acc[4][4] = {};
            mm_acc<4, 4>(acc, sN, 1, L64, sY, L64, 1, kChunk, tr, tc);
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const int r = tr + 16 * a, i = tc + 16 * b;
                    sM[r * L64 + i] = (i < r) ? -acc[a][b] : 0.f;
                }
        }
        __syncthreads();
    }
    if (tid < kChunk) {  // dbeta_r += sum_i dM[r][i] At[r][i];  dAt = Diag(beta) dM
        const int r = tid;
        float x = 0.f;
        for (int i = 0; i < r; ++i) {
            x = fmaf(sM[r * L64 + i], sAt[r * L64 + i], x);
            sM[r * L64 + i] *= sb[r];
        }
        sdb[r] += x;
    }
    __syncthreads();
    for (int r = tid; r < L; r += kSimtThreads) dbeta[(size_t)(t0 + r) * H + h] = sdb[r];

    // ---- step 4d: dV = T^T dU = Diag(beta) N^T dU
    if constexpr (TC) {
        bwd_ut_dv_tc(sN, sb, gdU, reinterpret_cast<__nv_bfloat16*>(dv_out), t0, L, H, h, tk);
    } else {
        for (int c0 = 0; c0 < dv; c0 += kBwdCT) {
            __syncthreads();
            bwd_load_scr_tile(gdU, dv, c0, tD);
            __syncthreads();
            float acc[4][2] = {};
            mm_acc<4, 2>(acc, sN, 1, L64, tD, LT, 1, kChunk, tr, tc);
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 2; ++b) {
                    const int i = tr + 16 * a, cc = tc + 16 * b;
                    if (i < L) dv_out[((size_t)(t0 + i) * H + h) * dv + c0 + cc] = from_f32<TIn>(sb[i] * acc[a][b]);
                }
        }
    }
    // N and dAt out for the gate half (U and dU are no longer read)
    __syncthreads();
    float* gN = o;
    float* gdAt = o + (size_t)kChunk * dv;
    for (int e = tid; e < kChunk * kChunk; e += kSimtThreads) {
        const int r = e / kChunk, i = e % kChunk;
        gN[e] = sN[r * L64 + i];
        gdAt[e] = sM[r * L64 + i];
    }
}

// Step 4, second half (one CTA per (chunk, head, 32-channel tile)): dq, dk and dlog_alpha through
// the gated products P = Qf Kb^T, At = Kf Kb^T and the gating itself.
template <typename TIn>
__global__ void __launch_bounds__(kSimtThreads, 2)
bwd_gate_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k, const void* __restrict__ log_alpha,
                const float* __restrict__ beta, const WsHeader* __restrict__ hdr, const int* __restrict__ off,
                const int32_t* __restrict__ cu, int Tseq, int N, int H, int Hk, unsigned pro, int dk, int dv,
                const float* __restrict__ scr, TIn* __restrict__ dq, TIn* __restrict__ dk_out,
                float* __restrict__ dla, float* __restrict__ dq_acc, float* __restrict__ dk_acc)
{
    extern __shared__ __align__(16) float smem[];
    const int j = blockIdx.x, h = blockIdx.y, c0 = blockIdx.z * kBwdCT, tid = threadIdx.x;
    if (hdr->bad || j >= hdr->total_chunks) return;
    int n, L;
    long long t0;
    locate_chunk(j, off, cu, Tseq, N, n, t0, L);
    const bool la16 = (pro & KDA_PROLOGUE_GATE_BF16) != 0;
    constexpr int M64 = kChunk * kBwdL64;
    constexpr int MT = kChunk * kBwdLT;
    constexpr int L64 = kBwdL64, LT = kBwdLT;
    float* sN = smem;             // [64][65] N
    float* sM = sN + M64;         // [64][65] dAt
    float* sdP = sM + M64;        // [64][65] dP
    float* tk = sdP + M64;        // tiles [64][33]: k, q, g, dW and three temporaries
    float* tq = tk + MT;
    float* tg = tq + MT;
    float* tA = tg + MT;
    float* tB = tA + MT;
    float* tC = tB + MT;
    float* tD = tC + MT;
    float* sb = tD + MT;          // [64] beta
    float* tref = sb + kChunk;    // [32]
    __shared__ int s_wide;

    const size_t u = (size_t)j * H + h;
    const float* o = scr + u * bwd_scr_floats(dk, dv);
    const float* gN = o;
    const float* gdAt = o + (size_t)kChunk * dv;
    const float* gdQg = o + 2 * (size_t)kChunk * dv;
    const float* gdW = gdQg + (size_t)kChunk * dk;
    const float* gdKd = gdW + (size_t)kChunk * dk;
    const float* gdP = gdKd + (size_t)kChunk * dk;
    const float* gdGam = gdP + (size_t)kChunk * kChunk;
    const int tr = tid >> 4, tc = tid & 15;

    if (tid == 0) s_wide = 0;
    // this thread's dQg and dKd (rows tr + 16 a, channels c0 + tc + 16 b), in flight from the start
    float pq[4][2], pk[4][2];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            const size_t gi = (size_t)(tr + 16 * a) * dk + c0 + tc + 16 * b;
            pq[a][b] = gdQg[gi];
            pk[a][b] = gdKd[gi];
        }
    for (int r = tid; r < kChunk; r += kSimtThreads) sb[r] = (r < L) ? beta[(size_t)(t0 + r) * H + h] : 0.f;
    for (int e = tid; e < kChunk * kChunk / 8; e += kSimtThreads) {
        float fn[8], fa[8], fp[8];
        load8(gN + 8 * e, fn);
        load8(gdAt + 8 * e, fa);
        load8(gdP + 8 * e, fp);
        const int x = ((8 * e) / kChunk) * L64 + (8 * e) % kChunk;
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            sN[x + m] = fn[m];
            sM[x + m] = fa[m];
            sdP[x + m] = fp[m];
        }
    }
    bwd_load_tile(k, t0, L, Hk, h / (H / Hk), dk, c0, tk);  // the q/k head of value head h
    bwd_load_tile(q, t0, L, Hk, h / (H / Hk), dk, c0, tq);
    bwd_load_scr_tile(gdW, dk, c0, tD);
    __syncthreads();  // s_wide zeroed before the gate tile flags it
    bwd_gate_tile(log_alpha, la16, t0, L, H, h, dk, c0, tg, tref, &s_wide);
    __syncthreads();
    const bool wide = s_wide != 0;
    if (!wide)
        for (int e = tid; e < kChunk * kBwdCT; e += kSimtThreads) {
            const int r = e / kBwdCT, cc = e % kBwdCT;
            const float x = tg[r * LT + cc] - tref[cc];
            const float ex = fast_exp(x), emx = fast_exp(-x);
            tA[r * LT + cc] = tk[r * LT + cc] * ex;   // Kf
            tB[r * LT + cc] = tk[r * LT + cc] * emx;  // Kb
            tC[r * LT + cc] = tq[r * LT + cc] * ex;   // Qf
        }
    __syncthreads();
    // per (row r, channel): rowP = sum_i dP[r][i] k_i E(r,i), rowA = sum_i dAt[r][i] k_i E(r,i),
    // col = sum_a (dP[a][r] q_a + dAt[a][r] k_a) E(a,r), dKt = beta_r sum_a N[a][r] dW[a]
    float rowP[4][2] = {}, rowA[4][2] = {}, col[4][2] = {}, dkt[4][2] = {};
    if (!wide) {
        mm_acc<4, 2>(rowP, sdP, L64, 1, tB, LT, 1, kChunk, tr, tc);
        mm_acc<4, 2>(rowA, sM, L64, 1, tB, LT, 1, kChunk, tr, tc);
        mm_acc<4, 2>(col, sdP, 1, L64, tC, LT, 1, kChunk, tr, tc);
        mm_acc<4, 2>(col, sM, 1, L64, tA, LT, 1, kChunk, tr, tc);
    } else {
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                const int r = tr + 16 * a, cc = tc + 16 * b;
                const float gr = tg[r * LT + cc];
                for (int i = 0; i <= r; ++i) {
                    const float ke = tk[i * LT + cc] * fast_exp(gr - tg[i * LT + cc]);
                    rowP[a][b] = fmaf(sdP[r * L64 + i], ke, rowP[a][b]);
                    rowA[a][b] = fmaf(sM[r * L64 + i], ke, rowA[a][b]);
                }
                for (int i = r; i < kChunk; ++i)
                    col[a][b] = fmaf(fmaf(sdP[i * L64 + r], tq[i * LT + cc], sM[i * L64 + r] * tk[i * LT + cc]),
                                     fast_exp(tg[i * LT + cc] - gr), col[a][b]);
            }
    }
    mm_acc<4, 2>(dkt, sN, 1, L64, tD, LT, 1, kChunk, tr, tc);
    float accg[4][2], accl[4][2];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            const int r = tr + 16 * a, cc = tc + 16 * b;
            const float g = tg[r * LT + cc], gl = tg[(kChunk - 1) * LT + cc];
            if (!wide) {
                const float x = g - tref[cc];
                const float ex = fast_exp(x);
                rowP[a][b] *= ex;
                rowA[a][b] *= ex;
                col[a][b] *= fast_exp(-x);
            }
            const float kt = dkt[a][b] * sb[r];
            const float eg = fast_exp(g), egl = fast_exp(gl - g);
            const float qv = tq[r * LT + cc], kv = tk[r * LT + cc];
            const float dQg = pq[a][b], dKd = pk[a][b];
            const float vq = rowP[a][b] + dQg * eg;
            const float vk = rowA[a][b] + col[a][b] + kt * eg + dKd * egl;
            accg[a][b] = qv * rowP[a][b] + kv * rowA[a][b] - kv * col[a][b] + (dQg * qv + kt * kv) * eg -
                         dKd * kv * egl;
            accl[a][b] = dKd * kv * egl;  // chunk-end term of g_last, summed below
            if (r < L) {
                const size_t oi = ((size_t)(t0 + r) * H + h) * dk + c0 + cc;
                if (dq_acc) {  // grouped heads: per value head, summed over each group afterwards
                    dq_acc[oi] = vq;
                    dk_acc[oi] = vk;
                } else {
                    dq[oi] = from_f32<TIn>(vq);
                    dk_out[oi] = from_f32<TIn>(vk);
                }
            }
        }
    __syncthreads();  // every thread is done with Kf / Kb / Qf
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            const int r = tr + 16 * a, cc = tc + 16 * b;
            tA[r * LT + cc] = accl[a][b];
            tB[r * LT + cc] = accg[a][b];
        }
    __syncthreads();
    if (tid < kBwdCT) {  // g_last terms, then dlog_alpha = reverse cumulative sum of dg
        const int cc = tid;
        float s = 0.f;
        for (int r = 0; r < kChunk; ++r) s += tA[r * LT + cc];
        s += gdGam[c0 + cc] * fast_exp(tg[(kChunk - 1) * LT + cc]);
        float acc = s;
        for (int r = kChunk - 1; r >= 0; --r) {
            acc += tB[r * LT + cc];
            if (r < L) dla[((size_t)(t0 + r) * H + h) * dk + c0 + cc] = acc;
        }
    }
}

// ------------------------------------------------------------------------------------------------
// Input prologue, forwards and backwards.  Before the backward proper, the transforms of the
// forward's prologue are applied once into the workspace (q/k normalised and rounded to the input
// precision as the forward does, log alpha = log sigmoid(a), beta = sigmoid(b)), so every kernel
// below sees the inputs the forward used.  Afterwards the gradients are carried back to the raw
// inputs: dx = dx_hat / n - x (x . dx_hat) / n^3 for the norm (n = sqrt(sum x^2 + eps); the
// rounding to the input precision is passed straight through), da = dlog_alpha sigmoid(-a),
// db = dbeta sigmoid(b) (1 - sigmoid(b)).
// ------------------------------------------------------------------------------------------------
constexpr int kRowWarps = 8;  // one warp per (token, head) row, 8 rows per CTA

template <typename TIn>
__global__ void __launch_bounds__(32 * kRowWarps)
bwd_qk_norm_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k, TIn* __restrict__ qn, TIn* __restrict__ kn,
                   long long rows, int dk)
{
    const long long row = (long long)blockIdx.x * kRowWarps + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31, per = dk / 32;
    if (row >= rows) return;
    const TIn* src = blockIdx.y ? k : q;
    TIn* dst = blockIdx.y ? kn : qn;
    float x[4], ss = 0.f;
    for (int m = 0; m < per; ++m) {
        x[m] = to_f32(src[(size_t)row * dk + lane + 32 * m]);
        ss = fmaf(x[m], x[m], ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = rsqrtf(ss + kQkNormEps);
    for (int m = 0; m < per; ++m) dst[(size_t)row * dk + lane + 32 * m] = from_f32<TIn>(x[m] * inv);
}

// log alpha = log sigmoid(a) (gate logits, fp32 or bf16) and beta = sigmoid(b), into fp32 buffers
__global__ void __launch_bounds__(256)
bwd_gate_act_kernel(const void* __restrict__ la, bool la16, bool logits, float* __restrict__ la_out, long long n_la,
                    const float* __restrict__ beta, float* __restrict__ beta_out, long long n_beta)
{
    const long long e = (long long)blockIdx.x * 256 + threadIdx.x;
    if (la_out && e < n_la) {
        const float x = la16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(la)[e])
                             : reinterpret_cast<const float*>(la)[e];
        la_out[e] = logits ? log_sigmoid_f(x) : x;
    }
    if (beta_out && e < n_beta) beta_out[e] = sigmoid_f(beta[e]);
}

// dq, dk of the raw q/k heads: sum over the G value heads of each q/k head (value head h reads q/k
// head h / G; rows t*H + hk*G + g are consecutive in acc), then, with the norm, its chain rule
template <typename TIn>
__global__ void __launch_bounds__(32 * kRowWarps)
bwd_qk_grad_kernel(const float* __restrict__ acc, const TIn* __restrict__ x_raw, TIn* __restrict__ out, long long rows,
                   int G, int dk, bool l2norm)
{
    const long long row = (long long)blockIdx.x * kRowWarps + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31, per = dk / 32;
    if (row >= rows) return;
    float g[4], x[4], ss = 0.f, dot = 0.f;
    for (int m = 0; m < per; ++m) {
        const int c = lane + 32 * m;
        float s = 0.f;
        for (int j = 0; j < G; ++j) s += acc[((size_t)row * G + j) * dk + c];
        g[m] = s;
        x[m] = l2norm ? to_f32(x_raw[(size_t)row * dk + c]) : 0.f;
        ss = fmaf(x[m], x[m], ss);
        dot = fmaf(x[m], g[m], dot);
    }
    if (l2norm) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            ss += __shfl_xor_sync(0xffffffffu, ss, o);
            dot += __shfl_xor_sync(0xffffffffu, dot, o);
        }
        const float inv = rsqrtf(ss + kQkNormEps), inv3 = inv * inv * inv;
        for (int m = 0; m < per; ++m) g[m] = g[m] * inv - x[m] * dot * inv3;
    }
    for (int m = 0; m < per; ++m) out[(size_t)row * dk + lane + 32 * m] = from_f32<TIn>(g[m]);
}

// in place: dlog_alpha *= sigmoid(-a) for gate logits a; dbeta *= sigmoid(b) (1 - sigmoid(b))
__global__ void __launch_bounds__(256)
bwd_gate_act_grad_kernel(const void* __restrict__ la, bool la16, float* __restrict__ dla, long long n_la,
                         const float* __restrict__ beta, float* __restrict__ dbeta, long long n_beta)
{
    const long long e = (long long)blockIdx.x * 256 + threadIdx.x;
    if (dla && e < n_la) {
        const float a = la16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(la)[e])
                             : reinterpret_cast<const float*>(la)[e];
        dla[e] *= sigmoid_f(-a);
    }
    if (dbeta && e < n_beta) {
        const float sb = sigmoid_f(beta[e]);
        dbeta[e] *= sb * (1.f - sb);
    }
}

inline size_t bwd_fwd_chain_smem(int dk, int dv)
{
    (void)dv;
    return sizeof(float) * ((size_t)dk * kSimtNV + 2 * kChunk * dk + 2 * kChunk * kSimtNV + dk);
}
inline size_t bwd_dstate_smem(int dk, int dv)
{
    (void)dv;
    return sizeof(float) * ((size_t)2 * dk * kSimtNV + 2 * kChunk * dk + 2 * kChunk * kSimtNV + dk);
}
inline size_t bwd_do_terms_smem(int dk, int dv)
{
    return sizeof(float) * ((size_t)kChunk * (kChunk + 1) + kChunk * (dk + 1) + kChunk * (dv + 1));
}
inline size_t bwd_state_side_smem(int dk, int dv)
{
    (void)dk;
    return sizeof(float) * (size_t)5 * kChunk * (dv + 1);
}
inline size_t bwd_ut_smem()
{
    return sizeof(float) * ((size_t)3 * kChunk * kBwdL64 + 6 * kChunk * kBwdLT + 2 * kChunk + kBwdCT);
}
inline size_t bwd_gate_smem()
{
    return sizeof(float) * ((size_t)3 * kChunk * kBwdL64 + 7 * kChunk * kBwdLT + kChunk + kBwdCT);
}

// the tensor-core kernels of the backward (backward_tc.cuh): bf16 inputs with dk = dv = 128
bool bwd_state_side_tc_ok(bool bf16, int dk, int dv);
cudaError_t launch_bwd_state_side_tc(const void* dout, const WsHeader* hdr, const int* off, const int32_t* cu,
                                     int Tseq, int N, int H, int max_chunks, const float* S_chunks,
                                     const float* dSn_chunks, float* scr, cudaStream_t stream);
cudaError_t launch_bwd_do_terms_tc(const void* dout, const WsHeader* hdr, const int* off, const int32_t* cu,
                                   int Tseq, int N, int H, int max_chunks, const float* slots, float* scr,
                                   float* F_chunks, cudaStream_t stream);
cudaError_t launch_bwd_chains_tc(const float* S0, const float* dS_final, float* dS0, const WsHeader* hdr,
                                 const int* off, int N, int H, int max_chunks, const float* slots, float* S_chunks,
                                 float* dSn_chunks, float* scr, const float* F_chunks, bool reverse,
                                 cudaStream_t stream);
cudaError_t launch_bwd_gate_tc(const void* q, const void* k, const void* la, bool la16, const float* beta,
                               const WsHeader* hdr, const int* off, const int32_t* cu, int Tseq, int N, int H,
                               int Hk, int max_chunks, const float* scr, void* dq, void* dk_out, float* dla,
                               float* dq_acc, float* dk_acc, cudaStream_t stream);

template <typename TIn, int DK, int DV>
cudaError_t launch_bwd_chains(const float* S0, const void* dout, const float* dS_final, float* dS0,
                              const WsHeader* hdr, const int* off, const int32_t* cu, int Tseq, int N, int H,
                              int max_chunks, const float* slots, float* S_chunks, float* dSn_chunks, float* scr,
                              float* F_chunks, cudaStream_t stream)
{
    const size_t smF = bwd_fwd_chain_smem(DK, DV), smD = bwd_dstate_smem(DK, DV), smT = bwd_do_terms_smem(DK, DV);
    cudaError_t e = cudaFuncSetAttribute(bwd_fwd_chain_kernel<DK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smF);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(bwd_dstate_kernel<DK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smD);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(bwd_do_terms_kernel<TIn, DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smT);
    if (e != cudaSuccess) return e;
    const dim3 grid(N, H, DV / kSimtNV);
    const bool tc = bwd_state_side_tc_ok(sizeof(TIn) == 2, DK, DV);
    if (tc) {
        e = launch_bwd_chains_tc(S0, dS_final, dS0, hdr, off, N, H, max_chunks, slots, S_chunks, dSn_chunks, scr,
                                 F_chunks, false, stream);
        if (e != cudaSuccess) return e;
    } else {
        LaunchScope ls("bwd_fwd_states", stream);
        bwd_fwd_chain_kernel<DK><<<grid, kSimtThreads, smF, stream>>>(S0, hdr, off, cu, Tseq, N, H, DV, slots,
                                                                      S_chunks, scr);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (max_chunks > 0 && bwd_state_side_tc_ok(sizeof(TIn) == 2, DK, DV)) {
        e = launch_bwd_do_terms_tc(dout, hdr, off, cu, Tseq, N, H, max_chunks, slots, scr, F_chunks, stream);
        if (e != cudaSuccess) return e;
    } else if (max_chunks > 0) {
        LaunchScope ls("bwd_do_terms", stream);
        bwd_do_terms_kernel<TIn, DK, DV><<<dim3(max_chunks, H), kSimtThreads, smT, stream>>>(
            (const TIn*)dout, hdr, off, cu, Tseq, N, H, slots, scr, F_chunks);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (tc)
        return launch_bwd_chains_tc(S0, dS_final, dS0, hdr, off, N, H, max_chunks, slots, S_chunks, dSn_chunks, scr,
                                    F_chunks, true, stream);
    LaunchScope ls("bwd_dstate", stream);
    bwd_dstate_kernel<DK><<<grid, kSimtThreads, smD, stream>>>(dS_final, dS0, hdr, off, N, H, DV, slots, dSn_chunks,
                                                               scr, F_chunks);
    return cudaGetLastError();
}

// Steps 1-4.  Workspace regions (all per (chunk, head) of the forward's chunk table): the
// CUDA-core forward slots, chunk start states, chunk end cotangents and the per-chunk scratch.

template <typename TIn>
cudaError_t launch_simt_backward(const void* q, const void* k, const void* v, const void* la, const float* beta,
                                 const float* S0, const void* dout, const float* dS_final, void* dq, void* dk_out,
                                 void* dv_out, float* dla, float* dbeta, float* dS0, const WsHeader* hdr,
                                 const int* off, const int32_t* cu, int Tseq, int N, int H, int Hk, unsigned pro_raw,
                                 int dk, int dv, int max_chunks, long long Ttot, float* slots, float* S_chunks,
                                 float* dSn_chunks, float* scr, float* F_chunks, float* dq_acc, float* dk_acc,
                                 void* qn, void* kn, float* la_act, float* beta_act, cudaStream_t stream)
{
    // the raw inputs, and the transformed ones every kernel below reads (the input prologue)
    const void *q_raw = q, *k_raw = k, *la_raw = la;
    const float* beta_raw = beta;
    const bool grouped = Hk != H, l2norm = (pro_raw & KDA_PROLOGUE_L2NORM_QK) != 0;
    unsigned pro = pro_raw & KDA_PROLOGUE_GATE_BF16;
    cudaError_t e0 = cudaSuccess;
    if (l2norm && Ttot > 0) {
        LaunchScope ls("bwd_qk_norm", stream);
        const long long rows = Ttot * Hk, blocks = (rows + kRowWarps - 1) / kRowWarps;
        if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
        bwd_qk_norm_kernel<TIn><<<dim3((unsigned)blocks, 2), 32 * kRowWarps, 0, stream>>>(
            (const TIn*)q, (const TIn*)k, (TIn*)qn, (TIn*)kn, rows, dk);
        if ((e0 = cudaGetLastError()) != cudaSuccess) return e0;
        q = qn;
        k = kn;
    }
    if ((pro_raw & (KDA_PROLOGUE_GATE_LOGITS | KDA_PROLOGUE_BETA_LOGITS)) && Ttot > 0) {
        LaunchScope ls("bwd_gate_act", stream);
        const bool gl = (pro_raw & KDA_PROLOGUE_GATE_LOGITS) != 0, bl = (pro_raw & KDA_PROLOGUE_BETA_LOGITS) != 0;
        const long long n_la = Ttot * H * dk, blocks = (n_la + 255) / 256;
        if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
        bwd_gate_act_kernel<<<(unsigned)blocks, 256, 0, stream>>>(la, (pro_raw & KDA_PROLOGUE_GATE_BF16) != 0, true,
                                                                   gl ? la_act : nullptr, n_la, beta,
                                                                   bl ? beta_act : nullptr, Ttot * H);
        if ((e0 = cudaGetLastError()) != cudaSuccess) return e0;
        if (gl) {
            la = la_act;
            pro = 0;  // the activated gates are fp32
        }
        if (bl) beta = beta_act;
    }
    const size_t smA = simt_intra_smem(dk, dv), smS = bwd_state_side_smem(dk, dv), smU = bwd_ut_smem(),
                 smG = bwd_gate_smem();
    const bool tcr = bwd_state_side_tc_ok(sizeof(TIn) == 2, dk, dv);  // the recompute's products on tcgen05
    auto* kintra = tcr ? simt_intra_kernel<TIn, sizeof(TIn) == 2> : simt_intra_kernel<TIn, false>;
    const size_t smAk = smA + (tcr ? 1024 : 0);
    cudaError_t e = cudaFuncSetAttribute(kintra, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smAk);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(bwd_state_side_kernel<TIn>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smS);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(bwd_ut_kernel<TIn, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smU);
    if (e == cudaSuccess && sizeof(TIn) == 2)
        e = cudaFuncSetAttribute(bwd_ut_kernel<TIn, sizeof(TIn) == 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smU);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(bwd_gate_kernel<TIn>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smG);
    if (e != cudaSuccess) return e;
    const TIn *qq = (const TIn*)q, *kk = (const TIn*)k, *vv = (const TIn*)v;
    if (max_chunks > 0) {
        LaunchScope ls(tcr ? "bwd_fwd_intra_tc" : "bwd_fwd_intra", stream);
        kintra<<<dim3(max_chunks, H), kSimtThreads, smAk, stream>>>(
            qq, kk, vv, la, beta, hdr, off, cu, Tseq, N, H, Hk, pro & KDA_PROLOGUE_GATE_BF16, dk, dv, slots);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
#define KDA_BWD_CHAINS(DKV, DVV)                                                                              \
    launch_bwd_chains<TIn, DKV, DVV>(S0, dout, dS_final, dS0, hdr, off, cu, Tseq, N, H, max_chunks, slots, S_chunks, \
                                     dSn_chunks, scr, F_chunks, stream)
    e = (dk == 128) ? (dv == 128 ? KDA_BWD_CHAINS(128, 128) : KDA_BWD_CHAINS(128, 64))
                    : (dv == 128 ? KDA_BWD_CHAINS(64, 128) : KDA_BWD_CHAINS(64, 64));
#undef KDA_BWD_CHAINS
    if (e != cudaSuccess) return e;
    if (max_chunks > 0) {
        if (bwd_state_side_tc_ok(sizeof(TIn) == 2, dk, dv)) {
            e = launch_bwd_state_side_tc(dout, hdr, off, cu, Tseq, N, H, max_chunks, S_chunks, dSn_chunks, scr,
                                         stream);
            if (e != cudaSuccess) return e;
        } else {
            LaunchScope ls("bwd_state_side", stream);
            bwd_state_side_kernel<TIn><<<dim3(max_chunks, H), kSimtThreads, smS, stream>>>(
                (const TIn*)dout, hdr, off, cu, Tseq, N, H, dk, dv, S_chunks, dSn_chunks, scr);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
        {
            const bool tc = bwd_state_side_tc_ok(sizeof(TIn) == 2, dk, dv);
            LaunchScope ls(tc ? "bwd_ut_tc" : "bwd_ut", stream);
            auto* kut = tc ? bwd_ut_kernel<TIn, sizeof(TIn) == 2> : bwd_ut_kernel<TIn, false>;
            kut<<<dim3(max_chunks, H), kSimtThreads, smU, stream>>>(
                kk, vv, la, beta, hdr, off, cu, Tseq, N, H, Hk, pro & KDA_PROLOGUE_GATE_BF16, dk, dv, scr,
                (TIn*)dv_out, dbeta);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
        if (bwd_state_side_tc_ok(sizeof(TIn) == 2, dk, dv)) {
            e = launch_bwd_gate_tc(qq, kk, la, (pro & KDA_PROLOGUE_GATE_BF16) != 0, beta, hdr, off, cu, Tseq, N, H,
                                   Hk, max_chunks, scr, dq, dk_out, dla, (grouped || l2norm) ? dq_acc : nullptr,
                                   (grouped || l2norm) ? dk_acc : nullptr, stream);
            if (e != cudaSuccess) return e;
        } else {
            LaunchScope ls("bwd_gate", stream);
            bwd_gate_kernel<TIn><<<dim3(max_chunks, H, dk / kBwdCT), kSimtThreads, smG, stream>>>(
                qq, kk, la, beta, hdr, off, cu, Tseq, N, H, Hk, pro & KDA_PROLOGUE_GATE_BF16, dk, dv, scr, (TIn*)dq,
                (TIn*)dk_out, dla, (grouped || l2norm) ? dq_acc : nullptr, (grouped || l2norm) ? dk_acc : nullptr);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
        if (grouped || l2norm) {  // per-value-head dq, dk -> the raw q/k heads
            LaunchScope ls("bwd_qk_grad", stream);
            const long long rows = Ttot * Hk, blocks = (rows + kRowWarps - 1) / kRowWarps;
            if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
            bwd_qk_grad_kernel<TIn><<<(unsigned)blocks, 32 * kRowWarps, 0, stream>>>(
                dq_acc, (const TIn*)q_raw, (TIn*)dq, rows, H / Hk, dk, l2norm);
            bwd_qk_grad_kernel<TIn><<<(unsigned)blocks, 32 * kRowWarps, 0, stream>>>(
                dk_acc, (const TIn*)k_raw, (TIn*)dk_out, rows, H / Hk, dk, l2norm);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
        if (pro_raw & (KDA_PROLOGUE_GATE_LOGITS | KDA_PROLOGUE_BETA_LOGITS)) {
            LaunchScope ls("bwd_gate_act_grad", stream);
            const long long n_la = Ttot * H * dk, n_b = Ttot * H;
            const long long blocks = (n_la + 255) / 256;
            if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
            const bool gl = (pro_raw & KDA_PROLOGUE_GATE_LOGITS) != 0, bl = (pro_raw & KDA_PROLOGUE_BETA_LOGITS) != 0;
            bwd_gate_act_grad_kernel<<<(unsigned)blocks, 256, 0, stream>>>(
                la_raw, (pro_raw & KDA_PROLOGUE_GATE_BF16) != 0, gl ? dla : nullptr, n_la, beta_raw,
                bl ? dbeta : nullptr, n_b);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
    }
    return cudaSuccess;
}

}  // namespace kda
