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
//      state S_c (the only forward intermediate kept).
//   2. reverse chain over chunks (one CTA per (sequence, head, 32 state columns), chunks last to
//      first), carrying D = dL/dS_next:
//          dU = P^T dO + Kd D
//          D <- Diag(gam) D + Qg^T dO - W^T dU          (= dL/dS at the chunk start)
//      storing every chunk's end cotangent D_c; D after the first chunk is dL/dS0.
//   3. chunk-parallel, state side (one CTA per (chunk, head)): with S_c and D_c,
//          U = Uv - W S_c,  dU = P^T dO + Kd D_c,
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
// Steps 3 and 4 work on 32-channel tiles of the key dimension, so each CTA holds a few 64 x 64
// matrices plus tiles.  The per-channel factors use the same centre-of-range reference as the
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

// fp32 scratch of one (chunk, head) between steps 3 and 4:
//   dU [64 x dv] | dQg [64 x dk] | dW [64 x dk] | dKd [64 x dk] | dP [64 x 64] | dgam [dk]
__host__ __device__ inline size_t bwd_scr_floats(int dk, int dv)
{
    return (size_t)kChunk * dv + 3 * (size_t)kChunk * dk + (size_t)kChunk * kChunk + dk;
}

// ------------------------------------------------------------------------------------------------
// Step 2: reverse chain of the state cotangent
// ------------------------------------------------------------------------------------------------
template <typename TIn>
__global__ void __launch_bounds__(kSimtThreads)
bwd_dstate_kernel(const TIn* __restrict__ dout, const float* __restrict__ dS_final, float* __restrict__ dS0,
                  const WsHeader* __restrict__ hdr, const int* __restrict__ off, const int32_t* __restrict__ cu,
                  int Tseq, int N, int H, int dk, int dv, const float* __restrict__ slots,
                  float* __restrict__ dSn_chunks)
{
    extern __shared__ __align__(16) float smem[];
    const int n = blockIdx.x, h = blockIdx.y, v0 = blockIdx.z * kSimtNV, tid = threadIdx.x;
    if (hdr->bad) return;
    constexpr int NV = kSimtNV;
    float* sD = smem;                       // [dk][NV]   D = dL/dS
    float* sW = sD + dk * NV;               // [64][dk]
    float* sQ = sW + kChunk * dk;           // [64][dk]
    float* sKd = sQ + kChunk * dk;          // [64][dk]
    float* sP = sKd + kChunk * dk;          // [64][64]
    float* sO = sP + kChunk * kChunk;       // [64][NV]   dO
    float* sU = sO + kChunk * NV;           // [64][NV]   dU
    float* sG = sU + kChunk * NV;           // [dk]

    const size_t sidx = ((size_t)n * H + h) * dk * dv;
    for (int e = tid; e < dk * NV; e += kSimtThreads) {
        const int c = e / NV, jj = e % NV;
        sD[e] = dS_final ? dS_final[sidx + (size_t)c * dv + v0 + jj] : 0.f;
    }
    long long s0, s1;
    seq_bounds(n, cu, Tseq, s0, s1);
    const size_t slot_f = simt_slot_floats(dk, dv);
    for (int j = off[n + 1] - 1; j >= off[n]; --j) {
        const long long t0 = s0 + (long long)(j - off[n]) * kChunk;
        const int L = (s1 - t0) < kChunk ? (int)(s1 - t0) : kChunk;
        const float* slot = slots + ((size_t)j * H + h) * slot_f;
        const float* gW = slot;
        const float* gQ = gW + (size_t)kChunk * dk;
        const float* gKd = gQ + (size_t)kChunk * dk;
        const float* gP = gKd + (size_t)kChunk * dk;
        const float* gGam = gP + (size_t)kChunk * kChunk + (size_t)kChunk * dv;
        __syncthreads();  // the previous chunk is done with the staged operands and D is final
        float* dst = dSn_chunks + ((size_t)j * H + h) * dk * dv + v0;
        for (int e = tid; e < dk * NV; e += kSimtThreads) dst[(size_t)(e / NV) * dv + (e % NV)] = sD[e];
        for (int e = tid; e < kChunk * dk; e += kSimtThreads) { sW[e] = gW[e]; sQ[e] = gQ[e]; sKd[e] = gKd[e]; }
        for (int e = tid; e < kChunk * kChunk; e += kSimtThreads) sP[e] = gP[e];
        for (int e = tid; e < kChunk * NV; e += kSimtThreads) {
            const int r = e / NV, jj = e % NV;
            sO[e] = (r < L) ? to_f32(dout[((size_t)(t0 + r) * H + h) * dv + v0 + jj]) : 0.f;
        }
        for (int e = tid; e < dk; e += kSimtThreads) sG[e] = gGam[e];
        __syncthreads();
        // dU = P^T dO + Kd D
        for (int e = tid; e < kChunk * NV; e += kSimtThreads) {
            const int i = e / NV, jj = e % NV;
            float x = 0.f;
            for (int r = i; r < kChunk; ++r) x = fmaf(sP[r * kChunk + i], sO[r * NV + jj], x);
            for (int c = 0; c < dk; ++c) x = fmaf(sKd[i * dk + c], sD[c * NV + jj], x);
            sU[e] = x;
        }
        __syncthreads();
        // D <- Diag(gam) D + Qg^T dO - W^T dU   (each thread rewrites only its own element)
        for (int e = tid; e < dk * NV; e += kSimtThreads) {
            const int c = e / NV, jj = e % NV;
            float s = sG[c] * sD[e];
            for (int r = 0; r < kChunk; ++r) {
                s = fmaf(sQ[r * dk + c], sO[r * NV + jj], s);
                s = fmaf(-sW[r * dk + c], sU[r * NV + jj], s);
            }
            sD[e] = s;
        }
    }
    __syncthreads();
    if (dS0)
        for (int e = tid; e < dk * NV; e += kSimtThreads)
            dS0[sidx + (size_t)(e / NV) * dv + v0 + (e % NV)] = sD[e];
}

// ------------------------------------------------------------------------------------------------
// Step 3: per-chunk gradients on the state side
// ------------------------------------------------------------------------------------------------
template <typename TIn>
__global__ void __launch_bounds__(kSimtThreads)
bwd_state_side_kernel(const TIn* __restrict__ dout, const WsHeader* __restrict__ hdr, const int* __restrict__ off,
                      const int32_t* __restrict__ cu, int Tseq, int N, int H, int dk, int dv,
                      const float* __restrict__ slots, const float* __restrict__ S_chunks,
                      const float* __restrict__ dSn_chunks, float* __restrict__ scr)
{
    extern __shared__ __align__(16) float smem[];
    const int j = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    if (hdr->bad || j >= hdr->total_chunks) return;
    int n, L;
    long long t0;
    locate_chunk(j, off, cu, Tseq, N, n, t0, L);
    const int LDV = dv + 1;
    float* sU = smem;                       // [64][dv+1]  U
    float* sdU = sU + kChunk * LDV;         // [64][dv+1]  dU
    float* sO = sdU + kChunk * LDV;         // [64][dv+1]  dO
    float* sP = sO + kChunk * LDV;          // [64][64]
    float* sS = sP + kChunk * kChunk;       // [32][dv+1]  tile of S_c
    float* sD = sS + kBwdCT * LDV;          // [32][dv+1]  tile of D_c
    float* sWt = sD + kBwdCT * LDV;         // [64][33]    tile of W
    float* sKt = sWt + kChunk * kBwdLT;     // [64][33]    tile of Kd

    const size_t u = (size_t)j * H + h;
    const float* slot = slots + u * simt_slot_floats(dk, dv);
    const float* gW = slot;
    const float* gKd = gW + 2 * (size_t)kChunk * dk;
    const float* gP = gKd + (size_t)kChunk * dk;
    const float* gUv = gP + (size_t)kChunk * kChunk;
    const float* Sc = S_chunks + u * dk * dv;
    const float* Dc = dSn_chunks + u * dk * dv;
    float* o = scr + u * bwd_scr_floats(dk, dv);
    float* oU = o;                                  // dU
    float* oQg = oU + (size_t)kChunk * dv;          // dQg
    float* oW = oQg + (size_t)kChunk * dk;          // dW
    float* oKd = oW + (size_t)kChunk * dk;          // dKd
    float* oP = oKd + (size_t)kChunk * dk;          // dP
    float* oGam = oP + (size_t)kChunk * kChunk;     // dgam

    for (int e = tid; e < kChunk * dv; e += kSimtThreads) {
        const int r = e / dv, jj = e % dv;
        sU[r * LDV + jj] = gUv[e];
        sO[r * LDV + jj] = (r < L) ? to_f32(dout[((size_t)(t0 + r) * H + h) * dv + jj]) : 0.f;
    }
    for (int e = tid; e < kChunk * kChunk; e += kSimtThreads) sP[e] = gP[e];
    __syncthreads();
    for (int e = tid; e < kChunk * dv; e += kSimtThreads) {  // dU = P^T dO
        const int i = e / dv, jj = e % dv;
        float x = 0.f;
        for (int r = i; r < kChunk; ++r) x = fmaf(sP[r * kChunk + i], sO[r * LDV + jj], x);
        sdU[i * LDV + jj] = x;
    }
    // U -= W S_c and dU += Kd D_c, one 32-row tile of the state at a time
    for (int c0 = 0; c0 < dk; c0 += kBwdCT) {
        __syncthreads();
        for (int e = tid; e < kBwdCT * dv; e += kSimtThreads) {
            const int cc = e / dv, jj = e % dv;
            sS[cc * LDV + jj] = Sc[(size_t)(c0 + cc) * dv + jj];
            sD[cc * LDV + jj] = Dc[(size_t)(c0 + cc) * dv + jj];
        }
        for (int e = tid; e < kChunk * kBwdCT; e += kSimtThreads) {
            const int r = e / kBwdCT, cc = e % kBwdCT;
            sWt[r * kBwdLT + cc] = gW[(size_t)r * dk + c0 + cc];
            sKt[r * kBwdLT + cc] = gKd[(size_t)r * dk + c0 + cc];
        }
        __syncthreads();
        for (int e = tid; e < kChunk * dv; e += kSimtThreads) {
            const int r = e / dv, jj = e % dv;
            float x = sU[r * LDV + jj], y = sdU[r * LDV + jj];
#pragma unroll 8
            for (int cc = 0; cc < kBwdCT; ++cc) {
                x = fmaf(-sWt[r * kBwdLT + cc], sS[cc * LDV + jj], x);
                y = fmaf(sKt[r * kBwdLT + cc], sD[cc * LDV + jj], y);
            }
            sU[r * LDV + jj] = x;
            sdU[r * LDV + jj] = y;
        }
    }
    __syncthreads();
    for (int e = tid; e < kChunk * kChunk; e += kSimtThreads) {  // dP = lower_incl(dO U^T)
        const int r = e / kChunk, i = e % kChunk;
        float x = 0.f;
        if (i <= r)
            for (int jj = 0; jj < dv; ++jj) x = fmaf(sO[r * LDV + jj], sU[i * LDV + jj], x);
        oP[e] = x;
    }
    for (int e = tid; e < kChunk * dv; e += kSimtThreads) oU[e] = sdU[(e / dv) * LDV + (e % dv)];
    // dQg = dO S_c^T, dW = -dU S_c^T, dKd = U D_c^T, dgam = rowsum(D_c * S_c), per tile of channels
    for (int c0 = 0; c0 < dk; c0 += kBwdCT) {
        __syncthreads();
        for (int e = tid; e < kBwdCT * dv; e += kSimtThreads) {
            const int cc = e / dv, jj = e % dv;
            sS[cc * LDV + jj] = Sc[(size_t)(c0 + cc) * dv + jj];
            sD[cc * LDV + jj] = Dc[(size_t)(c0 + cc) * dv + jj];
        }
        __syncthreads();
        for (int e = tid; e < kChunk * kBwdCT; e += kSimtThreads) {
            const int r = e / kBwdCT, cc = e % kBwdCT;
            float a = 0.f, b = 0.f, c = 0.f;
            for (int jj = 0; jj < dv; ++jj) {
                const float s = sS[cc * LDV + jj];
                a = fmaf(sO[r * LDV + jj], s, a);
                b = fmaf(sdU[r * LDV + jj], s, b);
                c = fmaf(sU[r * LDV + jj], sD[cc * LDV + jj], c);
            }
            oQg[(size_t)r * dk + c0 + cc] = a;
            oW[(size_t)r * dk + c0 + cc] = -b;
            oKd[(size_t)r * dk + c0 + cc] = c;
        }
        if (tid < kBwdCT) {
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
__device__ __forceinline__ void bwd_gate_tile(const void* __restrict__ log_alpha, bool la16, long long t0, int L,
                                              int H, int h, int dk, int c0, float* tg, float* tref, int* s_wide)
{
    const int tid = threadIdx.x;
    if (tid < kBwdCT) {
        float acc = 0.f, lo = 0.f, hi = 0.f;
        for (int r = 0; r < kChunk; ++r) {
            if (r < L) {
                const size_t ia = ((size_t)(t0 + r) * H + h) * dk + c0 + tid;
                acc += la16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(log_alpha)[ia])
                            : reinterpret_cast<const float*>(log_alpha)[ia];
            }
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
    for (int e = threadIdx.x; e < kChunk * kBwdCT; e += kSimtThreads) {
        const int r = e / kBwdCT, cc = e % kBwdCT;
        t[r * kBwdLT + cc] = (r < L) ? to_f32(x[((size_t)(t0 + r) * H + h) * d + c0 + cc]) : 0.f;
    }
}

template <typename TIn>
__global__ void __launch_bounds__(kSimtThreads)
bwd_input_side_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k, const TIn* __restrict__ v,
                      const void* __restrict__ log_alpha, const float* __restrict__ beta,
                      const WsHeader* __restrict__ hdr, const int* __restrict__ off, const int32_t* __restrict__ cu,
                      int Tseq, int N, int H, unsigned pro, int dk, int dv, const float* __restrict__ scr,
                      TIn* __restrict__ dq, TIn* __restrict__ dk_out, TIn* __restrict__ dv_out,
                      float* __restrict__ dla, float* __restrict__ dbeta)
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
    float* sAt = smem;            // [64][65] At = strict_lower(Kf Kb^T) (without beta)
    float* sN = sAt + M64;        // [64][65] N = (I + Diag(beta) At)^{-1}
    float* sM = sN + M64;         // [64][65] dT -> dN -> dM -> dAt
    float* sY = sM + M64;         // [64][65] dN N^T
    float* sdP = sY + M64;        // [64][65] dP
    float* tk = sdP + M64;        // tiles [64][33]: k, q, g and four temporaries
    float* tq = tk + MT;
    float* tg = tq + MT;
    float* tA = tg + MT;
    float* tB = tA + MT;
    float* tC = tB + MT;
    float* tD = tC + MT;
    float* sb = tD + MT;          // [64] beta
    float* sdb = sb + kChunk;     // [64] dbeta
    float* tref = sdb + kChunk;   // [32]
    __shared__ int s_wide;

    const size_t u = (size_t)j * H + h;
    const float* o = scr + u * bwd_scr_floats(dk, dv);
    const float* gdU = o;
    const float* gdQg = gdU + (size_t)kChunk * dv;
    const float* gdW = gdQg + (size_t)kChunk * dk;
    const float* gdKd = gdW + (size_t)kChunk * dk;
    const float* gdP = gdKd + (size_t)kChunk * dk;
    const float* gdGam = gdP + (size_t)kChunk * kChunk;

    for (int r = tid; r < kChunk; r += kSimtThreads) {
        sb[r] = (r < L) ? beta[(size_t)(t0 + r) * H + h] : 0.f;
        sdb[r] = 0.f;
    }
    for (int e = tid; e < kChunk * kChunk; e += kSimtThreads) {
        const int r = e / kChunk, i = e % kChunk;
        sAt[r * kBwdL64 + i] = 0.f;
        sM[r * kBwdL64 + i] = 0.f;
        sdP[r * kBwdL64 + i] = gdP[e];
    }

    // ---- step 4a: At and dT = dW Kt^T, accumulated over channel tiles; dT += dU V^T over value tiles
    for (int c0 = 0; c0 < dk; c0 += kBwdCT) {
        __syncthreads();
        if (tid == 0) s_wide = 0;
        __syncthreads();
        bwd_load_tile(k, t0, L, H, h, dk, c0, tk);
        bwd_gate_tile(log_alpha, la16, t0, L, H, h, dk, c0, tg, tref, &s_wide);
        for (int e = tid; e < kChunk * kBwdCT; e += kSimtThreads) {
            const int r = e / kBwdCT, cc = e % kBwdCT;
            tD[r * kBwdLT + cc] = gdW[(size_t)r * dk + c0 + cc];
        }
        __syncthreads();
        const bool wide = s_wide != 0;
        for (int e = tid; e < kChunk * kBwdCT; e += kSimtThreads) {
            const int r = e / kBwdCT, cc = e % kBwdCT;
            const float g = tg[r * kBwdLT + cc], x = g - tref[cc], kv = tk[r * kBwdLT + cc];
            tA[r * kBwdLT + cc] = kv * expf(x);   // Kf
            tB[r * kBwdLT + cc] = kv * expf(-x);  // Kb
            tC[r * kBwdLT + cc] = kv * expf(g);   // Kt
        }
        __syncthreads();
        for (int e = tid; e < kChunk * kChunk; e += kSimtThreads) {
            const int r = e / kChunk, i = e % kChunk;
            if (i > r) continue;
            float a = 0.f, t = 0.f;
            if (!wide) {
                for (int cc = 0; cc < kBwdCT; ++cc) a = fmaf(tA[r * kBwdLT + cc], tB[i * kBwdLT + cc], a);
            } else {
                for (int cc = 0; cc < kBwdCT; ++cc)
                    a = fmaf(tk[r * kBwdLT + cc] * tk[i * kBwdLT + cc],
                             expf(tg[r * kBwdLT + cc] - tg[i * kBwdLT + cc]), a);
            }
            for (int cc = 0; cc < kBwdCT; ++cc) t = fmaf(tD[r * kBwdLT + cc], tC[i * kBwdLT + cc], t);
            if (i < r) sAt[r * kBwdL64 + i] += a;
            sM[r * kBwdL64 + i] += t;
        }
    }
    for (int c0 = 0; c0 < dv; c0 += kBwdCT) {
        __syncthreads();
        bwd_load_tile(v, t0, L, H, h, dv, c0, tk);
        for (int e = tid; e < kChunk * kBwdCT; e += kSimtThreads) {
            const int r = e / kBwdCT, cc = e % kBwdCT;
            tD[r * kBwdLT + cc] = gdU[(size_t)r * dv + c0 + cc];
        }
        __syncthreads();
        for (int e = tid; e < kChunk * kChunk; e += kSimtThreads) {
            const int r = e / kChunk, i = e % kChunk;
            if (i > r) continue;
            float t = 0.f;
            for (int cc = 0; cc < kBwdCT; ++cc) t = fmaf(tD[r * kBwdLT + cc], tk[i * kBwdLT + cc], t);
            sM[r * kBwdL64 + i] += t;
        }
    }
    __syncthreads();

    // ---- step 4b: the UT transform backwards
    if (tid < kChunk) {  // N = (I + Diag(beta) At)^{-1}, column tid, rows in order
        const int jj = tid;
        for (int r = 0; r < kChunk; ++r) {
            float t = (r == jj) ? 1.f : 0.f;
            for (int i = jj; i < r; ++i) t = fmaf(-sb[r] * sAt[r * kBwdL64 + i], sN[i * kBwdL64 + jj], t);
            sN[r * kBwdL64 + jj] = (jj <= r) ? t : 0.f;
        }
    }
    __syncthreads();
    if (tid < kChunk) {  // dbeta_i += sum_r dT[r][i] N[r][i]   (T = N Diag(beta))
        float x = 0.f;
        for (int r = tid; r < kChunk; ++r) x = fmaf(sM[r * kBwdL64 + tid], sN[r * kBwdL64 + tid], x);
        sdb[tid] = x;
    }
    __syncthreads();
    for (int e = tid; e < kChunk * kChunk; e += kSimtThreads) {  // dN = dT Diag(beta)
        const int r = e / kChunk, i = e % kChunk;
        sM[r * kBwdL64 + i] = (i <= r) ? sM[r * kBwdL64 + i] * sb[i] : 0.f;
    }
    __syncthreads();
    for (int e = tid; e < kChunk * kChunk; e += kSimtThreads) {  // Y = dN N^T
        const int r = e / kChunk, b = e % kChunk;
        const int amax = r < b ? r : b;
        float x = 0.f;
        for (int a = 0; a <= amax; ++a) x = fmaf(sM[r * kBwdL64 + a], sN[b * kBwdL64 + a], x);
        sY[r * kBwdL64 + b] = x;
    }
    __syncthreads();
    for (int e = tid; e < kChunk * kChunk; e += kSimtThreads) {  // dM = -N^T Y, strictly lower
        const int r = e / kChunk, i = e % kChunk;
        float x = 0.f;
        if (i < r)
            for (int a = r; a < kChunk; ++a) x = fmaf(sN[a * kBwdL64 + r], sY[a * kBwdL64 + i], x);
        sM[r * kBwdL64 + i] = -x;
    }
    __syncthreads();
    if (tid < kChunk) {  // dbeta_r += sum_i dM[r][i] At[r][i];  dAt = Diag(beta) dM
        const int r = tid;
        float x = 0.f;
        for (int i = 0; i < r; ++i) {
            x = fmaf(sM[r * kBwdL64 + i], sAt[r * kBwdL64 + i], x);
            sM[r * kBwdL64 + i] *= sb[r];
        }
        sdb[r] += x;
    }
    __syncthreads();
    for (int r = tid; r < L; r += kSimtThreads) dbeta[(size_t)(t0 + r) * H + h] = sdb[r];

    // ---- step 4c: dq, dk, dlog_alpha per channel tile
    for (int c0 = 0; c0 < dk; c0 += kBwdCT) {
        __syncthreads();
        if (tid == 0) s_wide = 0;
        __syncthreads();
        bwd_load_tile(k, t0, L, H, h, dk, c0, tk);
        bwd_load_tile(q, t0, L, H, h, dk, c0, tq);
        bwd_gate_tile(log_alpha, la16, t0, L, H, h, dk, c0, tg, tref, &s_wide);
        for (int e = tid; e < kChunk * kBwdCT; e += kSimtThreads) {
            const int r = e / kBwdCT, cc = e % kBwdCT;
            tD[r * kBwdLT + cc] = gdW[(size_t)r * dk + c0 + cc];
        }
        __syncthreads();
        const bool wide = s_wide != 0;
        if (!wide)
            for (int e = tid; e < kChunk * kBwdCT; e += kSimtThreads) {
                const int r = e / kBwdCT, cc = e % kBwdCT;
                const float x = tg[r * kBwdLT + cc] - tref[cc];
                const float ex = expf(x), emx = expf(-x);
                tA[r * kBwdLT + cc] = tk[r * kBwdLT + cc] * ex;   // Kf
                tB[r * kBwdLT + cc] = tk[r * kBwdLT + cc] * emx;  // Kb
                tC[r * kBwdLT + cc] = tq[r * kBwdLT + cc] * ex;   // Qf
            }
        __syncthreads();
        // per (row, channel): RowP = sum_i dP[r][i] k_i E(r,i), RowA = sum_i dAt[r][i] k_i E(r,i),
        // Col = sum_r (dP[r][i] q_r + dAt[r][i] k_r) E(r,i), dKt = sum_r T[r][i] dW[r]
        constexpr int PT = (kChunk * kBwdCT) / kSimtThreads;  // elements per thread
        float accq[PT], acck[PT], accg[PT], accl[PT];
#pragma unroll
        for (int m = 0; m < PT; ++m) {
            const int e = tid + m * kSimtThreads;
            const int r = e / kBwdCT, cc = e % kBwdCT;
            float rowP = 0.f, rowA = 0.f, col = 0.f, dkt = 0.f;
            if (!wide) {
                float sp = 0.f, sa = 0.f;
                for (int i = 0; i <= r; ++i) {
                    const float kb = tB[i * kBwdLT + cc];
                    sp = fmaf(sdP[r * kBwdL64 + i], kb, sp);
                    sa = fmaf(sM[r * kBwdL64 + i], kb, sa);  // dAt is zero on the diagonal
                }
                float sc = 0.f;
                for (int a = r; a < kChunk; ++a)
                    sc = fmaf(sdP[a * kBwdL64 + r], tC[a * kBwdLT + cc], fmaf(sM[a * kBwdL64 + r], tA[a * kBwdLT + cc], sc));
                const float x = tg[r * kBwdLT + cc] - tref[cc];
                rowP = sp * expf(x);
                rowA = sa * expf(x);
                col = sc * expf(-x);
            } else {
                const float gr = tg[r * kBwdLT + cc];
                for (int i = 0; i <= r; ++i) {
                    const float ke = tk[i * kBwdLT + cc] * expf(gr - tg[i * kBwdLT + cc]);
                    rowP = fmaf(sdP[r * kBwdL64 + i], ke, rowP);
                    rowA = fmaf(sM[r * kBwdL64 + i], ke, rowA);
                }
                for (int a = r; a < kChunk; ++a) {
                    const float ea = expf(tg[a * kBwdLT + cc] - gr);
                    col = fmaf(fmaf(sdP[a * kBwdL64 + r], tq[a * kBwdLT + cc],
                                    sM[a * kBwdL64 + r] * tk[a * kBwdLT + cc]), ea, col);
                }
            }
            for (int a = r; a < kChunk; ++a) dkt = fmaf(sN[a * kBwdL64 + r], tD[a * kBwdLT + cc], dkt);
            dkt *= sb[r];
            const float g = tg[r * kBwdLT + cc], gl = tg[(kChunk - 1) * kBwdLT + cc];
            const float eg = expf(g), egl = expf(gl - g);
            const float qv = tq[r * kBwdLT + cc], kv = tk[r * kBwdLT + cc];
            const float dQg = gdQg[(size_t)r * dk + c0 + cc], dKd = gdKd[(size_t)r * dk + c0 + cc];
            accq[m] = rowP + dQg * eg;
            acck[m] = rowA + col + dkt * eg + dKd * egl;
            accg[m] = qv * rowP + kv * rowA - kv * col + (dQg * qv + dkt * kv) * eg - dKd * kv * egl;
            accl[m] = dKd * kv * egl;  // chunk-end term of g_last, summed below
        }
        __syncthreads();  // every thread is done with Kf / Kb / Qf
#pragma unroll
        for (int m = 0; m < PT; ++m) {
            const int e = tid + m * kSimtThreads;
            const int r = e / kBwdCT, cc = e % kBwdCT;
            tA[r * kBwdLT + cc] = accl[m];
            tB[r * kBwdLT + cc] = accg[m];
            if (r < L) {
                const size_t oi = ((size_t)(t0 + r) * H + h) * dk + c0 + cc;
                dq[oi] = from_f32<TIn>(accq[m]);
                dk_out[oi] = from_f32<TIn>(acck[m]);
            }
        }
        __syncthreads();
        if (tid < kBwdCT) {  // g_last terms, then dlog_alpha = reverse cumulative sum of dg
            const int cc = tid;
            float s = 0.f;
            for (int r = 0; r < kChunk; ++r) s += tA[r * kBwdLT + cc];
            const float gl = tg[(kChunk - 1) * kBwdLT + cc];
            s += gdGam[c0 + cc] * expf(gl);
            float acc = s;
            for (int r = kChunk - 1; r >= 0; --r) {
                acc += tB[r * kBwdLT + cc];
                if (r < L) dla[((size_t)(t0 + r) * H + h) * dk + c0 + cc] = acc;
            }
        }
    }

    // ---- step 4d: dV = T^T dU = Diag(beta) N^T dU
    for (int c0 = 0; c0 < dv; c0 += kBwdCT) {
        __syncthreads();
        for (int e = tid; e < kChunk * kBwdCT; e += kSimtThreads) {
            const int r = e / kBwdCT, cc = e % kBwdCT;
            tD[r * kBwdLT + cc] = gdU[(size_t)r * dv + c0 + cc];
        }
        __syncthreads();
        for (int e = tid; e < kChunk * kBwdCT; e += kSimtThreads) {
            const int i = e / kBwdCT, cc = e % kBwdCT;
            if (i >= L) continue;
            float x = 0.f;
            for (int a = i; a < kChunk; ++a) x = fmaf(sN[a * kBwdL64 + i], tD[a * kBwdLT + cc], x);
            dv_out[((size_t)(t0 + i) * H + h) * dv + c0 + cc] = from_f32<TIn>(sb[i] * x);
        }
    }
}

inline size_t bwd_dstate_smem(int dk, int dv) { return simt_inter_smem(dk, dv); }
inline size_t bwd_state_side_smem(int dk, int dv)
{
    (void)dk;
    return sizeof(float) * ((size_t)3 * kChunk * (dv + 1) + kChunk * kChunk + 2 * kBwdCT * (dv + 1) +
                            2 * kChunk * kBwdLT);
}
inline size_t bwd_input_side_smem()
{
    return sizeof(float) * ((size_t)5 * kChunk * kBwdL64 + 7 * kChunk * kBwdLT + 2 * kChunk + kBwdCT);
}

// Steps 1-4.  Workspace regions (all per (chunk, head) of the forward's chunk table): the
// CUDA-core forward slots, chunk start states, chunk end cotangents and the step-3 scratch.
template <typename TIn>
cudaError_t launch_simt_backward(const void* q, const void* k, const void* v, const void* la, const float* beta,
                                 const float* S0, const void* dout, const float* dS_final, void* dq, void* dk_out,
                                 void* dv_out, float* dla, float* dbeta, float* dS0, const WsHeader* hdr,
                                 const int* off, const int32_t* cu, int Tseq, int N, int H, unsigned pro, int dk,
                                 int dv, int max_chunks, float* slots, float* S_chunks, float* dSn_chunks, float* scr,
                                 cudaStream_t stream)
{
    const size_t smA = simt_intra_smem(dk, dv), smB = simt_inter_smem(dk, dv), smD = bwd_dstate_smem(dk, dv),
                 smS = bwd_state_side_smem(dk, dv), smI = bwd_input_side_smem();
    cudaError_t e = cudaFuncSetAttribute(simt_intra_kernel<TIn>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smA);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(simt_inter_kernel<TIn>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smB);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(bwd_dstate_kernel<TIn>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smD);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(bwd_state_side_kernel<TIn>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smS);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(bwd_input_side_kernel<TIn>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smI);
    if (e != cudaSuccess) return e;
    const TIn *qq = (const TIn*)q, *kk = (const TIn*)k, *vv = (const TIn*)v;
    if (max_chunks > 0) {
        LaunchScope ls("bwd_fwd_intra", stream);
        simt_intra_kernel<TIn><<<dim3(max_chunks, H), kSimtThreads, smA, stream>>>(
            qq, kk, vv, la, beta, hdr, off, cu, Tseq, N, H, H, pro & KDA_PROLOGUE_GATE_BF16, dk, dv, slots);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        LaunchScope ls("bwd_fwd_states", stream);
        simt_inter_kernel<TIn><<<dim3(N, H, dv / kSimtNV), kSimtThreads, smB, stream>>>(
            S0, nullptr, (TIn*)nullptr, hdr, off, cu, Tseq, N, H, dk, dv, slots, S_chunks);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        LaunchScope ls("bwd_dstate", stream);
        bwd_dstate_kernel<TIn><<<dim3(N, H, dv / kSimtNV), kSimtThreads, smD, stream>>>(
            (const TIn*)dout, dS_final, dS0, hdr, off, cu, Tseq, N, H, dk, dv, slots, dSn_chunks);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (max_chunks > 0) {
        {
            LaunchScope ls("bwd_state_side", stream);
            bwd_state_side_kernel<TIn><<<dim3(max_chunks, H), kSimtThreads, smS, stream>>>(
                (const TIn*)dout, hdr, off, cu, Tseq, N, H, dk, dv, slots, S_chunks, dSn_chunks, scr);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
        LaunchScope ls("bwd_input_side", stream);
        bwd_input_side_kernel<TIn><<<dim3(max_chunks, H), kSimtThreads, smI, stream>>>(
            qq, kk, vv, la, beta, hdr, off, cu, Tseq, N, H, pro & KDA_PROLOGUE_GATE_BF16, dk, dv, scr, (TIn*)dq,
            (TIn*)dk_out, (TIn*)dv_out, dla, dbeta);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace kda
