// prefill_simt.cuh -- chunked KDA prefill on CUDA cores in fp32 (any dt, dk/dv in {64, 128}).
//
// This is the full-precision path: it serves the fp32 dtype (where a tensor-core path would round
// operands to tf32 or bf16) and shapes the tensor-core path does not cover.  It follows the chunk
// form of the recurrence (chunk-parallel inside a chunk, recurrent between chunks, WY
// representation, UT transform -- "Kimi Linear" explainer, section "硬件效率的深度优化"):
//
//   phase A (one CTA per (chunk, head), all chunks in parallel):
//     g_r   = sum_{i<=r} log_alpha_i                       (restarted every chunk)
//     A     = strict_lower( beta_r sum_c k_rc k_ic e^{g_rc - g_ic} )
//     P     = lower_incl(  sum_c q_rc k_ic e^{g_rc - g_ic} )
//     T     = (I + A)^{-1} diag(beta)                      (forward substitution)
//     W     = T (k * e^{g}),  Uv = T v,  Qg = q * e^{g},  Kd = k * e^{g_last - g},  gam = e^{g_last}
//   phase B (one CTA per (sequence, head, 32-column slice of S), chunks in order):
//     U = Uv - W S;   O = Qg S + P U;   S <- Diag(gam) S + Kd^T U
//
// The intra-chunk products factor e^{g_r - g_i} = e^{g_r - ref} e^{ref - g_i} around the centre of
// each channel's in-chunk gate range, which keeps every factor within e^{+-80}; a chunk in which
// some channel decays by more than e^-160 uses the exact per-element factor instead (never larger
// than 1), so no gate value can overflow.  Padding rows of a partial chunk are identity steps
// (k = q = v = 0, log_alpha = 0, beta = 0).
#pragma once

#include "common.cuh"
#include "profile.cuh"

namespace kda {

constexpr int kSimtThreads = 256;

// e^x from the hardware's base-2 exponential (ex2.approx, relative error ~2^-22 over the normal
// range; results below 2^-126 flush to zero, which every use here can take: the factors are decays
// or the factorised halves of one, and the products they enter are sums of such terms)
__device__ __forceinline__ float fast_exp(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x * 1.4426950408889634f));
    return y;
}
constexpr int kSimtNV = 32;  // state columns per phase-B CTA

// fp32 workspace slot of one (chunk, head): W | Qg | Kd [64 x dk] | P [64 x 64] | Uv [64 x dv] | gam [dk]
__host__ __device__ inline size_t simt_slot_floats(int dk, int dv)
{
    return (size_t)kChunk * (3 * dk + kChunk + dv) + dk;
}

// Largest spread of the in-chunk cumulative gate (per channel) for which the factorised products
// below stay finite in fp32: each factor is e^{+-x} with |x| <= kFactorSpread / 2 <= 80.
constexpr float kFactorSpread = 160.f;

// 8 consecutive values widened to fp32 (the address is 16-byte aligned)
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* f)
{
    const uint4 r = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&r);
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const float2 t = __bfloat1622float2(b[m]);
        f[2 * m] = t.x;
        f[2 * m + 1] = t.y;
    }
}
__device__ __forceinline__ void load8(const float* p, float* f)
{
    const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

// acc[i][j] += sum_k A(tr + 16 i, k) B(k, tc + 16 j), with A(r, k) = A[r * ars + k * aks] and
// B(k, c) = B[k * bks + c * bcs] in shared memory (thread tid: tr = tid / 16, tc = tid % 16).  Each
// thread owns a TM x TN block of interleaved rows and columns, so the B reads of a warp fall on
// distinct banks whenever bcs = 1 or bcs is odd, and its A reads on two addresses.
template <int TM, int TN>
__device__ __forceinline__ void mm_acc(float (&acc)[TM][TN], const float* A, int ars, int aks, const float* B,
                                       int bks, int bcs, int K, int tr, int tc)
{
#pragma unroll 4
    for (int k = 0; k < K; ++k) {
        float a[TM], b[TN];
#pragma unroll
        for (int i = 0; i < TM; ++i) a[i] = A[(tr + 16 * i) * ars + k * aks];
#pragma unroll
        for (int j = 0; j < TN; ++j) b[j] = B[k * bks + (tc + 16 * j) * bcs];
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
            for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
}

// out[r][c] = sum_{i} T[r][i] X[i][c] for the 64 x D block (T in [64][65], X in [64][D+1]), written
// to a dense global [64][D] array
template <int D>
__device__ __forceinline__ void simt_apply_t(const float* sT, const float* X, float* __restrict__ out, int tr, int tc)
{
    float acc[4][D / 16] = {};
    mm_acc<4, D / 16>(acc, sT, kChunk + 1, 1, X, D + 1, 1, kChunk, tr, tc);
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < D / 16; ++b) out[(size_t)(tr + 16 * a) * D + tc + 16 * b] = acc[a][b];
}

// X = (I + A)^{-1} for a strictly lower-triangular 64 x 64 A (row stride 65), in place of A, by
// block doubling on all 256 threads: the four 16 x 16 diagonal blocks by forward substitution, then
// X_10 = -X_11 A_10 X_00 for the 16-row pairs and again for the two 32-row halves.  Above the
// diagonal the result holds zeros (A does), on it ones.  Y: scratch of 32 x 33 floats.
__device__ __forceinline__ void simt_unit_lower_inverse(float* __restrict__ A, float* __restrict__ Y)
{
    constexpr int LS = kChunk + 1;
    const int tid = threadIdx.x;
    {   // diagonal blocks: thread (block b, column jj), rows in order
        const int b = 16 * (tid >> 4), jj = tid & 15;
        float x[16];
        if (tid < 64) {
            float sacc[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) sacc[r] = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                x[i] = (i == jj) ? 1.f : ((i < jj) ? 0.f : -sacc[i]);
#pragma unroll
                for (int r = i + 1; r < 16; ++r) sacc[r] = fmaf(A[(b + r) * LS + b + i], x[i], sacc[r]);
            }
        }
        __syncthreads();
        if (tid < 64)
#pragma unroll
            for (int r = 0; r < 16; ++r) A[(b + r) * LS + b + jj] = x[r];
        __syncthreads();
    }
    {   // blocks (1,0) and (3,2) of 16: thread (pair p, row rr, columns cc, cc + 1)
        const int p = tid >> 7, rr = (tid >> 3) & 15, cc = (tid & 7) * 2;
        const int bi = 16 * (2 * p + 1), bj = 16 * (2 * p);
        float y0 = 0.f, y1 = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float a = A[(bi + rr) * LS + bj + k];
            y0 = fmaf(a, A[(bj + k) * LS + bj + cc], y0);
            y1 = fmaf(a, A[(bj + k) * LS + bj + cc + 1], y1);
        }
        Y[(p * 16 + rr) * 33 + cc] = y0;
        Y[(p * 16 + rr) * 33 + cc + 1] = y1;
        __syncthreads();
        float x0 = 0.f, x1 = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float xi = A[(bi + rr) * LS + bi + k];
            x0 = fmaf(xi, Y[(p * 16 + k) * 33 + cc], x0);
            x1 = fmaf(xi, Y[(p * 16 + k) * 33 + cc + 1], x1);
        }
        A[(bi + rr) * LS + bj + cc] = -x0;
        A[(bi + rr) * LS + bj + cc + 1] = -x1;
        __syncthreads();
    }
    {   // rows 32..63 x columns 0..31: thread (row rr, columns cc .. cc + 3)
        const int rr = tid >> 3, cc = (tid & 7) * 4;
        float y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
        for (int k = 0; k < 32; ++k) {
            const float a = A[(32 + rr) * LS + k];
#pragma unroll
            for (int m = 0; m < 4; ++m) y[m] = fmaf(a, A[k * LS + cc + m], y[m]);
        }
#pragma unroll
        for (int m = 0; m < 4; ++m) Y[rr * 33 + cc + m] = y[m];
        __syncthreads();
        float x[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
        for (int k = 0; k < 32; ++k) {
            const float xi = A[(32 + rr) * LS + 32 + k];
#pragma unroll
            for (int m = 0; m < 4; ++m) x[m] = fmaf(xi, Y[k * 33 + cc + m], x[m]);
        }
#pragma unroll
        for (int m = 0; m < 4; ++m) A[(32 + rr) * LS + cc + m] = -x[m];
        __syncthreads();
    }
}

// the product stages on the tensor cores, for the backward's recompute with bf16 inputs and
// dk = dv = 128 (defined with the backward's tensor-core kernels)
__device__ void simt_intra_tc_setup(uint32_t* s_tm, uint64_t* s_mb);
__device__ void simt_intra_ap_tc(const float* sk, const float* sq, const float* sg, float* sv, const float* sb,
                                 float* sA, float* sP, uint32_t* s_tm, uint64_t* s_mb);
__device__ void simt_intra_wuv_tc(const float* sT, const float* sKt, const __nv_bfloat16* __restrict__ v, long long t0,
                                  int L, int H, int h, float* tiles, float* __restrict__ gW, float* __restrict__ gUv,
                                  uint32_t* s_tm, uint64_t* s_mb, uint32_t phase);

template <typename TIn, bool TC = false>
__global__ void __launch_bounds__(kSimtThreads)
simt_intra_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k, const TIn* __restrict__ v,
                  const void* __restrict__ log_alpha, const float* __restrict__ beta, const WsHeader* __restrict__ hdr,
                  const int* __restrict__ off, const int32_t* __restrict__ cu, int Tseq, int N, int H, int Hk,
                  unsigned pro, int dk, int dv, float* __restrict__ slots)
{
    extern __shared__ __align__(16) float smem[];
    const int j = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    if (hdr->bad || j >= hdr->total_chunks) return;
    int n, L;
    long long t0;
    locate_chunk(j, off, cu, Tseq, N, n, t0, L);

    // row strides padded by one float, so column walks of a warp hit distinct banks
    const int LK = dk + 1, LV = dv + 1;
    constexpr int L64 = kChunk + 1;
    // (TC: the layout starts on a 1024-byte boundary, so that the operand tiles placed over its dead
    // regions are aligned and stay inside them; the launch adds 1024 bytes)
    float* sk = TC ? reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(smem) + 1023) & ~uintptr_t(1023))
                   : smem;                  // [64][dk+1]  k, later k e^{g - ref}
    float* sq = sk + kChunk * LK;           // [64][dk+1]  q, later q e^{g - ref}
    float* sg = sq + kChunk * LK;           // [64][dk+1]  g, later k e^{ref - g}
    float* sv = sg + kChunk * LK;           // [64][dv+1]
    float* sKt = sv + kChunk * LV;          // [64][dk+1]  k e^{g}
    float* sA = sKt + kChunk * LK;          // [64][65]
    float* sP = sA + kChunk * L64;          // [64][65]
    float* sT = sP + kChunk * L64;          // [64][65]
    float* sb = sT + kChunk * L64;          // [64]
    float* sref = sb + kChunk;              // [dk]
    __shared__ int s_wide;
    __shared__ uint32_t s_tm;  // TC: TMEM base address and the MMA-completion barrier
    __shared__ uint64_t s_mb;
    const int tr = tid >> 4, tc = tid & 15;

    if (tid == 0) s_wide = 0;
    if constexpr (TC) simt_intra_tc_setup(&s_tm, &s_mb);
    // 8 consecutive channels per thread and step (16- or 32-byte loads); rows past the end read as 0
    for (int e = tid; e < kChunk * dk / 8; e += kSimtThreads) {
        const int r = e / (dk / 8), c = 8 * (e % (dk / 8));
        float kv[8] = {}, qv[8] = {}, lv[8] = {};
        if (r < L) {
            const size_t gi = ((size_t)(t0 + r) * H + h) * dk + c;
            const size_t qi = ((size_t)(t0 + r) * Hk + h / (H / Hk)) * dk + c;  // q/k head of value head h
            load8(k + qi, kv);
            load8(q + qi, qv);
            if (pro & KDA_PROLOGUE_GATE_BF16) load8(reinterpret_cast<const __nv_bfloat16*>(log_alpha) + gi, lv);
            else load8(reinterpret_cast<const float*>(log_alpha) + gi, lv);
            if (pro & KDA_PROLOGUE_GATE_LOGITS)  // rows past the end stay 0 (identity)
                for (int m = 0; m < 8; ++m) lv[m] = log_sigmoid_f(lv[m]);
        }
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            sk[r * LK + c + m] = kv[m];
            sq[r * LK + c + m] = qv[m];
            sg[r * LK + c + m] = lv[m];
        }
    }
    for (int e = tid; e < kChunk * dv / 8; e += kSimtThreads) {
        const int r = e / (dv / 8), c = 8 * (e % (dv / 8));
        float vv[8] = {};
        if (r < L) load8(v + ((size_t)(t0 + r) * H + h) * dv + c, vv);
#pragma unroll
        for (int m = 0; m < 8; ++m) sv[r * LV + c + m] = vv[m];
    }
    for (int r = tid; r < kChunk; r += kSimtThreads) {
        float b = 0.f;
        if (r < L) {
            b = beta[(size_t)(t0 + r) * H + h];
            if (pro & KDA_PROLOGUE_BETA_LOGITS) b = sigmoid_f(b);
        }
        sb[r] = b;
    }
    __syncthreads();
    if (pro & KDA_PROLOGUE_L2NORM_QK) {  // rows of k (i < 64) and q (i >= 64), normalised at the input precision
        for (int i = tid; i < 2 * kChunk; i += kSimtThreads) {
            float* row = (i < kChunk ? sk : sq) + (i & (kChunk - 1)) * LK;
            float ss = 0.f;
            for (int c0 = 0; c0 < dk; ++c0) {
                const float x = row[(c0 + i) & (dk - 1)];  // rotated start: fewer bank conflicts
                ss = fmaf(x, x, ss);
            }
            const float inv = rsqrtf(ss + kQkNormEps);
            for (int c0 = 0; c0 < dk; ++c0) {
                const int c = (c0 + i) & (dk - 1);
                row[c] = to_f32(from_f32<TIn>(row[c] * inv));
            }
        }
        __syncthreads();
    }

    // cumulative gate per channel; reference point = centre of the channel's range
    for (int c = tid; c < dk; c += kSimtThreads) {
        float acc = 0.f, lo = 0.f, hi = 0.f;
        for (int r = 0; r < kChunk; ++r) {
            acc += sg[r * LK + c];
            sg[r * LK + c] = acc;
            lo = fminf(lo, acc);
            hi = fmaxf(hi, acc);
        }
        sref[c] = 0.5f * (lo + hi);
        if (!(hi - lo <= kFactorSpread)) atomicOr(&s_wide, 1);
    }
    __syncthreads();

    const size_t slot_f = simt_slot_floats(dk, dv);
    float* slot = slots + ((size_t)j * H + h) * slot_f;
    float* gW = slot;
    float* gQ = gW + (size_t)kChunk * dk;
    float* gKd = gQ + (size_t)kChunk * dk;
    float* gP = gKd + (size_t)kChunk * dk;
    float* gUv = gP + (size_t)kChunk * kChunk;
    float* gGam = gUv + (size_t)kChunk * dv;

    // gated operands that never overflow (every exponent <= 0)
    for (int e = tid; e < kChunk * dk; e += kSimtThreads) {
        const int r = e / dk, c = e % dk, x = r * LK + c;
        const float gl = sg[(kChunk - 1) * LK + c];
        const float eg = fast_exp(sg[x]);
        gQ[e] = sq[x] * eg;
        gKd[e] = sk[x] * fast_exp(gl - sg[x]);
        sKt[x] = sk[x] * eg;
        if (r == 0) gGam[c] = fast_exp(gl);
    }
    __syncthreads();

    const bool wide = s_wide != 0;
    if (!wide) {
        // factorised form: e^{g_r - g_i} = e^{g_r - ref} e^{ref - g_i}, both factors within e^{+-80}
        for (int e = tid; e < kChunk * dk; e += kSimtThreads) {
            const int r = e / dk, c = e % dk, x0 = r * LK + c;
            const float x = sg[x0] - sref[c];
            const float kv = sk[x0];
            sk[x0] = kv * fast_exp(x);
            sq[x0] = sq[x0] * fast_exp(x);
            sg[x0] = kv * fast_exp(-x);
        }
        __syncthreads();
        if constexpr (TC) {
            simt_intra_ap_tc(sk, sq, sg, sv, sb, sA, sP, &s_tm, &s_mb);
        } else {
        // A = Kf Kb^T and P = Qf Kb^T, register-tiled (4 x 4 per thread, shared Kb reads)
        float a_[4][4] = {}, p_[4][4] = {};
#pragma unroll 2
        for (int c = 0; c < dk; ++c) {
            float kf[4], qf[4], kb[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                kf[a] = sk[(tr + 16 * a) * LK + c];
                qf[a] = sq[(tr + 16 * a) * LK + c];
                kb[a] = sg[(tc + 16 * a) * LK + c];
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    a_[a][b] = fmaf(kf[a], kb[b], a_[a][b]);
                    p_[a][b] = fmaf(qf[a], kb[b], p_[a][b]);
                }
        }
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int r = tr + 16 * a, i = tc + 16 * b;
                sA[r * L64 + i] = (i < r) ? sb[r] * a_[a][b] : 0.f;
                sP[r * L64 + i] = (i <= r) ? p_[a][b] : 0.f;
            }
        }
    } else {
        // some channel decays by more than e^-160 inside the chunk: exact per-element factors
        for (int e = tid; e < kChunk * kChunk; e += kSimtThreads) {
            const int r = e / kChunk, i = e % kChunk;
            float a = 0.f, p = 0.f;
            if (i <= r) {
                for (int c = 0; c < dk; ++c) {
                    const float kk = sk[i * LK + c] * fast_exp(sg[r * LK + c] - sg[i * LK + c]);
                    a = fmaf(sk[r * LK + c], kk, a);
                    p = fmaf(sq[r * LK + c], kk, p);
                }
            }
            sA[r * L64 + i] = (i < r) ? sb[r] * a : 0.f;
            sP[r * L64 + i] = p;
        }
    }
    __syncthreads();

    // T = (I + A)^{-1} diag(beta): the inverse in place of A (Kf, Qf and Kb are dead: sg is scratch)
    simt_unit_lower_inverse(sA, sg);
    for (int e = tid; e < kChunk * kChunk; e += kSimtThreads) {
        const int r = e / kChunk, i = e % kChunk;
        sT[r * L64 + i] = (i <= r) ? sA[r * L64 + i] * sb[i] : 0.f;
        gP[e] = sP[r * L64 + i];
    }
    __syncthreads();

    // W = T Kt, Uv = T V (T is lower triangular with zeros above the diagonal)
    if constexpr (TC) {  // the barrier's phase 0 was stage 1's (factorised chunks only)
        simt_intra_wuv_tc(sT, sKt, reinterpret_cast<const __nv_bfloat16*>(v), t0, L, H, h, sk, gW, gUv, &s_tm, &s_mb,
                          wide ? 0u : 1u);
    } else {
        if (dk == 128) simt_apply_t<128>(sT, sKt, gW, tr, tc);
        else simt_apply_t<64>(sT, sKt, gW, tr, tc);
        if (dv == 128) simt_apply_t<128>(sT, sv, gUv, tr, tc);
        else simt_apply_t<64>(sT, sv, gUv, tr, tc);
    }
}

// 16-byte asynchronous global -> shared copies in commit groups (phase B's operand prefetch)
__device__ __forceinline__ void simt_cp16(float* dst, const float* src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void simt_cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void simt_cp_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void simt_cp_wait0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// rows x cols floats from a dense global array into a shared array of row stride ld (cols and ld
// multiples of 4)
__device__ __forceinline__ void simt_cp_rows(float* dst, int ld, const float* src, int src_ld, int rows, int cols)
{
    const int per = cols / 4;
    for (int e = threadIdx.x; e < rows * per; e += kSimtThreads) {
        const int r = e / per, c = 4 * (e % per);
        simt_cp16(dst + r * ld + c, src + (size_t)r * src_ld + c);
    }
}

// Phase B: one CTA per (sequence, head, 32 state columns), chunks in order.  Chunk c's W and its Uv
// columns arrive in one cp.async group, Qg, P, Kd and gam in another, each while the previous
// chunk's other half computes.  Products are register-tiled (rows tr + 16 a, columns tc + 16 b).
template <typename TOut, int DK>
__global__ void __launch_bounds__(kSimtThreads)
simt_inter_kernel(const float* S0, float* S_final, TOut* __restrict__ out, const WsHeader* __restrict__ hdr,
                  const int* __restrict__ off, const int32_t* __restrict__ cu, int Tseq, int N, int H, int dv,
                  const float* __restrict__ slots)
{
    extern __shared__ __align__(16) float smem[];
    const int n = blockIdx.x, h = blockIdx.y, v0 = blockIdx.z * kSimtNV, tid = threadIdx.x;
    if (hdr->bad) return;
    constexpr int NV = kSimtNV, TMD = DK / 16;
    constexpr int LK = DK + 4, LP = kChunk + 4;  // padded rows: the two rows a warp reads sit on distinct banks
    float* sS = smem;                 // [DK][NV]
    float* sW = sS + DK * NV;         // [64][DK+4]
    float* sQ = sW + kChunk * LK;     // [64][DK+4]
    float* sKd = sQ + kChunk * LK;    // [64][DK+4]
    float* sP = sKd + kChunk * LK;    // [64][68]
    float* sUv = sP + kChunk * LP;    // [64][NV]
    float* sU = sUv + kChunk * NV;    // [64][NV]
    float* sG = sU + kChunk * NV;     // [DK]
    const int tr = tid >> 4, tc = tid & 15;
    const size_t slot_f = simt_slot_floats(DK, dv);
    const size_t sidx = ((size_t)n * H + h) * DK * dv;
    for (int e = tid; e < DK * NV; e += kSimtThreads)
        sS[e] = S0 ? S0[sidx + (size_t)(e / NV) * dv + v0 + (e % NV)] : 0.f;
    long long s0, s1;
    seq_bounds(n, cu, Tseq, s0, s1);
    const int j0 = off[n], j1 = off[n + 1];
    auto issue_w = [&](int j) {  // W and the Uv columns of chunk j
        const float* slot = slots + ((size_t)j * H + h) * slot_f;
        simt_cp_rows(sW, LK, slot, DK, kChunk, DK);
        simt_cp_rows(sUv, NV, slot + (size_t)kChunk * (3 * DK + kChunk) + v0, dv, kChunk, NV);
        simt_cp_commit();
    };
    auto issue_q = [&](int j) {  // Qg, Kd, P and gam of chunk j
        const float* slot = slots + ((size_t)j * H + h) * slot_f;
        simt_cp_rows(sQ, LK, slot + (size_t)kChunk * DK, DK, kChunk, DK);
        simt_cp_rows(sKd, LK, slot + 2 * (size_t)kChunk * DK, DK, kChunk, DK);
        simt_cp_rows(sP, LP, slot + 3 * (size_t)kChunk * DK, kChunk, kChunk, kChunk);
        simt_cp_rows(sG, DK, slot + (size_t)kChunk * (3 * DK + kChunk + dv), DK, 1, DK);
        simt_cp_commit();
    };
    if (j0 < j1) {
        issue_w(j0);
        issue_q(j0);
    }
    for (int j = j0; j < j1; ++j) {
        const long long t0 = s0 + (long long)(j - j0) * kChunk;
        const int L = (s1 - t0) < kChunk ? (int)(s1 - t0) : kChunk;
        simt_cp_wait1();  // W and Uv of chunk j (Qg, Kd, P may still be in flight)
        __syncthreads();
        {   // U = Uv - W S
            float x[4][2] = {};
            mm_acc<4, 2>(x, sW, LK, 1, sS, NV, 1, DK, tr, tc);
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 2; ++b) {
                    const int r = tr + 16 * a, jj = tc + 16 * b;
                    sU[r * NV + jj] = sUv[r * NV + jj] - x[a][b];
                }
        }
        __syncthreads();
        if (j + 1 < j1) issue_w(j + 1);
        else simt_cp_commit();  // one group per step keeps the wait counts aligned
        simt_cp_wait1();        // Qg, Kd, P, gam of chunk j
        __syncthreads();
        {   // out = Qg S + P U (rows past the end are not written)
            float o[4][2] = {};
            mm_acc<4, 2>(o, sQ, LK, 1, sS, NV, 1, DK, tr, tc);
            mm_acc<4, 2>(o, sP, LP, 1, sU, NV, 1, kChunk, tr, tc);
            if (out)
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    const int r = tr + 16 * a;
                    if (r < L)
#pragma unroll
                        for (int b = 0; b < 2; ++b)
                            out[((size_t)(t0 + r) * H + h) * dv + v0 + tc + 16 * b] = from_f32<TOut>(o[a][b]);
                }
        }
        {   // S <- Diag(gam) S + Kd^T U
            float acc[TMD][2];
#pragma unroll
            for (int a = 0; a < TMD; ++a)
#pragma unroll
                for (int b = 0; b < 2; ++b) acc[a][b] = sG[tr + 16 * a] * sS[(tr + 16 * a) * NV + tc + 16 * b];
            mm_acc<TMD, 2>(acc, sKd, 1, LK, sU, NV, 1, kChunk, tr, tc);
            __syncthreads();  // every thread has read the old S (and Qg, P, Kd)
#pragma unroll
            for (int a = 0; a < TMD; ++a)
#pragma unroll
                for (int b = 0; b < 2; ++b) sS[(tr + 16 * a) * NV + tc + 16 * b] = acc[a][b];
        }
        __syncthreads();
        if (j + 1 < j1) issue_q(j + 1);
        else simt_cp_commit();
    }
    simt_cp_wait0();
    __syncthreads();
    if (S_final)
        for (int e = tid; e < DK * NV; e += kSimtThreads)
            S_final[sidx + (size_t)(e / NV) * dv + v0 + (e % NV)] = sS[e];
}

inline size_t simt_intra_smem(int dk, int dv)
{
    return sizeof(float) * ((size_t)kChunk * (4 * (dk + 1) + dv + 1) + 3 * kChunk * (kChunk + 1) + kChunk + dk);
}
inline size_t simt_inter_smem(int dk, int dv)
{
    (void)dv;
    return sizeof(float) * ((size_t)dk * kSimtNV + 3 * kChunk * (dk + 4) + kChunk * (kChunk + 4) +
                            2 * kChunk * kSimtNV + dk);
}

template <typename TIn>
cudaError_t launch_simt_prefill(const void* q, const void* k, const void* v, const void* la, const float* beta,
                                const float* S0, float* S_final, void* out, const WsHeader* hdr, const int* off,
                                const int32_t* cu, int Tseq, int N, int H, int Hk, unsigned pro, int dk, int dv,
                                int max_chunks, float* slots, cudaStream_t stream)
{
    const size_t smA = simt_intra_smem(dk, dv), smB = simt_inter_smem(dk, dv);
    cudaError_t e = cudaFuncSetAttribute(simt_intra_kernel<TIn>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smA);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(dk == 128 ? simt_inter_kernel<TIn, 128> : simt_inter_kernel<TIn, 64>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smB);
    if (e != cudaSuccess) return e;
    if (max_chunks > 0) {
        LaunchScope ls("simt_intra", stream);
        simt_intra_kernel<TIn><<<dim3(max_chunks, H), kSimtThreads, smA, stream>>>(
            (const TIn*)q, (const TIn*)k, (const TIn*)v, la, beta, hdr, off, cu, Tseq, N, H, Hk, pro, dk, dv, slots);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    LaunchScope ls("simt_inter", stream);
    auto* inter = dk == 128 ? simt_inter_kernel<TIn, 128> : simt_inter_kernel<TIn, 64>;
    inter<<<dim3(N, H, dv / kSimtNV), kSimtThreads, smB, stream>>>(S0, S_final, (TIn*)out, hdr, off, cu, Tseq, N, H,
                                                                   dv, slots);
    return cudaGetLastError();
}

}  // namespace kda
