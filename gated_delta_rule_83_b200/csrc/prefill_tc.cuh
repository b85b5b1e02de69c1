// prefill_tc.cuh -- tensor-core (tcgen05 / TMEM) chunked KDA prefill for bf16 q/k/v, dk = dv = 128.
//
// The chunk form of the recurrence ("Kimi Linear" explainer, section "硬件效率的深度优化":
// chunk-parallel work inside a chunk, recurrent state passing between chunks, WY representation,
// UT transform; chunk size 64), split into two kernels:
//
// Phase A, one CTA per (chunk, head), every chunk in parallel (128 threads, thread c = channel c):
//   g_r = sum_{i<=r} log_alpha_i (fp32, restarted every chunk); ref_c = centre of channel c's range
//   Kf = k e^{g-ref}, Qf = q e^{g-ref}, Kb = k e^{ref-g}   (bf16 operands; every factor <= e^80)
//   A' = Kf Kb^T, P' = Qf Kb^T                       tcgen05, M=64 N=64 K=128, fp32 in TMEM
//   A = strict_lower(diag(beta) A'), P = lower_incl(P')     (= the exact e^{g_r - g_i} products)
//   T = (I + A)^{-1} diag(beta)                      fp32 blocked triangular inverse (UT transform)
//   W = T (k e^g), Uv = T v                          tcgen05, M=64 N=128 K=64 (B operands MN-major)
//   writes bf16 operand images of W, Qg = q e^g, Kd^T = (k e^{g_last-g})^T, P, Uv and fp32 e^{g_last}
//   to the workspace, already in the swizzled shared-memory layout phase B consumes.
//   A chunk in which some channel's gate spreads over more than e^160 (far outside any trained
//   gate) computes A and P with exact per-element factors on CUDA cores instead.
//
// Phase B, one CTA per (sequence, head, 32-column slice of S), chunks in order (128 threads):
//   a 3-stage bulk-copy (cp.async.bulk) pipeline streams each chunk's operand images into shared
//   memory; per chunk
//     X = W S, O = Qg S                 tcgen05 M=64 N=32 K=128
//     U = Uv - X  (-> bf16 U^T tile)
//     O += P U, Y = Kd^T U              tcgen05 M=64/128 N=32 K=64
//     S <- Diag(e^{g_last}) S + Y       fp32 in registers (thread c owns row c of the slice)
//   out = O (bf16), S_final = S (fp32).
#pragma once

#include "common.cuh"
#include "profile.cuh"
#include "tc_common.cuh"

namespace kda {

constexpr bool kTcPathReady = true;

// ---- workspace slot of one (chunk, head), bytes ------------------------------------------------
constexpr uint32_t kSlotW = 0;          // W    [64 x 128] bf16, SW128 tile (2 atom columns)
constexpr uint32_t kSlotQ = 16384;      // Qg   [64 x 128] bf16, SW128 tile
constexpr uint32_t kSlotKd = 32768;     // Kd^T [128 x 64] bf16, SW128 tile
constexpr uint32_t kSlotP = 49152;      // P    [64 x 64]  bf16, SW128 tile
constexpr uint32_t kSlotUv = 57344;     // Uv   [4 slices][64][32] bf16, plain row-major
constexpr uint32_t kSlotGam = 73728;    // e^{g_last} [128] fp32
constexpr uint32_t kSlotBytes = 74240;
inline size_t tc_slot_bytes() { return kSlotBytes; }

constexpr int kTcNV = 32;               // state columns per phase-B CTA

constexpr float kTcFactorSpread = 160.f;

// ------------------------------------------------------------------------------------------------
// small device helpers
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ float lds_bf16(const uint8_t* p) { return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p)); }
__device__ __forceinline__ void sts_bf16(uint8_t* p, float x) { *reinterpret_cast<__nv_bfloat16*>(p) = __float2bfloat16_rn(x); }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all()
{
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p)
{
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// ------------------------------------------------------------------------------------------------
// UT transform: X = (I + A)^{-1} for a strictly lower 64 x 64 A (fp32, row stride 65), by 16 x 16
// blocks: the diagonal blocks by forward substitution, then block row by block row
// X_ij = -X_ii sum_{k=j}^{i-1} A_ik X_kj.  128 threads.  Y is 3 x 16 x 17 floats of scratch.
// ------------------------------------------------------------------------------------------------
constexpr int kTS = 65;  // row stride of A and X

__device__ __forceinline__ void ut_inverse_64(const float* __restrict__ sA, float* __restrict__ sX, float* __restrict__ sY)
{
    const int tid = threadIdx.x;
    // zero X (upper blocks stay zero)
    for (int e = tid; e < 64 * kTS; e += 128) sX[e] = 0.f;
    __syncthreads();
    // diagonal blocks: warp kb inverts block kb, lane jj < 16 owns column jj
    {
        const int kb = tid >> 5, jj = tid & 31;
        if (jj < 16) {
            const int b = 16 * kb;
            float x[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float s = 0.f;
#pragma unroll
                for (int i = 0; i < r; ++i) s = fmaf(sA[(b + r) * kTS + b + i], x[i], s);
                x[r] = (r == jj) ? 1.f : ((r < jj) ? 0.f : -s);
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) sX[(b + r) * kTS + b + jj] = x[r];
        }
    }
    __syncthreads();
    // block rows 1..3
    for (int bi = 1; bi < 4; ++bi) {
        // Y_j = sum_{k=j}^{bi-1} A_{bi,k} X_{k,j}, for j = 0..bi-1 (bi blocks of 16 x 16)
        for (int e = tid; e < bi * 256; e += 128) {
            const int bj = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
            float s = 0.f;
            for (int kk = 16 * bj; kk < 16 * bi; ++kk) s = fmaf(sA[(16 * bi + rr) * kTS + kk], sX[kk * kTS + 16 * bj + cc], s);
            sY[(bj * 16 + rr) * 17 + cc] = s;
        }
        __syncthreads();
        // X_{bi,j} = -X_{bi,bi} Y_j
        for (int e = tid; e < bi * 256; e += 128) {
            const int bj = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
            float s = 0.f;
#pragma unroll
            for (int kk = 0; kk < 16; ++kk) s = fmaf(sX[(16 * bi + rr) * kTS + 16 * bi + kk], sY[(bj * 16 + kk) * 17 + cc], s);
            sX[(16 * bi + rr) * kTS + 16 * bj + cc] = -s;
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------------------------------------------
// Phase A
// ------------------------------------------------------------------------------------------------
constexpr int kAThreads = 128;
constexpr uint32_t kA_K = 0;        // Kf (raw k on load)                       16 KB
constexpr uint32_t kA_Q = 16384;    // Qf (raw q on load)                       16 KB
constexpr uint32_t kA_Kb = 32768;   // Kb; later T (bf16, 8 KB); wide case: g rows 0..31
constexpr uint32_t kA_Kt = 49152;   // k e^g (B operand of W); wide case: g rows 32..63
constexpr uint32_t kA_V = 65536;    // v                                        16 KB
constexpr uint32_t kA_A = 81920;    // A fp32 [64][65]                          16640 B
constexpr uint32_t kA_Y = 98560;    // solve scratch 3 x 16 x 17 fp32           3264 B
constexpr uint32_t kA_Misc = 101888;// beta[64] ref[128] E[128] D[128] + tmem addr, flag, mbarrier
constexpr uint32_t kA_Smem = kA_Misc + 2048 + 1024;  // + 1024 for aligning the dynamic base
// X = (I+A)^{-1}, fp32 [64][65], overlays Kf/Qf (dead by then)

__global__ void __launch_bounds__(kAThreads, 2)
tc_intra_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                const __nv_bfloat16* __restrict__ v, const float* __restrict__ log_alpha,
                const float* __restrict__ beta, const WsHeader* __restrict__ hdr, const int* __restrict__ off,
                const int32_t* __restrict__ cu, int Tseq, int N, int H, uint8_t* __restrict__ slots)
{
    using namespace tc;
    extern __shared__ uint8_t smem_raw[];
    const int j = blockIdx.x, h = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (hdr->bad || j >= hdr->total_chunks) return;
    int n, L;
    long long t0;
    locate_chunk(j, off, cu, Tseq, N, n, t0, L);

    uint8_t* sm = align1024(smem_raw);
    const uint32_t sb = smem_u32(sm);
    float* s_beta = reinterpret_cast<float*>(sm + kA_Misc);            // [64]
    float* s_E = reinterpret_cast<float*>(sm + kA_Misc + 256);         // [128] e^{ref}
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + kA_Misc + 768);
    int* s_wide = reinterpret_cast<int*>(sm + kA_Misc + 772);
    const uint32_t mbar = smem_u32(sm + kA_Misc + 1024);
    float* sA = reinterpret_cast<float*>(sm + kA_A);
    float* sX = reinterpret_cast<float*>(sm + kA_K);
    float* sY = reinterpret_cast<float*>(sm + kA_Y);
    uint8_t* slot = slots + ((size_t)j * H + h) * kSlotBytes;

    if (tid == 0) {
        *s_wide = 0;
        mbar_init(mbar, 1);
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(s_tmem), 256);
        tmem_relinquish();
    }
    // raw k, q, v -> SW128 tiles (rows >= L zero-filled)
    for (int e = tid; e < 64 * 16; e += kAThreads) {
        const int r = e >> 4, ch = e & 15;
        const uint32_t o = sw128_chunk_off(r, ch, 64);
        const int rr = r < L ? r : 0;
        const size_t gi = ((size_t)(t0 + rr) * H + h) * 128 + ch * 8;
        const uint32_t nb = r < L ? 16u : 0u;
        cp_async16(sb + kA_K + o, k + gi, nb);
        cp_async16(sb + kA_Q + o, q + gi, nb);
        cp_async16(sb + kA_V + o, v + gi, nb);
    }
    if (tid < 64) s_beta[tid] = tid < L ? beta[(size_t)(t0 + tid) * H + h] : 0.f;
    __syncthreads();  // s_wide / mbarrier init / TMEM address visible

    // cumulative gate of channel c = tid
    const int c = tid;
    float g[64];
    float lo = 0.f, hi = 0.f;
    {
        float acc = 0.f;
#pragma unroll
        for (int r = 0; r < 64; ++r) {
            const int rr = r < L ? r : L - 1;
            float x = log_alpha[((size_t)(t0 + rr) * H + h) * 128 + c];
            if (r >= L) x = 0.f;
            acc += x;
            g[r] = acc;
            lo = fminf(lo, acc);
            hi = fmaxf(hi, acc);
        }
    }
    const float ref = 0.5f * (lo + hi);
    const float glast = g[63];
    if (!(hi - lo <= kTcFactorSpread)) atomicOr(s_wide, 1);
    const float Ec = expf(ref);
    const float Dc = expf(glast - ref);
    s_E[c] = Ec;
    *reinterpret_cast<float*>(slot + kSlotGam + 4 * c) = expf(glast);
    cp_async_wait_all();
    __syncthreads();
    const bool wide = *s_wide != 0;
    const uint32_t tmem = *s_tmem;
    uint32_t phase = 0;
    bool ok = true;

    if (!wide) {
        // gated operands in place + Kd^T image (row c of the [128 x 64] tile, 16-byte stores)
#pragma unroll
        for (int rb = 0; rb < 64; rb += 8) {
            uint32_t pk[4];
#pragma unroll
            for (int m = 0; m < 8; m += 2) {
                float kd[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int r = rb + m + u;
                    const uint32_t o = sw128_off(r, c, 64);
                    const float kv = lds_bf16(sm + kA_K + o), qv = lds_bf16(sm + kA_Q + o);
                    const float x = g[r] - ref;
                    const float ef = exp_fast(x), eb = exp_fast(-x);
                    sts_bf16(sm + kA_K + o, kv * ef);
                    sts_bf16(sm + kA_Q + o, qv * ef);
                    sts_bf16(sm + kA_Kb + o, kv * eb);
                    sts_bf16(sm + kA_Kt + o, kv * ef * Ec);
                    kd[u] = kv * eb * Dc;
                }
                pk[m >> 1] = pack_bf16(kd[0], kd[1]);
            }
            *reinterpret_cast<uint4*>(slot + kSlotKd + sw128_chunk_off(c, rb >> 3, 128)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        fence_proxy_async();
        __syncthreads();
        if (tid == 0) {
            fence_after_sync();
            const uint32_t id = idesc_bf16(64, 64, false, false);
#pragma unroll
            for (int kk = 0; kk < 128; kk += 16) {
                mma_bf16(tmem + 0, desc_kmajor(sb + kA_K, 64, kk), desc_kmajor(sb + kA_Kb, 64, kk), id, kk > 0);
                mma_bf16(tmem + 64, desc_kmajor(sb + kA_Q, 64, kk), desc_kmajor(sb + kA_Kb, 64, kk), id, kk > 0);
            }
            mma_commit(mbar);
        }
        // Qg image = Qf * e^{ref} (same swizzled layout), while the MMAs run
        for (int e = tid; e < 64 * 16; e += kAThreads) {
            const int r = e >> 4, ch = e & 15;
            const uint32_t o = sw128_chunk_off(r, ch, 64);
            const uint4 raw = *reinterpret_cast<const uint4*>(sm + kA_Q + o);
            const __nv_bfloat16* hv = reinterpret_cast<const __nv_bfloat16*>(&raw);
            uint32_t pk[4];
#pragma unroll
            for (int m = 0; m < 8; m += 2)
                pk[m >> 1] = pack_bf16(__bfloat162float(hv[m]) * s_E[ch * 8 + m],
                                       __bfloat162float(hv[m + 1]) * s_E[ch * 8 + m + 1]);
            *reinterpret_cast<uint4*>(slot + kSlotQ + o) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        ok = mbar_wait(mbar, phase);
        phase ^= 1;
        fence_after_sync();
        // A' and P' rows (M = 64 layout: row 16*warp + lane at TMEM lane 32*warp + lane, lane < 16)
        const int r = 16 * warp + (lane & 15);
        const uint32_t trow = tmem + ((uint32_t)(32 * warp) << 16);
        const float br = s_beta[r];
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
            float a[16];
            tmem_ld16(trow + blk * 16, a);
            tmem_wait_ld();
            if (lane < 16) {
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    const int i = blk * 16 + m;
                    sA[r * kTS + i] = (i < r) ? br * a[m] : 0.f;
                }
            }
        }
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
            float a[16];
            tmem_ld16(trow + 64 + blk * 16, a);
            tmem_wait_ld();
            if (lane < 16) {
                uint32_t pk[8];
#pragma unroll
                for (int m = 0; m < 16; m += 2) {
                    const int i = blk * 16 + m;
                    pk[m >> 1] = pack_bf16(i <= r ? a[m] : 0.f, i + 1 <= r ? a[m + 1] : 0.f);
                }
                *reinterpret_cast<uint4*>(slot + kSlotP + sw128_chunk_off(r, 2 * blk, 64)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                *reinterpret_cast<uint4*>(slot + kSlotP + sw128_chunk_off(r, 2 * blk + 1, 64)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
        }
        fence_before_sync();
    } else {
        // exact per-element factors on CUDA cores; g goes to shared memory (Kb and Kt areas)
        float* sg = reinterpret_cast<float*>(sm + kA_Kb);
#pragma unroll
        for (int r = 0; r < 64; ++r) sg[r * 128 + c] = g[r];
        __syncthreads();
        for (int e = tid; e < 64 * 64; e += kAThreads) {
            const int r = e >> 6, i = e & 63;
            float a = 0.f, p = 0.f;
            if (i <= r) {
                for (int cc = 0; cc < 128; ++cc) {
                    const float kk = lds_bf16(sm + kA_K + sw128_off(i, cc, 64)) * expf(sg[r * 128 + cc] - sg[i * 128 + cc]);
                    a = fmaf(lds_bf16(sm + kA_K + sw128_off(r, cc, 64)), kk, a);
                    p = fmaf(lds_bf16(sm + kA_Q + sw128_off(r, cc, 64)), kk, p);
                }
            }
            sA[r * kTS + i] = (i < r) ? s_beta[r] * a : 0.f;
            *reinterpret_cast<__nv_bfloat16*>(slot + kSlotP + sw128_off(r, i, 64)) = __float2bfloat16_rn(p);
        }
        __syncthreads();  // g in shared memory no longer needed
#pragma unroll
        for (int rb = 0; rb < 64; rb += 8) {
            uint32_t pk[4];
#pragma unroll
            for (int m = 0; m < 8; m += 2) {
                float kd[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int r = rb + m + u;
                    const uint32_t o = sw128_off(r, c, 64);
                    const float kv = lds_bf16(sm + kA_K + o), qv = lds_bf16(sm + kA_Q + o);
                    const float eg = expf(g[r]);
                    sts_bf16(sm + kA_Kt + o, kv * eg);
                    *reinterpret_cast<__nv_bfloat16*>(slot + kSlotQ + o) = __float2bfloat16_rn(qv * eg);
                    kd[u] = kv * expf(glast - g[r]);
                }
                pk[m >> 1] = pack_bf16(kd[0], kd[1]);
            }
            *reinterpret_cast<uint4*>(slot + kSlotKd + sw128_chunk_off(c, rb >> 3, 128)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
    }
    ok = __syncthreads_and(ok);

    // UT transform, then T = X diag(beta) as a bf16 K-major tile (over Kb)
    if (ok) ut_inverse_64(sA, sX, sY);
    for (int e = tid; e < 64 * 8 && ok; e += kAThreads) {
        const int r = e >> 3, ch = e & 7;
        uint32_t pk[4];
#pragma unroll
        for (int m = 0; m < 8; m += 2) {
            const int i = ch * 8 + m;
            pk[m >> 1] = pack_bf16(sX[r * kTS + i] * s_beta[i], sX[r * kTS + i + 1] * s_beta[i + 1]);
        }
        *reinterpret_cast<uint4*>(sm + kA_Kb + sw128_chunk_off(r, ch, 64)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
    fence_proxy_async();
    __syncthreads();
    if (ok && tid == 0) {
        fence_after_sync();
        const uint32_t id = idesc_bf16(64, 128, false, true);
#pragma unroll
        for (int kk = 0; kk < 64; kk += 16) {
            mma_bf16(tmem + 0, desc_kmajor(sb + kA_Kb, 64, kk), desc_mnmajor(sb + kA_Kt, 64, kk), id, kk > 0);
            mma_bf16(tmem + 128, desc_kmajor(sb + kA_Kb, 64, kk), desc_mnmajor(sb + kA_V, 64, kk), id, kk > 0);
        }
        mma_commit(mbar);
    }
    if (ok) {
        ok = mbar_wait(mbar, phase);
        fence_after_sync();
    }
    ok = __syncthreads_and(ok);
    if (ok) {
        const int r = 16 * warp + (lane & 15);
        const uint32_t trow = tmem + ((uint32_t)(32 * warp) << 16);
#pragma unroll
        for (int blk = 0; blk < 8; ++blk) {  // W row r -> image
            float a[16];
            tmem_ld16(trow + blk * 16, a);
            tmem_wait_ld();
            if (lane < 16) {
                uint32_t pk[8];
#pragma unroll
                for (int m = 0; m < 16; m += 2) pk[m >> 1] = pack_bf16(a[m], a[m + 1]);
                *reinterpret_cast<uint4*>(slot + kSlotW + sw128_chunk_off(r, 2 * blk, 64)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                *reinterpret_cast<uint4*>(slot + kSlotW + sw128_chunk_off(r, 2 * blk + 1, 64)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
        }
#pragma unroll
        for (int blk = 0; blk < 8; ++blk) {  // Uv row r -> [slice][64][32]
            float a[16];
            tmem_ld16(trow + 128 + blk * 16, a);
            tmem_wait_ld();
            if (lane < 16) {
                uint32_t pk[8];
#pragma unroll
                for (int m = 0; m < 16; m += 2) pk[m >> 1] = pack_bf16(a[m], a[m + 1]);
                const int col = blk * 16, sl = col >> 5;
                uint8_t* dst = slot + kSlotUv + (size_t)(sl * 64 + r) * 64 + (col & 31) * 2;
                *reinterpret_cast<uint4*>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                *reinterpret_cast<uint4*>(dst + 16) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// ------------------------------------------------------------------------------------------------
// Phase B
// ------------------------------------------------------------------------------------------------
constexpr int kBThreads = 128;
constexpr int kBStages = 3;
constexpr uint32_t kStageBytes = 62464;     // W | Qg | Kd^T | P (57344 B) + Uv slice (4096 B) + e^{g_last} (512 B)
constexpr uint32_t kStUv = 57344, kStGam = 61440, kStTx = 61952;
constexpr uint32_t kB_S = kBStages * kStageBytes;  // S^T tile [32 x 128] bf16 (8 KB)
constexpr uint32_t kB_U = kB_S + 8192;             // U^T tile [32 x 64]  bf16 (4 KB)
constexpr uint32_t kB_Misc = kB_U + 4096;          // mbarriers + TMEM address
constexpr uint32_t kB_Smem = kB_Misc + 256 + 1024;

__device__ __forceinline__ void tc_issue_stage(uint32_t stage_addr, uint32_t full_bar, const uint8_t* slot, int vt)
{
    using namespace tc;
    mbar_arrive_expect_tx(full_bar, kStTx);
    bulk_g2s(stage_addr, slot, kSlotUv, full_bar);
    bulk_g2s(stage_addr + kStUv, slot + kSlotUv + vt * 4096, 4096, full_bar);
    bulk_g2s(stage_addr + kStGam, slot + kSlotGam, 512, full_bar);
}

__global__ void __launch_bounds__(kBThreads, 1)
tc_inter_kernel(const float* S0, float* S_final, __nv_bfloat16* __restrict__ out, const WsHeader* __restrict__ hdr,
                const int* __restrict__ off, const int32_t* __restrict__ cu, int Tseq, int N, int H,
                const uint8_t* __restrict__ slots)
{
    using namespace tc;
    extern __shared__ uint8_t smem_raw[];
    const int n = blockIdx.x, h = blockIdx.y, vt = blockIdx.z, v0 = vt * kTcNV;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (hdr->bad) return;
    uint8_t* sm = align1024(smem_raw);
    const uint32_t sb = smem_u32(sm);
    const uint32_t bar_full = smem_u32(sm + kB_Misc);       // kBStages barriers
    const uint32_t bar_mma = bar_full + 8 * kBStages;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + kB_Misc + 64);

    const int jb = off[n], je = off[n + 1], nch = je - jb;
    long long s0, s1;
    seq_bounds(n, cu, Tseq, s0, s1);

    if (tid == 0) {
        for (int s = 0; s < kBStages; ++s) mbar_init(bar_full + 8 * s, 1);
        mbar_init(bar_mma, 1);
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(s_tmem), 128);
        tmem_relinquish();
    }
    // state slice: thread c owns row c, columns v0 .. v0+31
    const int c = tid;
    float S[kTcNV];
    const size_t srow = (((size_t)n * H + h) * 128 + c) * 128 + v0;
    if (S0) {
#pragma unroll
        for (int m = 0; m < kTcNV; m += 4) {
            const float4 x = *reinterpret_cast<const float4*>(S0 + srow + m);
            S[m] = x.x; S[m + 1] = x.y; S[m + 2] = x.z; S[m + 3] = x.w;
        }
    } else {
#pragma unroll
        for (int m = 0; m < kTcNV; ++m) S[m] = 0.f;
    }
#pragma unroll
    for (int m = 0; m < kTcNV; ++m) sts_bf16(sm + kB_S + sw128_off(m, c, 32), S[m]);
    __syncthreads();  // barriers initialised, TMEM address visible
    if (tid == 0)
        for (int s = 0; s < kBStages && s < nch; ++s)
            tc_issue_stage(sb + s * kStageBytes, bar_full + 8 * s, slots + ((size_t)(jb + s) * H + h) * kSlotBytes, vt);
    fence_proxy_async();
    __syncthreads();
    const uint32_t tmem = *s_tmem;
    const uint32_t tw = tmem + ((uint32_t)(32 * warp) << 16);
    const int r = 16 * warp + (lane & 15);
    uint32_t mphase = 0;
    bool ok = true;

    for (int it = 0; it < nch && ok; ++it) {
        const int s = it % kBStages;
        const uint32_t st = sb + s * kStageBytes;
        const uint8_t* stp = sm + s * kStageBytes;
        const long long t0 = s0 + (long long)it * 64;
        const int L = (s1 - t0) < 64 ? (int)(s1 - t0) : 64;
        ok = mbar_wait(bar_full + 8 * s, (uint32_t)(it / kBStages) & 1u);
        if (ok && tid == 0) {
            fence_after_sync();
            const uint32_t id = idesc_bf16(64, kTcNV, false, false);
#pragma unroll
            for (int kk = 0; kk < 128; kk += 16) {
                mma_bf16(tmem + 0, desc_kmajor(st + kSlotW, 64, kk), desc_kmajor(sb + kB_S, 32, kk), id, kk > 0);
                mma_bf16(tmem + 32, desc_kmajor(st + kSlotQ, 64, kk), desc_kmajor(sb + kB_S, 32, kk), id, kk > 0);
            }
            mma_commit(bar_mma);
        }
        ok = ok && mbar_wait(bar_mma, mphase);
        mphase ^= 1;
        fence_after_sync();
        {   // U = Uv - X  ->  U^T tile
            float x[32];
            tmem_ld16(tw + 0, x);
            tmem_ld16(tw + 16, x + 16);
            tmem_wait_ld();
            if (lane < 16) {
                const uint8_t* uv = stp + kStUv + r * 64;
#pragma unroll
                for (int m = 0; m < 32; m += 8) {
                    const uint4 raw = *reinterpret_cast<const uint4*>(uv + 2 * m);
                    const __nv_bfloat16* hv = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        sts_bf16(sm + kB_U + sw128_off(m + u, r, 32), __bfloat162float(hv[u]) - x[m + u]);
                }
            }
        }
        fence_proxy_async();
        fence_before_sync();
        ok = __syncthreads_and(ok);
        if (ok && tid == 0) {
            fence_after_sync();
            const uint32_t id64 = idesc_bf16(64, kTcNV, false, false);
            const uint32_t id128 = idesc_bf16(128, kTcNV, false, false);
#pragma unroll
            for (int kk = 0; kk < 64; kk += 16) {
                mma_bf16(tmem + 32, desc_kmajor(st + kSlotP, 64, kk), desc_kmajor(sb + kB_U, 32, kk), id64, 1u);
                mma_bf16(tmem + 64, desc_kmajor(st + kSlotKd, 128, kk), desc_kmajor(sb + kB_U, 32, kk), id128, kk > 0);
            }
            mma_commit(bar_mma);
        }
        ok = ok && mbar_wait(bar_mma, mphase);
        mphase ^= 1;
        fence_after_sync();
        {   // S <- e^{g_last} S + Y
            float y[32];
            tmem_ld16(tw + 64, y);
            tmem_ld16(tw + 80, y + 16);
            tmem_wait_ld();
            const float gam = *reinterpret_cast<const float*>(stp + kStGam + 4 * c);
#pragma unroll
            for (int m = 0; m < kTcNV; ++m) {
                S[m] = fmaf(gam, S[m], y[m]);
                sts_bf16(sm + kB_S + sw128_off(m, c, 32), S[m]);
            }
        }
        {   // O -> out
            float o[32];
            tmem_ld16(tw + 32, o);
            tmem_ld16(tw + 48, o + 16);
            tmem_wait_ld();
            if (lane < 16 && r < L && ok) {
                __nv_bfloat16* dst = out + ((size_t)(t0 + r) * H + h) * 128 + v0;
#pragma unroll
                for (int m = 0; m < 32; m += 8)
                    *reinterpret_cast<uint4*>(dst + m) = make_uint4(pack_bf16(o[m], o[m + 1]), pack_bf16(o[m + 2], o[m + 3]),
                                                                    pack_bf16(o[m + 4], o[m + 5]), pack_bf16(o[m + 6], o[m + 7]));
            }
        }
        fence_proxy_async();
        fence_before_sync();
        ok = __syncthreads_and(ok);
        if (ok && tid == 0 && it + kBStages < nch)
            tc_issue_stage(st, bar_full + 8 * s, slots + ((size_t)(jb + it + kBStages) * H + h) * kSlotBytes, vt);
    }
    if (S_final && ok) {
#pragma unroll
        for (int m = 0; m < kTcNV; m += 4)
            *reinterpret_cast<float4*>(S_final + srow + m) = make_float4(S[m], S[m + 1], S[m + 2], S[m + 3]);
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 128);
}

inline cudaError_t launch_tc_prefill(const void* q, const void* k, const void* v, const float* la, const float* beta,
                                     const float* S0, float* S_final, void* out, const WsHeader* hdr, const int* off,
                                     const int32_t* cu, int Tseq, int N, int H, int max_chunks, char* slots,
                                     cudaStream_t stream)
{
    cudaError_t e = cudaFuncSetAttribute(tc_intra_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kA_Smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(tc_inter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kB_Smem);
    if (e != cudaSuccess) return e;
    if (max_chunks > 0) {
        LaunchScope ls("tc_intra", stream);
        tc_intra_kernel<<<dim3(max_chunks, H), kAThreads, kA_Smem, stream>>>(
            (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, la, beta, hdr, off, cu, Tseq, N,
            H, (uint8_t*)slots);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    LaunchScope ls("tc_inter", stream);
    tc_inter_kernel<<<dim3(N, H, 128 / kTcNV), kBThreads, kB_Smem, stream>>>(
        S0, S_final, (__nv_bfloat16*)out, hdr, off, cu, Tseq, N, H, (const uint8_t*)slots);
    return cudaGetLastError();
}

}  // namespace kda
