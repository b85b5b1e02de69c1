// prefill_tc.cuh -- tensor-core (tcgen05 / TMEM) chunked KDA prefill for bf16 q/k/v, dk = dv = 128.
//
// The chunk form of the recurrence ("Kimi Linear" explainer, section "硬件效率的深度优化":
// chunk-parallel work inside a chunk, recurrent state passing between chunks, WY representation,
// UT transform; chunk size 64), split into two kernels.
//
// Phase A, persistent (two 256-thread CTAs per SM), one (chunk, head) unit at a time per CTA, units
// claimed from a work counter one ahead so that the next unit's inputs load during this one:
//   g_r = sum_{i<=r} log_alpha_i (fp32, log2 units, restarted every chunk); ref_c = centre of channel c's range
//   Kf = k e^{g-ref}, Qf = q e^{g-ref}, Kb = k e^{ref-g}   (bf16 operands; every factor <= e^80)
//   A' = Kf Kb^T, P' = Qf Kb^T                          tcgen05 M=64 N=64 K=128, fp32 in TMEM
//   A = strict_lower(diag(beta) A'), P = lower_incl(P')        (= the exact e^{g_r - g_i} products)
//   T = (I + A)^{-1} diag(beta)                         fp32 recursive-doubling triangular inverse (in place)
//   [W' | Uv] = T [Kf | v], W = W' diag(e^ref)         tcgen05 M=64 N=256 K=64 (B operand MN-major)
//   [P W | P Uv] = P [W | Uv]                           tcgen05 M=64 N=256 K=64
//   Q' = q e^g - P W,  O0 = P Uv                        (the intra-chunk part of the output, folded in)
//   writes bf16 operand images -- [W; Q'] stacked (128 rows), Kd = k e^{g_last-g}, Uv, O0 -- and fp32
//   e^{g_last} to the workspace, already in the swizzled shared-memory layout phase B consumes.
//   A chunk in which some channel's gate spreads over more than e^160 (far outside any trained
//   gate) computes A and P with exact per-element factors on CUDA cores instead.
//
// Phase B, one CTA per (sequence, head, 32-column slice of S), chunks in order, longest sequences
// launched first.  Warp roles: four
// compute warps, one MMA-issue warp, one bulk-copy warp.  A 3-stage cp.async.bulk pipeline streams
// each chunk's images into shared memory; per chunk
//     [X; O'] = [W; Q'] S               tcgen05 M=128 N=32 K=128   (one 8-instruction batch)
//     U = Uv - X  (-> bf16 U tile)      out = O' + O0  (off the critical path)
//     Y = Kd^T U                        tcgen05 M=128 N=32 K=64
//     S <- Diag(e^{g_last}) S + Y       fp32 in registers (thread c owns row c of the slice)
// which equals O = Qg S + P U with U = Uv - W S, the chunk form of o_t = S_t^T q_t.
#pragma once

#include <cuda.h>  // CUtensorMap and its enums (the encoder is fetched through the runtime)

#include "common.cuh"
#include "profile.cuh"
#include "tc_common.cuh"

namespace kda {

constexpr bool kTcPathReady = true;

// ---- workspace slot of one (chunk, head), bytes ------------------------------------------------
// Every image is a 64-row SW128 tile, bf16 [64 x 128] (two 8 KB atom columns), exactly as phase A
// holds it in shared memory, so phase A writes each with bulk copies.  The slot of unit u = chunk * H
// + head is slot u: the slots of one chunk row (all heads) are adjacent.
constexpr uint32_t kSlotW = 0;          // W
constexpr uint32_t kSlotQ = 16384;      // Q'
constexpr uint32_t kSlotKd = 32768;     // Kd  (MN-major A operand of Kd^T U)
constexpr uint32_t kSlotUv = 49152;     // Uv
constexpr uint32_t kSlotO0 = 65536;     // O0
constexpr uint32_t kSlotGam = 81920;    // e^{g_last} [128] fp32
constexpr uint32_t kSlotBytes = 82432;
inline size_t tc_slot_bytes() { return kSlotBytes; }

constexpr int kTcNV = 32;               // state columns per phase-B CTA

constexpr float kTcFactorSpread = 230.f;  // log2 units (about e^159): every factor 2^(+-(g2 - ref2)) <= 2^115

// ------------------------------------------------------------------------------------------------
// small device helpers
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ float lds_bf16(const uint8_t* p) { return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p)); }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, uint32_t src_bytes)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all()
{
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ uint8_t* align1024(uint8_t* p)
{
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}
__device__ __forceinline__ void unpack8(const uint4& raw, float* f)
{
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const float2 t = __bfloat1622float2(h[m]);
        f[2 * m] = t.x;
        f[2 * m + 1] = t.y;
    }
}
__device__ __forceinline__ uint4 pack8(const float* f)
{
    return make_uint4(tc::pack_bf16(f[0], f[1]), tc::pack_bf16(f[2], f[3]), tc::pack_bf16(f[4], f[5]),
                      tc::pack_bf16(f[6], f[7]));
}
__device__ __forceinline__ void named_sync(int id, int threads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
__device__ __forceinline__ void named_arrive(int id, int threads)
{
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// ------------------------------------------------------------------------------------------------
// UT transform: from a strictly lower 64 x 64 A (fp32, row stride 68, zero on and above the diagonal)
// to T = (I + A)^{-1} diag(beta), written as a bf16 K-major SW128 64 x 64 tile (the A operand of
// [W' | Uv] = T [Kf | v]).  X = (I + A)^{-1} by recursive doubling: the four 16 x 16 diagonal blocks
// by forward substitution; then, inside each 32 x 32 half, X_10 = -X_11 A_10 X_00; then the 32 x 32
// off-diagonal block X_10 = -X_11 A_10 X_00 of the whole.  X overwrites A in place where a later
// level reads it.  Each level also writes its blocks of T as soon as they are final, and threads idle
// in the first level zero the blocks above the diagonal, so no separate pass packs T.  256 threads;
// the levels use 64, 64 and 128 of them (with two CTAs per SM the idle warps' issue slots go to the
// other CTA).  sY: scratch of 32 x 36 floats (16-byte aligned rows).
// ------------------------------------------------------------------------------------------------
constexpr int kAS = 68;  // row stride of A / X

__device__ __forceinline__ void ut_transform_T(float* __restrict__ sA, float* __restrict__ sY,
                                               const float* __restrict__ s_beta, uint8_t* __restrict__ tT)
{
    const int tid = threadIdx.x;
    {   // diagonal 16 x 16 blocks: thread -> (block, column jj); written back once every block is read
        const int b = 16 * (tid >> 4), jj = tid & 15;
        float x[16];
        if (tid < 64) {  // left-looking: x_r = -sum_{i<r} A[r][i] x_i, row r read as 128-bit words;
                         // each sum takes x_{r-1} last, so the rows' chains overlap
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float s = 0.f;
#pragma unroll
                for (int i4 = 0; i4 < r; i4 += 4) {
                    const float4 a4 = *reinterpret_cast<const float4*>(sA + (b + r) * kAS + b + i4);
                    const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        if (i4 + j < r) s = fmaf(av[j], x[i4 + j], s);
                }
                x[r] = (r == jj) ? 1.f : ((r < jj) ? 0.f : -s);
            }
        } else if (tid < 64 + 192) {  // the blocks of T above the diagonal: 192 chunks of 16 bytes
            const int z = tid - 64;
            int row, ch;
            if (z < 96) { row = z / 6; ch = 2 + z % 6; }
            else if (z < 160) { row = 16 + (z - 96) / 4; ch = 4 + (z - 96) % 4; }
            else { row = 32 + (z - 160) / 2; ch = 6 + (z - 160) % 2; }
            *reinterpret_cast<uint4*>(tT + tc::sw128_chunk_off(row, ch, 64)) = make_uint4(0, 0, 0, 0);
        }
        __syncthreads();
        if (tid < 64) {
            const float bj = s_beta[b + jj];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                sA[(b + r) * kAS + b + jj] = x[r];
                *reinterpret_cast<__nv_bfloat16*>(tT + tc::sw128_off(b + r, b + jj, 64)) = __float2bfloat16_rn(x[r] * bj);
            }
        }
        __syncthreads();
    }
    {   // level 1: blocks (1,0) and (3,2) on warps 0-1: thread -> (pair p, rows ra and ra + 8,
        // columns cc..cc+3); rows ra = 0..7 of a warp sit on distinct banks (row stride 68)
        const int p = tid >> 5, ra = (tid >> 2) & 7, cc = (tid & 3) * 4;
        const int bi = 16 * (2 * p + 1), bj = 16 * (2 * p);
        if (tid < 64) {
            float y0[4] = {0.f, 0.f, 0.f, 0.f}, y1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const float a0 = sA[(bi + ra) * kAS + bj + k], a1 = sA[(bi + ra + 8) * kAS + bj + k];
                const float4 xv = *reinterpret_cast<const float4*>(sA + (bj + k) * kAS + bj + cc);
                y0[0] = fmaf(a0, xv.x, y0[0]); y0[1] = fmaf(a0, xv.y, y0[1]); y0[2] = fmaf(a0, xv.z, y0[2]); y0[3] = fmaf(a0, xv.w, y0[3]);
                y1[0] = fmaf(a1, xv.x, y1[0]); y1[1] = fmaf(a1, xv.y, y1[1]); y1[2] = fmaf(a1, xv.z, y1[2]); y1[3] = fmaf(a1, xv.w, y1[3]);
            }
            *reinterpret_cast<float4*>(sY + (p * 16 + ra) * 36 + cc) = make_float4(y0[0], y0[1], y0[2], y0[3]);
            *reinterpret_cast<float4*>(sY + (p * 16 + ra + 8) * 36 + cc) = make_float4(y1[0], y1[1], y1[2], y1[3]);
        }
        __syncthreads();  // A_10 read: X_10 takes its place
        if (tid < 64) {
            float x0[4] = {0.f, 0.f, 0.f, 0.f}, x1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const float a0 = sA[(bi + ra) * kAS + bi + k], a1 = sA[(bi + ra + 8) * kAS + bi + k];
                const float4 yv = *reinterpret_cast<const float4*>(sY + (p * 16 + k) * 36 + cc);
                x0[0] = fmaf(a0, yv.x, x0[0]); x0[1] = fmaf(a0, yv.y, x0[1]); x0[2] = fmaf(a0, yv.z, x0[2]); x0[3] = fmaf(a0, yv.w, x0[3]);
                x1[0] = fmaf(a1, yv.x, x1[0]); x1[1] = fmaf(a1, yv.y, x1[1]); x1[2] = fmaf(a1, yv.z, x1[2]); x1[3] = fmaf(a1, yv.w, x1[3]);
            }
            *reinterpret_cast<float4*>(sA + (bi + ra) * kAS + bj + cc) = make_float4(-x0[0], -x0[1], -x0[2], -x0[3]);
            *reinterpret_cast<float4*>(sA + (bi + ra + 8) * kAS + bj + cc) = make_float4(-x1[0], -x1[1], -x1[2], -x1[3]);
            const float4 be = *reinterpret_cast<const float4*>(s_beta + bj + cc);
            *reinterpret_cast<uint2*>(tT + tc::sw128_off(bi + ra, bj + cc, 64)) =
                make_uint2(tc::pack_bf16(-x0[0] * be.x, -x0[1] * be.y), tc::pack_bf16(-x0[2] * be.z, -x0[3] * be.w));
            *reinterpret_cast<uint2*>(tT + tc::sw128_off(bi + ra + 8, bj + cc, 64)) =
                make_uint2(tc::pack_bf16(-x1[0] * be.x, -x1[1] * be.y), tc::pack_bf16(-x1[2] * be.z, -x1[3] * be.w));
        }
        __syncthreads();
    }
    {   // level 2: rows 32..63, columns 0..31, on warps 0-3: thread -> (rows r0, r0 + 1, columns
        // cc..cc+3).  Each right-hand float4 serves two rows, which halves the shared-memory
        // wavefronts of the 128-bit loads; X22 is lower triangular, so warp w stops at row 8 w + 7.
        // The block is final here: only its T values are written.
        const int r0 = 2 * (tid >> 3), cc = (tid & 7) * 4;
        if (tid < 128) {
            float y0[4] = {0.f, 0.f, 0.f, 0.f}, y1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
            for (int k = 0; k < 32; ++k) {
                const float a0 = sA[(32 + r0) * kAS + k], a1 = sA[(33 + r0) * kAS + k];
                const float4 xv = *reinterpret_cast<const float4*>(sA + k * kAS + cc);
                y0[0] = fmaf(a0, xv.x, y0[0]); y0[1] = fmaf(a0, xv.y, y0[1]); y0[2] = fmaf(a0, xv.z, y0[2]); y0[3] = fmaf(a0, xv.w, y0[3]);
                y1[0] = fmaf(a1, xv.x, y1[0]); y1[1] = fmaf(a1, xv.y, y1[1]); y1[2] = fmaf(a1, xv.z, y1[2]); y1[3] = fmaf(a1, xv.w, y1[3]);
            }
            *reinterpret_cast<float4*>(sY + r0 * 36 + cc) = make_float4(y0[0], y0[1], y0[2], y0[3]);
            *reinterpret_cast<float4*>(sY + (r0 + 1) * 36 + cc) = make_float4(y1[0], y1[1], y1[2], y1[3]);
        }
        __syncthreads();
        if (tid < 128) {
            const int kend = 8 * (tid >> 5) + 8;  // rows of this warp: 8 w .. 8 w + 7 (X22[r][k] = 0 for k > r)
            float x0[4] = {0.f, 0.f, 0.f, 0.f}, x1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
            for (int k = 0; k < kend; ++k) {
                const float a0 = sA[(32 + r0) * kAS + 32 + k], a1 = sA[(33 + r0) * kAS + 32 + k];
                const float4 yv = *reinterpret_cast<const float4*>(sY + k * 36 + cc);
                x0[0] = fmaf(a0, yv.x, x0[0]); x0[1] = fmaf(a0, yv.y, x0[1]); x0[2] = fmaf(a0, yv.z, x0[2]); x0[3] = fmaf(a0, yv.w, x0[3]);
                x1[0] = fmaf(a1, yv.x, x1[0]); x1[1] = fmaf(a1, yv.y, x1[1]); x1[2] = fmaf(a1, yv.z, x1[2]); x1[3] = fmaf(a1, yv.w, x1[3]);
            }
            const float4 be = *reinterpret_cast<const float4*>(s_beta + cc);
            *reinterpret_cast<uint2*>(tT + tc::sw128_off(32 + r0, cc, 64)) =
                make_uint2(tc::pack_bf16(-x0[0] * be.x, -x0[1] * be.y), tc::pack_bf16(-x0[2] * be.z, -x0[3] * be.w));
            *reinterpret_cast<uint2*>(tT + tc::sw128_off(33 + r0, cc, 64)) =
                make_uint2(tc::pack_bf16(-x1[0] * be.x, -x1[1] * be.y), tc::pack_bf16(-x1[2] * be.z, -x1[3] * be.w));
        }
    }
    tc::fence_proxy_async();  // T is read by the tensor core
    __syncthreads();
}

// ------------------------------------------------------------------------------------------------
// Phase A
// ------------------------------------------------------------------------------------------------
// Persistent: CTA b starts with (chunk, head) unit b (unit u = chunk * H + head) and claims each
// further unit from a work counter one unit ahead, so that its inputs can be prefetched.
// Each input buffer is refilled with the next unit's data as soon as the current unit is done with
// it: log_alpha once MMA3 has read P (the last tenant of its region); k, q and v once the last images
// (Q' in the q rows, O0 in the v tile) have left for the workspace.
constexpr int kAThreads = 256;
constexpr uint32_t kA_KQ = 0;        // 32 KB: [k; q] -> [Kf; Qf] stacked (128 rows, atom columns at 0 / 16384)
                                     //   -> W in the k rows, Q' in the q rows
constexpr uint32_t kA_V = 32768;     // 16 KB: v -> O0
constexpr uint32_t kA_B = 49152;     // 16 KB: Kb -> T -> Uv
constexpr uint32_t kA_G = 65536;     // 32 KB: log_alpha (fp32, or bf16 in the upper 16 KB) -> g fp32 [64][128]
                                     //   -> A / X fp32 [64][68] + scratch + P tile
constexpr uint32_t kA_Ysc = kA_G + 17408;   // solve scratch 32 x 36 fp32
constexpr uint32_t kA_P = kA_G + 22528;     // P bf16 [64][64] tile (1024-aligned)
constexpr uint32_t kA_Misc = kA_G + 32768;  // small arrays, TMEM address, flags, mbarriers (4 KB)
constexpr uint32_t kA_Smem = kA_Misc + 4096 + 1024;  // + 1024 for aligning the dynamic base
constexpr int kGS = 128;             // row stride of the g tile (floats)
constexpr int kACopyThread = 160;    // warp 5, lane 0: issues the next log_alpha load
constexpr uint32_t kKQ_LBO = 16384;  // distance between the atom columns of the stacked [k; q] tile

__device__ __forceinline__ void bulk_s2g(void* dst, uint32_t src_smem, uint32_t bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src_smem), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// (chunk, head) unit u = chunk * H + head -> head, sequence, first token, length
__device__ __forceinline__ void tc_unit(long long u, int H, const int* __restrict__ off, const int32_t* __restrict__ cu,
                                        int Tseq, int N, int& h, int& n, long long& t0, int& L)
{
    const long long j = u / H;
    h = (int)(u - j * H);
    if (cu == nullptr) {  // regular batches of Tseq tokens: the chunk follows from j alone
        const int cpb = (Tseq + kChunk - 1) / kChunk;
        n = (int)(j / cpb);
        const int c = (int)(j - (long long)n * cpb);
        t0 = (long long)n * Tseq + (long long)c * kChunk;
        L = min(kChunk, Tseq - c * kChunk);
    } else {
        locate_chunk((int)j, off, cu, Tseq, N, n, t0, L);
    }
}

// PRO: some q/k or beta/gate-activation prologue bit is set (the plain instance carries none of that code)
// LA16: log_alpha arrives as bf16 (16 KB per unit, landed in the upper half of the gate region and
// widened to the fp32 g tile by the gate scan)
template <bool PRO, bool LA16>
__global__ void __launch_bounds__(kAThreads, 2)
tc_intra_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_la,
                const float* __restrict__ beta, WsHeader* __restrict__ hdr, const int* __restrict__ off,
                const int32_t* __restrict__ cu, int Tseq, int N, int H, int G, unsigned pro,
                uint8_t* __restrict__ slots)
{
    using namespace tc;
    extern __shared__ uint8_t smem_raw[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    long long nunits;
    if (cu == nullptr) {
        nunits = (long long)N * ((Tseq + kChunk - 1) / kChunk) * H;
    } else {
        if (hdr->bad) return;
        nunits = (long long)hdr->total_chunks * H;
    }
    if ((long long)blockIdx.x >= nunits) return;

    uint8_t* sm = align1024(smem_raw);
    const uint32_t sb = smem_u32(sm);
    float* s_beta = reinterpret_cast<float*>(sm + kA_Misc);          // [64]
    float* s_ref = reinterpret_cast<float*>(sm + kA_Misc + 256);     // [128] (log2 units)
    float* s_E = reinterpret_cast<float*>(sm + kA_Misc + 768);       // [128] e^{ref} (1 in the wide case)
    float* s_D = reinterpret_cast<float*>(sm + kA_Misc + 1280);      // [128] e^{g_last - ref}
    float* s_carry = reinterpret_cast<float*>(sm + kA_Misc + 1792);  // [128] rows 0..31 total
    float* s_lo = reinterpret_cast<float*>(sm + kA_Misc + 2304);     // [128] rows 32..63 min
    float* s_hi = reinterpret_cast<float*>(sm + kA_Misc + 2816);     // [128] rows 32..63 max
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + kA_Misc + 3328);
    int* s_wide = reinterpret_cast<int*>(sm + kA_Misc + 3332);
    volatile int* s_abort = reinterpret_cast<volatile int*>(sm + kA_Misc + 3336);
    const uint32_t mbar = smem_u32(sm + kA_Misc + 3344);     // MMA completions
    const uint32_t mbar_la = smem_u32(sm + kA_Misc + 3352);  // log_alpha landed
    const uint32_t mbar_kq = mbar_la + 8, mbar_v = mbar_la + 16;
    // the unit after this one, claimed and decoded by thread 0: {u, t0} and {head, length}
    long long* s_next = reinterpret_cast<long long*>(sm + kA_Misc + 3376);
    int* s_next_hl = reinterpret_cast<int*>(sm + kA_Misc + 3392);
    float* sG = reinterpret_cast<float*>(sm + kA_G);
    float* sA = reinterpret_cast<float*>(sm + kA_G);                 // after the gating pass
    float* sY = reinterpret_cast<float*>(sm + kA_Ysc);

    // TMA boxes of 64 tokens of one head; tokens past the tensor's end arrive as zeros
    auto issue_la = [&](int hh, long long tt) {
        mbar_arrive_expect_tx(mbar_la, LA16 ? 16384 : 32768);
        tma_load_3d(sb + kA_G + (LA16 ? 16384 : 0), &tm_la, 0, hh, (int)tt, mbar_la);
    };
    auto issue_kq = [&](int hh, long long tt) {  // stacked tile: atom column a = k rows then q rows
        const int hq = hh / G;                         // the q/k head of value head hh (grouped heads)
        mbar_arrive_expect_tx(mbar_kq, 4 * 8192);
        tma_load_3d(sb + kA_KQ, &tm_k, 0, hq, (int)tt, mbar_kq);
        tma_load_3d(sb + kA_KQ + 8192, &tm_q, 0, hq, (int)tt, mbar_kq);
        tma_load_3d(sb + kA_KQ + kKQ_LBO, &tm_k, 64, hq, (int)tt, mbar_kq);
        tma_load_3d(sb + kA_KQ + kKQ_LBO + 8192, &tm_q, 64, hq, (int)tt, mbar_kq);
    };
    auto issue_v = [&](int hh, long long tt) {
        mbar_arrive_expect_tx(mbar_v, 2 * 8192);
        tma_load_3d(sb + kA_V, &tm_v, 0, hh, (int)tt, mbar_v);
        tma_load_3d(sb + kA_V + 8192, &tm_v, 64, hh, (int)tt, mbar_v);
    };
    auto issue_beta = [&](int hh, long long tt, int LL) {  // threads 0..63; rows past the end read as 0
        cp_async4(sb + kA_Misc + 4 * tid, beta + (size_t)(tt + (tid < LL ? tid : 0)) * H + hh, tid < LL ? 4u : 0u);
    };

    int h, n, L;
    long long t0;
    tc_unit(blockIdx.x, H, off, cu, Tseq, N, h, n, t0, L);
    if (tid == 0) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        prefetch_tensormap(&tm_la);
        *s_abort = 0;
        mbar_init(mbar, 1);
        mbar_init(mbar_la, 1);
        mbar_init(mbar_kq, 1);
        mbar_init(mbar_v, 1);
        mbar_fence_init();
        issue_la(h, t0);
        issue_kq(h, t0);
        issue_v(h, t0);
    }
    if (tid < 64) issue_beta(h, t0, L);
    if (warp == 0) {
        tmem_alloc(smem_u32(s_tmem), 256);
        tmem_relinquish();
    }
    fence_before_sync();
    __syncthreads();  // mbarriers initialised, TMEM address visible
    fence_after_sync();
    const uint32_t tmem = *s_tmem;
    const int ch = tid & 15, rb = tid >> 4;  // element-wise passes: chunk ch of rows rb + 16 jj
    const int wq = warp & 3;
    const int rowq = 16 * wq + (lane & 15);  // M = 64 accumulator row held by this thread
    const int hc = (lane >> 4) * 64;         // ... and its half of the 128 columns
    const uint32_t trow = tmem + ((uint32_t)(32 * wq) << 16);
    const int c = tid & 127, hf = tid >> 7;  // gate scan: channel c, rows 32 hf .. 32 hf + 31
    uint32_t mphase = 0;
    bool ok = true, has_next = false;
    int it = 0;

    for (long long u = blockIdx.x; u < nunits; ++it) {
        int claim = 0;  // thread 0: the next unit (gridDim.x + claim), from the work counter
        if (tid == 0) claim = atomicAdd(&hdr->next_unit, 1);
        const uint32_t par = (uint32_t)it & 1u;
        uint8_t* slot = slots + (size_t)u * kSlotBytes;

        if (tid == 0) *s_wide = 0;
        ok = mbar_wait_ab(mbar_la, par, s_abort) && ok;
        if (L < 64) {  // rows past the sequence (another sequence's tokens, or zeros): identity steps
            ok = mbar_wait_ab(mbar_kq, par, s_abort) && ok;
            ok = mbar_wait_ab(mbar_v, par, s_abort) && ok;
            for (int e = tid; e < (64 - L) * 16; e += kAThreads) {
                const int r = L + (e >> 4), chh = e & 15;
                *reinterpret_cast<uint4*>(sm + kA_KQ + sw128_chunk_off(r, chh, 128)) = make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4*>(sm + kA_KQ + sw128_chunk_off(64 + r, chh, 128)) = make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4*>(sm + kA_V + sw128_chunk_off(r, chh, 64)) = make_uint4(0, 0, 0, 0);
            }
            if (!LA16)
                for (int e = tid; e < (64 - L) * 32; e += kAThreads)
                    *reinterpret_cast<float4*>(sG + (L + (e >> 5)) * kGS + 4 * (e & 31)) = make_float4(0.f, 0.f, 0.f, 0.f);
            __syncthreads();
        }

        // cumulative gate in log2 units (g2 = log2(e) g): thread (c, hf) scans rows 32 hf .. 32 hf + 31
        float gl[32];
        {
            // rows past the sequence contribute nothing (identity steps), whatever their input
            const bool logits = PRO && (pro & KDA_PROLOGUE_GATE_LOGITS) != 0;
            const __nv_bfloat16* sG16 = reinterpret_cast<const __nv_bfloat16*>(sm + kA_G + 16384);
            float acc = 0.f;
#pragma unroll
            for (int u2 = 0; u2 < 32; ++u2) {
                const float x = LA16 ? __bfloat162float(sG16[(32 * hf + u2) * 128 + c]) : sG[(32 * hf + u2) * kGS + c];
                const float l2 = logits ? log2_sigmoid(x) : x * kLog2e;
                acc += (32 * hf + u2 < L) ? l2 : 0.f;
                gl[u2] = acc;
            }
        }
        if (hf == 0) s_carry[c] = gl[31];
        __syncthreads();
        float lo, hi;
        if (hf == 1) {
            const float cr = s_carry[c];
            lo = hi = cr;
#pragma unroll
            for (int u2 = 0; u2 < 32; ++u2) {
                gl[u2] += cr;
                lo = fminf(lo, gl[u2]);
                hi = fmaxf(hi, gl[u2]);
            }
            s_lo[c] = lo;
            s_hi[c] = hi;
            s_D[c] = gl[31];  // g_last, turned into e^{g_last - ref} below
        } else {
            lo = hi = 0.f;  // the chunk start (g = 0) is part of the range
#pragma unroll
            for (int u2 = 0; u2 < 32; ++u2) {
                lo = fminf(lo, gl[u2]);
                hi = fmaxf(hi, gl[u2]);
            }
        }
#pragma unroll
        // (LA16: the bf16 source under rows 32..63 has been read by every thread before the barrier above)
        for (int u2 = 0; u2 < 32; ++u2) sG[(32 * hf + u2) * kGS + c] = gl[u2];
        __syncthreads();
        if (hf == 0) {
            lo = fminf(lo, s_lo[c]);
            hi = fmaxf(hi, s_hi[c]);
            const float ref = 0.5f * (lo + hi);
            const float glast = s_D[c];
            s_ref[c] = ref;
            s_E[c] = ex2_approx(ref);
            s_D[c] = ex2_approx(glast - ref);
            *reinterpret_cast<float*>(slot + kSlotGam + 4 * c) = ex2_approx(glast);
            if (!(hi - lo <= kTcFactorSpread)) atomicOr(s_wide, 1);
        }
        if (tid == 0) {  // decode the claimed next unit for the prefetches below
            int hh = 0, nn = 0, LL = 0;
            long long tt = 0;
            const long long un = (long long)gridDim.x + claim;
            if (un < nunits) tc_unit(un, H, off, cu, Tseq, N, hh, nn, tt, LL);
            s_next[0] = un;
            s_next[1] = tt;
            s_next_hl[0] = hh;
            s_next_hl[1] = LL;
        }
        ok = mbar_wait_ab(mbar_kq, par, s_abort) && ok;  // k and q in place
        cp_async_wait_all();                             // beta in place
        if (PRO && (pro & KDA_PROLOGUE_BETA_LOGITS) && tid < 64) s_beta[tid] = tid < L ? sigmoid_f(s_beta[tid]) : 0.f;
        __syncthreads();
        has_next = s_next[0] < nunits;
        const bool wide = *s_wide != 0;
        if (PRO && (pro & KDA_PROLOGUE_L2NORM_QK)) {
            // k and q rows normalised in place (fp32 norms over the 128 channels held by the 16 threads
            // of a half-warp, then rounded back to bf16) before anything reads them
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const int r = rb + 16 * jj;
                uint4* pk = reinterpret_cast<uint4*>(sm + kA_KQ + sw128_chunk_off(r, ch, 128));
                uint4* pq = reinterpret_cast<uint4*>(sm + kA_KQ + sw128_chunk_off(64 + r, ch, 128));
                float kv[8], qv[8];
                unpack8(*pk, kv);
                unpack8(*pq, qv);
                float sk = 0.f, sq = 0.f;
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    sk = fmaf(kv[m], kv[m], sk);
                    sq = fmaf(qv[m], qv[m], sq);
                }
#pragma unroll
                for (int o = 1; o < 16; o <<= 1) {
                    sk += __shfl_xor_sync(0xffffffffu, sk, o);
                    sq += __shfl_xor_sync(0xffffffffu, sq, o);
                }
                const float ik = rsqrtf(sk + kQkNormEps), iq = rsqrtf(sq + kQkNormEps);
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    kv[m] *= ik;
                    qv[m] *= iq;
                }
                *pk = pack8(kv);
                *pq = pack8(qv);
            }
            __syncthreads();
        }

        if (!wide) {
            // a lane's 8 channels span 32 bytes of fp32 rows: lanes 4-7 of each quarter-warp read their
            // upper 16 bytes first, so that one 128-bit load instruction covers all eight 16-byte bank
            // groups of a 128-byte line (no two-way conflict)
            const int h0 = 4 * ((ch >> 2) & 1);
            float ref8[8], d8[8];
            {
                const float4 a0 = *reinterpret_cast<const float4*>(s_ref + 8 * ch + h0);
                const float4 a1 = *reinterpret_cast<const float4*>(s_ref + 8 * ch + (h0 ^ 4));
                const float4 b0 = *reinterpret_cast<const float4*>(s_D + 8 * ch + h0);
                const float4 b1 = *reinterpret_cast<const float4*>(s_D + 8 * ch + (h0 ^ 4));
                const float x0[4] = {a0.x, a0.y, a0.z, a0.w}, x1[4] = {a1.x, a1.y, a1.z, a1.w};
                const float y0[4] = {b0.x, b0.y, b0.z, b0.w}, y1[4] = {b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    ref8[m] = h0 ? x1[m] : x0[m];
                    ref8[m + 4] = h0 ? x0[m] : x1[m];
                    d8[m] = h0 ? y1[m] : y0[m];
                    d8[m + 4] = h0 ? y0[m] : y1[m];
                }
            }
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const int r = rb + 16 * jj;
                const uint32_t ok_ = sw128_chunk_off(r, ch, 128), oq = sw128_chunk_off(64 + r, ch, 128);
                float kv[8], qv[8];
                unpack8(*reinterpret_cast<const uint4*>(sm + kA_KQ + ok_), kv);
                unpack8(*reinterpret_cast<const uint4*>(sm + kA_KQ + oq), qv);
                const float4 ga = *reinterpret_cast<const float4*>(sG + r * kGS + 8 * ch + h0);
                const float4 gb = *reinterpret_cast<const float4*>(sG + r * kGS + 8 * ch + (h0 ^ 4));
                const float gx[4] = {ga.x, ga.y, ga.z, ga.w}, gy[4] = {gb.x, gb.y, gb.z, gb.w};
                float g8[8];
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    g8[m] = h0 ? gy[m] : gx[m];
                    g8[m + 4] = h0 ? gx[m] : gy[m];
                }
                float kf[8], qf[8], kb[8], kd[8];
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const float x = g8[m] - ref8[m];
                    const float ef = ex2_approx(x), eb = ex2_approx(-x);
                    kf[m] = kv[m] * ef;
                    qf[m] = qv[m] * ef;
                    kb[m] = kv[m] * eb;
                    kd[m] = kb[m] * d8[m];
                }
                const uint32_t okd = sw128_chunk_off(r, ch, 64);
                *reinterpret_cast<uint4*>(sm + kA_KQ + ok_) = pack8(kf);
                *reinterpret_cast<uint4*>(sm + kA_KQ + oq) = pack8(qf);
                *reinterpret_cast<uint4*>(sm + kA_B + okd) = pack8(kb);
                *reinterpret_cast<uint4*>(slot + kSlotKd + okd) = pack8(kd);  // Kd = Kb diag(e^{g_last - ref})
            }
            fence_proxy_async();
            __syncthreads();
            if (tid == 0 && ok) {  // [A'; P'] = [Kf; Qf] Kb^T: one M = 128 batch
                fence_after_sync();
                const uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
                for (int kk = 0; kk < 128; kk += 16)
                    mma_bf16(tmem + 0, desc_kmajor(sb + kA_KQ, 128, kk), desc_kmajor(sb + kA_B, 64, kk), id, kk > 0);
                mma_commit(mbar);
            }
            ok = mbar_wait_ab(mbar, mphase, s_abort) && ok;
            mphase ^= 1;
            fence_after_sync();
            {   // warps 0,1 (and 4,5): A' rows 0..63; warps 2,3 (and 6,7): P' rows; warps < 4 columns 0..31, >= 4 32..63
                const int col0 = (warp >> 2) * 32;
                float a[32];
                tmem_ld16(tmem + ((uint32_t)(32 * wq) << 16) + col0, a);
                tmem_ld16(tmem + ((uint32_t)(32 * wq) << 16) + col0 + 16, a + 16);
                tmem_wait_ld();
                if (wq < 2) {
                    const int r = 32 * wq + lane;
                    const float br = s_beta[r];
#pragma unroll
                    for (int m = 0; m < 32; m += 4) {
                        const int i = col0 + m;
                        *reinterpret_cast<float4*>(sA + r * kAS + i) =
                            make_float4(i < r ? br * a[m] : 0.f, i + 1 < r ? br * a[m + 1] : 0.f,
                                        i + 2 < r ? br * a[m + 2] : 0.f, i + 3 < r ? br * a[m + 3] : 0.f);
                    }
                } else {
                    const int r = 32 * (wq - 2) + lane;
#pragma unroll
                    for (int m = 0; m < 32; ++m) a[m] = (col0 + m <= r) ? a[m] : 0.f;
#pragma unroll
                    for (int m = 0; m < 4; ++m)
                        *reinterpret_cast<uint4*>(sm + kA_P + sw128_chunk_off(r, (col0 >> 3) + m, 64)) = pack8(a + 8 * m);
                }
            }
        } else {
            // some channel's gate spreads beyond e^159: exact per-element factors on CUDA cores
            float av[16], pv[16];
#pragma unroll 1
            for (int m = 0; m < 16; ++m) {
                const int e = tid + kAThreads * m;
                const int r = e >> 6, i = e & 63;
                float a = 0.f, p = 0.f;
                if (i <= r) {
                    for (int cc = 0; cc < 128; ++cc) {
                        const float kk = lds_bf16(sm + kA_KQ + sw128_off(i, cc, 128)) * ex2_approx(sG[r * kGS + cc] - sG[i * kGS + cc]);
                        a = fmaf(lds_bf16(sm + kA_KQ + sw128_off(r, cc, 128)), kk, a);
                        p = fmaf(lds_bf16(sm + kA_KQ + sw128_off(64 + r, cc, 128)), kk, p);
                    }
                }
                av[m] = (i < r) ? s_beta[r] * a : 0.f;
                pv[m] = p;
            }
            __syncthreads();  // every thread is done reading raw k and q across rows
            // in place: k -> k e^g (B operand of W), q -> q e^g; Kd = k e^{g_last - g} straight to the slot
#pragma unroll 1
            for (int jj = 0; jj < 4; ++jj) {
                const int r = rb + 16 * jj;
                const uint32_t ok_ = sw128_chunk_off(r, ch, 128), oq = sw128_chunk_off(64 + r, ch, 128);
                float kv[8], qv[8], kt[8], kd[8], qg[8];
                unpack8(*reinterpret_cast<const uint4*>(sm + kA_KQ + ok_), kv);
                unpack8(*reinterpret_cast<const uint4*>(sm + kA_KQ + oq), qv);
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const float gv = sG[r * kGS + 8 * ch + m], gz = sG[63 * kGS + 8 * ch + m];
                    const float eg = ex2_approx(gv);
                    kt[m] = kv[m] * eg;
                    qg[m] = qv[m] * eg;
                    kd[m] = kv[m] * ex2_approx(gz - gv);
                }
                *reinterpret_cast<uint4*>(sm + kA_KQ + ok_) = pack8(kt);
                *reinterpret_cast<uint4*>(sm + kA_KQ + oq) = pack8(qg);
                *reinterpret_cast<uint4*>(slot + kSlotKd + sw128_chunk_off(r, ch, 64)) = pack8(kd);
            }
            __syncthreads();  // g no longer read: A and the P tile take its place
            for (int cc = tid; cc < 128; cc += kAThreads) s_E[cc] = 1.f;
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                const int e = tid + kAThreads * m;
                const int r = e >> 6, i = e & 63;
                sA[r * kAS + i] = av[m];
                *reinterpret_cast<__nv_bfloat16*>(sm + kA_P + sw128_off(r, i, 64)) = __float2bfloat16_rn(pv[m]);
            }
        }
        fence_before_sync();
        ok = __syncthreads_and(ok);  // A and the P tile complete; the tensor core is done with Kb

        // UT transform: T = (I + A)^{-1} diag(beta) as a bf16 K-major tile over Kb (MMA1 has read Kb)
        if (ok) ut_transform_T(sA, sY, s_beta, sm + kA_B);
        if (tid == 0) ok = mbar_wait_ab(mbar_v, par, s_abort) && ok;  // v in place
        if (ok && tid == 0) {  // W' = T Kf (B: k rows of the stacked tile), Uv = T v
            fence_after_sync();
            const uint32_t id = idesc_bf16(64, 128, false, true);
#pragma unroll
            for (int kk = 0; kk < 64; kk += 16) {
                mma_bf16(tmem + 0, desc_kmajor(sb + kA_B, 64, kk), desc_sw128(sb + kA_KQ + kk * 128, kKQ_LBO, 1024u), id, kk > 0);
                mma_bf16(tmem + 128, desc_kmajor(sb + kA_B, 64, kk), desc_mnmajor(sb + kA_V, 64, kk), id, kk > 0);
            }
            mma_commit(mbar);
        }
        ok = mbar_wait_ab(mbar, mphase, s_abort) && ok;
        mphase ^= 1;
        ok = mbar_wait_ab(mbar_v, par, s_abort) && ok;  // (long complete) orders this thread after the v copy
        fence_after_sync();
        ok = __syncthreads_and(ok);
        if (ok) {
            if (warp < 4) {  // W = W' diag(e^ref) -> the k rows of the stacked tile (Kf consumed)
#pragma unroll
                for (int b2 = 0; b2 < 64; b2 += 32) {
                    float a2[32];
                    tmem_ld16_pair<64>(trow + b2, a2);
                    tmem_ld16_pair<64>(trow + b2 + 16, a2 + 16);
                    tmem_wait_ld();
#pragma unroll
                    for (int m = 0; m < 32; m += 4) {
                        const float4 e4 = *reinterpret_cast<const float4*>(s_E + hc + b2 + m);
                        a2[m] *= e4.x; a2[m + 1] *= e4.y; a2[m + 2] *= e4.z; a2[m + 3] *= e4.w;
                    }
#pragma unroll
                    for (int m = 0; m < 4; ++m)
                        *reinterpret_cast<uint4*>(sm + kA_KQ + sw128_chunk_off(rowq, (hc + b2) / 8 + m, 128)) = pack8(a2 + 8 * m);
                }
            } else {  // Uv -> the T tile's place (T consumed)
#pragma unroll
                for (int b2 = 0; b2 < 64; b2 += 32) {
                    float a2[32];
                    tmem_ld16_pair<64>(trow + 128 + b2, a2);
                    tmem_ld16_pair<64>(trow + 128 + b2 + 16, a2 + 16);
                    tmem_wait_ld();
#pragma unroll
                    for (int m = 0; m < 4; ++m)
                        *reinterpret_cast<uint4*>(sm + kA_B + sw128_chunk_off(rowq, (hc + b2) / 8 + m, 64)) = pack8(a2 + 8 * m);
                }
            }
        }
        fence_proxy_async();
        fence_before_sync();
        ok = __syncthreads_and(ok);
        if (tid == 0) {
            if (ok) {
                // W and Uv images out (bulk), then [P W | P Uv] = P [W | Uv]
                bulk_s2g(slot + kSlotW, sb + kA_KQ, 8192);
                bulk_s2g(slot + kSlotW + 8192, sb + kA_KQ + kKQ_LBO, 8192);
                bulk_s2g(slot + kSlotUv, sb + kA_B, 16384);
                bulk_commit();
                fence_after_sync();
                const uint32_t id = idesc_bf16(64, 128, false, true);
#pragma unroll
                for (int kk = 0; kk < 64; kk += 16) {
                    mma_bf16(tmem + 0, desc_kmajor(sb + kA_P, 64, kk), desc_sw128(sb + kA_KQ + kk * 128, kKQ_LBO, 1024u), id, kk > 0);
                    mma_bf16(tmem + 128, desc_kmajor(sb + kA_P, 64, kk), desc_mnmajor(sb + kA_B, 64, kk), id, kk > 0);
                }
                mma_commit(mbar);
            }
        }
        ok = mbar_wait_ab(mbar, mphase, s_abort) && ok;
        mphase ^= 1;
        fence_after_sync();
        ok = __syncthreads_and(ok);
        if (has_next) {  // the log_alpha region is free (P consumed) and beta has been read.  Copies are
                         // issued by lanes of different warps, so that no single thread on the
                         // critical path waits for all of them.
            if (tid == kACopyThread) issue_la(s_next_hl[0], s_next[1]);
            if (tid < 64) issue_beta(s_next_hl[0], s_next[1], s_next_hl[1]);
        }
        if (ok) {
            if (warp < 4) {  // Q' = Qf e^ref - P W -> the q rows of the stacked tile, in place
#pragma unroll
                for (int b2 = 0; b2 < 64; b2 += 32) {
                    float a2[32];
                    tmem_ld16_pair<64>(trow + b2, a2);
                    tmem_ld16_pair<64>(trow + b2 + 16, a2 + 16);
                    tmem_wait_ld();
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        uint4* p = reinterpret_cast<uint4*>(sm + kA_KQ + sw128_chunk_off(64 + rowq, (hc + b2) / 8 + m, 128));
                        float qf[8];
                        unpack8(*p, qf);
                        const float4 e0 = *reinterpret_cast<const float4*>(s_E + hc + b2 + 8 * m);
                        const float4 e1 = *reinterpret_cast<const float4*>(s_E + hc + b2 + 8 * m + 4);
                        const float ev[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
#pragma unroll
                        for (int e = 0; e < 8; ++e) qf[e] = qf[e] * ev[e] - a2[8 * m + e];
                        *p = pack8(qf);
                    }
                }
            } else {  // O0 = P Uv -> the v tile's place (MMA2 has read v; the Uv image may still be leaving)
#pragma unroll
                for (int b2 = 0; b2 < 64; b2 += 32) {
                    float a2[32];
                    tmem_ld16_pair<64>(trow + 128 + b2, a2);
                    tmem_ld16_pair<64>(trow + 128 + b2 + 16, a2 + 16);
                    tmem_wait_ld();
#pragma unroll
                    for (int m = 0; m < 4; ++m)
                        *reinterpret_cast<uint4*>(sm + kA_V + sw128_chunk_off(rowq, (hc + b2) / 8 + m, 64)) = pack8(a2 + 8 * m);
                }
            }
            // the warp's 16 rows of its image (Q' or O0) leave at once: one 2 KB run per atom column.
            // The issuing lane waits until they have been read (bulk groups are per thread); thread 0's
            // wait also covers the W and Uv images.
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) {
                const uint32_t src = warp < 4 ? sb + kA_KQ + 8192 + 2048 * wq : sb + kA_V + 2048 * wq;
                const uint32_t lbo = warp < 4 ? kKQ_LBO : 8192u;
                uint8_t* dst = slot + (warp < 4 ? kSlotQ : kSlotO0) + 2048 * wq;
                bulk_s2g(dst, src, 2048);
                bulk_s2g(dst + 8192, src + lbo, 2048);
                bulk_commit();
            }
        }
        if (lane == 0) bulk_wait_read();  // every image of this unit has been read out of shared memory
        fence_before_sync();
        ok = __syncthreads_and(ok);  // the next chunk's tiles (k, q, v; Kb over the Uv image) may land from here on
        if (has_next) {
            if (tid == 0) issue_kq(s_next_hl[0], s_next[1]);
            if (tid == 32) issue_v(s_next_hl[0], s_next[1]);
        }
        if (!ok) break;
        u = s_next[0];
        t0 = s_next[1];
        h = s_next_hl[0];
        L = s_next_hl[1];
    }
    if (tid == 0 && !ok && has_next) {  // loads for the next chunk may still be landing: bounded waits
        const uint32_t pn = ((uint32_t)it + 1u) & 1u;
        (void)mbar_wait(mbar_la, pn);
        (void)mbar_wait(mbar_kq, pn);
        (void)mbar_wait(mbar_v, pn);
    }
    if (lane == 0) bulk_wait_all();  // every lane that issued image stores
    cp_async_wait_all();
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// ------------------------------------------------------------------------------------------------
// Phase B
// ------------------------------------------------------------------------------------------------
constexpr int kBCompute = 128;              // 4 compute warps: thread c owns row c of the state slice
constexpr int kBThreads = kBCompute + 64;   // + MMA-issue warp (4) + bulk-copy warp (5)
constexpr int kBStages = 3;
// stage: [W; Q'] stacked 128-row tile (32 KB) | Kd (16 KB) | the Uv and O0 atom columns holding this
// CTA's 32-column slice (8 KB each) | e^{g_last} (512 B)
constexpr uint32_t kStWQ = 0, kStKd = 32768, kStUv = 49152, kStO0 = 57344, kStGam = 65536;
constexpr uint32_t kStTx = 66048;           // bytes landing per stage
constexpr uint32_t kStageBytes = 66560;     // 65 KB, 1024-aligned
constexpr uint32_t kB_S = kBStages * kStageBytes;  // S slice: bf16 [128 rows][64] SW128 (32 columns used)
constexpr uint32_t kB_U = kB_S + 16384;            // U:       bf16 [64 rows][64]  SW128 (32 columns used)
constexpr uint32_t kB_Misc = kB_U + 8192;          // mbarriers + TMEM address
constexpr uint32_t kB_Smem = kB_Misc + 256 + 1024;
constexpr uint32_t kTmD1 = 0, kTmY = 32;           // TMEM columns: [X; O'] and Y

// The output gate in phase B's epilogue, y = o / sqrt(mean_group(o^2) + eps) * w * act(z) (the grouped,
// gated RMS norm of the attention review's GDN/KDA pseudo-code and Ring-linear notes), computed from the
// fp32 o = O' + O0 before it is rounded: o is never written.  A group of 8, 16 or 32 channels lies inside
// one CTA's 32-column slice (kGateLocal); a group of 64 or 128 spans 2 or 4 slices, whose CTAs run as one
// 4-CTA cluster and trade per-row partial sums of squares through distributed shared memory (kGateCluster).
struct OutGate {
    const __nv_bfloat16* z;  // [tokens][H][128], the layout of out
    const float* w;          // [128] fp32, or nullptr (= ones)
    float inv_g, eps;        // 1 / group, eps
    int group;               // channels per norm group: 8, 16, 32, 64 or 128
    int sigmoid;             // act = sigmoid (1) or identity (0)
};
constexpr int kGateNone = 0, kGateLocal = 1, kGateCluster = 2;
// gated variants: the slice of w at kB_Misc + 256 (128 B); partial sums xs[2 parities][4 slices][64 rows]
// fp32 at kB_Misc + 512 (2 KB); two exchange mbarriers at kB_Misc + 64; the next chunk's z rows (64 x 64 B,
// 16-byte chunk m of row r at chunk m ^ ((r >> 1) & 3)) at kB_Z
constexpr uint32_t kB_W = kB_Misc + 256, kB_X = kB_Misc + 512, kB_Z = kB_X + 2048;
constexpr uint32_t kB_SmemGate = kB_Z + 4096 + 1024;
static_assert(kB_SmemGate <= 232448, "phase B shared memory");

__device__ __forceinline__ void tc_issue_stage(uint32_t stage_addr, uint32_t full_bar, const uint8_t* slot, int vt)
{
    using namespace tc;
    mbar_arrive_expect_tx(full_bar, kStTx);
    // [W; Q'] as one 128-row tile: atom column a holds W rows then Q' rows
    bulk_g2s(stage_addr + kStWQ, slot + kSlotW, 8192, full_bar);
    bulk_g2s(stage_addr + kStWQ + 8192, slot + kSlotQ, 8192, full_bar);
    bulk_g2s(stage_addr + kStWQ + 16384, slot + kSlotW + 8192, 8192, full_bar);
    bulk_g2s(stage_addr + kStWQ + 24576, slot + kSlotQ + 8192, 8192, full_bar);
    bulk_g2s(stage_addr + kStKd, slot + kSlotKd, 16384, full_bar);
    bulk_g2s(stage_addr + kStUv, slot + kSlotUv + (vt >> 1) * 8192, 8192, full_bar);
    bulk_g2s(stage_addr + kStO0, slot + kSlotO0 + (vt >> 1) * 8192, 8192, full_bar);
    bulk_g2s(stage_addr + kStGam, slot + kSlotGam, 512, full_bar);
}

// the same regions of a chunk's slot, into L2 only, a few chunks before tc_issue_stage needs them
__device__ __forceinline__ void tc_prefetch_stage(const uint8_t* slot, int vt)
{
    using namespace tc;
    bulk_prefetch_l2(slot + kSlotW, 16384);
    bulk_prefetch_l2(slot + kSlotQ, 16384);
    bulk_prefetch_l2(slot + kSlotKd, 16384);
    bulk_prefetch_l2(slot + kSlotUv + (vt >> 1) * 8192, 8192);
    bulk_prefetch_l2(slot + kSlotO0 + (vt >> 1) * 8192, 8192);
    bulk_prefetch_l2(slot + kSlotGam, 512);
}
constexpr int kBPrefetch = 4;  // L2 prefetch distance beyond the shared-memory stages (chunks)

// row r of chunk j of the sequence [s0, s1): this CTA's 32 columns of z, copied asynchronously into the
// row's 64 bytes at kB_Z (cp.async: no register waits on the load; rows past the end are zero-filled)
__device__ __forceinline__ void copy_z_row(uint32_t zbuf, const __nv_bfloat16* z, long long s0, long long s1, int j,
                                           int r, int H, int h, int v0)
{
    const long long t0 = s0 + (long long)j * 64;
    const bool in = t0 + r < s1;
    const uint8_t* src = reinterpret_cast<const uint8_t*>(z + ((size_t)(t0 + (in ? r : 0)) * H + h) * 128 + v0);
#pragma unroll
    for (int m = 0; m < 4; ++m)
        cp_async16(zbuf + (uint32_t)(r * 64 + ((m ^ ((r >> 1) & 3)) << 4)), src + 16 * m, in ? 16u : 0u);
}

template <int GATE>
__global__ void __launch_bounds__(GATE == kGateNone ? kBThreads : kBThreads + 64, 1)
tc_inter_kernel(const float* S0, float* S_final, __nv_bfloat16* __restrict__ out, const WsHeader* __restrict__ hdr,
                const int* __restrict__ off, const int32_t* __restrict__ cu, int Tseq, int N, int H,
                const uint8_t* __restrict__ slots, OutGate gate)
{
    using namespace tc;
    extern __shared__ uint8_t smem_raw[];
    // 1-D grid, longest sequences first: CTA L -> (sequence order[L / (4H)], head, 32-column slice)
    const int L_cta = blockIdx.x, per_seq = 4 * H;
    const int rank = L_cta / per_seq, rem = L_cta - rank * per_seq;
    const int n = off[N + 1 + rank], h = rem >> 2, vt = rem & 3, v0 = vt * kTcNV;
    const int cq = 4 * (vt & 1);  // first 16-byte chunk of this slice inside its Uv / O0 atom column
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (hdr->bad) return;
    uint8_t* sm = align1024(smem_raw);
    const uint32_t sb = smem_u32(sm);
    const uint32_t bar_full = smem_u32(sm + kB_Misc);   // kBStages barriers
    const uint32_t bar_d1 = bar_full + 8 * kBStages;    // [X; O'] ready
    const uint32_t bar_y = bar_d1 + 8;                  // Y ready
    const uint32_t bar_empty = bar_y + 8;               // kBStages barriers: stage consumed (128 arrivals)
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + kB_Misc + 128);
    volatile int* s_abort = reinterpret_cast<volatile int*>(sm + kB_Misc + 132);
    const uint32_t bar_x = smem_u32(sm + kB_Misc + 64);  // kGateCluster: 2 exchange barriers (by chunk parity)
    volatile int* s_xabort = reinterpret_cast<volatile int*>(sm + kB_Misc + 136);  // the exchange gave up

    const int jb = off[n], je = off[n + 1], nch = je - jb;
    const uint8_t* hslots = slots + (size_t)h * kSlotBytes;  // this head's slots, H slots apart
    long long s0, s1;
    seq_bounds(n, cu, Tseq, s0, s1);

    if (tid == 0) {
        for (int s = 0; s < kBStages; ++s) mbar_init(bar_full + 8 * s, 1);
        mbar_init(bar_d1, 1);
        mbar_init(bar_y, 1);
        for (int s = 0; s < kBStages; ++s) mbar_init(bar_empty + 8 * s, GATE == kGateNone ? kBCompute : kBCompute + 64);
        if (GATE == kGateCluster) {  // one local arrival (with the expected bytes) per phase
            mbar_init(bar_x, 1);
            mbar_init(bar_x + 8, 1);
        }
        mbar_fence_init();
        *s_abort = 0;
        if (GATE == kGateCluster) *s_xabort = 0;
    }
    if (GATE != kGateNone && tid < kTcNV)
        reinterpret_cast<float*>(sm + kB_W)[tid] = gate.w ? gate.w[v0 + tid] : 1.f;
    if (warp == 0) {
        tmem_alloc(smem_u32(s_tmem), 64);
        tmem_relinquish();
    }
    const int c = tid;  // compute threads: state row
    float S[kTcNV];
    const size_t srow = (((size_t)n * H + h) * 128 + (c & 127)) * 128 + v0;
    if (warp < 4) {
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
        for (int m = 0; m < 4; ++m) *reinterpret_cast<uint4*>(sm + kB_S + sw128_chunk_off(c, m, 128)) = pack8(S + 8 * m);
    }
    fence_proxy_async();
    if (GATE == kGateCluster)
        cluster_sync();  // also every peer's exchange barriers initialised before the first remote arrival
    else
        __syncthreads();  // barriers initialised, TMEM address visible, S tile written
    if (warp == 5 && lane == 0) {
        for (int s = 0; s < kBStages && s < nch; ++s)
            tc_issue_stage(sb + s * kStageBytes, bar_full + 8 * s, hslots + (size_t)(jb + s) * H * kSlotBytes, vt);
        for (int s = kBStages; s < kBStages + kBPrefetch && s < nch; ++s)
            tc_prefetch_stage(hslots + (size_t)(jb + s) * H * kSlotBytes, vt);
    }
    const uint32_t tmem = *s_tmem;
    const uint32_t tw = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
    const uint32_t id_d1 = idesc_bf16(128, kTcNV, false, true);  // [W; Q'] S   (S MN-major)
    const uint32_t id_y = idesc_bf16(128, kTcNV, true, true);    // Kd^T U      (Kd, U MN-major)
    // descriptor bases; per K step only the 14-bit start address field advances (never carries)
    const uint64_t dS = desc_sw128(sb + kB_S, 128 * 128, 1024u), dU = desc_sw128(sb + kB_U, 64 * 128, 1024u);
    bool ok = true;
    if (GATE != kGateNone && warp >= 6 && nch > 0)  // gated epilogue warps: the first chunk's z rows
        copy_z_row(sb + kB_Z, gate.z, s0, s1, 0, tid - kBThreads, H, h, v0);
    // kGateCluster: the partial-sum array and exchange barriers of the other CTAs of this CTA's group, as
    // shared::cluster addresses (the same offsets in every CTA)
    uint32_t peer_x[3] = {0, 0, 0}, peer_bar[3] = {0, 0, 0};
    const int npeer = gate.group == 128 ? 3 : 1;  // a 128-channel group spans all four slices, 64 a pair
    if (GATE == kGateCluster && warp >= 6) {
#pragma unroll
        for (int q = 0; q < 3; ++q) {
            const uint32_t pv = gate.group == 128 ? (uint32_t)((vt + 1 + q) & 3) : (uint32_t)(vt ^ 1);
            peer_x[q] = cluster_map(smem_u32(sm + kB_X), pv);
            peer_bar[q] = cluster_map(bar_x, pv);
        }
    }

    // Roles per chunk (no CTA-wide barrier inside the loop):
    //   warp 4 (MMA)     : [X; O'] = [W; Q'] S once the S tile is ready (barrier 2), Y = Kd^T U once
    //                      the U tile is ready (barrier 1)
    //   warps 0-1        : U = Uv - X -> U tile, arrive on barrier 1
    //   warps 2-3        : out = O' + O0 (ungated)
    //   warps 0-3        : S <- e^{g_last} S + Y -> S tile; arrive on the stage's "empty" mbarrier
    //                      (stage read) and on barrier 2 (S ready)
    //   warp 5 (copies)  : refills the stage of chunk it with chunk it+3 once it is empty
    //   warps 6-7 (gated): read O' and O0, arrive on barrier 2 and the stage's "empty" mbarrier, then
    //                      form o = O' + O0 and the gated output while the next chunk runs
    // A bounded wait that gives up raises the CTA's abort flag; every later wait then fails at once,
    // so the loop still runs its barriers to the end without hanging and exits quickly.
    for (int it = 0; it < nch; ++it) {
        const int s = it % kBStages;
        const uint32_t st = sb + s * kStageBytes;
        const uint8_t* stp = sm + s * kStageBytes;
        const long long t0 = s0 + (long long)it * 64;
        const int L = (s1 - t0) < 64 ? (int)(s1 - t0) : 64;
        const uint32_t par = (uint32_t)it & 1u;
        const bool refill = it + kBStages < nch;
        if (warp == 4) {
            if (it > 0) named_sync(2, GATE == kGateNone ? 160 : 224);  // S tile written (and, gated, O' read)
            if (lane == 0) {
                ok = ok && mbar_wait_ab(bar_full + 8 * s, (uint32_t)(it / kBStages) & 1u, s_abort);
                fence_after_sync();
                if (ok) {
                    const uint64_t dA = desc_sw128(st + kStWQ, 16u, 1024u);
#pragma unroll
                    for (int kk = 0; kk < 128; kk += 16)
                        mma_bf16(tmem + kTmD1, dA + (uint64_t)((((kk >> 6) * 16384) + ((kk & 63) << 1)) >> 4),
                                 dS + (uint64_t)((kk * 128) >> 4), id_d1, kk > 0);
                    mma_commit(bar_d1);
                }
            }
            named_sync(1, 96);  // U tile written by warps 0 and 1
            if (lane == 0 && ok) {
                fence_after_sync();
                const uint64_t dK = desc_sw128(st + kStKd, 64 * 128, 1024u);
#pragma unroll
                for (int kk = 0; kk < 64; kk += 16)
                    mma_bf16(tmem + kTmY, dK + (uint64_t)((kk * 128) >> 4), dU + (uint64_t)((kk * 128) >> 4), id_y, kk > 0);
                mma_commit(bar_y);
            }
        } else if (warp == 5) {
            if (refill && lane == 0) {  // stage s fully consumed (every reader arrived) -> refill
                ok = ok && mbar_wait_ab(bar_empty + 8 * s, (uint32_t)(it / kBStages) & 1u, s_abort);
                if (ok) {
                    tc_issue_stage(st, bar_full + 8 * s, hslots + (size_t)(jb + it + kBStages) * H * kSlotBytes, vt);
                    if (it + kBStages + kBPrefetch < nch)
                        tc_prefetch_stage(hslots + (size_t)(jb + it + kBStages + kBPrefetch) * H * kSlotBytes, vt);
                }
            }
        } else if (GATE != kGateNone && warp >= 6) {
            // epilogue warps (gated): row r of O' is TMEM lane 64 + r, which warps 6 and 7 address
            const int r = tid - kBThreads;
            ok = ok && mbar_wait_ab(bar_full + 8 * s, (uint32_t)(it / kBStages) & 1u, s_abort);
            uint4 raw[4];
#pragma unroll
            for (int m = 0; m < 4; ++m)
                raw[m] = *reinterpret_cast<const uint4*>(stp + kStO0 + sw128_chunk_off(r, cq + m, 64));
            ok = ok && mbar_wait_ab(bar_d1, par, s_abort);
            fence_after_sync();
            float x[32];
            tmem_ld16(tw + kTmD1, x);
            tmem_ld16(tw + kTmD1 + 16, x + 16);
            tmem_wait_ld();
            fence_before_sync();
            if (it + 1 < nch) named_arrive(2, 224);      // O' read: the next MMA1 may overwrite it
            if (refill) mbar_arrive(bar_empty + 8 * s);  // O0 read
#pragma unroll
            for (int m = 0; m < 4; ++m) {  // o = O' + O0, kept in fp32
                float u[8];
                unpack8(raw[m], u);
#pragma unroll
                for (int e = 0; e < 8; ++e) x[8 * m + e] += u[e];
            }
            float p[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                p[m] = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) p[m] = fmaf(x[8 * m + e], x[8 * m + e], p[m]);
            }
            float rs[4];
            bool xok = true;
            const int g0 = gate.group == 128 ? 0 : (vt & 2), g1 = gate.group == 128 ? 4 : (vt & 2) + 2;
            const uint32_t bx = bar_x + 8u * (uint32_t)(it & 1);
            // this slice's share of the row's sum of squares -> its own slot and the other CTAs of the group.
            // The exchange runs whatever `ok` says, so that every CTA's phases stay matched; it stops only
            // after one of its own waits has timed out (s_xabort).
            if (GATE == kGateCluster && !*s_xabort) {
                const float part = (p[0] + p[1]) + (p[2] + p[3]);
                const uint32_t xo = 4u * (uint32_t)((it & 1) * 256 + vt * 64 + r), bo = 8u * (uint32_t)(it & 1);
                *reinterpret_cast<float*>(sm + kB_X + xo) = part;
                if (r == 0) mbar_arrive_expect_tx(bx, (uint32_t)(g1 - g0 - 1) * 64u * 4u);
#pragma unroll
                for (int q = 0; q < 3; ++q)
                    if (q < npeer) st_async_cluster_f32(peer_x[q] + xo, part, peer_bar[q] + bo);
            }
            // g = act(z) w while the partial sums travel; the next chunk's z row goes into the same shared
            // bytes as soon as this one is in registers (unpacked), a whole chunk ahead of its use
            cp_async_wait_all();
            float gz[32];
#pragma unroll
            for (int m = 0; m < 4; ++m)
                unpack8(*reinterpret_cast<const uint4*>(sm + kB_Z + r * 64 + ((m ^ ((r >> 1) & 3)) << 4)), gz + 8 * m);
            if (it + 1 < nch) copy_z_row(sb + kB_Z, gate.z, s0, s1, it + 1, r, H, h, v0);
            {
                const float4* sw = reinterpret_cast<const float4*>(sm + kB_W);
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const float4 wa = sw[2 * m], wb = sw[2 * m + 1];
                    const float w8[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        gz[8 * m + e] = w8[e] * (gate.sigmoid ? sigmoid_tanh(gz[8 * m + e]) : gz[8 * m + e]);
                }
            }
            if (GATE == kGateCluster) {
                const float* xs = reinterpret_cast<const float*>(sm + kB_X) + (it & 1) * 256 + r;
                xok = !*s_xabort && mbar_wait(bx, (uint32_t)(it >> 1) & 1u);
                if (!xok) *s_xabort = 1;
                const float ss = gate.group == 128 ? (xs[0] + xs[64]) + (xs[128] + xs[192]) : xs[g0 * 64] + xs[g0 * 64 + 64];
                rs[0] = rs[1] = rs[2] = rs[3] = rsqrtf(ss * gate.inv_g + gate.eps);
            } else {
                if (gate.group >= 16) {
                    p[0] = p[1] = p[0] + p[1];
                    p[2] = p[3] = p[2] + p[3];
                }
                if (gate.group >= 32) p[0] = p[1] = p[2] = p[3] = p[0] + p[2];
#pragma unroll
                for (int m = 0; m < 4; ++m) rs[m] = rsqrtf(p[m] * gate.inv_g + gate.eps);
            }
            if (r < L && ok && xok) {
                uint4* dst = reinterpret_cast<uint4*>(out + ((size_t)(t0 + r) * H + h) * 128 + v0);
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    float yv[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) yv[e] = x[8 * m + e] * rs[m] * gz[8 * m + e];
                    dst[m] = pack8(yv);
                }
            }
        } else {
            ok = ok && mbar_wait_ab(bar_full + 8 * s, (uint32_t)(it / kBStages) & 1u, s_abort);
            // this thread's Uv (warps 0-1) or O0 (warps 2-3) row and e^{g_last} are read before MMA1 is waited for
            uint4 raw[4];
            if (GATE == kGateNone || warp < 2) {
#pragma unroll
                for (int m = 0; m < 4; ++m)
                    raw[m] = *reinterpret_cast<const uint4*>(stp + (warp < 2 ? kStUv : kStO0) + sw128_chunk_off(c & 63, cq + m, 64));
            }
            const float gam = *reinterpret_cast<const float*>(stp + kStGam + 4 * c);
            if (GATE == kGateNone || warp < 2) {  // gated: warps 2-3 only carry the state
                ok = ok && mbar_wait_ab(bar_d1, par, s_abort);
                fence_after_sync();
                float x[32];
                tmem_ld16(tw + kTmD1, x);
                tmem_ld16(tw + kTmD1 + 16, x + 16);
                tmem_wait_ld();
                if (warp < 2) {  // U = Uv - X, row r = c
                    uint4 pk[4];
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        float u[8];
                        unpack8(raw[m], u);
#pragma unroll
                        for (int e = 0; e < 8; ++e) u[e] -= x[8 * m + e];
                        pk[m] = pack8(u);
                    }
#pragma unroll
                    for (int m = 0; m < 4; ++m) *reinterpret_cast<uint4*>(sm + kB_U + sw128_chunk_off(c, m, 64)) = pk[m];
                    fence_proxy_async();
                    named_arrive(1, 96);
                } else {  // out = O' + O0, row r = c - 64
                    const int r = c - 64;
                    if (r < L && ok) {
                        uint4* dst = reinterpret_cast<uint4*>(out + ((size_t)(t0 + r) * H + h) * 128 + v0);
#pragma unroll
                        for (int m = 0; m < 4; ++m) {
                            float u[8];
                            unpack8(raw[m], u);
#pragma unroll
                            for (int e = 0; e < 8; ++e) u[e] += x[8 * m + e];
                            dst[m] = pack8(u);
                        }
                    }
                }
            }
            ok = ok && mbar_wait_ab(bar_y, par, s_abort);
            fence_after_sync();
            if (refill) mbar_arrive(bar_empty + 8 * s);  // last read of stage s done (MMAs on it complete)
            float y[32];
            tmem_ld16(tw + kTmY, y);
            tmem_ld16(tw + kTmY + 16, y + 16);
            tmem_wait_ld();
#pragma unroll
            for (int m = 0; m < kTcNV; ++m) S[m] = fmaf(gam, S[m], y[m]);
            uint4 pk[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) pk[m] = pack8(S + 8 * m);
#pragma unroll
            for (int m = 0; m < 4; ++m) *reinterpret_cast<uint4*>(sm + kB_S + sw128_chunk_off(c, m, 128)) = pk[m];
            fence_proxy_async();
            fence_before_sync();
            if (it + 1 < nch) named_arrive(2, GATE == kGateNone ? 160 : 224);  // S tile ready for the next chunk
        }
    }
    ok = __syncthreads_and(ok && !*s_abort);
    if (warp < 4 && S_final && ok) {
#pragma unroll
        for (int m = 0; m < kTcNV; m += 4)
            *reinterpret_cast<float4*>(S_final + srow + m) = make_float4(S[m], S[m + 1], S[m + 2], S[m + 3]);
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 64);
    if (GATE == kGateCluster) cluster_sync();  // no CTA leaves while a peer may still write its shared memory
}

// cuTensorMapEncodeTiled, fetched from the driver through the runtime (no link against libcuda)
typedef CUresult (*TensorMapEncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                      const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                      CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline TensorMapEncodeFn tensor_map_encoder()
{
    static TensorMapEncodeFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        cudaDriverEntryPointQueryResult res;
        void* p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &res) == cudaSuccess &&
            res == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<TensorMapEncodeFn>(p);
    }
    return fn;
}

// [tokens][H][128] row-major tensor as a 3-D map (d, head, token), box = 64 tokens x 1 head x box_d;
// bf16 tiles of 64 channels land 128B-swizzled (MMA operands), every other box unswizzled
inline bool make_token_map(CUtensorMap* m, const void* base, bool bf16, int H, long long ntok, int box_d)
{
    TensorMapEncodeFn enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t esz = bf16 ? 2 : 4;
    const bool swz = bf16 && box_d * esz == 128;
    const cuuint64_t dims[3] = {128, (cuuint64_t)H, (cuuint64_t)ntok};
    const cuuint64_t strides[2] = {128 * esz, 128 * esz * (cuuint64_t)H};
    const cuuint32_t box[3] = {(cuuint32_t)box_d, 1, 64};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base),
               dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               swz ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline cudaError_t launch_tc_prefill(const void* q, const void* k, const void* v, const void* la, const float* beta,
                                     const float* S0, float* S_final, void* out, const WsHeader* hdr, const int* off,
                                     const int32_t* cu, int Tseq, int N, int H, int Hk, unsigned pro, int max_chunks,
                                     long long Ttot,
                                     char* slots, const OutGate* gate, cudaStream_t stream)
{
    // instance: (any q/k, beta or gate-activation bit, bf16 gates)
    const bool la16 = (pro & KDA_PROLOGUE_GATE_BF16) != 0, pr = (pro & ~KDA_PROLOGUE_GATE_BF16) != 0;
    auto* kern = pr ? (la16 ? tc_intra_kernel<true, true> : tc_intra_kernel<true, false>)
                    : (la16 ? tc_intra_kernel<false, true> : tc_intra_kernel<false, false>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kA_Smem);
    if (e != cudaSuccess) return e;
    const int gmode = !gate ? kGateNone : gate->group <= kTcNV ? kGateLocal : kGateCluster;
    auto* kernB = gmode == kGateNone ? tc_inter_kernel<kGateNone>
                : gmode == kGateLocal ? tc_inter_kernel<kGateLocal> : tc_inter_kernel<kGateCluster>;
    const uint32_t smemB = gmode == kGateNone ? kB_Smem : kB_SmemGate;
    e = cudaFuncSetAttribute(kernB, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smemB);
    if (e != cudaSuccess) return e;
    if (max_chunks > 0 && Ttot > 0) {
        alignas(64) CUtensorMap tq, tk, tv, tla;
        if (!make_token_map(&tq, q, true, Hk, Ttot, 64) || !make_token_map(&tk, k, true, Hk, Ttot, 64) ||
            !make_token_map(&tv, v, true, H, Ttot, 64) || !make_token_map(&tla, la, la16, H, Ttot, 128))
            return cudaErrorInvalidValue;
        // persistent: two CTAs per SM (the register and shared-memory budget of one CTA is half an SM)
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const long long units = (long long)max_chunks * H;
        const unsigned grid = (unsigned)(units < 2LL * sms ? units : 2LL * sms);
        LaunchScope ls("tc_intra", stream);
        kern<<<grid, kAThreads, kA_Smem, stream>>>(tq, tk, tv, tla, beta, const_cast<WsHeader*>(hdr), off, cu, Tseq,
                                                  N, H, H / Hk, pro, (uint8_t*)slots);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    LaunchScope ls("tc_inter", stream);
    const long long nb = (long long)N * H * (128 / kTcNV);
    if (nb > 0x7fffffffLL) return cudaErrorInvalidValue;
    const OutGate g = gate ? *gate : OutGate{nullptr, nullptr, 0.f, 0.f, 0, 0};
    // the four slice CTAs of one (sequence, head) are consecutive in the grid: a cluster of 4 along x
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)nb);
    cfg.blockDim = dim3(gmode == kGateNone ? kBThreads : kBThreads + 64);
    cfg.dynamicSmemBytes = smemB;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 128 / kTcNV;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = gmode == kGateCluster ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernB, S0, S_final, (__nv_bfloat16*)out, hdr, off, cu, Tseq, N, H,
                              (const uint8_t*)slots, g);
}

}  // namespace kda
