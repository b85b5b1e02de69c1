// backward_tc.cuh -- the state side of the chunked KDA backward on the tensor cores (tcgen05 / TMEM),
// for bf16 inputs with dk = dv = 128.
//
// Per (chunk, head), with the chunk's start state S_c, its end cotangent D_c, the corrected values U
// and their cotangent dU (all fp32, from the backward's chains) and the output cotangent dO (bf16):
//     dQg = dO S_c^T,   dW = -dU S_c^T,   dKd = U D_c^T,   dP = lower_incl(dO U^T),
//     dgam = rowsum(D_c * S_c)
// (the reverse-mode derivative of U = Uv - W S, O = Qg S + P U, S_next = Diag(gam) S + Kd^T U; the
// CUDA-core bwd_state_side_kernel computes the same).  The four products are tcgen05 MMAs with fp32
// accumulators in TMEM.  To keep the backward's fp32 accuracy, every fp32 operand x is split into two
// bf16 parts, x = hi + lo with hi = bf16(x) and lo = bf16(x - hi), and each product is formed as
// hi*hi + hi*lo + lo*hi: the three-term bf16 splitting of Henry, Tang and Heinecke, "Leveraging the
// bfloat16 artificial intelligence datatype for higher-precision computations" (ARITH 2019), which
// carries about 16 significant bits per operand.  dO is bf16 already (its lo part is zero).  dgam is
// an fp32 dot product on the CUDA cores, taken while the states are converted.
//
// Persistent CTAs of 256 threads, one per SM (the operands of a unit take 208 KB of shared memory),
// each prefetching its next unit into L2.  Per unit, phase 1: the threads load and split dO, dU and
// S_c into SW128 K-major tiles and thread 0 issues the 24 MMAs of S_c [dO; dU]^T.  Phase 2, while those
// run: U and D_c, and dgam.  Thread 0 then issues the 40 MMAs of D_c U^T and dO U^T, and all eight
// warps drain the first product from TMEM into the unit's fp32 scratch while the second batch runs,
// then the rest.  The first two products are formed transposed (key channel on the TMEM lane), so
// that a warp's stores cover 32 consecutive channels of one token row.
#pragma once

#include "backward_simt.cuh"
#include "prefill_tc.cuh"

namespace kda {

// shared memory (bytes; every tile 1024-aligned).  X = [dO; dU] stacked, 128 rows x 128 (K = value
// channel), and the lo part of its dU rows (dO has none); S, D: 128 rows (key channel) x 128; U: 64
// rows x 128.
constexpr uint32_t kBX_hi = 0, kBX_lo = 32768;
constexpr uint32_t kBS_hi = 49152, kBS_lo = 81920;
constexpr uint32_t kBD_hi = 114688, kBD_lo = 147456;
constexpr uint32_t kBU_hi = 180224, kBU_lo = 196608;
constexpr uint32_t kBMisc = 212992;                   // 2 mbarriers (16 B) | TMEM base address (4 B)
constexpr uint32_t kBStateSmem = kBMisc + 64 + 1024;  // + alignment slack
static_assert(kBStateSmem <= 232448, "state-side shared memory");
// TMEM columns (lane = key channel i for the first two): [dO; dU] S_c^T transposed (N = 128 token rows),
// U D_c^T transposed (N = 64), and dO U^T (M = 64, N = 64)
constexpr uint32_t kTmQW = 0, kTmKd = 128, kTmP = 192;

// 8 fp32 values -> their bf16 hi and lo parts, as two 16-byte chunks
__device__ __forceinline__ void split8(const float* f, uint4& hi, uint4& lo)
{
    float h[8], l[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        h[m] = __bfloat162float(__float2bfloat16_rn(f[m]));
        l[m] = f[m] - h[m];
    }
    hi = pack8(h);
    lo = pack8(l);
}

// Persistent: one CTA per SM walks the (chunk, head) units u = blockIdx.x + k gridDim.x and prefetches
// the next unit's operands into L2 while it works on the current one.
__global__ void __launch_bounds__(256, 1)
bwd_state_side_tc_kernel(const __nv_bfloat16* __restrict__ dout, const WsHeader* __restrict__ hdr,
                         const int* __restrict__ off, const int32_t* __restrict__ cu, int Tseq, int N, int H,
                         const float* __restrict__ S_chunks, const float* __restrict__ dSn_chunks,
                         float* __restrict__ scr)
{
    using namespace tc;
    constexpr int D = 128;
    extern __shared__ uint8_t smem_raw[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (hdr->bad) return;
    const long long units = (long long)hdr->total_chunks * H;
    if ((long long)blockIdx.x >= units) return;
    uint8_t* sm = align1024(smem_raw);
    const uint32_t sb = smem_u32(sm);
    const uint32_t mbar = sb + kBMisc;  // two mbarriers: the S_c products, then the others
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + kBMisc + 16);
    const size_t scr_unit = bwd_scr_floats(D, D);

    if (tid == 0) {
        mbar_init(mbar, 1);
        mbar_init(mbar + 8, 1);
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(s_tmem), 256);
        tmem_relinquish();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *s_tmem;
    const int ch = tid & 15, rq = tid >> 4;  // a thread's load tasks: 16-byte chunk ch of rows rq + 16 m
    const int q = warp & 3, half = warp >> 2;
    const uint32_t tl = tmem + ((uint32_t)(32 * q) << 16);
    const uint4 z4 = make_uint4(0, 0, 0, 0);
    bool ok = true;
    uint32_t ph = 0;

    for (long long u = blockIdx.x; u < units; u += gridDim.x, ph ^= 1u) {
        const int j = (int)(u / H), h = (int)(u - (long long)j * H);
        int n, L;
        long long t0;
        locate_chunk(j, off, cu, Tseq, N, n, t0, L);
        const float* Sc = S_chunks + (size_t)u * D * D;
        const float* Dc = dSn_chunks + (size_t)u * D * D;
        float* o = scr + (size_t)u * scr_unit;
        const float* oU = o;
        const float* odU = oU + (size_t)kChunk * D;
        float* oQg = o + 2 * (size_t)kChunk * D;
        float* oW = oQg + (size_t)kChunk * D;
        float* oKd = oW + (size_t)kChunk * D;
        float* oP = oKd + (size_t)kChunk * D;
        float* oGam = oP + (size_t)kChunk * kChunk;
        {  // the next unit's operands into L2 (warp 0: its states and U, dU; warp 1: its dO rows)
            const long long un = u + gridDim.x;
            if (un < units) {
                if (tid == 0) {
                    bulk_prefetch_l2(S_chunks + (size_t)un * D * D, D * D * 4);
                    bulk_prefetch_l2(dSn_chunks + (size_t)un * D * D, D * D * 4);
                    bulk_prefetch_l2(scr + (size_t)un * scr_unit, 2 * kChunk * D * 4);
                }
                if (warp == 1) {
                    const int jn = (int)(un / H), hn = (int)(un - (long long)jn * H);
                    int nn, Ln;
                    long long tn;
                    locate_chunk(jn, off, cu, Tseq, N, nn, tn, Ln);
                    for (int r = lane; r < Ln; r += 32) bulk_prefetch_l2(dout + ((size_t)(tn + r) * H + hn) * D, D * 2);
                }
            }
        }
        // phase 1: X = [dO; dU] and S_c -> SW128 K-major bf16 tiles (every load issued before any use)
        {
            uint4 dov[4];
            float du[4][8], fs[8][8];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int r = rq + 16 * m;
                dov[m] = r < L ? *reinterpret_cast<const uint4*>(dout + ((size_t)(t0 + r) * H + h) * D + 8 * ch) : z4;
                load8(odU + (size_t)r * D + 8 * ch, du[m]);
            }
#pragma unroll
            for (int m = 0; m < 8; ++m) load8(Sc + (size_t)(rq + 16 * m) * D + 8 * ch, fs[m]);
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int r = rq + 16 * m;
                uint4 hi, lo;
                *reinterpret_cast<uint4*>(sm + kBX_hi + sw128_chunk_off(r, ch, 128)) = dov[m];  // exact in bf16
                split8(du[m], hi, lo);
                *reinterpret_cast<uint4*>(sm + kBX_hi + sw128_chunk_off(64 + r, ch, 128)) = hi;
                *reinterpret_cast<uint4*>(sm + kBX_lo + sw128_chunk_off(r, ch, 64)) = lo;
            }
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                uint4 hi, lo;
                split8(fs[m], hi, lo);
                *reinterpret_cast<uint4*>(sm + kBS_hi + sw128_chunk_off(rq + 16 * m, ch, 128)) = hi;
                *reinterpret_cast<uint4*>(sm + kBS_lo + sw128_chunk_off(rq + 16 * m, ch, 128)) = lo;
            }
        }
        fence_proxy_async();  // the tiles, written by the threads, are read by the tensor cores
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (tid == 0) {  // (S_c [dO; dU]^T)[i][r] = hi*hi + lo*hi over all rows, + hi*lo over the dU rows
            const uint32_t idA = idesc_bf16(128, 128, false, false), idB = idesc_bf16(128, 64, false, false);
#pragma unroll
            for (int k0 = 0; k0 < D; k0 += 16)
                mma_bf16(tmem + kTmQW, desc_kmajor(sb + kBS_hi, 128, k0), desc_kmajor(sb + kBX_hi, 128, k0), idA,
                         k0 > 0 ? 1u : 0u);
#pragma unroll
            for (int k0 = 0; k0 < D; k0 += 16)
                mma_bf16(tmem + kTmQW, desc_kmajor(sb + kBS_lo, 128, k0), desc_kmajor(sb + kBX_hi, 128, k0), idA, 1u);
#pragma unroll
            for (int k0 = 0; k0 < D; k0 += 16)
                mma_bf16(tmem + kTmQW + 64, desc_kmajor(sb + kBS_hi, 128, k0), desc_kmajor(sb + kBX_lo, 64, k0), idB,
                         1u);
            mma_commit(mbar);
        }
        // phase 2 (while those run): U and D_c; dgam[i] = sum_j D_c[i][j] S_c[i][j] with S_c = hi + lo read
        // back from its tiles (the 16 chunks of row i are the 16 consecutive threads of a half-warp)
        {
            float fu[4][8], fd[8][8];
#pragma unroll
            for (int m = 0; m < 4; ++m) load8(oU + (size_t)(rq + 16 * m) * D + 8 * ch, fu[m]);
#pragma unroll
            for (int m = 0; m < 8; ++m) load8(Dc + (size_t)(rq + 16 * m) * D + 8 * ch, fd[m]);
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                uint4 hi, lo;
                split8(fu[m], hi, lo);
                *reinterpret_cast<uint4*>(sm + kBU_hi + sw128_chunk_off(rq + 16 * m, ch, 64)) = hi;
                *reinterpret_cast<uint4*>(sm + kBU_lo + sw128_chunk_off(rq + 16 * m, ch, 64)) = lo;
            }
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const int i = rq + 16 * m;
                float sh[8], sl[8];
                unpack8(*reinterpret_cast<const uint4*>(sm + kBS_hi + sw128_chunk_off(i, ch, 128)), sh);
                unpack8(*reinterpret_cast<const uint4*>(sm + kBS_lo + sw128_chunk_off(i, ch, 128)), sl);
                float g = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) g = fmaf(fd[m][e], sh[e] + sl[e], g);
#pragma unroll
                for (int s2 = 1; s2 < 16; s2 <<= 1) g += __shfl_xor_sync(0xffffffffu, g, s2);
                if (ch == 0) oGam[i] = g;
                uint4 hi, lo;
                split8(fd[m], hi, lo);
                *reinterpret_cast<uint4*>(sm + kBD_hi + sw128_chunk_off(i, ch, 128)) = hi;
                *reinterpret_cast<uint4*>(sm + kBD_lo + sw128_chunk_off(i, ch, 128)) = lo;
            }
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (tid == 0) {
            // (D_c U^T)[i][r]: hi*hi + lo*hi + hi*lo
            const uint32_t idB = idesc_bf16(128, 64, false, false), idP = idesc_bf16(64, 64, false, false);
            const uint32_t da[3] = {kBD_hi, kBD_lo, kBD_hi}, ub[3] = {kBU_hi, kBU_hi, kBU_lo};
#pragma unroll
            for (int t = 0; t < 3; ++t)
#pragma unroll
                for (int k0 = 0; k0 < D; k0 += 16)
                    mma_bf16(tmem + kTmKd, desc_kmajor(sb + da[t], 128, k0), desc_kmajor(sb + ub[t], 64, k0), idB,
                             (t > 0 || k0 > 0) ? 1u : 0u);
            // (dO U^T)[r][i] (dO is the first 64 rows of X_hi; it has no lo part)
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int k0 = 0; k0 < D; k0 += 16)
                    mma_bf16(tmem + kTmP, desc_kmajor(sb + kBX_hi, 128, k0),
                             desc_kmajor(sb + (t ? kBU_lo : kBU_hi), 64, k0), idP, (t > 0 || k0 > 0) ? 1u : 0u);
            mma_commit(mbar + 8);
        }
        ok = mbar_wait(mbar, ph) && ok;
        fence_after_sync();
        if (ok) {  // lane = key channel i = 32 q + lane; columns = token rows: dQg (half 0) or dW = -(...) (half 1)
            const int i = 32 * q + lane;
            float* dst = (half == 0 ? oQg : oW) + i;
            const float sgn = half == 0 ? 1.f : -1.f;
#pragma unroll
            for (int t = 0; t < 4; t += 2) {
                float v[32];
                tmem_ld16(tl + kTmQW + 64 * half + 16 * t, v);
                tmem_ld16(tl + kTmQW + 64 * half + 16 * t + 16, v + 16);
                tmem_wait_ld();
#pragma unroll
                for (int m = 0; m < 32; ++m) dst[(size_t)(16 * t + m) * D] = sgn * v[m];
            }
        }
        ok = mbar_wait(mbar + 8, ph) && ok;
        fence_after_sync();
        if (ok) {
            {  // dKd[r][i]: lane = i, columns r = 32 half .. +31
                const int i = 32 * q + lane;
                float v[32];
                tmem_ld16(tl + kTmKd + 32 * half, v);
                tmem_ld16(tl + kTmKd + 32 * half + 16, v + 16);
                tmem_wait_ld();
#pragma unroll
                for (int m = 0; m < 32; ++m) oKd[(size_t)(32 * half + m) * D + i] = v[m];
            }
            {  // dP = lower_incl(dO U^T) (M = 64: row 16 q + lane % 16; columns 32 half + 16 (lane / 16) .. +15)
                const int r = 16 * q + (lane & 15), c0 = 32 * half + 16 * (lane >> 4);
                float v[16];
                tmem_ld16_pair<16>(tl + kTmP + 32 * half, v);
                tmem_wait_ld();
#pragma unroll
                for (int m = 0; m < 16; m += 4) {
                    float4 x;
                    x.x = (c0 + m <= r) ? v[m] : 0.f;
                    x.y = (c0 + m + 1 <= r) ? v[m + 1] : 0.f;
                    x.z = (c0 + m + 2 <= r) ? v[m + 2] : 0.f;
                    x.w = (c0 + m + 3 <= r) ? v[m + 3] : 0.f;
                    *reinterpret_cast<float4*>(oP + (size_t)r * kChunk + c0 + m) = x;
                }
            }
        }
        fence_before_sync();
        __syncthreads();  // TMEM drained and the tiles free for the next unit
        fence_after_sync();
    }
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// ------------------------------------------------------------------------------------------------
// The dO terms of the reverse chain, chunk-parallel (one CTA per (chunk, head)):
//     E = P^T dO  (64 x dv, into the unit's dU scratch),   F = Qg^T dO  (dk x dv)
// formed as one transposed product dO^T [P | Qg] (M = 128 value channels, N = 64 + 128, K = 64
// tokens; both operands MN-major, i.e. the row-major token tiles as they are), so that the value
// channel lands on the TMEM lane and the stores of E and F coalesce.  dO is exact in bf16; P and Qg
// (fp32, from the forward's slot) are split into bf16 hi and lo parts: dO [P | Qg]_hi + dO [P | Qg]_lo.
// ------------------------------------------------------------------------------------------------
constexpr uint32_t kTO = 0;             // dO: 64 token rows x 128 (two atom columns), 16 KB
constexpr uint32_t kTB_hi = 16384;      // [P | Qg] hi: 64 token rows x 192 (three atom columns), 24 KB
constexpr uint32_t kTB_lo = 40960;      // ... lo
constexpr uint32_t kTMisc = 65536;      // mbarrier | TMEM base address
// 100 KB requested (64 KB used) so that at most two CTAs share an SM: two 256-column TMEM allocations
constexpr uint32_t kDoTermsSmem = 102400;

__global__ void __launch_bounds__(128)
bwd_do_terms_tc_kernel(const __nv_bfloat16* __restrict__ dout, const WsHeader* __restrict__ hdr,
                       const int* __restrict__ off, const int32_t* __restrict__ cu, int Tseq, int N, int H,
                       const float* __restrict__ slots, float* __restrict__ scr, float* __restrict__ F_chunks)
{
    using namespace tc;
    constexpr int D = 128;
    extern __shared__ uint8_t smem_raw[];
    const int j = blockIdx.x, h = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (hdr->bad || j >= hdr->total_chunks) return;
    int n, L;
    long long t0;
    locate_chunk(j, off, cu, Tseq, N, n, t0, L);
    uint8_t* sm = align1024(smem_raw);
    const uint32_t sb = smem_u32(sm);
    const uint32_t mbar = sb + kTMisc;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + kTMisc + 8);
    const size_t u = (size_t)j * H + h;
    const float* slot = slots + u * simt_slot_floats(D, D);
    const float* gQ = slot + (size_t)kChunk * D;
    const float* gP = slot + 3 * (size_t)kChunk * D;
    float* gE = scr + u * bwd_scr_floats(D, D) + (size_t)kChunk * D;
    float* gF = F_chunks + u * D * D;

    if (tid == 0) {
        mbar_init(mbar, 1);
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(s_tmem), 256);
        tmem_relinquish();
    }
    // token rows -> SW128 tiles with 64-element atom columns (chunk ch of row r: 8 consecutive columns)
    const uint4 z4 = make_uint4(0, 0, 0, 0);
    {
        const int ch = tid & 15, rq = tid >> 4;  // dO and Qg: rows rq + 8 m, chunk ch of 16
        uint4 dov[8];
        float fq[8][8];
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const int r = rq + 8 * m;
            dov[m] = r < L ? *reinterpret_cast<const uint4*>(dout + ((size_t)(t0 + r) * H + h) * D + 8 * ch) : z4;
            load8(gQ + (size_t)r * D + 8 * ch, fq[m]);
        }
        const int cp = tid & 7, rp = tid >> 3;   // P: rows rp + 16 m, chunk cp of 8
        float fp[4][8];
#pragma unroll
        for (int m = 0; m < 4; ++m) load8(gP + (size_t)(rp + 16 * m) * kChunk + 8 * cp, fp[m]);
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const int r = rq + 8 * m;
            uint4 hi, lo;
            *reinterpret_cast<uint4*>(sm + kTO + sw128_chunk_off(r, ch, 64)) = dov[m];
            split8(fq[m], hi, lo);
            *reinterpret_cast<uint4*>(sm + kTB_hi + sw128_chunk_off(r, 8 + ch, 64)) = hi;
            *reinterpret_cast<uint4*>(sm + kTB_lo + sw128_chunk_off(r, 8 + ch, 64)) = lo;
        }
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            uint4 hi, lo;
            split8(fp[m], hi, lo);
            *reinterpret_cast<uint4*>(sm + kTB_hi + sw128_chunk_off(rp + 16 * m, cp, 64)) = hi;
            *reinterpret_cast<uint4*>(sm + kTB_lo + sw128_chunk_off(rp + 16 * m, cp, 64)) = lo;
        }
    }
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *s_tmem;
    if (tid == 0) {
        const uint32_t id = idesc_bf16(128, 192, true, true);
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int k0 = 0; k0 < kChunk; k0 += 16)
                mma_bf16(tmem, desc_mnmajor(sb + kTO, kChunk, k0), desc_mnmajor(sb + (t ? kTB_lo : kTB_hi), kChunk, k0),
                         id, (t > 0 || k0 > 0) ? 1u : 0u);
        mma_commit(mbar);
    }
    const bool ok = mbar_wait(mbar, 0);
    fence_after_sync();
    if (ok) {  // lane = value channel jv; columns 0-63: E[i][jv], 64-191: F[c][jv]
        const int jv = 32 * warp + lane;
        const uint32_t tl = tmem + ((uint32_t)(32 * warp) << 16);
#pragma unroll
        for (int cb = 0; cb < 192; cb += 32) {
            float v[32];
            tmem_ld16(tl + cb, v);
            tmem_ld16(tl + cb + 16, v + 16);
            tmem_wait_ld();
#pragma unroll
            for (int m = 0; m < 32; ++m) {
                const int col = cb + m;
                if (col < kChunk) gE[(size_t)col * D + jv] = v[m];
                else gF[(size_t)(col - kChunk) * D + jv] = v[m];
            }
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

inline cudaError_t launch_bwd_do_terms_tc(const void* dout, const WsHeader* hdr, const int* off, const int32_t* cu,
                                          int Tseq, int N, int H, int max_chunks, const float* slots, float* scr,
                                          float* F_chunks, cudaStream_t stream)
{
    cudaError_t e = cudaFuncSetAttribute(bwd_do_terms_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kDoTermsSmem);
    if (e != cudaSuccess) return e;
    LaunchScope ls("bwd_do_terms_tc", stream);
    bwd_do_terms_tc_kernel<<<dim3(max_chunks, H), 128, kDoTermsSmem, stream>>>(
        (const __nv_bfloat16*)dout, hdr, off, cu, Tseq, N, H, slots, scr, F_chunks);
    return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------------
// The input side's second half (per (chunk, head, 64-channel half)): dq, dk and dlog_alpha
// through the gated products P = Qf Kb^T, At = Kf Kb^T and the gating (bwd_gate_kernel computes the
// same on CUDA cores).  The five products, each M = 64 token rows, N = 64 channels, K = 64 tokens,
//     rowP = dP Kb,  rowA = dAt Kb,  col = dP^T Qf + dAt^T Kf,  dkt = N^T dW,
// are tcgen05 MMAs with split-bf16 operands (hi*hi + hi*lo + lo*hi).  dP, dAt and N are stored once as
// row-major tiles: K-major for the first two products and read MN-major (the same bytes) for the
// transposed ones.  A 32-channel tile whose in-chunk gate spread exceeds kFactorSpread takes the
// exact per-element factors on the CUDA cores instead, as the CUDA-core kernel does.
// ------------------------------------------------------------------------------------------------
constexpr uint32_t kG_Phi = 0, kG_Plo = 8192, kG_Ahi = 16384, kG_Alo = 24576, kG_Nhi = 32768, kG_Nlo = 40960;
constexpr uint32_t kG_Kbhi = 49152, kG_Kblo = 57344, kG_Qfhi = 65536, kG_Qflo = 73728, kG_Kfhi = 81920,
                   kG_Kflo = 90112, kG_Whi = 98304, kG_Wlo = 106496;
constexpr uint32_t kG_G = 114688;                   // fp32 [64][64]: the cumulative gate g (natural log)
constexpr uint32_t kG_K = 131072, kG_Q = 139264;    // bf16 [64][64] k and q, row-major
constexpr uint32_t kG_Misc = 147456;                // beta [64] | ref [64] | quarter totals, lo, hi [4][64] x3 | flags
constexpr uint32_t kG_Smem = kG_Misc + 4096 + 1024;
constexpr int kG_LS = 68;                           // row stride (floats) of the dg staging over the B tiles
static_assert(kG_Smem <= 232448, "gate shared memory");

// One CTA per item (unit, half) = blockIdx.x (a persistent variant that prefetched its next item into
// L2 measured slower: 4.25 against 3.77 ms per 32K step).
template <bool LA16>
__global__ void __launch_bounds__(256, 1)
bwd_gate_tc_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                   const void* __restrict__ log_alpha, const float* __restrict__ beta, const WsHeader* __restrict__ hdr,
                   const int* __restrict__ off, const int32_t* __restrict__ cu, int Tseq, int N, int H, int Hk,
                   const float* __restrict__ scr, __nv_bfloat16* __restrict__ dq, __nv_bfloat16* __restrict__ dk_out,
                   float* __restrict__ dla, float* __restrict__ dq_acc, float* __restrict__ dk_acc)
{
    using namespace tc;
    constexpr int D = 128;
    extern __shared__ uint8_t smem_raw[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (hdr->bad) return;
    const long long items = (long long)hdr->total_chunks * H * 2;
    if ((long long)blockIdx.x >= items) return;
    uint8_t* sm = align1024(smem_raw);
    const uint32_t sb = smem_u32(sm);
    float* sG = reinterpret_cast<float*>(sm + kG_G);
    const __nv_bfloat16* sK = reinterpret_cast<const __nv_bfloat16*>(sm + kG_K);
    const __nv_bfloat16* sQ = reinterpret_cast<const __nv_bfloat16*>(sm + kG_Q);
    float* sbeta = reinterpret_cast<float*>(sm + kG_Misc);
    float* sref = sbeta + 64;
    float* stot = sref + 64;    // [4][64] quarter totals (gate scan), then [4][64] dg partial sums
    float* slo = stot + 256;    // [4][64]
    float* shi = slo + 256;     // [4][64]
    int* swide = reinterpret_cast<int*>(shi + 256);  // [2] one flag per 32-channel tile
    const uint32_t mbar = smem_u32(swide + 4);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(swide + 6);
    float* sAccG = reinterpret_cast<float*>(sm + kG_Kbhi);  // dg staging over the B tiles (after the MMAs)
    float* sAccL = sAccG + 64 * kG_LS;
    const size_t scr_unit = bwd_scr_floats(D, D);

    if (tid == 0) {
        mbar_init(mbar, 1);
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(s_tmem), 256);
        tmem_relinquish();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *s_tmem;
    // epilogue mapping: row r = 16 qd + lane % 16, channels cb .. cb + 15 (one 32-channel tile hh)
    const int qd = warp & 3, hh = warp >> 2;
    const int r = 16 * qd + (lane & 15), cb = 32 * hh + 16 * (lane >> 4);
    uint32_t ph = 0;

    for (long long it = blockIdx.x; it < items; it += gridDim.x, ph ^= 1u) {
        const long long uu = it >> 1;
        const int j = (int)(uu / H), h = (int)(uu - (long long)j * H), c0 = 64 * (int)(it & 1);
        int n, L;
        long long t0;
        locate_chunk(j, off, cu, Tseq, N, n, t0, L);
        const float* o = scr + (size_t)uu * scr_unit;
        const float* gN = o;
        const float* gdAt = o + (size_t)kChunk * D;
        const float* gdQg = o + 2 * (size_t)kChunk * D;
        const float* gdW = gdQg + (size_t)kChunk * D;
        const float* gdKd = gdW + (size_t)kChunk * D;
        const float* gdP = gdKd + (size_t)kChunk * D;
        const float* gdGam = gdP + (size_t)kChunk * kChunk;
        const int hq = h / (H / Hk);  // the q/k head of value head h
        if (tid == 0) swide[0] = swide[1] = 0;
        if (tid < 64) sbeta[tid] = tid < L ? beta[(size_t)(t0 + tid) * H + h] : 0.f;
        // this thread's dQg and dKd, in flight from the start
        float dqg[16], dkd[16];
#pragma unroll
        for (int x = 0; x < 16; x += 4) {
            const float4 a = *reinterpret_cast<const float4*>(gdQg + (size_t)r * D + c0 + cb + x);
            const float4 b = *reinterpret_cast<const float4*>(gdKd + (size_t)r * D + c0 + cb + x);
            dqg[x] = a.x; dqg[x + 1] = a.y; dqg[x + 2] = a.z; dqg[x + 3] = a.w;
            dkd[x] = b.x; dkd[x + 1] = b.y; dkd[x + 2] = b.z; dkd[x + 3] = b.w;
        }
        // loads: task e = tid + 256 m -> row e / 8, 8-element chunk e % 8 of the 64 columns
        {
            float fP[2][8], fA[2][8], fN[2][8], fW[2][8], fg[2][8];
            uint4 kr[2], qr[2];
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                const int e = tid + 256 * m, rr = e >> 3, ch = e & 7;
                load8(gdP + (size_t)rr * kChunk + 8 * ch, fP[m]);
                load8(gdAt + (size_t)rr * kChunk + 8 * ch, fA[m]);
                load8(gN + (size_t)rr * kChunk + 8 * ch, fN[m]);
                load8(gdW + (size_t)rr * D + c0 + 8 * ch, fW[m]);
                const bool in = rr < L;
                const size_t ia = ((size_t)(t0 + (in ? rr : 0)) * H + h) * D + c0 + 8 * ch;
                if (LA16) load8(reinterpret_cast<const __nv_bfloat16*>(log_alpha) + ia, fg[m]);
                else load8(reinterpret_cast<const float*>(log_alpha) + ia, fg[m]);
                if (!in)
#pragma unroll
                    for (int x = 0; x < 8; ++x) fg[m][x] = 0.f;  // rows past the chunk's end add nothing
                const size_t iq = ((size_t)(t0 + (in ? rr : 0)) * Hk + hq) * D + c0 + 8 * ch;
                kr[m] = in ? *reinterpret_cast<const uint4*>(k + iq) : make_uint4(0, 0, 0, 0);
                qr[m] = in ? *reinterpret_cast<const uint4*>(q + iq) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                const int e = tid + 256 * m, rr = e >> 3, ch = e & 7;
                const uint32_t so = sw128_chunk_off(rr, ch, 64);
                uint4 hi, lo;
                split8(fP[m], hi, lo);
                *reinterpret_cast<uint4*>(sm + kG_Phi + so) = hi;
                *reinterpret_cast<uint4*>(sm + kG_Plo + so) = lo;
                split8(fA[m], hi, lo);
                *reinterpret_cast<uint4*>(sm + kG_Ahi + so) = hi;
                *reinterpret_cast<uint4*>(sm + kG_Alo + so) = lo;
                split8(fN[m], hi, lo);
                *reinterpret_cast<uint4*>(sm + kG_Nhi + so) = hi;
                *reinterpret_cast<uint4*>(sm + kG_Nlo + so) = lo;
                split8(fW[m], hi, lo);
                *reinterpret_cast<uint4*>(sm + kG_Whi + so) = hi;
                *reinterpret_cast<uint4*>(sm + kG_Wlo + so) = lo;
                *reinterpret_cast<float4*>(sG + rr * 64 + 8 * ch) = make_float4(fg[m][0], fg[m][1], fg[m][2], fg[m][3]);
                *reinterpret_cast<float4*>(sG + rr * 64 + 8 * ch + 4) = make_float4(fg[m][4], fg[m][5], fg[m][6], fg[m][7]);
                *reinterpret_cast<uint4*>(sm + kG_K + (rr * 64 + 8 * ch) * 2) = kr[m];
                *reinterpret_cast<uint4*>(sm + kG_Q + (rr * 64 + 8 * ch) * 2) = qr[m];
            }
        }
        __syncthreads();
        // cumulative gate per channel: thread (channel c, quarter qt) scans rows 16 qt .. 16 qt + 15, then
        // adds the totals of the quarters before it; the reference is the centre of [min, max] over the
        // chunk (the chunk start g = 0 included), as in the CUDA-core kernel
        {
            const int c = tid & 63, qt = tid >> 6;
            float gv[16], acc = 0.f;
#pragma unroll
            for (int x = 0; x < 16; ++x) {
                acc += sG[(16 * qt + x) * 64 + c];
                gv[x] = acc;
            }
            stot[qt * 64 + c] = acc;
            __syncthreads();
            float carry = 0.f;
            for (int p2 = 0; p2 < qt; ++p2) carry += stot[p2 * 64 + c];
            float lo = qt == 0 ? 0.f : carry, hi = lo;
#pragma unroll
            for (int x = 0; x < 16; ++x) {
                gv[x] += carry;
                lo = fminf(lo, gv[x]);
                hi = fmaxf(hi, gv[x]);
                sG[(16 * qt + x) * 64 + c] = gv[x];
            }
            slo[qt * 64 + c] = lo;
            shi[qt * 64 + c] = hi;
            __syncthreads();
            if (tid < 64) {
                lo = fminf(fminf(slo[c], slo[64 + c]), fminf(slo[128 + c], slo[192 + c]));
                hi = fmaxf(fmaxf(shi[c], shi[64 + c]), fmaxf(shi[128 + c], shi[192 + c]));
                sref[c] = 0.5f * (lo + hi);
                if (!(hi - lo <= kFactorSpread)) atomicOr(&swide[c >> 5], 1);
            }
            __syncthreads();
        }
        // Kf = k e^{g - ref}, Kb = k e^{ref - g}, Qf = q e^{g - ref} (zero in a wide tile: unused there)
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            const int e = tid + 256 * m, a = e >> 3, ch = e & 7;
            const bool wide = swide[ch >> 2] != 0;
            float kf[8], kb[8], qf[8];
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                const int c = 8 * ch + x;
                const float xx = sG[a * 64 + c] - sref[c];
                const float ex = wide ? 0.f : fast_exp(xx), emx = wide ? 0.f : fast_exp(-xx);
                const float kv = __bfloat162float(sK[a * 64 + c]), qv = __bfloat162float(sQ[a * 64 + c]);
                kf[x] = kv * ex;
                kb[x] = kv * emx;
                qf[x] = qv * ex;
            }
            const uint32_t so = sw128_chunk_off(a, ch, 64);
            uint4 hi, lo;
            split8(kb, hi, lo);
            *reinterpret_cast<uint4*>(sm + kG_Kbhi + so) = hi;
            *reinterpret_cast<uint4*>(sm + kG_Kblo + so) = lo;
            split8(qf, hi, lo);
            *reinterpret_cast<uint4*>(sm + kG_Qfhi + so) = hi;
            *reinterpret_cast<uint4*>(sm + kG_Qflo + so) = lo;
            split8(kf, hi, lo);
            *reinterpret_cast<uint4*>(sm + kG_Kfhi + so) = hi;
            *reinterpret_cast<uint4*>(sm + kG_Kflo + so) = lo;
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (tid == 0) {
            const uint32_t idK = idesc_bf16(64, 64, false, true), idT = idesc_bf16(64, 64, true, true);
            // three split terms of one product: (A_hi, B_hi), (A_hi, B_lo), (A_lo, B_hi)
            auto prod = [&](uint32_t d, uint32_t ahi, uint32_t alo, bool amn, uint32_t bhi, uint32_t blo, uint32_t id,
                            bool first) {
                const uint32_t as[3] = {ahi, ahi, alo}, bs[3] = {bhi, blo, bhi};
#pragma unroll
                for (int t = 0; t < 3; ++t)
#pragma unroll
                    for (int k0 = 0; k0 < kChunk; k0 += 16)
                        mma_bf16(tmem + d, amn ? desc_mnmajor(sb + as[t], 64, k0) : desc_kmajor(sb + as[t], 64, k0),
                                 desc_mnmajor(sb + bs[t], 64, k0), id, (first && t == 0 && k0 == 0) ? 0u : 1u);
            };
            prod(0, kG_Phi, kG_Plo, false, kG_Kbhi, kG_Kblo, idK, true);     // rowP = dP Kb
            prod(64, kG_Ahi, kG_Alo, false, kG_Kbhi, kG_Kblo, idK, true);    // rowA = dAt Kb
            prod(128, kG_Phi, kG_Plo, true, kG_Qfhi, kG_Qflo, idT, true);    // col = dP^T Qf
            prod(128, kG_Ahi, kG_Alo, true, kG_Kfhi, kG_Kflo, idT, false);   //     + dAt^T Kf
            prod(192, kG_Nhi, kG_Nlo, true, kG_Whi, kG_Wlo, idT, true);      // dkt = N^T dW
            mma_commit(mbar);
        }
        const bool ok = mbar_wait(mbar, ph);
        fence_after_sync();
        const bool wide = swide[hh] != 0;
        float rowP[16], rowA[16], col[16], dkt[16];
        {
            const uint32_t tl = tmem + ((uint32_t)(32 * qd) << 16) + 32 * hh;
            tmem_ld16_pair<16>(tl, rowP);
            tmem_ld16_pair<16>(tl + 64, rowA);
            tmem_ld16_pair<16>(tl + 128, col);
            tmem_ld16_pair<16>(tl + 192, dkt);
            tmem_wait_ld();
        }
        if (wide) {  // exact per-element factors e^{g_r - g_i} (never above 1), dP and dAt as hi + lo
#pragma unroll
            for (int x = 0; x < 16; ++x) {
                const int c = cb + x;
                const float gr = sG[r * 64 + c];
                float p = 0.f, a = 0.f, cl = 0.f;
                for (int i = 0; i <= r; ++i) {
                    const float ke = __bfloat162float(sK[i * 64 + c]) * fast_exp(gr - sG[i * 64 + c]);
                    const uint32_t oi = sw128_off(r, i, 64);
                    const float dpv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + kG_Phi + oi)) +
                                      __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + kG_Plo + oi));
                    const float dav = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + kG_Ahi + oi)) +
                                      __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + kG_Alo + oi));
                    p = fmaf(dpv, ke, p);
                    a = fmaf(dav, ke, a);
                }
                for (int i = r; i < kChunk; ++i) {
                    const uint32_t oi = sw128_off(i, r, 64);
                    const float dpv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + kG_Phi + oi)) +
                                      __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + kG_Plo + oi));
                    const float dav = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + kG_Ahi + oi)) +
                                      __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + kG_Alo + oi));
                    cl = fmaf(fmaf(dpv, __bfloat162float(sQ[i * 64 + c]), dav * __bfloat162float(sK[i * 64 + c])),
                              fast_exp(sG[i * 64 + c] - gr), cl);
                }
                rowP[x] = p;
                rowA[x] = a;
                col[x] = cl;
            }
        }
        // the element-wise gradients (as in the CUDA-core kernel); dg staged over the B tiles (the MMAs
        // that read them are complete) for the reverse cumulative sum
        {
            float vq[16], vk[16];
#pragma unroll
            for (int x = 0; x < 16; ++x) {
                const int c = cb + x;
                const float g = sG[r * 64 + c], gl = sG[63 * 64 + c];
                float rp = rowP[x], ra = rowA[x], cl = col[x];
                if (!wide) {
                    const float xx = g - sref[c];
                    const float ex = fast_exp(xx);
                    rp *= ex;
                    ra *= ex;
                    cl *= fast_exp(-xx);
                }
                const float kt = dkt[x] * sbeta[r];
                const float eg = fast_exp(g), egl = fast_exp(gl - g);
                const float qv = __bfloat162float(sQ[r * 64 + c]), kv = __bfloat162float(sK[r * 64 + c]);
                vq[x] = rp + dqg[x] * eg;
                vk[x] = ra + cl + kt * eg + dkd[x] * egl;
                sAccG[r * kG_LS + c] = qv * rp + kv * ra - kv * cl + (dqg[x] * qv + kt * kv) * eg - dkd[x] * kv * egl;
                sAccL[r * kG_LS + c] = dkd[x] * kv * egl;  // chunk-end term of g_last, summed below
            }
            if (r < L && ok) {
                const size_t oi = ((size_t)(t0 + r) * H + h) * D + c0 + cb;
                if (dq_acc) {  // grouped heads or the q/k norm: per value head, summed afterwards
#pragma unroll
                    for (int x = 0; x < 16; x += 4) {
                        *reinterpret_cast<float4*>(dq_acc + oi + x) = make_float4(vq[x], vq[x + 1], vq[x + 2], vq[x + 3]);
                        *reinterpret_cast<float4*>(dk_acc + oi + x) = make_float4(vk[x], vk[x + 1], vk[x + 2], vk[x + 3]);
                    }
                } else {
#pragma unroll
                    for (int x = 0; x < 16; x += 8) {
                        *reinterpret_cast<uint4*>(dq + oi + x) = pack8(vq + x);
                        *reinterpret_cast<uint4*>(dk_out + oi + x) = pack8(vk + x);
                    }
                }
            }
        }
        fence_before_sync();
        __syncthreads();
        // dlog_alpha = reverse cumulative sum of dg (plus the g_last terms), channel c = tid % 64 over the
        // row quarter qt = tid / 64: quarter sums first, then each quarter's suffix
        {
            const int c = tid & 63, qt = tid >> 6;
            float sl = 0.f, sg = 0.f;
#pragma unroll
            for (int x = 0; x < 16; ++x) {
                sl += sAccL[(16 * qt + x) * kG_LS + c];
                sg += sAccG[(16 * qt + x) * kG_LS + c];
            }
            slo[qt * 64 + c] = sl;  // the scan's scratch is free again
            shi[qt * 64 + c] = sg;
            __syncthreads();
            float acc = gdGam[c0 + c] * fast_exp(sG[63 * 64 + c]);
            for (int p2 = 0; p2 < 4; ++p2) acc += slo[p2 * 64 + c];
            for (int p2 = qt + 1; p2 < 4; ++p2) acc += shi[p2 * 64 + c];
            if (ok)
                for (int x = 15; x >= 0; --x) {
                    const int rr = 16 * qt + x;
                    acc += sAccG[rr * kG_LS + c];
                    if (rr < L) dla[((size_t)(t0 + rr) * H + h) * D + c0 + c] = acc;
                }
        }
        fence_before_sync();
        __syncthreads();  // the tiles, the staging and TMEM free for the next item
        fence_after_sync();
    }
    if (warp == 0) tmem_dealloc(tmem, 256);
}

inline cudaError_t launch_bwd_gate_tc(const void* q, const void* k, const void* la, bool la16, const float* beta,
                                      const WsHeader* hdr, const int* off, const int32_t* cu, int Tseq, int N, int H,
                                      int Hk, int max_chunks, const float* scr, void* dq, void* dk_out, float* dla,
                                      float* dq_acc, float* dk_acc, cudaStream_t stream)
{
    auto* kern = la16 ? bwd_gate_tc_kernel<true> : bwd_gate_tc_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kG_Smem);
    if (e != cudaSuccess) return e;
    const long long items = (long long)max_chunks * H * 2;
    if (items == 0) return cudaSuccess;
    if (items > 0x7fffffffLL) return cudaErrorInvalidValue;
    const unsigned grid = (unsigned)items;
    LaunchScope ls("bwd_gate_tc", stream);
    kern<<<grid, 256, kG_Smem, stream>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, la, beta, hdr, off, cu, Tseq, N, H, Hk, scr,
        (__nv_bfloat16*)dq, (__nv_bfloat16*)dk_out, dla, dq_acc, dk_acc);
    return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------------
// Step 4a of the input side's first half on the tensor cores (called by bwd_ut_kernel<bf16, true>):
//     At = strict_lower(Kf Kb^T),   dT = lower_incl(dW Kt^T + dU V^T)
// over two 64-channel blocks of the key dimension and two of the value dimension, accumulated in
// TMEM by split-bf16 MMAs (M = N = K = 64 per block).  The scratch is the kernel's own shared memory
// below its beta array, which the UT step reuses afterwards for its fp32 matrices.  A 32-channel
// tile with a wide gate spread contributes to At through exact per-element factors on the CUDA cores
// (accA, at the thread's (tr + 16 a, tc + 16 b) elements), as in the CUDA-core loop.
// ------------------------------------------------------------------------------------------------
constexpr uint32_t kU_Kfhi = 0, kU_Kflo = 8192, kU_Kbhi = 16384, kU_Kblo = 24576;  // K-major [token][64 ch]
constexpr uint32_t kU_Ahi = 32768, kU_Alo = 40960;  // dW or dU block [token r][64]
constexpr uint32_t kU_Bhi = 49152, kU_Blo = 57344;  // Kt or V block [token i][64]
constexpr uint32_t kU_G = 65536;                    // fp32 [64][64] cumulative gate of the block
constexpr uint32_t kU_K = 81920;                    // bf16 [64][64] k of the block
constexpr uint32_t kU_S = 90112;                    // scan scratch: totals, lo, hi [4][64] x 3 | ref [64] | wide [2]
constexpr uint32_t kU_End = kU_S + 3072 + 256 + 16;
static_assert(kU_End + 1024 <= sizeof(float) * (3 * kChunk * kBwdL64 + 6 * kChunk * kBwdLT),
              "step 4a scratch must fit below bwd_ut_kernel's beta array");

__device__ void bwd_ut_step4a_tc(const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                                 const void* __restrict__ log_alpha, bool la16, long long t0, int L, int H, int Hk,
                                 int h, const float* __restrict__ gdW, const float* __restrict__ gdU, float* smem,
                                 float* sAt, float* sM, float (&accA)[4][4])
{
    using namespace tc;
    constexpr int D = 128, L64 = kBwdL64;
    __shared__ uint64_t s_mbar;
    __shared__ uint32_t s_tm;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, tr = tid >> 4, tcc = tid & 15;
    uint8_t* ab = align1024(reinterpret_cast<uint8_t*>(smem));
    const uint32_t sbs = smem_u32(ab);
    const uint32_t mbar = smem_u32(&s_mbar);
    float* sG = reinterpret_cast<float*>(ab + kU_G);
    __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(ab + kU_K);
    float* stot = reinterpret_cast<float*>(ab + kU_S);
    float* slo = stot + 256;
    float* shi = slo + 256;
    float* sref = shi + 256;
    int* swide = reinterpret_cast<int*>(sref + 64);
    const int hq = h / (H / Hk);  // the q/k head of value head h
    const uint4 z4 = make_uint4(0, 0, 0, 0);

    __syncthreads();  // the caller is done with this memory
    if (tid == 0) {
        mbar_init(mbar, 1);
        mbar_fence_init();
    }
    if (warp == 0) tmem_alloc(smem_u32(&s_tm), 128);  // no relinquish: the UT stages allocate again
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = s_tm;  // At in columns 0..63, dT in 64..127 (M = 64 accumulators)
    const uint32_t idK = idesc_bf16(64, 64, false, false);
    uint32_t ph = 0;
    bool ok = true;

    // key-channel blocks: At += Kf Kb^T, dT += dW Kt^T
    for (int blk = 0; blk < 2; ++blk, ph ^= 1u) {
        const int c0 = 64 * blk;
        if (tid == 0) swide[0] = swide[1] = 0;
        {
            float fw[2][8], fg[2][8];
            uint4 kr[2];
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                const int e = tid + 256 * m, rr = e >> 3, ch = e & 7;
                load8(gdW + (size_t)rr * D + c0 + 8 * ch, fw[m]);
                const bool in = rr < L;
                const size_t ia = ((size_t)(t0 + (in ? rr : 0)) * H + h) * D + c0 + 8 * ch;
                if (la16) load8(reinterpret_cast<const __nv_bfloat16*>(log_alpha) + ia, fg[m]);
                else load8(reinterpret_cast<const float*>(log_alpha) + ia, fg[m]);
                if (!in)
#pragma unroll
                    for (int x = 0; x < 8; ++x) fg[m][x] = 0.f;  // rows past the chunk's end add nothing
                kr[m] = in ? *reinterpret_cast<const uint4*>(k + ((size_t)(t0 + rr) * Hk + hq) * D + c0 + 8 * ch) : z4;
            }
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                const int e = tid + 256 * m, rr = e >> 3, ch = e & 7;
                uint4 hi, lo;
                split8(fw[m], hi, lo);
                *reinterpret_cast<uint4*>(ab + kU_Ahi + sw128_chunk_off(rr, ch, 64)) = hi;
                *reinterpret_cast<uint4*>(ab + kU_Alo + sw128_chunk_off(rr, ch, 64)) = lo;
                *reinterpret_cast<float4*>(sG + rr * 64 + 8 * ch) = make_float4(fg[m][0], fg[m][1], fg[m][2], fg[m][3]);
                *reinterpret_cast<float4*>(sG + rr * 64 + 8 * ch + 4) = make_float4(fg[m][4], fg[m][5], fg[m][6], fg[m][7]);
                *reinterpret_cast<uint4*>(sK + rr * 64 + 8 * ch) = kr[m];
            }
        }
        __syncthreads();
        {  // cumulative gate: thread (channel c, quarter qt), as in the gate kernel
            const int c = tid & 63, qt = tid >> 6;
            float gv[16], acc = 0.f;
#pragma unroll
            for (int x = 0; x < 16; ++x) {
                acc += sG[(16 * qt + x) * 64 + c];
                gv[x] = acc;
            }
            stot[qt * 64 + c] = acc;
            __syncthreads();
            float carry = 0.f;
            for (int p2 = 0; p2 < qt; ++p2) carry += stot[p2 * 64 + c];
            float lo = qt == 0 ? 0.f : carry, hi = lo;
#pragma unroll
            for (int x = 0; x < 16; ++x) {
                gv[x] += carry;
                lo = fminf(lo, gv[x]);
                hi = fmaxf(hi, gv[x]);
                sG[(16 * qt + x) * 64 + c] = gv[x];
            }
            slo[qt * 64 + c] = lo;
            shi[qt * 64 + c] = hi;
            __syncthreads();
            if (tid < 64) {
                lo = fminf(fminf(slo[c], slo[64 + c]), fminf(slo[128 + c], slo[192 + c]));
                hi = fmaxf(fmaxf(shi[c], shi[64 + c]), fmaxf(shi[128 + c], shi[192 + c]));
                sref[c] = 0.5f * (lo + hi);
                if (!(hi - lo <= kFactorSpread)) atomicOr(&swide[c >> 5], 1);
            }
            __syncthreads();
        }
        // Kf = k e^{g - ref}, Kb = k e^{ref - g} (zero in a wide tile), Kt = k e^{g}
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            const int e = tid + 256 * m, a = e >> 3, ch = e & 7;
            const bool wide = swide[ch >> 2] != 0;
            float kf[8], kb[8], kt[8];
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                const int c = 8 * ch + x;
                const float g = sG[a * 64 + c], xx = g - sref[c], kv = __bfloat162float(sK[a * 64 + c]);
                kf[x] = wide ? 0.f : kv * fast_exp(xx);
                kb[x] = wide ? 0.f : kv * fast_exp(-xx);
                kt[x] = kv * fast_exp(g);
            }
            const uint32_t so = sw128_chunk_off(a, ch, 64);
            uint4 hi, lo;
            split8(kf, hi, lo);
            *reinterpret_cast<uint4*>(ab + kU_Kfhi + so) = hi;
            *reinterpret_cast<uint4*>(ab + kU_Kflo + so) = lo;
            split8(kb, hi, lo);
            *reinterpret_cast<uint4*>(ab + kU_Kbhi + so) = hi;
            *reinterpret_cast<uint4*>(ab + kU_Kblo + so) = lo;
            split8(kt, hi, lo);
            *reinterpret_cast<uint4*>(ab + kU_Bhi + so) = hi;
            *reinterpret_cast<uint4*>(ab + kU_Blo + so) = lo;
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (tid == 0) {
            const uint32_t fa[3] = {kU_Kfhi, kU_Kfhi, kU_Kflo}, fb[3] = {kU_Kbhi, kU_Kblo, kU_Kbhi};
            const uint32_t wa[3] = {kU_Ahi, kU_Ahi, kU_Alo}, wb[3] = {kU_Bhi, kU_Blo, kU_Bhi};
#pragma unroll
            for (int t = 0; t < 3; ++t)
#pragma unroll
                for (int k0 = 0; k0 < 64; k0 += 16) {
                    const uint32_t acc = (blk > 0 || t > 0 || k0 > 0) ? 1u : 0u;
                    mma_bf16(tmem, desc_kmajor(sbs + fa[t], 64, k0), desc_kmajor(sbs + fb[t], 64, k0), idK, acc);
                    mma_bf16(tmem + 64, desc_kmajor(sbs + wa[t], 64, k0), desc_kmajor(sbs + wb[t], 64, k0), idK, acc);
                }
            mma_commit(mbar);
        }
        // a wide tile's At terms, exactly: sum over its channels of k_r k_i e^{g_r - g_i} (i < r)
#pragma unroll 1
        for (int w = 0; w < 2; ++w) {
            if (!swide[w]) continue;
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const int r = tr + 16 * a, i = tcc + 16 * b;
                    if (i >= r) continue;
                    float x = 0.f;
                    for (int cc = 32 * w; cc < 32 * w + 32; ++cc)
                        x = fmaf(__bfloat162float(sK[r * 64 + cc]) * __bfloat162float(sK[i * 64 + cc]),
                                 fast_exp(sG[r * 64 + cc] - sG[i * 64 + cc]), x);
                    accA[a][b] += x;
                }
        }
        ok = mbar_wait(mbar, ph) && ok;
        fence_after_sync();
        __syncthreads();  // the tiles are free for the next block
    }
    // value blocks: dT += dU V^T (V is exact in bf16: dU_hi V + dU_lo V)
    for (int blk = 0; blk < 2; ++blk, ph ^= 1u) {
        const int c0 = 64 * blk;
        {
            float fu[2][8];
            uint4 vr[2];
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                const int e = tid + 256 * m, rr = e >> 3, ch = e & 7;
                load8(gdU + (size_t)rr * D + c0 + 8 * ch, fu[m]);
                vr[m] = rr < L ? *reinterpret_cast<const uint4*>(v + ((size_t)(t0 + rr) * H + h) * D + c0 + 8 * ch) : z4;
            }
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                const int e = tid + 256 * m, rr = e >> 3, ch = e & 7;
                const uint32_t so = sw128_chunk_off(rr, ch, 64);
                uint4 hi, lo;
                split8(fu[m], hi, lo);
                *reinterpret_cast<uint4*>(ab + kU_Ahi + so) = hi;
                *reinterpret_cast<uint4*>(ab + kU_Alo + so) = lo;
                *reinterpret_cast<uint4*>(ab + kU_Bhi + so) = vr[m];
            }
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (tid == 0) {
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int k0 = 0; k0 < 64; k0 += 16)
                    mma_bf16(tmem + 64, desc_kmajor(sbs + (t ? kU_Alo : kU_Ahi), 64, k0), desc_kmajor(sbs + kU_Bhi, 64, k0),
                             idK, 1u);
            mma_commit(mbar);
        }
        ok = mbar_wait(mbar, ph) && ok;
        fence_after_sync();
        __syncthreads();
    }
    // At (strictly lower) and dT (lower, inclusive) from TMEM (M = 64: row 16 q + lane % 16, columns
    // 32 half + 16 (lane / 16) .. +15), over the dead tiles
    {
        const int q = warp & 3, half = warp >> 2;
        const int r = 16 * q + (lane & 15), cb = 32 * half + 16 * (lane >> 4);
        const uint32_t tl = tmem + ((uint32_t)(32 * q) << 16) + 32 * half;
        float va[16], vt[16];
        tmem_ld16_pair<16>(tl, va);
        tmem_ld16_pair<16>(tl + 64, vt);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 16; ++x) {
            const int i = cb + x;
            sAt[r * L64 + i] = (i < r && ok) ? va[x] : 0.f;
            sM[r * L64 + i] = (i <= r && ok) ? vt[x] : 0.f;
        }
    }
    fence_before_sync();
    __syncthreads();
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int r = tr + 16 * a, i = tcc + 16 * b;
            if (i < r) sAt[r * L64 + i] += accA[a][b];  // the wide tiles' exact terms (zero elsewhere)
        }
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 128);
}

// ------------------------------------------------------------------------------------------------
// The two chains of the backward on the tensor cores.  Per (sequence, head, 32-column slice), chunks
// in order (forward) or in reverse (reverse chain), with the carried matrix Z (the state S, or its
// cotangent D) fp32 in registers (thread c owns row c):
//   forward:  X = W S,   U = Uv - X,  S <- Diag(gam) S + Kd^T U          (stores S_c and U)
//   reverse:  Z = Kd D,  dU = E + Z,  D <- Diag(gam) D + F - W^T dU      (stores D_c and dU)
// the recurrences of bwd_fwd_chain_kernel and bwd_dstate_kernel.  Both products are split-bf16
// tcgen05 MMAs (24 + 12 per chunk): W and Kd as bf16 hi/lo images written once per unit by
// bwd_wk_images_kernel, Z and U split by the compute threads every chunk.  Warp roles as in the
// forward's phase B: four compute warps, one MMA warp, one copy warp streaming the images through two
// shared-memory stages.
// ------------------------------------------------------------------------------------------------
// the unit's image region inside its scratch (over dQg and dW, which the state side writes later):
// W hi | W lo | Kd hi | Kd lo, each a 64-row x 128 SW128 tile (two 8 KB atom columns)
__host__ __device__ inline size_t bwd_wk_image_offset_floats() { return 2 * (size_t)kChunk * 128; }
constexpr uint32_t kImgW = 0, kImgWlo = 16384, kImgKd = 32768, kImgKdlo = 49152, kImgBytes = 65536;

__global__ void __launch_bounds__(256)
bwd_wk_images_kernel(const WsHeader* __restrict__ hdr, int H, const float* __restrict__ slots, float* __restrict__ scr)
{
    using namespace tc;
    constexpr int D = 128;
    const int j = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    if (hdr->bad || j >= hdr->total_chunks) return;
    const size_t u = (size_t)j * H + h;
    const float* slot = slots + u * simt_slot_floats(D, D);
    uint8_t* img = reinterpret_cast<uint8_t*>(scr + u * bwd_scr_floats(D, D) + bwd_wk_image_offset_floats());
#pragma unroll
    for (int m = 0; m < 8; ++m) {  // task e: matrix e / 1024 (W, Kd), row (e % 1024) / 16, chunk e % 16
        const int e = tid + 256 * m, mat = e >> 10, r = (e >> 4) & 63, ch = e & 15;
        float f[8];
        load8(slot + (size_t)mat * 2 * kChunk * D + (size_t)r * D + 8 * ch, f);
        uint4 hi, lo;
        split8(f, hi, lo);
        const uint32_t o = (mat ? kImgKd : kImgW) + sw128_chunk_off(r, ch, 64);
        *reinterpret_cast<uint4*>(img + o) = hi;
        *reinterpret_cast<uint4*>(img + o + 16384) = lo;
    }
}

constexpr int kChThreads = 192;                       // compute warps 0-3, MMA warp 4, copy warp 5
constexpr uint32_t kChStage = 65536;                  // one unit's four images
constexpr uint32_t kChZ = 2 * kChStage;               // Z hi, lo: 128 rows (K = key channel) x 32 (SW128, 16 KB each)
constexpr uint32_t kChU = kChZ + 32768;               // U hi, lo: 64 rows (K = token) x 32 (8 KB each)
constexpr uint32_t kChMisc = kChU + 16384;            // mbarriers | TMEM address | abort flag
constexpr uint32_t kChSmem = kChMisc + 256 + 1024;
static_assert(kChSmem <= 232448, "chain shared memory");

template <bool REV>
__global__ void __launch_bounds__(kChThreads, 1)
bwd_chain_tc_kernel(const float* __restrict__ Z_init, float* __restrict__ Z_final, const WsHeader* __restrict__ hdr,
                    const int* __restrict__ off, int N, int H, const float* __restrict__ slots, float* __restrict__ scr,
                    float* __restrict__ Z_chunks, const float* __restrict__ F_chunks)
{
    using namespace tc;
    constexpr int D = 128, NV = 32;
    extern __shared__ uint8_t smem_raw[];
    const int n = blockIdx.x, h = blockIdx.y, v0 = blockIdx.z * NV, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (hdr->bad) return;
    uint8_t* sm = align1024(smem_raw);
    const uint32_t sb = smem_u32(sm);
    const uint32_t bar_full = sb + kChMisc;   // [2]
    const uint32_t bar_empty = bar_full + 16;  // [2]: the stage's MMAs are complete
    const uint32_t bar_p1 = bar_full + 32, bar_p2 = bar_full + 40;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + kChMisc + 64);
    volatile int* s_abort = reinterpret_cast<volatile int*>(sm + kChMisc + 68);
    const size_t slot_f = simt_slot_floats(D, D), scr_f = bwd_scr_floats(D, D);
    const size_t zidx = ((size_t)n * H + h) * D * D;
    const int j0 = off[n], j1 = off[n + 1], nch = j1 - j0;
    auto chunk = [&](int it) { return REV ? j1 - 1 - it : j0 + it; };
    auto img_of = [&](int j) {
        return reinterpret_cast<const uint8_t*>(scr + ((size_t)j * H + h) * scr_f + bwd_wk_image_offset_floats());
    };

    if (tid == 0) {
        mbar_init(bar_full, 1);
        mbar_init(bar_full + 8, 1);
        mbar_init(bar_empty, 1);
        mbar_init(bar_empty + 8, 1);
        mbar_init(bar_p1, 1);
        mbar_init(bar_p2, 1);
        mbar_fence_init();
        *s_abort = 0;
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(s_tmem), 64);
        tmem_relinquish();
    }
    // the carried matrix: thread c < 128 owns row c of this slice
    const int c = tid;
    float Z[NV];
    if (warp < 4) {
#pragma unroll
        for (int m = 0; m < NV; m += 4) {
            const float4 x = Z_init ? *reinterpret_cast<const float4*>(Z_init + zidx + (size_t)c * D + v0 + m)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
            Z[m] = x.x; Z[m + 1] = x.y; Z[m + 2] = x.z; Z[m + 3] = x.w;
        }
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            uint4 hi, lo;
            split8(Z + 8 * m, hi, lo);
            *reinterpret_cast<uint4*>(sm + kChZ + sw128_chunk_off(c, m, 128)) = hi;
            *reinterpret_cast<uint4*>(sm + kChZ + 16384 + sw128_chunk_off(c, m, 128)) = lo;
        }
    }
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();  // barriers initialised, TMEM address visible, Z tiles written
    fence_after_sync();
    if (warp == 5 && lane == 0) {
        for (int s = 0; s < 2 && s < nch; ++s) {
            const uint8_t* img = img_of(chunk(s));
            mbar_arrive_expect_tx(bar_full + 8 * s, kImgBytes);
            for (int q4 = 0; q4 < 4; ++q4) bulk_g2s(sb + s * kChStage + 16384 * q4, img + 16384 * q4, 16384, bar_full + 8 * s);
        }
        for (int s = 2; s < 4 && s < nch; ++s) bulk_prefetch_l2(img_of(chunk(s)), kImgBytes);
    }
    const uint32_t tmem = *s_tmem;  // P1 result in columns 0..31 (M = 64), P2 in 32..63 (M = 128)
    bool ok = true;
    // compute threads: a chunk's inputs (Uv or E at the first epilogue's row rr and columns cb .. cb + 15,
    // gam of row c, and for REV the row c of F), loaded one chunk ahead
    const int rr = 16 * (warp & 3) + (lane & 15), cb = 16 * (lane >> 4);
    float ua[16], gam = 0.f, fr[NV];
    auto load_inputs = [&](int it, float* ua_, float& gam_, float* fr_) {
        const size_t uu = (size_t)chunk(it) * H + h;
        const float* slot = slots + uu * slot_f;
        const float* uin = REV ? scr + uu * scr_f + (size_t)kChunk * D : slot + (size_t)kChunk * (3 * D + kChunk);
#pragma unroll
        for (int m = 0; m < 16; m += 4) {
            const float4 x = *reinterpret_cast<const float4*>(uin + (size_t)rr * D + v0 + cb + m);
            ua_[m] = x.x; ua_[m + 1] = x.y; ua_[m + 2] = x.z; ua_[m + 3] = x.w;
        }
        gam_ = slot[(size_t)kChunk * (3 * D + kChunk + D) + c];
        if (REV) {
            const float* gF = F_chunks + uu * D * D + (size_t)c * D + v0;
#pragma unroll
            for (int m = 0; m < NV; m += 4) {
                const float4 x = *reinterpret_cast<const float4*>(gF + m);
                fr_[m] = x.x; fr_[m + 1] = x.y; fr_[m + 2] = x.z; fr_[m + 3] = x.w;
            }
        }
    };
    if (warp < 4 && nch > 0) load_inputs(0, ua, gam, fr);

    for (int it = 0; it < nch; ++it) {
        const int j = chunk(it), s = it & 1;
        const uint32_t par = (uint32_t)it & 1u, spar = (uint32_t)(it >> 1) & 1u;
        const size_t u = (size_t)j * H + h;
        const uint32_t st = sb + s * kChStage;
        // A of the first product (K-major) and of the second (its MN-major view): W and Kd, swapped for REV
        const uint32_t a1 = REV ? kImgKd : kImgW, a2 = REV ? kImgW : kImgKd;
        if (warp == 4) {
            if (it > 0) named_sync(2, 160);  // Z tiles of this chunk written
            if (lane == 0) {
                ok = ok && mbar_wait_ab(bar_full + 8 * s, spar, s_abort);
                fence_after_sync();
                if (ok) {
                    const uint32_t id1 = idesc_bf16(64, NV, false, true);
                    const uint32_t as[3] = {a1, a1, a1 + 16384}, bs[3] = {kChZ, kChZ + 16384, kChZ};
#pragma unroll
                    for (int t = 0; t < 3; ++t)
#pragma unroll
                        for (int k0 = 0; k0 < D; k0 += 16)
                            mma_bf16(tmem, desc_kmajor(st + as[t], 64, k0), desc_mnmajor(sb + bs[t], 128, k0), id1,
                                     (t > 0 || k0 > 0) ? 1u : 0u);
                    mma_commit(bar_p1);
                }
            }
            named_sync(1, 160);  // U tiles written
            if (lane == 0 && ok) {
                fence_after_sync();
                const uint32_t id2 = idesc_bf16(128, NV, true, true);
                const uint32_t as[3] = {a2, a2, a2 + 16384}, bs[3] = {kChU, kChU + 8192, kChU};
#pragma unroll
                for (int t = 0; t < 3; ++t)
#pragma unroll
                    for (int k0 = 0; k0 < kChunk; k0 += 16)
                        mma_bf16(tmem + 32, desc_mnmajor(st + as[t], 64, k0), desc_mnmajor(sb + bs[t], 64, k0), id2,
                                 (t > 0 || k0 > 0) ? 1u : 0u);
                mma_commit(bar_p2);
                mma_commit(bar_empty + 8 * s);  // the stage's images are read
            }
        } else if (warp == 5) {
            if (lane == 0 && it + 2 < nch) {
                ok = ok && mbar_wait_ab(bar_empty + 8 * s, spar, s_abort);
                if (ok) {
                    const uint8_t* img = img_of(chunk(it + 2));
                    mbar_arrive_expect_tx(bar_full + 8 * s, kImgBytes);
                    for (int q4 = 0; q4 < 4; ++q4) bulk_g2s(st + 16384 * q4, img + 16384 * q4, 16384, bar_full + 8 * s);
                    if (it + 4 < nch) bulk_prefetch_l2(img_of(chunk(it + 4)), kImgBytes);
                }
            }
        } else {
            // Z_c out (the chunk's start state, or the cotangent at its end) before the update
            float* zc = Z_chunks + u * D * D + (size_t)c * D + v0;
#pragma unroll
            for (int m = 0; m < NV; m += 4) *reinterpret_cast<float4*>(zc + m) = make_float4(Z[m], Z[m + 1], Z[m + 2], Z[m + 3]);
            const int q = warp;
            float* o = scr + u * scr_f;
            float* uout = REV ? o + (size_t)kChunk * D : o;  // dU (over E) : U
            float ua_n[16], gam_n = 0.f, fr_n[NV];          // the next chunk's inputs, in flight meanwhile
            if (it + 1 < nch) load_inputs(it + 1, ua_n, gam_n, fr_n);
            ok = ok && mbar_wait_ab(bar_p1, par, s_abort);
            fence_after_sync();
            {  // U = Uv - X, or dU = E + Z (M = 64: row rr, columns cb .. cb + 15)
                float x[16];
                tmem_ld16_pair<16>(tmem + ((uint32_t)(32 * q) << 16), x);
                tmem_wait_ld();
#pragma unroll
                for (int m = 0; m < 16; ++m) ua[m] = REV ? ua[m] + x[m] : ua[m] - x[m];
                if (ok)
#pragma unroll
                    for (int m = 0; m < 16; m += 4)
                        *reinterpret_cast<float4*>(uout + (size_t)rr * D + v0 + cb + m) =
                            make_float4(ua[m], ua[m + 1], ua[m + 2], ua[m + 3]);
#pragma unroll
                for (int m = 0; m < 2; ++m) {
                    uint4 hi, lo;
                    split8(ua + 8 * m, hi, lo);
                    *reinterpret_cast<uint4*>(sm + kChU + sw128_chunk_off(rr, cb / 8 + m, 64)) = hi;
                    *reinterpret_cast<uint4*>(sm + kChU + 8192 + sw128_chunk_off(rr, cb / 8 + m, 64)) = lo;
                }
                fence_proxy_async();
                fence_before_sync();
                named_arrive(1, 160);
            }
            ok = ok && mbar_wait_ab(bar_p2, par, s_abort);
            fence_after_sync();
            {  // S <- Diag(gam) S + Kd^T U, or D <- Diag(gam) D + F - W^T dU (row c)
                float y[NV];
                const uint32_t tw = tmem + ((uint32_t)(32 * q) << 16) + 32;
                tmem_ld16(tw, y);
                tmem_ld16(tw + 16, y + 16);
                tmem_wait_ld();
#pragma unroll
                for (int m = 0; m < NV; ++m) Z[m] = REV ? fmaf(gam, Z[m], fr[m] - y[m]) : fmaf(gam, Z[m], y[m]);
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    uint4 hi, lo;
                    split8(Z + 8 * m, hi, lo);
                    *reinterpret_cast<uint4*>(sm + kChZ + sw128_chunk_off(c, m, 128)) = hi;
                    *reinterpret_cast<uint4*>(sm + kChZ + 16384 + sw128_chunk_off(c, m, 128)) = lo;
                }
                fence_proxy_async();
                fence_before_sync();
                if (it + 1 < nch) named_arrive(2, 160);
            }
            if (it + 1 < nch) {
#pragma unroll
                for (int m = 0; m < 16; ++m) ua[m] = ua_n[m];
                gam = gam_n;
                if (REV)
#pragma unroll
                    for (int m = 0; m < NV; ++m) fr[m] = fr_n[m];
            }
        }
    }
    ok = __syncthreads_and(ok && !*s_abort);
    if (REV && Z_final && warp < 4 && ok) {  // dS0
#pragma unroll
        for (int m = 0; m < NV; m += 4)
            *reinterpret_cast<float4*>(Z_final + zidx + (size_t)c * D + v0 + m) = make_float4(Z[m], Z[m + 1], Z[m + 2], Z[m + 3]);
    }
    if (tid == 0 && !ok) {  // copies still in flight after a wait gave up: bounded waits for them
        for (int s = 0; s < 2; ++s) (void)mbar_wait(bar_full + 8 * s, 0);
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 64);
}

// ------------------------------------------------------------------------------------------------
// bwd_ut's UT step and dV on the tensor cores (bwd_ut_kernel<bf16, true>), split-bf16 as above, with
// the operand tiles over the kernel's per-tile scratch (free after the inverse; 48 KB at most):
//   Y = dN N^T  ->  dM = strict_lower(-N^T Y)  (into sM)          dV = Diag(beta) N^T dU
// N and dN stay fp32 in sN / sM for the beta sums; N's tile serves K-major for Y and MN-major (its
// transpose) for dM and dV.
// ------------------------------------------------------------------------------------------------
// 64 x 64 fp32 rows (stride 65) -> bf16 hi / lo SW128 tiles (one atom column)
__device__ __forceinline__ void split_64x64(const float* src, uint8_t* hi, uint8_t* lo)
{
    constexpr int L64 = kChunk + 1;
#pragma unroll
    for (int m = 0; m < 2; ++m) {
        const int e = threadIdx.x + 256 * m, r = e >> 3, ch = e & 7;
        float f[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) f[x] = src[r * L64 + 8 * ch + x];
        uint4 h4, l4;
        split8(f, h4, l4);
        *reinterpret_cast<uint4*>(hi + tc::sw128_chunk_off(r, ch, 64)) = h4;
        *reinterpret_cast<uint4*>(lo + tc::sw128_chunk_off(r, ch, 64)) = l4;
    }
}

__device__ void bwd_ut_y_dm_tc(const float* sN, float* sM, float* tiles)
{
    using namespace tc;
    constexpr int L64 = kChunk + 1;
    __shared__ uint64_t s_mb;
    __shared__ uint32_t s_tm;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint8_t* ab = align1024(reinterpret_cast<uint8_t*>(tiles));  // dN | N | Y, hi and lo (8 KB each)
    const uint32_t tb = smem_u32(ab), mbar = smem_u32(&s_mb);
    __syncthreads();  // dN in sM, N in sM's neighbour, and the inverse's scratch is free
    if (tid == 0) {
        mbar_init(mbar, 1);
        mbar_fence_init();
    }
    if (warp == 0) tmem_alloc(smem_u32(&s_tm), 128);  // no relinquish: the dV stage allocates again
    split_64x64(sM, ab, ab + 8192);           // dN
    split_64x64(sN, ab + 16384, ab + 24576);  // N
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = s_tm;
    const int q = warp & 3, half = warp >> 2, r = 16 * q + (lane & 15), cb = 32 * half + 16 * (lane >> 4);
    const uint32_t tl = tmem + ((uint32_t)(32 * q) << 16) + 32 * half;
    if (tid == 0) {  // Y[r][i'] = sum_i dN[r][i] N[i'][i]
        const uint32_t id = idesc_bf16(64, 64, false, false);
        const uint32_t as[3] = {0u, 0u, 8192u}, bs[3] = {16384u, 24576u, 16384u};
#pragma unroll
        for (int t = 0; t < 3; ++t)
#pragma unroll
            for (int k0 = 0; k0 < kChunk; k0 += 16)
                mma_bf16(tmem, desc_kmajor(tb + as[t], 64, k0), desc_kmajor(tb + bs[t], 64, k0), id,
                         (t > 0 || k0 > 0) ? 1u : 0u);
        mma_commit(mbar);
    }
    bool ok = mbar_wait(mbar, 0);
    fence_after_sync();
    {  // Y -> hi / lo tiles (row r, columns cb .. cb + 15): the B operand of dM, read MN-major
        float y[16];
        tmem_ld16_pair<16>(tl, y);
        tmem_wait_ld();
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            uint4 h4, l4;
            split8(y + 8 * m, h4, l4);
            *reinterpret_cast<uint4*>(ab + 32768 + sw128_chunk_off(r, cb / 8 + m, 64)) = h4;
            *reinterpret_cast<uint4*>(ab + 40960 + sw128_chunk_off(r, cb / 8 + m, 64)) = l4;
        }
    }
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (tid == 0) {  // (N^T Y)[r][i] = sum_a N[a][r] Y[a][i]
        const uint32_t id = idesc_bf16(64, 64, true, true);
        const uint32_t as[3] = {16384u, 16384u, 24576u}, bs[3] = {32768u, 40960u, 32768u};
#pragma unroll
        for (int t = 0; t < 3; ++t)
#pragma unroll
            for (int k0 = 0; k0 < kChunk; k0 += 16)
                mma_bf16(tmem + 64, desc_mnmajor(tb + as[t], 64, k0), desc_mnmajor(tb + bs[t], 64, k0), id,
                         (t > 0 || k0 > 0) ? 1u : 0u);
        mma_commit(mbar);
    }
    ok = mbar_wait(mbar, 1) && ok;
    fence_after_sync();
    {
        float d[16];
        tmem_ld16_pair<16>(tl + 64, d);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 16; ++x) {
            const int i = cb + x;
            sM[r * L64 + i] = (i < r && ok) ? -d[x] : 0.f;
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 128);
}

__device__ void bwd_ut_dv_tc(const float* sN, const float* sb, const float* __restrict__ gdU, __nv_bfloat16* dv_out,
                             long long t0, int L, int H, int h, float* tiles)
{
    using namespace tc;
    constexpr int D = 128;
    __shared__ uint64_t s_mb;
    __shared__ uint32_t s_tm;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint8_t* ab = align1024(reinterpret_cast<uint8_t*>(tiles));  // N hi | lo (8 KB each), dU hi | lo (16 KB each)
    const uint32_t tb = smem_u32(ab), mbar = smem_u32(&s_mb);
    __syncthreads();
    if (tid == 0) {
        mbar_init(mbar, 1);
        mbar_fence_init();
    }
    if (warp == 0) {  // the CTA's last allocation: the permit can go
        tmem_alloc(smem_u32(&s_tm), 128);
        tmem_relinquish();
    }
    split_64x64(sN, ab, ab + 8192);
#pragma unroll
    for (int m = 0; m < 4; ++m) {  // dU [a][j] (MN-major B: rows a = K)
        const int e = tid + 256 * m, a = e >> 4, ch = e & 15;
        float f[8];
        load8(gdU + (size_t)a * D + 8 * ch, f);
        uint4 h4, l4;
        split8(f, h4, l4);
        *reinterpret_cast<uint4*>(ab + 16384 + sw128_chunk_off(a, ch, 64)) = h4;
        *reinterpret_cast<uint4*>(ab + 32768 + sw128_chunk_off(a, ch, 64)) = l4;
    }
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = s_tm;
    if (tid == 0) {  // (N^T dU)[i][j] = sum_a N[a][i] dU[a][j]
        const uint32_t id = idesc_bf16(64, 128, true, true);
        const uint32_t as[3] = {0u, 0u, 8192u}, bs[3] = {16384u, 32768u, 16384u};
#pragma unroll
        for (int t = 0; t < 3; ++t)
#pragma unroll
            for (int k0 = 0; k0 < kChunk; k0 += 16)
                mma_bf16(tmem, desc_mnmajor(tb + as[t], 64, k0), desc_mnmajor(tb + bs[t], 64, k0), id,
                         (t > 0 || k0 > 0) ? 1u : 0u);
        mma_commit(mbar);
    }
    const bool ok = mbar_wait(mbar, 0);
    fence_after_sync();
    // M = 64: row i = 16 q + lane % 16; warps 0-3 columns 0..63, warps 4-7 64..127
    const int q = warp & 3, half = warp >> 2, i = 16 * q + (lane & 15);
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        float x[16];
        tmem_ld16_pair<16>(tmem + ((uint32_t)(32 * q) << 16) + 64 * half + 32 * t, x);
        tmem_wait_ld();
        if (i < L && ok) {
            const int c0 = 64 * half + 32 * t + 16 * (lane >> 4);
            const float bi = sb[i];
#pragma unroll
            for (int m = 0; m < 16; ++m) x[m] *= bi;
            uint4* dst = reinterpret_cast<uint4*>(dv_out + ((size_t)(t0 + i) * H + h) * D + c0);
            dst[0] = pack8(x);
            dst[1] = pack8(x + 8);
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 128);
}

// ------------------------------------------------------------------------------------------------
// The backward's forward recompute (simt_intra_kernel<bf16, true>, dk = dv = 128): its two product
// stages as split-bf16 tcgen05 MMAs, with the operand tiles over regions of the kernel's own shared
// memory that are dead at that point (its fp32 layout, which starts 1024-aligned in this variant:
// k, q, g, v, Kt at 33,024-byte strides, then A, P, T at 16,640): Qf over k (32 KB from offset 0),
// Kf over v (from 99,328 to 132,096, the start of Kt), Kb over A and P (from 165,888; its last
// 256 bytes reach into T, unused until the inverse), and in the second stage T, [Kt | V] and Kt's
// lo part over k and q (64 KB from offset 0):
//   A = strict_lower(diag(beta) Kf Kb^T), P = lower_incl(Qf Kb^T)     (factorised chunks only)
//   [W | Uv] = T [Kt | V]                                             (one N = 256 product)
// ------------------------------------------------------------------------------------------------
// the MMA-completion barrier and 256 TMEM columns, at the kernel's start (read after its barriers)
__device__ void simt_intra_tc_setup(uint32_t* s_tm, uint64_t* s_mb)
{
    using namespace tc;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(s_mb), 1);
        mbar_fence_init();
    }
    if ((threadIdx.x >> 5) == 0) {
        tmem_alloc(smem_u32(s_tm), 256);
        tmem_relinquish();
    }
}

__device__ void simt_intra_ap_tc(const float* sk, const float* sq, const float* sg, float* sv, const float* sb,
                                 float* sA, float* sP, uint32_t* s_tm, uint64_t* s_mb)
{
    using namespace tc;
    constexpr int LK = 129, L64 = kChunk + 1;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint8_t* tq = align1024(reinterpret_cast<uint8_t*>(const_cast<float*>(sk)));  // Qf hi | lo (over k)
    uint8_t* tf = align1024(reinterpret_cast<uint8_t*>(sv));                       // Kf hi | lo (over v)
    uint8_t* tb = align1024(reinterpret_cast<uint8_t*>(sA));                       // Kb hi | lo (over A, P)
    const uint32_t mbar = smem_u32(s_mb);
    // 64 rows x 16 chunks of 8 channels; rows are padded fp32 (stride 129), read as scalars
    auto split_rows = [&](const float* src, uint8_t* dst) {
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int e = tid + 256 * m, r = e >> 4, ch = e & 15;
            float f[8];
#pragma unroll
            for (int x = 0; x < 8; ++x) f[x] = src[r * LK + 8 * ch + x];
            uint4 hi, lo;
            split8(f, hi, lo);
            *reinterpret_cast<uint4*>(dst + sw128_chunk_off(r, ch, 64)) = hi;
            *reinterpret_cast<uint4*>(dst + 16384 + sw128_chunk_off(r, ch, 64)) = lo;
        }
    };
    split_rows(sk, tf);  // Kf (in sk) -> over v
    split_rows(sg, tb);  // Kb (in sg) -> over A, P
    __syncthreads();     // every read of sk is done
    split_rows(sq, tq);  // Qf -> over k
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *s_tm;
    if (tid == 0) {
        const uint32_t id = idesc_bf16(64, 64, false, false);
        const uint32_t ta = smem_u32(tf), tqq = smem_u32(tq), tbb = smem_u32(tb);
#pragma unroll
        for (int t = 0; t < 3; ++t) {
            const uint32_t ao = t == 2 ? 16384u : 0u, bo = t == 1 ? 16384u : 0u;
#pragma unroll
            for (int k0 = 0; k0 < 128; k0 += 16) {
                const uint32_t acc = (t > 0 || k0 > 0) ? 1u : 0u;
                mma_bf16(tmem, desc_kmajor(ta + ao, 64, k0), desc_kmajor(tbb + bo, 64, k0), id, acc);       // Kf Kb^T
                mma_bf16(tmem + 64, desc_kmajor(tqq + ao, 64, k0), desc_kmajor(tbb + bo, 64, k0), id, acc);  // Qf Kb^T
            }
        }
        mma_commit(mbar);
    }
    const bool ok = mbar_wait(mbar, 0);
    fence_after_sync();
    // M = 64 accumulators: row 16 q + lane % 16, columns 32 half + 16 (lane / 16) .. +15
    const int q = warp & 3, half = warp >> 2, r = 16 * q + (lane & 15), cb = 32 * half + 16 * (lane >> 4);
    float va[16], vp[16];
    const uint32_t tl = tmem + ((uint32_t)(32 * q) << 16) + 32 * half;
    tmem_ld16_pair<16>(tl, va);
    tmem_ld16_pair<16>(tl + 64, vp);
    tmem_wait_ld();
    __syncthreads();  // the Kb tiles under sA / sP are no longer read by anyone
#pragma unroll
    for (int x = 0; x < 16; ++x) {
        const int i = cb + x;
        sA[r * L64 + i] = (i < r && ok) ? sb[r] * va[x] : 0.f;
        sP[r * L64 + i] = (i <= r && ok) ? vp[x] : 0.f;
    }
}

__device__ void simt_intra_wuv_tc(const float* sT, const float* sKt, const __nv_bfloat16* __restrict__ v, long long t0,
                                  int L, int H, int h, float* tiles, float* __restrict__ gW, float* __restrict__ gUv,
                                  uint32_t* s_tm, uint64_t* s_mb, uint32_t phase)
{
    using namespace tc;
    constexpr int LK = 129, L64 = kChunk + 1, D = 128;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint8_t* tt = align1024(reinterpret_cast<uint8_t*>(tiles));  // T hi | lo (8 KB each)
    uint8_t* bh = tt + 16384;                                    // [Kt | V] hi: four atom columns (32 KB)
    uint8_t* bl = bh + 32768;                                    // Kt lo: two atom columns (16 KB)
    const uint32_t mbar = smem_u32(s_mb);
    // T [r][i] (K-major, 64 x 64): 512 tasks of 8
#pragma unroll
    for (int m = 0; m < 2; ++m) {
        const int e = tid + 256 * m, r = e >> 3, ch = e & 7;
        float f[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) f[x] = sT[r * L64 + 8 * ch + x];
        uint4 hi, lo;
        split8(f, hi, lo);
        *reinterpret_cast<uint4*>(tt + sw128_chunk_off(r, ch, 64)) = hi;
        *reinterpret_cast<uint4*>(tt + 8192 + sw128_chunk_off(r, ch, 64)) = lo;
    }
    // Kt [i][c] and V [i][j] (MN-major: rows i = K): 1,024 tasks of 8 each
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int e = tid + 256 * m, i = e >> 4, ch = e & 15;
        float f[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) f[x] = sKt[i * LK + 8 * ch + x];
        uint4 hi, lo;
        split8(f, hi, lo);
        *reinterpret_cast<uint4*>(bh + sw128_chunk_off(i, ch, 64)) = hi;
        *reinterpret_cast<uint4*>(bl + sw128_chunk_off(i, ch, 64)) = lo;
        *reinterpret_cast<uint4*>(bh + sw128_chunk_off(i, 16 + ch, 64)) =
            i < L ? *reinterpret_cast<const uint4*>(v + ((size_t)(t0 + i) * H + h) * D + 8 * ch) : make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *s_tm;
    if (tid == 0) {
        const uint32_t id256 = idesc_bf16(64, 256, false, true), id128 = idesc_bf16(64, 128, false, true);
        const uint32_t ta = smem_u32(tt), bhh = smem_u32(bh), bll = smem_u32(bl);
#pragma unroll
        for (int k0 = 0; k0 < kChunk; k0 += 16)
            mma_bf16(tmem, desc_kmajor(ta, 64, k0), desc_mnmajor(bhh, 64, k0), id256, k0 > 0 ? 1u : 0u);  // T_hi B_hi
#pragma unroll
        for (int k0 = 0; k0 < kChunk; k0 += 16)
            mma_bf16(tmem, desc_kmajor(ta, 64, k0), desc_mnmajor(bll, 64, k0), id128, 1u);  // T_hi Kt_lo
#pragma unroll
        for (int k0 = 0; k0 < kChunk; k0 += 16)
            mma_bf16(tmem, desc_kmajor(ta + 8192, 64, k0), desc_mnmajor(bhh, 64, k0), id256, 1u);  // T_lo B_hi
        mma_commit(mbar);
    }
    const bool ok = mbar_wait(mbar, phase);
    fence_after_sync();
    // M = 64: row 16 q + lane % 16; warps 0-3 columns 0..127 (W), warps 4-7 columns 128..255 (Uv)
    const int q = warp & 3, half = warp >> 2, r = 16 * q + (lane & 15);
    float* dst = (half == 0 ? gW : gUv) + (size_t)r * D;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        float x[16];
        tmem_ld16_pair<16>(tmem + ((uint32_t)(32 * q) << 16) + 128 * half + 32 * t, x);
        tmem_wait_ld();
        const int c0 = 32 * t + 16 * (lane >> 4);
        if (ok)
#pragma unroll
            for (int m = 0; m < 16; m += 4)
                *reinterpret_cast<float4*>(dst + c0 + m) = make_float4(x[m], x[m + 1], x[m + 2], x[m + 3]);
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

inline bool bwd_state_side_tc_ok(bool bf16, int dk, int dv) { return kTcPathReady && bf16 && dk == 128 && dv == 128; }

inline cudaError_t launch_bwd_chains_tc(const float* S0, const float* dS_final, float* dS0, const WsHeader* hdr,
                                       const int* off, int N, int H, int max_chunks, const float* slots,
                                       float* S_chunks, float* dSn_chunks, float* scr, const float* F_chunks,
                                       bool reverse, cudaStream_t stream)
{
    cudaError_t e;
    if (!reverse) {
        if (max_chunks > 0) {
            LaunchScope ls("bwd_wk_images", stream);
            bwd_wk_images_kernel<<<dim3(max_chunks, H), 256, 0, stream>>>(hdr, H, slots, scr);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
        e = cudaFuncSetAttribute(bwd_chain_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kChSmem);
        if (e != cudaSuccess) return e;
        LaunchScope ls("bwd_fwd_states_tc", stream);
        bwd_chain_tc_kernel<false><<<dim3(N, H, 4), kChThreads, kChSmem, stream>>>(S0, nullptr, hdr, off, N, H, slots,
                                                                                   scr, S_chunks, nullptr);
        return cudaGetLastError();
    }
    e = cudaFuncSetAttribute(bwd_chain_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kChSmem);
    if (e != cudaSuccess) return e;
    LaunchScope ls("bwd_dstate_tc", stream);
    bwd_chain_tc_kernel<true><<<dim3(N, H, 4), kChThreads, kChSmem, stream>>>(dS_final, dS0, hdr, off, N, H, slots, scr,
                                                                              dSn_chunks, F_chunks);
    return cudaGetLastError();
}

inline cudaError_t launch_bwd_state_side_tc(const void* dout, const WsHeader* hdr, const int* off, const int32_t* cu,
                                            int Tseq, int N, int H, int max_chunks, const float* S_chunks,
                                            const float* dSn_chunks, float* scr, cudaStream_t stream)
{
    cudaError_t e = cudaFuncSetAttribute(bwd_state_side_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kBStateSmem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long units = (long long)max_chunks * H;
    const unsigned grid = (unsigned)(units < sms ? units : sms);
    if (grid == 0) return cudaSuccess;
    LaunchScope ls("bwd_state_side_tc", stream);
    bwd_state_side_tc_kernel<<<grid, 256, kBStateSmem, stream>>>(
        (const __nv_bfloat16*)dout, hdr, off, cu, Tseq, N, H, S_chunks, dSn_chunks, scr);
    return cudaGetLastError();
}

}  // namespace kda
