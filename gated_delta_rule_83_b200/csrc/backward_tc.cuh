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

inline bool bwd_state_side_tc_ok(bool bf16, int dk, int dv) { return kTcPathReady && bf16 && dk == 128 && dv == 128; }

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
