// tc_common.cuh -- thin wrappers over the sm_100a tensor-core (tcgen05 / TMEM), mbarrier and
// bulk-copy instructions used by the tensor-core prefill, plus the shared-memory operand layout.
//
// Operand layout ("SW128 tile"): a bf16 matrix with R rows and 64*A columns is stored as A "atom
// columns", each R rows x 128 bytes, atom column a at byte a*R*128.  Inside an atom column row r
// starts at r*128 and its eight 16-byte chunks are permuted by chunk' = chunk ^ (r % 8) (the
// 128-byte swizzle).  Tiles start on 1024-byte boundaries.  The same bytes serve as
//   * a K-major operand (rows = M or N, K contiguous): descriptor start = atom column + 2*k0 bytes,
//     stride between 8-row groups (SBO) = 1024 B;
//   * an MN-major operand (rows = K, M/N contiguous): start = tile + 128*k0 bytes, SBO = 1024 B
//     between 8-row K groups, LBO = R*128 B between 64-column atom columns.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"

namespace kda {
namespace tc {

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// byte offset of element (r, c) of a SW128 tile with R rows
__host__ __device__ __forceinline__ uint32_t sw128_off(int r, int c, int R)
{
    return (uint32_t)((c >> 6) * R * 128 + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + ((c & 7) << 1));
}
// byte offset of the 16-byte chunk holding columns 8*ch .. 8*ch+7 of row r
__host__ __device__ __forceinline__ uint32_t sw128_chunk_off(int r, int ch, int R)
{
    return (uint32_t)((ch >> 3) * R * 128 + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
}

// ---- shared-memory matrix descriptors (tcgen05 "version 1", SWIZZLE_128B) ---------------------
__device__ __forceinline__ uint64_t desc_sw128(uint32_t start_addr, uint32_t lbo_bytes, uint32_t sbo_bytes)
{
    uint64_t d = 0;
    d |= (uint64_t)((start_addr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;  // descriptor version for sm_100
    d |= (uint64_t)2u << 61;  // SWIZZLE_128B
    return d;
}
// K-major operand: tile of R rows, K offset k0 (multiple of 16 elements)
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile_addr, int R, int k0)
{
    return desc_sw128(tile_addr + (uint32_t)((k0 >> 6) * R * 128 + ((k0 & 63) << 1)), 16u, 1024u);
}
// MN-major operand: tile of R = K rows, K offset k0 (multiple of 16 rows)
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t tile_addr, int R, int k0)
{
    return desc_sw128(tile_addr + (uint32_t)(k0 * 128), (uint32_t)(R * 128), 1024u);
}

// ---- instruction descriptor, kind::f16 with bf16 inputs and fp32 accumulation -----------------
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ---- tcgen05 ---------------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem_addr, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem_addr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem desc] * B[smem desc]; issued by one thread
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// arrive (once) on an mbarrier when all previously issued MMAs of this thread have completed
__device__ __forceinline__ void mma_commit(uint32_t mbar_addr)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar_addr)
                 : "memory");
}
// 32 lanes x 32 bit, 16 consecutive columns per thread (thread i of the warp <- lane base+i)
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v)
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
// M = 64 accumulators keep row r in lane (r % 16) + 32 (r / 16): the 16x32bx2 shape reads lanes
// base .. base+15 twice, threads 0-15 at columns [taddr, +16) and threads 16-31 at columns
// [taddr + OFF, +16), so every thread of the warp receives a row.
template <int OFF>
__device__ __forceinline__ void tmem_ld16_pair(uint32_t taddr, float* v)
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16], %17;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr), "n"(OFF)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// 32 lanes x 32 bit, 16 consecutive columns per thread (thread i of the warp -> lane base+i)
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float* v)
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
        "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
        "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
        "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
        "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15]))
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// generic-proxy shared-memory writes -> visible to the async proxy (tensor core, bulk copy)
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ---- mbarrier --------------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t addr, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(addr), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void mbar_arrive(uint32_t addr)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(addr) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t addr, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(addr), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t addr, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(addr), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait: gives up after 4e8 SM cycles (~0.2 s, far beyond any legitimate wait here),
// records KDA_ERR_TIMEOUT in the device error word and returns false.
__device__ __forceinline__ bool mbar_wait(uint32_t addr, uint32_t parity)
{
    if (mbar_try_wait(addr, parity)) return true;
    const long long start = clock64();
    while (clock64() - start < 400000000LL)
        if (mbar_try_wait(addr, parity)) return true;
    set_error(KDA_ERR_TIMEOUT);
    return false;
}

// As mbar_wait, but also gives up at once when *abort is set, and sets it when it gives up itself:
// after one wait in a CTA times out, every later wait in that CTA returns false immediately.
__device__ __forceinline__ bool mbar_wait_ab(uint32_t addr, uint32_t parity, volatile int* abort)
{
    if (mbar_try_wait(addr, parity)) return true;
    const long long start = clock64();
    while (clock64() - start < 400000000LL) {
        if (mbar_try_wait(addr, parity)) return true;
        if (*abort) return false;
    }
    set_error(KDA_ERR_TIMEOUT);
    *abort = 1;
    return false;
}

// ---- thread-block cluster: distributed shared memory between the CTAs of one cluster ----------
__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// the shared::cluster address of `local_addr` (a shared::cta address) in the CTA of rank `rank`
__device__ __forceinline__ uint32_t cluster_map(uint32_t local_addr, uint32_t rank)
{
    uint32_t a;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(local_addr), "r"(rank));
    return a;
}
// Asynchronous 4-byte store into the shared memory of another CTA of the cluster (both addresses are
// shared::cluster addresses in that CTA).  Its completion counts 4 bytes of transactions on that CTA's
// mbarrier, which the receiver waits on like on a bulk copy; the sender neither waits nor fences, so
// the store does not wait for this thread's outstanding global loads and stores.
__device__ __forceinline__ void st_async_cluster_f32(uint32_t cluster_addr, float v, uint32_t cluster_bar)
{
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(cluster_addr),
                 "r"(__float_as_uint(v)), "r"(cluster_bar)
                 : "memory");
}
// every thread of every CTA of the cluster (release / acquire at cluster scope)
__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// ---- bulk copy global -> shared (completion counted on an mbarrier) ---------------------------
// bulk prefetch of a global range into L2 (no shared memory, no completion to wait for); address and
// size multiples of 16 bytes
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst_smem, const void* src, uint32_t bytes, uint32_t mbar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     dst_smem),
                 "l"(src), "r"(bytes), "r"(mbar)
                 : "memory");
}

// ---- TMA tiled load (3-D tensor map), completion counted on an mbarrier -----------------------
// The innermost coordinate c0 times the element size is always a multiple of 16 bytes here.
__device__ __forceinline__ void tma_load_3d(uint32_t dst_smem, const void* tmap, int c0, int c1, int c2, uint32_t mbar)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::
            "r"(dst_smem),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(mbar)
        : "memory");
}

// brings a tensor map (kernel parameter space) into the descriptor cache ahead of its first use
__device__ __forceinline__ void prefetch_tensormap(const void* tmap)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// ---- small helpers ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t pack_bf16(float a, float b)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float exp_fast(float x) { return exp2f(x * 1.4426950408889634f); }
// 2^x with the hardware's approximate base-2 exponential (relative error ~2^-22 over the normal
// range; results below 2^-126 flush to zero).
__device__ __forceinline__ float ex2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
constexpr float kLog2e = 1.4426950408889634f;
// sigmoid(x) = 0.5 + 0.5 tanh(x / 2), the tanh from the hardware's approximation (tanh.approx.f32, one
// instruction; relative error about 2^-11, below a bf16 rounding of the result)
__device__ __forceinline__ float sigmoid_tanh(float x)
{
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
    return fmaf(0.5f, t, 0.5f);
}
// log2(x) with the hardware's approximate base-2 logarithm (x > 0, normal range)
__device__ __forceinline__ float lg2_approx(float x)
{
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// log2 sigmoid(a) = min(a, 0) log2(e) - log2(1 + 2^{-|a| log2(e)}): the gate logit's log-space
// forget gate, in the log2 units the tensor-core path accumulates
__device__ __forceinline__ float log2_sigmoid(float a)
{
    return fminf(a, 0.f) * kLog2e - lg2_approx(1.f + ex2_approx(-fabsf(a) * kLog2e));
}

}  // namespace tc
}  // namespace kda
