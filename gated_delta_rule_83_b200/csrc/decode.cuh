// decode.cuh -- fused single-token KDA decode step (state read once, written once).
//
// Per (sequence, head) the step is, in the order of the per-token loop in the attention review's
// GDN/KDA pseudo-code (lanjinlin.com.cn, entry on Qwen3-Next GDN, the block that loads the
// per-sequence state): decay S' = Diag(alpha) S; r = S'^T k; u = beta (v - r); S = S' + k u^T;
// o = S^T q = S'^T q + u (q . k).  Both column reductions (r and S'^T q) come out of the single
// read of S, and the rank-1 update is applied to the values still held in registers, so the
// 64 KiB fp32 state of a 128x128 head crosses HBM exactly twice (one read, one write).
//
// Work decomposition: one CTA of 256 threads owns a 64-column slice of one head's state
// (columns of S evolve independently).  A warp reads two 256-byte row segments per 128-bit load
// instruction (lanes 0-15 row a, lanes 16-31 row a+1; each lane 4 consecutive columns), so every
// state access is a fully coalesced, 16-byte-vectorised streaming load/store (ld.global.cs /
// st.global.cs: the state is touched once per step and is far larger than L2).
#pragma once

#include "common.cuh"
#include "profile.cuh"

namespace kda {

constexpr int kDecodeThreads = 256;
constexpr int kDecodeSlice = 64;  // columns of S per CTA

template <typename TIn, int DK, bool GROUPED, bool PRO>
__global__ void __launch_bounds__(kDecodeThreads, 3)
decode_step_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k, const TIn* __restrict__ v,
                   const void* __restrict__ log_alpha, const float* __restrict__ beta, float* __restrict__ S,
                   TIn* __restrict__ out, int dv, int H, int G, unsigned pro)
{
    constexpr int RPT = DK / 16;  // state rows held per thread
    const int nslices = dv / kDecodeSlice;
    const int p = blockIdx.x / nslices;            // (sequence, head) pair, = n*H + h
    const int pq = GROUPED ? (p / H) * (H / G) + (p % H) / G : p;  // its q/k head: n*Hk + h/G (G = H/Hk)
    const int j0 = (blockIdx.x % nslices) * kDecodeSlice;
    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
    const int cg = l & 15;                         // columns j0 + 4cg .. j0 + 4cg + 3
    const int rb = 2 * w + (l >> 4);               // rows rb + 16 i

    __shared__ float s_a[DK], s_k[DK], s_q[DK];
    __shared__ __align__(16) float s_red[8][16][8];
    __shared__ float s_qk[8];  // per-warp partial q . k

    float* Sp = S + (size_t)p * DK * dv + j0;
    float4 st[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i)
        st[i] = __ldcs(reinterpret_cast<const float4*>(Sp + (size_t)(rb + 16 * i) * dv) + cg);

    // the step's small inputs, loaded alongside the state so that no load sits on the critical path
    const float b = (PRO && (pro & KDA_PROLOGUE_BETA_LOGITS)) ? sigmoid_f(beta[p]) : beta[p];
    const TIn* vp = v + (size_t)p * dv + j0 + 4 * cg;
    const float v0 = to_f32(vp[0]), v1 = to_f32(vp[1]), v2 = to_f32(vp[2]), v3 = to_f32(vp[3]);
    for (int c = tid; c < DK; c += kDecodeThreads) {
        const size_t ia = (size_t)p * DK + c;  // gates fp32, or bf16 with the bf16-gate bit
        const float la = (PRO && (pro & KDA_PROLOGUE_GATE_BF16))
                             ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(log_alpha)[ia])
                             : reinterpret_cast<const float*>(log_alpha)[ia];
        s_a[c] = (PRO && (pro & KDA_PROLOGUE_GATE_LOGITS)) ? sigmoid_f(la) : expf(la);  // alpha = sigmoid(logit)
        s_k[c] = to_f32(k[(size_t)pq * DK + c]);
        s_q[c] = to_f32(q[(size_t)pq * DK + c]);
    }
    if (PRO && (pro & KDA_PROLOGUE_L2NORM_QK)) {  // q and k normalised over d_k (threads 0..DK-1 hold them)
        __shared__ float s_nrm[DK / 32][2];
        float kk = 0.f, qq = 0.f;
        if (tid < DK) {
            kk = s_k[tid] * s_k[tid];
            qq = s_q[tid] * s_q[tid];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            kk += __shfl_xor_sync(0xffffffffu, kk, o);
            qq += __shfl_xor_sync(0xffffffffu, qq, o);
        }
        if (tid < DK && l == 0) {
            s_nrm[w][0] = kk;
            s_nrm[w][1] = qq;
        }
        __syncthreads();
        if (tid < DK) {
            float sk = 0.f, sq = 0.f;
#pragma unroll
            for (int i = 0; i < DK / 32; ++i) {
                sk += s_nrm[i][0];
                sq += s_nrm[i][1];
            }
            s_k[tid] = to_f32(from_f32<TIn>(s_k[tid] * rsqrtf(sk + kQkNormEps)));
            s_q[tid] = to_f32(from_f32<TIn>(s_q[tid] * rsqrtf(sq + kQkNormEps)));
        }
    }
    __syncthreads();

    float r0 = 0.f, r1 = 0.f, r2 = 0.f, r3 = 0.f, q0 = 0.f, q1 = 0.f, q2 = 0.f, q3 = 0.f, qk = 0.f;
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int c = rb + 16 * i;
        const float a = s_a[c], kc = s_k[c], qc = s_q[c];
        qk = fmaf(qc, kc, qk);  // rows rb + 16 i: the two half-warps together cover this warp's rows
        st[i].x *= a; st[i].y *= a; st[i].z *= a; st[i].w *= a;
        r0 = fmaf(st[i].x, kc, r0); r1 = fmaf(st[i].y, kc, r1); r2 = fmaf(st[i].z, kc, r2); r3 = fmaf(st[i].w, kc, r3);
        q0 = fmaf(st[i].x, qc, q0); q1 = fmaf(st[i].y, qc, q1); q2 = fmaf(st[i].z, qc, q2); q3 = fmaf(st[i].w, qc, q3);
    }
    r0 += __shfl_xor_sync(0xffffffffu, r0, 16); r1 += __shfl_xor_sync(0xffffffffu, r1, 16);
    r2 += __shfl_xor_sync(0xffffffffu, r2, 16); r3 += __shfl_xor_sync(0xffffffffu, r3, 16);
    q0 += __shfl_xor_sync(0xffffffffu, q0, 16); q1 += __shfl_xor_sync(0xffffffffu, q1, 16);
    q2 += __shfl_xor_sync(0xffffffffu, q2, 16); q3 += __shfl_xor_sync(0xffffffffu, q3, 16);
    if (l < 16) {
        float4* dst = reinterpret_cast<float4*>(&s_red[w][cg][0]);
        dst[0] = make_float4(r0, r1, r2, r3);
        dst[1] = make_float4(q0, q1, q2, q3);
    }
    qk += __shfl_xor_sync(0xffffffffu, qk, 16);  // lanes l and l ^ 16 hold the warp's two rows of each pair
    if (l == 0) s_qk[w] = qk;
    __syncthreads();

    float4 rr = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int ww = 0; ww < 8; ++ww) {
        const float4 x = reinterpret_cast<const float4*>(&s_red[ww][cg][0])[0];
        rr.x += x.x; rr.y += x.y; rr.z += x.z; rr.w += x.w;
    }
    const float u0 = b * (v0 - rr.x), u1 = b * (v1 - rr.y);
    const float u2 = b * (v2 - rr.z), u3 = b * (v3 - rr.w);

#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int c = rb + 16 * i;
        const float kc = s_k[c];
        float4 x = st[i];
        x.x = fmaf(kc, u0, x.x); x.y = fmaf(kc, u1, x.y); x.z = fmaf(kc, u2, x.z); x.w = fmaf(kc, u3, x.w);
        __stcs(reinterpret_cast<float4*>(Sp + (size_t)c * dv) + cg, x);
    }

    if (w == 0 && l < 16) {
        float qk_all = 0.f;
#pragma unroll
        for (int ww = 0; ww < 8; ++ww) qk_all += s_qk[ww];
        float4 ss = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int ww = 0; ww < 8; ++ww) {
            const float4 x = reinterpret_cast<const float4*>(&s_red[ww][cg][4])[0];
            ss.x += x.x; ss.y += x.y; ss.z += x.z; ss.w += x.w;
        }
        TIn* op = out + (size_t)p * dv + j0 + 4 * cg;
        op[0] = from_f32<TIn>(fmaf(u0, qk_all, ss.x));
        op[1] = from_f32<TIn>(fmaf(u1, qk_all, ss.y));
        op[2] = from_f32<TIn>(fmaf(u2, qk_all, ss.z));
        op[3] = from_f32<TIn>(fmaf(u3, qk_all, ss.w));
    }
}

template <typename TIn>
cudaError_t launch_decode(const void* q, const void* k, const void* v, const void* la, const float* beta, float* S,
                          void* out, int N, int H, int Hk, unsigned pro, int dk, int dv, cudaStream_t stream)
{
    const long long pairs = (long long)N * H;
    const long long blocks = pairs * (dv / kDecodeSlice);
    if (blocks == 0) return cudaSuccess;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    LaunchScope ls("decode_step", stream);
    const int G = H / Hk;
    const dim3 grid((unsigned)blocks);
    const TIn *qq = (const TIn*)q, *kk = (const TIn*)k, *vv = (const TIn*)v;
    TIn* oo = (TIn*)out;
    // one instantiation per (d_k, grouped, prologue) so that the plain step carries none of the options
#define KDA_DECODE_LAUNCH(DKV, GR, PR) \
    decode_step_kernel<TIn, DKV, GR, PR><<<grid, kDecodeThreads, 0, stream>>>(qq, kk, vv, la, beta, S, oo, dv, H, G, pro)
    const bool gr = G != 1, pr = pro != 0;
    if (dk == 128) {
        if (!gr && !pr) KDA_DECODE_LAUNCH(128, false, false);
        else if (gr && !pr) KDA_DECODE_LAUNCH(128, true, false);
        else if (!gr) KDA_DECODE_LAUNCH(128, false, true);
        else KDA_DECODE_LAUNCH(128, true, true);
    } else {
        if (!gr && !pr) KDA_DECODE_LAUNCH(64, false, false);
        else if (gr && !pr) KDA_DECODE_LAUNCH(64, true, false);
        else if (!gr) KDA_DECODE_LAUNCH(64, false, true);
        else KDA_DECODE_LAUNCH(64, true, true);
    }
#undef KDA_DECODE_LAUNCH
    return cudaGetLastError();
}

}  // namespace kda
