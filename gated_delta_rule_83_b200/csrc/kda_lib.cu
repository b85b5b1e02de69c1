// kda_lib.cu -- the C ABI of libkda.so (declared in include/kda.h): argument validation,
// workspace carving and kernel dispatch.  Every step of the operator runs in the kernels
// included below; this file only checks arguments and launches.
#include <cstdio>
#include <cstring>
#include <memory>
#include <mutex>
#include <vector>

#include "kda.h"
#include "backward_simt.cuh"
#include "backward_tc.cuh"
#include "common.cuh"
#include "chunks.cuh"
#include "decode.cuh"
#include "gated_norm.cuh"
#include "prefill_simt.cuh"
#include "prefill_tc.cuh"
#include "profile.cuh"

using namespace kda;

namespace kda {
// Waits on an mbarrier that nothing ever completes, through the same bounded wait the
// tensor-core kernels use: the wait gives up, records KDA_ERR_TIMEOUT and the kernel returns.
__global__ void selftest_timeout_kernel()
{
    __shared__ __align__(8) uint64_t bar;
    const uint32_t a = tc::smem_u32(&bar);
    if (threadIdx.x == 0) {
        tc::mbar_init(a, 1);
        tc::mbar_fence_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)tc::mbar_wait(a, 0);
    __syncthreads();
}
}  // namespace kda

namespace {

constexpr size_t kAlign = 256;

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

bool dims_supported(int dk, int dv) { return (dk == 64 || dk == 128) && (dv == 64 || dv == 128); }

// The tensor-core path covers bf16 with dk = dv = 128; everything else runs the fp32 CUDA-core path.
bool use_tc_path(kda_dtype dt, int dk, int dv) { return kTcPathReady && dt == KDA_BF16 && dk == 128 && dv == 128; }

struct Plan {
    int N;            // number of sequences
    int Tseq;         // tokens per sequence (regular batches); 0 for varlen
    long long Ttot;   // total tokens
    int max_chunks;   // upper bound on the number of chunks
    bool tc;
    size_t off_bytes, slot_bytes, total_bytes;
};

kda_status make_plan(int B, int T, int H, int dk, int dv, bool varlen, int num_seqs, kda_dtype dt, Plan& p)
{
    if (dt != KDA_BF16 && dt != KDA_F32) return KDA_ERR_INVALID_ARG;
    if (H <= 0 || T < 0 || B <= 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
    if (!dims_supported(dk, dv)) return KDA_ERR_UNSUPPORTED;
    if (H > 65535) return KDA_ERR_UNSUPPORTED;
    if (varlen) {
        if (B != 1 || num_seqs <= 0) return KDA_ERR_INVALID_ARG;
        p.N = num_seqs;
        p.Tseq = 0;
        p.Ttot = T;
        p.max_chunks = T / kChunk + num_seqs;
    } else {
        p.N = B;
        p.Tseq = T;
        p.Ttot = (long long)B * T;
        const long long mc = (long long)B * ((T + kChunk - 1) / kChunk);
        if (mc > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
        p.max_chunks = (int)mc;
    }
    if (p.Ttot > 0x7fffffffLL || p.N > 65535 * 64) return KDA_ERR_UNSUPPORTED;
    p.tc = use_tc_path(dt, dk, dv);
    p.off_bytes = round_up(sizeof(int) * (2 * (size_t)p.N + 1), kAlign);  // off[N+1] + order[N]
    p.slot_bytes = p.tc ? tc_slot_bytes() : round_up(sizeof(float) * simt_slot_floats(dk, dv), kAlign);
    p.total_bytes = sizeof(WsHeader) + p.off_bytes + (size_t)p.max_chunks * (size_t)H * p.slot_bytes;
    return KDA_OK;
}

// Backward workspace: the forward's header and chunk table, then per (chunk, head) the CUDA-core
// forward slot, the chunk's start state, its end cotangent and the state-side scratch.
struct BwdPlan {
    Plan f;
    size_t slot_bytes, state_bytes, scr_bytes, acc_bytes, qk_bytes, la_bytes, beta_bytes, total_bytes;
};

// Hk < H (grouped q/k heads) or the q/k norm adds two fp32 per-value-head buffers for dq and dk;
// the prologue bits add buffers for the transformed inputs (normalised q, k; activated gates, beta)
kda_status make_bwd_plan(int B, int T, int H, int Hk, unsigned pro, int dk, int dv, bool varlen, int num_seqs,
                         kda_dtype dt, BwdPlan& p)
{
    const kda_status st = make_plan(B, T, H, dk, dv, varlen, num_seqs, dt, p.f);
    if (st != KDA_OK) return st;
    const size_t units = (size_t)p.f.max_chunks * (size_t)H;
    // dense per-unit strides: the kernels index these regions as float arrays
    p.slot_bytes = sizeof(float) * simt_slot_floats(dk, dv);
    p.state_bytes = sizeof(float) * (size_t)dk * dv;
    p.scr_bytes = sizeof(float) * bwd_scr_floats(dk, dv);
    const size_t Tt = (size_t)p.f.Ttot, esz = dt == KDA_BF16 ? 2 : 4;
    const bool l2 = (pro & KDA_PROLOGUE_L2NORM_QK) != 0;
    p.acc_bytes = (Hk != H || l2) ? round_up(sizeof(float) * Tt * H * dk, kAlign) : 0;
    p.qk_bytes = l2 ? round_up(esz * Tt * Hk * dk, kAlign) : 0;
    p.la_bytes = (pro & KDA_PROLOGUE_GATE_LOGITS) ? round_up(sizeof(float) * Tt * H * dk, kAlign) : 0;
    p.beta_bytes = (pro & KDA_PROLOGUE_BETA_LOGITS) ? round_up(sizeof(float) * Tt * H, kAlign) : 0;
    p.total_bytes = round_up(sizeof(WsHeader) + p.f.off_bytes +
                             units * (p.slot_bytes + 3 * p.state_bytes + p.scr_bytes), kAlign) +
                    2 * p.acc_bytes + 2 * p.qk_bytes + p.la_bytes + p.beta_bytes;
    return KDA_OK;
}

// Options of the extended entry points: Hk = q/k heads (0 -> H), prologue bits; reserved fields
// must be zero.
kda_status parse_options(const kda_options* opt, int H, int& Hk, unsigned& pro)
{
    Hk = H;
    pro = 0;
    if (!opt) return KDA_OK;
    for (int r : opt->reserved)
        if (r != 0) return KDA_ERR_INVALID_ARG;
    if (opt->num_qk_heads != 0) {
        if (opt->num_qk_heads < 0 || H % opt->num_qk_heads != 0) return KDA_ERR_INVALID_ARG;
        Hk = opt->num_qk_heads;
    }
    const unsigned known =
        KDA_PROLOGUE_L2NORM_QK | KDA_PROLOGUE_GATE_LOGITS | KDA_PROLOGUE_BETA_LOGITS | KDA_PROLOGUE_GATE_BF16;
    if (opt->prologue & ~known) return KDA_ERR_INVALID_ARG;
    pro = opt->prologue;
    return KDA_OK;
}

}  // namespace

extern "C" {

const char* kda_status_string(kda_status s)
{
    switch (s) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG";
        case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
        case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT";
        case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE";
        case KDA_ERR_BAD_SEQLENS: return "KDA_ERR_BAD_SEQLENS";
    }
    return "KDA_ERR_UNKNOWN";
}

const char* kda_version(void) { return "kda-b200 0.1 sm_100a"; }

kda_status kda_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv, int varlen, int num_seqs,
                                        kda_dtype dt, size_t* bytes)
{
    if (!bytes) return KDA_ERR_INVALID_ARG;
    Plan p;
    const kda_status st = make_plan(B, T, H, dk, dv, varlen != 0, num_seqs, dt, p);
    if (st != KDA_OK) return st;
    *bytes = p.total_bytes;
    return KDA_OK;
}

kda_status kda_chunk_fwd_gated(const void* q, const void* k, const void* v, const void* log_alpha, const float* beta,
                               const float* S0, const int32_t* cu_seqlens, int num_seqs, void* out, float* S_final,
                               int B, int T, int H, int dk, int dv, kda_dtype dt, const kda_options* opt,
                               const kda_output_gate* gate, void* workspace, size_t workspace_bytes,
                               kda_stream_t stream_)
{
    cudaStream_t stream = (cudaStream_t)stream_;
    int Hk = H;
    unsigned pro = 0;
    const kda_status so = parse_options(opt, H, Hk, pro);
    if (so != KDA_OK) return so;
    Plan p;
    const kda_status st = make_plan(B, T, H, dk, dv, cu_seqlens != nullptr, num_seqs, dt, p);
    if (st != KDA_OK) return st;
    int group = 0;
    if (gate) {
        for (int r : gate->reserved)
            if (r != 0) return KDA_ERR_INVALID_ARG;
        group = gate->group == 0 ? dv : gate->group;
        if (group < 8 || group > dv || (group & (group - 1)) != 0) return KDA_ERR_INVALID_ARG;
        if (!(gate->eps > 0.f) || (gate->act != KDA_GATE_IDENTITY && gate->act != KDA_GATE_SIGMOID))
            return KDA_ERR_INVALID_ARG;
        if (p.Ttot > 0 && (!gate->z || !aligned16(gate->z))) return KDA_ERR_INVALID_ARG;
        if (gate->weight && !aligned16(gate->weight)) return KDA_ERR_INVALID_ARG;
    }
    if (p.Ttot > 0 && (!q || !k || !v || !log_alpha || !beta || !out)) return KDA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, log_alpha, beta, S0, out, S_final};
    for (const void* x : ptrs)
        if (x && !aligned16(x)) return KDA_ERR_INVALID_ARG;
    if (cu_seqlens && ((uintptr_t)cu_seqlens & 3u)) return KDA_ERR_INVALID_ARG;
    if (!workspace || ((uintptr_t)workspace % kAlign) || workspace_bytes < p.total_bytes) return KDA_ERR_WORKSPACE;

    char* ws = (char*)workspace;
    WsHeader* hdr = (WsHeader*)ws;
    int* off = (int*)(ws + sizeof(WsHeader));
    char* slots = ws + sizeof(WsHeader) + p.off_bytes;

    {
        LaunchScope ls("chunk_table", stream);
        chunk_table_kernel<<<1, kTableThreads, 0, stream>>>(cu_seqlens, p.N, p.Tseq, p.Ttot, hdr, off,
                                                             off + p.N + 1);
        if (cudaGetLastError() != cudaSuccess) return KDA_ERR_CUDA;
    }

    cudaError_t e;
    if (p.tc) {
        // the tensor-core path applies the gate in phase B's epilogue, from the fp32 output
        OutGate og{};
        if (gate)
            og = OutGate{(const __nv_bfloat16*)gate->z, gate->weight, 1.f / (float)group, gate->eps, group,
                         gate->act == KDA_GATE_SIGMOID ? 1 : 0};
        e = launch_tc_prefill(q, k, v, log_alpha, beta, S0, S_final, out, hdr, off, cu_seqlens, p.Tseq, p.N, H, Hk, pro,
                              p.max_chunks, p.Ttot, slots, gate ? &og : nullptr, stream);
    } else {
        e = dt == KDA_BF16
            ? launch_simt_prefill<__nv_bfloat16>(q, k, v, log_alpha, beta, S0, S_final, out, hdr, off, cu_seqlens,
                                                 p.Tseq, p.N, H, Hk, pro, dk, dv, p.max_chunks, (float*)slots, stream)
            : launch_simt_prefill<float>(q, k, v, log_alpha, beta, S0, S_final, out, hdr, off, cu_seqlens, p.Tseq,
                                         p.N, H, Hk, pro, dk, dv, p.max_chunks, (float*)slots, stream);
        // the CUDA-core path writes o, then the gate runs over it in place
        if (e == cudaSuccess && gate && p.Ttot > 0) {
            const long long rows = p.Ttot * H;
            const int sg = gate->act == KDA_GATE_SIGMOID ? 1 : 0;
            e = dt == KDA_BF16
                ? launch_gated_rmsnorm<__nv_bfloat16>(out, gate->z, gate->weight, out, rows, dv, group, gate->eps, sg,
                                                      stream)
                : launch_gated_rmsnorm<float>(out, gate->z, gate->weight, out, rows, dv, group, gate->eps, sg, stream);
        }
    }
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_chunk_fwd_ex(const void* q, const void* k, const void* v, const void* log_alpha, const float* beta,
                            const float* S0, const int32_t* cu_seqlens, int num_seqs, void* out, float* S_final,
                            int B, int T, int H, int dk, int dv, kda_dtype dt, const kda_options* opt,
                            void* workspace, size_t workspace_bytes, kda_stream_t stream)
{
    return kda_chunk_fwd_gated(q, k, v, log_alpha, beta, S0, cu_seqlens, num_seqs, out, S_final, B, T, H, dk, dv, dt,
                               opt, nullptr, workspace, workspace_bytes, stream);
}

kda_status kda_chunk_fwd(const void* q, const void* k, const void* v, const float* log_alpha, const float* beta,
                         const float* S0, const int32_t* cu_seqlens, int num_seqs, void* out, float* S_final,
                         int B, int T, int H, int dk, int dv, kda_dtype dt, void* workspace,
                         size_t workspace_bytes, kda_stream_t stream)
{
    return kda_chunk_fwd_ex(q, k, v, log_alpha, beta, S0, cu_seqlens, num_seqs, out, S_final, B, T, H, dk, dv, dt,
                            nullptr, workspace, workspace_bytes, stream);
}

kda_status kda_decode_step_ex(const void* q, const void* k, const void* v, const void* log_alpha,
                              const float* beta, float* S_inout, void* out, int N, int H, int dk, int dv,
                              kda_dtype dt, const kda_options* opt, kda_stream_t stream_)
{
    cudaStream_t stream = (cudaStream_t)stream_;
    if (dt != KDA_BF16 && dt != KDA_F32) return KDA_ERR_INVALID_ARG;
    if (N < 0 || H <= 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
    int Hk = H;
    unsigned pro = 0;
    const kda_status so = parse_options(opt, H, Hk, pro);
    if (so != KDA_OK) return so;
    if (!dims_supported(dk, dv)) return KDA_ERR_UNSUPPORTED;
    if (N == 0) return KDA_OK;
    if (!q || !k || !v || !log_alpha || !beta || !S_inout || !out) return KDA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, log_alpha, beta, S_inout, out};
    for (const void* x : ptrs)
        if (!aligned16(x)) return KDA_ERR_INVALID_ARG;
    const cudaError_t e = (dt == KDA_BF16)
        ? launch_decode<__nv_bfloat16>(q, k, v, log_alpha, beta, S_inout, out, N, H, Hk, pro, dk, dv, stream)
        : launch_decode<float>(q, k, v, log_alpha, beta, S_inout, out, N, H, Hk, pro, dk, dv, stream);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_decode_step(const void* q, const void* k, const void* v, const float* log_alpha, const float* beta,
                           float* S_inout, void* out, int N, int H, int dk, int dv, kda_dtype dt,
                           kda_stream_t stream)
{
    return kda_decode_step_ex(q, k, v, log_alpha, beta, S_inout, out, N, H, dk, dv, dt, nullptr, stream);
}

kda_status kda_chunk_bwd_workspace_size(int B, int T, int H, int dk, int dv, int varlen, int num_seqs,
                                        kda_dtype dt, const kda_options* opt, size_t* bytes)
{
    if (!bytes) return KDA_ERR_INVALID_ARG;
    int Hk = H;
    unsigned pro = 0;
    const kda_status so = parse_options(opt, H, Hk, pro);
    if (so != KDA_OK) return so;
    BwdPlan p;
    const kda_status st = make_bwd_plan(B, T, H, Hk, pro, dk, dv, varlen != 0, num_seqs, dt, p);
    if (st != KDA_OK) return st;
    *bytes = p.total_bytes;
    return KDA_OK;
}

kda_status kda_chunk_bwd(const void* q, const void* k, const void* v, const void* log_alpha, const float* beta,
                         const float* S0, const int32_t* cu_seqlens, int num_seqs, const void* dout,
                         const float* dS_final, void* dq, void* dk_out, void* dv_out, float* dlog_alpha, float* dbeta,
                         float* dS0, int B, int T, int H, int dk, int dv, kda_dtype dt, const kda_options* opt,
                         void* workspace, size_t workspace_bytes, kda_stream_t stream_)
{
    cudaStream_t stream = (cudaStream_t)stream_;
    int Hk = H;
    unsigned pro = 0;
    const kda_status so = parse_options(opt, H, Hk, pro);
    if (so != KDA_OK) return so;
    BwdPlan p;
    const kda_status st = make_bwd_plan(B, T, H, Hk, pro, dk, dv, cu_seqlens != nullptr, num_seqs, dt, p);
    if (st != KDA_OK) return st;
    if (p.f.Ttot > 0 && (!q || !k || !v || !log_alpha || !beta || !dout || !dq || !dk_out || !dv_out ||
                         !dlog_alpha || !dbeta))
        return KDA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, log_alpha, beta, S0, dout, dS_final, dq, dk_out, dv_out, dlog_alpha, dbeta, dS0};
    for (const void* x : ptrs)
        if (x && !aligned16(x)) return KDA_ERR_INVALID_ARG;
    if (cu_seqlens && ((uintptr_t)cu_seqlens & 3u)) return KDA_ERR_INVALID_ARG;
    if (!workspace || ((uintptr_t)workspace % kAlign) || workspace_bytes < p.total_bytes) return KDA_ERR_WORKSPACE;

    char* ws = (char*)workspace;
    WsHeader* hdr = (WsHeader*)ws;
    int* off = (int*)(ws + sizeof(WsHeader));
    const size_t units = (size_t)p.f.max_chunks * (size_t)H;
    char* slots = ws + sizeof(WsHeader) + p.f.off_bytes;
    char* states = slots + units * p.slot_bytes;
    char* cot = states + units * p.state_bytes;
    char* scr = cot + units * p.state_bytes;
    char* fdo = scr + units * p.scr_bytes;  // F = Qg^T dO per chunk
    char* acc = ws + round_up(sizeof(WsHeader) + p.f.off_bytes +
                              units * (p.slot_bytes + 3 * p.state_bytes + p.scr_bytes), kAlign);
    char* qn = acc + 2 * p.acc_bytes;  // prologue buffers (empty when their bit is off)
    char* kn = qn + p.qk_bytes;
    char* la_act = kn + p.qk_bytes;
    char* beta_act = la_act + p.la_bytes;
    {
        LaunchScope ls("chunk_table", stream);
        chunk_table_kernel<<<1, kTableThreads, 0, stream>>>(cu_seqlens, p.f.N, p.f.Tseq, p.f.Ttot, hdr, off,
                                                             off + p.f.N + 1);
        if (cudaGetLastError() != cudaSuccess) return KDA_ERR_CUDA;
    }
    // the per-unit regions are indexed by (chunk, head) with the dense strides of the kernels
    const cudaError_t e = (dt == KDA_BF16)
        ? launch_simt_backward<__nv_bfloat16>(q, k, v, log_alpha, beta, S0, dout, dS_final, dq, dk_out, dv_out,
                                              dlog_alpha, dbeta, dS0, hdr, off, cu_seqlens, p.f.Tseq, p.f.N, H, Hk,
                                              pro, dk, dv, p.f.max_chunks, p.f.Ttot, (float*)slots, (float*)states,
                                              (float*)cot, (float*)scr, (float*)fdo, (float*)acc,
                                              (float*)(acc + p.acc_bytes), qn, kn, (float*)la_act,
                                              (float*)beta_act, stream)
        : launch_simt_backward<float>(q, k, v, log_alpha, beta, S0, dout, dS_final, dq, dk_out, dv_out, dlog_alpha,
                                      dbeta, dS0, hdr, off, cu_seqlens, p.f.Tseq, p.f.N, H, Hk, pro, dk, dv,
                                      p.f.max_chunks, p.f.Ttot, (float*)slots, (float*)states, (float*)cot,
                                      (float*)scr, (float*)fdo, (float*)acc, (float*)(acc + p.acc_bytes), qn,
                                      kn, (float*)la_act, (float*)beta_act, stream);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_gated_rmsnorm(const void* o, const void* z, const float* weight, void* y, long long rows, int d,
                             int group, float eps, kda_gate_act act, kda_dtype dt, kda_stream_t stream_)
{
    if (dt != KDA_BF16 && dt != KDA_F32) return KDA_ERR_INVALID_ARG;
    if (rows < 0 || d <= 0) return KDA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return KDA_ERR_UNSUPPORTED;
    const int g = group == 0 ? d : group;
    if (g < 8 || g > d || (g & (g - 1)) != 0 || d % g != 0) return KDA_ERR_INVALID_ARG;
    if (!(eps > 0.f) || (act != KDA_GATE_IDENTITY && act != KDA_GATE_SIGMOID)) return KDA_ERR_INVALID_ARG;
    if (rows == 0) return KDA_OK;
    if (!o || !z || !y || !aligned16(o) || !aligned16(z) || !aligned16(y) || (weight && !aligned16(weight)))
        return KDA_ERR_INVALID_ARG;
    cudaStream_t stream = (cudaStream_t)stream_;
    const int sg = act == KDA_GATE_SIGMOID ? 1 : 0;
    const cudaError_t e = dt == KDA_BF16
        ? launch_gated_rmsnorm<__nv_bfloat16>(o, z, weight, y, rows, d, g, eps, sg, stream)
        : launch_gated_rmsnorm<float>(o, z, weight, y, rows, d, g, eps, sg, stream);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_profile_begin(void)
{
    Profiler& p = profiler();
    std::lock_guard<std::mutex> g(p.mu);
    p.recs.clear();
    p.used = 0;
    p.on = true;
    return KDA_OK;
}

kda_status kda_profile_end(void)
{
    Profiler& p = profiler();
    std::lock_guard<std::mutex> g(p.mu);
    p.on = false;
    return KDA_OK;
}

int kda_profile_kernels(int max_kernels, const char** names, int* launches, double* total_ms)
{
    Profiler& p = profiler();
    std::lock_guard<std::mutex> g(p.mu);
    int n = 0;
    for (const ProfRecord& r : p.recs) {
        float ms = 0.f;
        if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess)
            return -1;
        int i = 0;
        while (i < n && std::strcmp(names[i], r.name) != 0) ++i;
        if (i == n) {
            if (n == max_kernels) return -1;
            names[n] = r.name;
            launches[n] = 0;
            total_ms[n] = 0.0;
            ++n;
        }
        launches[i] += 1;
        total_ms[i] += ms;
    }
    return n;
}

kda_status kda_selftest_timeout(kda_stream_t stream_)
{
    LaunchScope ls("selftest_timeout", (cudaStream_t)stream_);
    selftest_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream_>>>();
    return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_check(kda_stream_t stream_)
{
    cudaStream_t stream = (cudaStream_t)stream_;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return KDA_ERR_CUDA;
    int word = 0;
    if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(int)) != cudaSuccess) return KDA_ERR_CUDA;
    if (word != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(int)) != cudaSuccess) return KDA_ERR_CUDA;
        return (kda_status)word;
    }
    return KDA_OK;
}

}  // extern "C"

// ------------------------------------------------------------------------------------------------
// Allocation-free variant of kda_chunk_fwd (declared in include/kda.h).
//
// For hosts that cannot allocate device memory at call time (engines that reserve all memory in
// their own pool up front, plugin hooks that forbid cudaMalloc, fixed memory budgets), the
// workspace comes from a static device array compiled into this file instead of from the caller.
// The array exists once per GPU that loads the library and lives until the process exits.  In
// host code its name is only a host-side stand-in, so its device address is looked up with
// cudaGetSymbolAddress on every call, on the device current at the call, and passed to the
// kernels like any other workspace pointer (a host-side lookup: no allocation, no stream work;
// looking it up each time also follows the module if the device's context is ever recreated).
// All calls on a device share the array; calls that overlap on the GPU race.  Every scratch byte
// a kernel reads is written earlier in the same call, so nothing needs clearing between calls.
// ------------------------------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[KDA_NOALLOC_SCRATCH_BYTES];

namespace {

kda_status noalloc_scratch_address(void** ptr)
{
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return KDA_ERR_CUDA;
    *ptr = p;
    return KDA_OK;
}

}  // namespace

extern "C" kda_status kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const float* log_alpha,
                                            const float* beta, const float* S0, const int32_t* cu_seqlens,
                                            int num_seqs, void* out, float* S_final, int B, int T, int H, int dk,
                                            int dv, kda_dtype dt, kda_stream_t stream)
{
    Plan p;
    const kda_status st = make_plan(B, T, H, dk, dv, cu_seqlens != nullptr, num_seqs, dt, p);
    if (st != KDA_OK) return st;
    if (p.total_bytes > (size_t)KDA_NOALLOC_SCRATCH_BYTES) return KDA_ERR_WORKSPACE;
    void* scratch = nullptr;
    const kda_status sa = noalloc_scratch_address(&scratch);
    if (sa != KDA_OK) return sa;
    return kda_chunk_fwd(q, k, v, log_alpha, beta, S0, cu_seqlens, num_seqs, out, S_final, B, T, H, dk, dv, dt,
                         scratch, (size_t)KDA_NOALLOC_SCRATCH_BYTES, stream);
}

// ------------------------------------------------------------------------------------------------
// Host-resident inputs: segments of the token axis stream in on one copy stream, run on the
// caller's stream and stream out on another, double-buffered, with the state carried on the device.
// ------------------------------------------------------------------------------------------------
namespace {

struct HostPlan {
    int nseg, seg;
    size_t in_bytes[5];  // q, k, v, log_alpha, beta of a full segment
    size_t slot_in, slot_out, state, fwd_ws, total;
};

kda_status make_host_plan(int B, int T, int H, int Hk, int dk, int dv, kda_dtype dt, unsigned pro, int seg,
                          HostPlan& p)
{
    if (seg <= 0 || seg % kChunk != 0 || T <= 0) return KDA_ERR_INVALID_ARG;
    Plan f;
    const int s = seg < T ? seg : T;
    const kda_status st = make_plan(B, s, H, dk, dv, false, 0, dt, f);
    if (st != KDA_OK) return st;
    const size_t esz = dt == KDA_BF16 ? 2 : 4, lsz = (pro & KDA_PROLOGUE_GATE_BF16) ? 2 : 4;
    const size_t tok = (size_t)B * s;
    p.seg = s;
    p.nseg = (T + s - 1) / s;
    p.in_bytes[0] = p.in_bytes[1] = tok * Hk * dk * esz;
    p.in_bytes[2] = tok * H * dv * esz;
    p.in_bytes[3] = tok * H * dk * lsz;
    p.in_bytes[4] = tok * H * sizeof(float);
    p.slot_in = 0;
    for (size_t b : p.in_bytes) p.slot_in += round_up(b, kAlign);
    p.slot_out = round_up(tok * H * dv * esz, kAlign);
    p.state = round_up(sizeof(float) * (size_t)B * H * dk * dv, kAlign);
    p.fwd_ws = round_up(f.total_bytes, kAlign);
    p.total = 2 * (p.slot_in + p.slot_out) + p.state + p.fwd_ws;
    return KDA_OK;
}

}  // namespace

namespace {

// Copy streams and events of kda_chunk_fwd_host, created on the first call for a (device, caller
// stream) pair and reused by every later call on that pair (kda_host_release() destroys them).
struct HostRes {
    int dev = -1;
    cudaStream_t caller = nullptr;
    cudaStream_t cin = nullptr, cout = nullptr;
    cudaEvent_t ev_in[2] = {}, ev_comp[2] = {}, ev_out[2] = {}, ev_start = nullptr;
    std::mutex mu;
};

std::mutex g_host_mu;
std::vector<std::unique_ptr<HostRes>> g_host_res;

void destroy_host_res(HostRes& r)
{
    for (int i = 0; i < 2; ++i) {
        if (r.ev_in[i]) cudaEventDestroy(r.ev_in[i]);
        if (r.ev_comp[i]) cudaEventDestroy(r.ev_comp[i]);
        if (r.ev_out[i]) cudaEventDestroy(r.ev_out[i]);
    }
    if (r.ev_start) cudaEventDestroy(r.ev_start);
    if (r.cin) cudaStreamDestroy(r.cin);
    if (r.cout) cudaStreamDestroy(r.cout);
}

HostRes* host_resources(cudaStream_t caller)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
    std::lock_guard<std::mutex> g(g_host_mu);
    for (auto& r : g_host_res)
        if (r->dev == dev && r->caller == caller) return r.get();
    auto r = std::make_unique<HostRes>();
    r->dev = dev;
    r->caller = caller;
    bool ok = cudaStreamCreateWithFlags(&r->cin, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&r->cout, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&r->ev_start, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; i < 2 && ok; ++i)
        ok = cudaEventCreateWithFlags(&r->ev_in[i], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&r->ev_comp[i], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&r->ev_out[i], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
        destroy_host_res(*r);
        return nullptr;
    }
    g_host_res.push_back(std::move(r));
    return g_host_res.back().get();
}

}  // namespace

extern "C" kda_status kda_host_release(void)
{
    std::lock_guard<std::mutex> g(g_host_mu);
    int cur = -1;
    const bool have_cur = cudaGetDevice(&cur) == cudaSuccess;
    kda_status st = KDA_OK;
    for (auto& r : g_host_res) {
        std::lock_guard<std::mutex> call_guard(r->mu);
        if (cudaSetDevice(r->dev) != cudaSuccess) st = KDA_ERR_CUDA;
        // work queued on these streams completes first; then they are released
        if (cudaStreamSynchronize(r->cin) != cudaSuccess || cudaStreamSynchronize(r->cout) != cudaSuccess)
            st = KDA_ERR_CUDA;
        destroy_host_res(*r);
    }
    g_host_res.clear();
    if (have_cur) cudaSetDevice(cur);
    return st;
}

extern "C" kda_status kda_chunk_fwd_host_workspace_size(int B, int T, int H, int dk, int dv, kda_dtype dt,
                                                        const kda_options* opt, int segment_tokens, size_t* bytes)
{
    if (!bytes) return KDA_ERR_INVALID_ARG;
    int Hk = H;
    unsigned pro = 0;
    const kda_status so = parse_options(opt, H, Hk, pro);
    if (so != KDA_OK) return so;
    HostPlan p;
    const kda_status st = make_host_plan(B, T, H, Hk, dk, dv, dt, pro, segment_tokens, p);
    if (st != KDA_OK) return st;
    *bytes = p.total;
    return KDA_OK;
}

extern "C" kda_status kda_chunk_fwd_host(const void* q, const void* k, const void* v, const void* log_alpha,
                                         const float* beta, const float* S0, void* out, float* S_final, int B,
                                         int T, int H, int dk, int dv, kda_dtype dt, const kda_options* opt,
                                         int segment_tokens, void* workspace, size_t workspace_bytes,
                                         kda_stream_t stream_)
{
    cudaStream_t stream = (cudaStream_t)stream_;
    int Hk = H;
    unsigned pro = 0;
    const kda_status so = parse_options(opt, H, Hk, pro);
    if (so != KDA_OK) return so;
    HostPlan p;
    const kda_status st = make_host_plan(B, T, H, Hk, dk, dv, dt, pro, segment_tokens, p);
    if (st != KDA_OK) return st;
    if (!q || !k || !v || !log_alpha || !beta || !out) return KDA_ERR_INVALID_ARG;
    if (!workspace || ((uintptr_t)workspace % kAlign) || workspace_bytes < p.total) return KDA_ERR_WORKSPACE;

    char* ws = (char*)workspace;
    char* slot_in[2] = {ws, ws + p.slot_in};
    char* slot_out[2] = {ws + 2 * p.slot_in, ws + 2 * p.slot_in + p.slot_out};
    float* state = (float*)(ws + 2 * (p.slot_in + p.slot_out));
    char* fwd_ws = ws + 2 * (p.slot_in + p.slot_out) + p.state;
    const size_t esz = dt == KDA_BF16 ? 2 : 4, lsz = (pro & KDA_PROLOGUE_GATE_BF16) ? 2 : 4;
    // per token of one sequence: bytes of q, k, v, log_alpha, beta, out
    const size_t per_tok[6] = {(size_t)Hk * dk * esz, (size_t)Hk * dk * esz, (size_t)H * dv * esz,
                               (size_t)H * dk * lsz, (size_t)H * sizeof(float), (size_t)H * dv * esz};
    const char* src[5] = {(const char*)q, (const char*)k, (const char*)v, (const char*)log_alpha,
                          (const char*)beta};

    HostRes* hr = host_resources(stream);
    if (!hr) return KDA_ERR_CUDA;
    std::lock_guard<std::mutex> call_guard(hr->mu);  // one call at a time on these copy streams
    cudaStream_t cin = hr->cin, cout = hr->cout;
    cudaEvent_t* ev_in = hr->ev_in;
    cudaEvent_t* ev_comp = hr->ev_comp;
    cudaEvent_t* ev_out = hr->ev_out;
    kda_status rs = KDA_ERR_CUDA;
    // the copy streams start after everything already queued on the caller's stream
    bool ok = cudaEventRecord(hr->ev_start, stream) == cudaSuccess &&
              cudaStreamWaitEvent(cin, hr->ev_start, 0) == cudaSuccess &&
              cudaStreamWaitEvent(cout, hr->ev_start, 0) == cudaSuccess;
    const size_t sbytes = sizeof(float) * (size_t)B * H * dk * dv;
    if (ok) ok = (S0 ? cudaMemcpyAsync(state, S0, sbytes, cudaMemcpyHostToDevice, stream)
                     : cudaMemsetAsync(state, 0, sbytes, stream)) == cudaSuccess;
    kda_options o2 = opt ? *opt : kda_options{};
    for (int i = 0; i < p.nseg && ok; ++i) {
        const int b = i & 1;
        const long long t0 = (long long)i * p.seg;
        const int len = (int)((T - t0) < p.seg ? (T - t0) : p.seg);
        // inputs of segment i into slot b, once segment i - 2 has finished reading it
        if (i >= 2) ok = cudaStreamWaitEvent(cin, ev_comp[b], 0) == cudaSuccess;
        char* dst = slot_in[b];
        void* dptr[5];
        for (int f = 0; f < 5 && ok; ++f) {
            dptr[f] = dst;
            const size_t w = per_tok[f] * (size_t)len;
            ok = cudaMemcpy2DAsync(dst, w, src[f] + per_tok[f] * (size_t)t0, per_tok[f] * (size_t)T, w, B,
                                   cudaMemcpyHostToDevice, cin) == cudaSuccess;
            dst += round_up(p.in_bytes[f], kAlign);
        }
        ok = ok && cudaEventRecord(ev_in[b], cin) == cudaSuccess;
        // compute on the caller's stream, once the inputs landed and slot b's previous output left
        ok = ok && cudaStreamWaitEvent(stream, ev_in[b], 0) == cudaSuccess;
        if (ok && i >= 2) ok = cudaStreamWaitEvent(stream, ev_out[b], 0) == cudaSuccess;
        if (!ok) break;
        const kda_status fs = kda_chunk_fwd_ex(dptr[0], dptr[1], dptr[2], dptr[3], (const float*)dptr[4], state,
                                               nullptr, 0, slot_out[b], state, B, len, H, dk, dv, dt, &o2, fwd_ws,
                                               p.fwd_ws, stream);
        if (fs != KDA_OK) {
            rs = fs;
            ok = false;
            break;
        }
        ok = cudaEventRecord(ev_comp[b], stream) == cudaSuccess;
        // outputs of segment i back to the host
        ok = ok && cudaStreamWaitEvent(cout, ev_comp[b], 0) == cudaSuccess;
        ok = ok && cudaMemcpy2DAsync((char*)out + per_tok[5] * (size_t)t0, per_tok[5] * (size_t)T, slot_out[b],
                                     per_tok[5] * (size_t)len, per_tok[5] * (size_t)len, B, cudaMemcpyDeviceToHost,
                                     cout) == cudaSuccess;
        ok = ok && cudaEventRecord(ev_out[b], cout) == cudaSuccess;
    }
    if (ok && S_final) ok = cudaMemcpyAsync(S_final, state, sbytes, cudaMemcpyDeviceToHost, stream) == cudaSuccess;
    // the caller's stream completes only after every copy of this call
    for (int b = 0; b < 2 && ok; ++b)
        if (p.nseg > b) ok = cudaStreamWaitEvent(stream, ev_out[b], 0) == cudaSuccess;
    if (ok) rs = KDA_OK;
    return rs;
}
