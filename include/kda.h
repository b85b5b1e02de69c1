/*
 * kda.h -- C ABI of libkda.so: the Kimi Delta Attention (KDA) operator on NVIDIA B200 (sm_100a).
 *
 * The operator (forward only).  Per sequence n and head h a state S of shape d_k x d_v
 * (row = key channel, fp32) evolves over the tokens t of the sequence as
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,     o_t = S_t^T q_t
 *
 * with alpha_t = exp(log_alpha_t) a per-key-channel forget gate and beta_t a per-head scalar.
 * Source: "Kimi Linear: redefining long-context inference efficiency" (xugj520.cn), section
 * "Kimi Delta Attention的技术内核" (the recurrent-form update) and the 2025 attention/MoE review
 * (lanjinlin.com.cn), entry "KLA 25.10 kimi" (the per-channel Diag(alpha_t) form and the
 * readout o_t = S_t^T q_t).  No scaling of q is applied (callers pre-scale q if they want one).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers, 16-byte aligned, contiguous, row-major.
 *   - q, k, v, out use the element type `dt` (KDA_BF16 or KDA_F32); log_alpha, beta and every
 *     state are fp32.  Accumulation is fp32.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream) and
 *     never synchronise.  The caller owns every buffer.  The library allocates no device memory.
 *   - Host-checkable argument errors return KDA_ERR_INVALID_ARG / KDA_ERR_UNSUPPORTED before
 *     anything is launched.  A launch failure returns KDA_ERR_CUDA.  Errors found on the device
 *     (a malformed cu_seqlens array, a bounded wait that gave up) are recorded in a device error
 *     word and reported by kda_check().
 *   - Thread safety: calls on different streams are independent; each call only touches the
 *     buffers it is given (and the workspace it is given).
 */
#ifndef KDA_H
#define KDA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;                         /* = cudaStream_t */
typedef struct CUstream_st* kda_stream_t;

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size, inconsistent arguments    */
    KDA_ERR_UNSUPPORTED = 2,   /* valid but not implemented here (e.g. d_k not in {64, 128})    */
    KDA_ERR_CUDA = 3,          /* a CUDA runtime call or kernel launch failed                  */
    KDA_ERR_TIMEOUT = 4,       /* a bounded device-side wait gave up (reported by kda_check)   */
    KDA_ERR_WORKSPACE = 5,     /* workspace pointer NULL/misaligned or smaller than required  */
    KDA_ERR_BAD_SEQLENS = 6    /* cu_seqlens not 0 = c0 <= c1 <= ... <= cN = T (device check)  */
} kda_status;

typedef enum {
    KDA_BF16 = 0,              /* q, k, v, out are bf16 */
    KDA_F32 = 1                /* q, k, v, out are fp32 */
} kda_dtype;

/* Human-readable name of a status code (static string, never NULL). */
const char* kda_status_string(kda_status s);

/* Library version string, e.g. "kda-b200 0.1 sm_100a". */
const char* kda_version(void);

/*
 * kda_chunk_fwd_workspace_size -- bytes of device workspace kda_chunk_fwd needs.
 *
 * Same shape arguments as kda_chunk_fwd (`num_seqs` is used only when `varlen` is nonzero).
 * The bound holds for every cu_seqlens with the given total T and num_seqs.  Writes the size to
 * *bytes.  Returns KDA_ERR_INVALID_ARG / KDA_ERR_UNSUPPORTED for arguments kda_chunk_fwd would
 * reject.
 */
kda_status kda_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv, int varlen, int num_seqs,
                                        kda_dtype dt, size_t* bytes);

/*
 * kda_chunk_fwd -- chunked-parallel prefill (chunk size 64).
 *
 * The algorithm is the chunk form of the recurrence: inside each 64-token chunk the cumulative
 * log-gate g_r = sum_{i<=r} log_alpha_i is restarted, the chunk's rank-1 updates are packed into
 * a WY representation through the UT transform T = (I + strict_lower(diag(beta) (k*e^g)(k*e^-g)^T))^-1
 * diag(beta), the intra-chunk products are dense tensor-core GEMMs, and the state is carried
 * from chunk to chunk ("Kimi Linear" explainer, section "硬件效率的深度优化": chunked parallel
 * computation, WY representation, UT transform; chunk size 64 as in the coreui.cn article,
 * section 2.2 "硬件感知的块状计算").  The result equals the token-by-token recurrence up to
 * rounding.
 *
 * Layout (token-major):
 *   q, k       [B, T, H, dk]  dt
 *   v          [B, T, H, dv]  dt
 *   log_alpha  [B, T, H, dk]  fp32   (log of the forget gate, <= 0 expected; any finite value works)
 *   beta       [B, T, H]      fp32
 *   S0         [N, H, dk, dv] fp32 or NULL (= zero state)                  N = B, or num_seqs
 *   out        [B, T, H, dv]  dt     (written)
 *   S_final    [N, H, dk, dv] fp32 or NULL (not written); may alias S0 (in-place state passing)
 * Varlen: if cu_seqlens (DEVICE int32 [num_seqs+1]) is non-NULL, B must be 1, the T tokens are
 *   num_seqs packed sequences, sequence n = tokens cu_seqlens[n] .. cu_seqlens[n+1]-1, with its
 *   own S0[n] / S_final[n].  Chunks restart at every sequence boundary.  A malformed array is
 *   detected on the device: nothing is computed, out/S_final are left untouched, and
 *   kda_check() returns KDA_ERR_BAD_SEQLENS.
 * Supported: dk, dv in {64, 128}; dt in {KDA_BF16, KDA_F32}; T >= 0 (T = 0 copies S0 to S_final).
 * Workspace: device memory of at least kda_chunk_fwd_workspace_size() bytes, 256-byte aligned,
 *   owned by the caller, contents irrelevant on entry; it must not be used by another call that
 *   runs concurrently.
 */
kda_status kda_chunk_fwd(const void* q, const void* k, const void* v, const float* log_alpha, const float* beta,
                         const float* S0, const int32_t* cu_seqlens, int num_seqs, void* out, float* S_final,
                         int B, int T, int H, int dk, int dv, kda_dtype dt, void* workspace,
                         size_t workspace_bytes, kda_stream_t stream);

/*
 * kda_decode_step -- one token for each of N independent sequences, state updated in place.
 *
 * Follows the per-token loop of the attention review's GDN/KDA pseudo-code (lanjinlin.com.cn,
 * the block that starts from the loaded per-sequence state): (a) decay S' = Diag(alpha) S,
 * (b) value modification u = beta (v - S'^T k), (c) rank-1 update S = S' + k u^T, (d) output from
 * the UPDATED state o = S^T q.  One read and one write of the state per call.
 *
 * Layout:
 *   q, k, log_alpha [N, H, dk] (q, k: dt; log_alpha: fp32);  v [N, H, dv] dt;  beta [N, H] fp32;
 *   S_inout [N, H, dk, dv] fp32 (read, then overwritten with the new state);  out [N, H, dv] dt.
 * Supported: dk, dv in {64, 128}; N >= 0 (N = 0 is a no-op).
 */
kda_status kda_decode_step(const void* q, const void* k, const void* v, const float* log_alpha, const float* beta,
                           float* S_inout, void* out, int N, int H, int dk, int dv, kda_dtype dt,
                           kda_stream_t stream);

/*
 * Options of the extended entry points kda_chunk_fwd_ex and kda_decode_step_ex.  Zero-initialise
 * the struct, then set the fields that differ from the plain entry points:
 *
 *   num_qk_heads  Grouped q/k heads.  q and k hold Hk = num_qk_heads heads ([B, T, Hk, dk] for the
 *                 prefill, [N, Hk, dk] for decode) and value head h reads q/k head h / (H / Hk).
 *                 Every other tensor (v, log_alpha, beta, out, S0, S_final, S_inout) keeps its H
 *                 heads: the gates and the state belong to the value head.  0 means H (one q/k
 *                 head per value head, the plain entry points).  H must be a multiple of Hk,
 *                 else KDA_ERR_INVALID_ARG.  The attention review's GDN pseudo-code
 *                 (lanjinlin.com.cn, entry on Qwen3-Next GDN) comments its q/k and value head
 *                 counts separately; this is that layout.
 *   prologue      Input transforms applied inside the kernels, so the caller can pass the raw
 *                 projections (a set of KDA_PROLOGUE_* bits; 0 = inputs used as given):
 *                   KDA_PROLOGUE_L2NORM_QK    q and k are normalised per (token, q/k head) over the
 *                                             d_k axis in fp32, x / sqrt(sum x^2 + 1e-6), then used
 *                                             at the input precision (bf16 inputs: rounded to bf16).
 *                   KDA_PROLOGUE_GATE_LOGITS  the log_alpha argument holds raw gate logits a:
 *                                             log_alpha = log sigmoid(a) (the log-space forget gate
 *                                             of the coreui.cn article, section 4.2).
 *                   KDA_PROLOGUE_BETA_LOGITS  the beta argument holds raw logits b: beta = sigmoid(b).
 *                   KDA_PROLOGUE_GATE_BF16    the log_alpha argument (log alpha, or gate logits with
 *                                             KDA_PROLOGUE_GATE_LOGITS) points at bf16 values in the
 *                                             same [.., H, dk] layout instead of fp32.  Each value is
 *                                             widened to fp32 exactly on load, so the result is
 *                                             bit-identical to the fp32 call on the same values; the
 *                                             largest input of the prefill is halved.  Any dt.
 *                 Other bits: KDA_ERR_INVALID_ARG.
 *   reserved      Must be zero (KDA_ERR_INVALID_ARG otherwise).
 */
#define KDA_PROLOGUE_L2NORM_QK 1u
#define KDA_PROLOGUE_GATE_LOGITS 2u
#define KDA_PROLOGUE_BETA_LOGITS 4u
#define KDA_PROLOGUE_GATE_BF16 8u
typedef struct {
    int num_qk_heads;
    unsigned prologue;
    int reserved[6];
} kda_options;

/*
 * kda_chunk_fwd_ex -- kda_chunk_fwd with options (`opt` may be NULL: the plain behaviour).
 * Same arguments, layout, workspace (kda_chunk_fwd_workspace_size with the value-head count H),
 * errors and asynchrony as kda_chunk_fwd; with opt->num_qk_heads = Hk, q and k are [B, T, Hk, dk].
 * log_alpha is fp32, or bf16 with KDA_PROLOGUE_GATE_BF16.
 */
kda_status kda_chunk_fwd_ex(const void* q, const void* k, const void* v, const void* log_alpha, const float* beta,
                            const float* S0, const int32_t* cu_seqlens, int num_seqs, void* out, float* S_final,
                            int B, int T, int H, int dk, int dv, kda_dtype dt, const kda_options* opt,
                            void* workspace, size_t workspace_bytes, kda_stream_t stream);

/*
 * kda_decode_step_ex -- kda_decode_step with options (`opt` may be NULL: the plain behaviour).
 * Same arguments, layout and errors as kda_decode_step; with opt->num_qk_heads = Hk, q and k are
 * [N, Hk, dk].  log_alpha is fp32, or bf16 with KDA_PROLOGUE_GATE_BF16.
 */
kda_status kda_decode_step_ex(const void* q, const void* k, const void* v, const void* log_alpha,
                              const float* beta, float* S_inout, void* out, int N, int H, int dk, int dv,
                              kda_dtype dt, const kda_options* opt, kda_stream_t stream);

/*
 * kda_chunk_fwd_host -- kda_chunk_fwd on HOST-resident inputs and outputs, pipelined.
 *
 * A deployment path of this library (the pages describe none): when q, k, v, log_alpha, beta (and
 * S0) live in host memory, the call splits the token axis into segments of `segment_tokens` and
 * runs them through a double-buffered pipeline.  Segment i + 1 is copied in on a copy stream while
 * segment i runs on `stream` and segment i - 1 is copied out on a second copy stream, so the host
 * link's two directions and the kernels overlap.  The state is carried from segment to segment on
 * the device; results are bit-identical to one kda_chunk_fwd_ex call on the whole input, because
 * the segments start on chunk boundaries.
 *   q, k, v, log_alpha, beta, S0, out, S_final: HOST pointers, layouts as kda_chunk_fwd /
 *                kda_chunk_fwd_ex (regular batches of B sequences of T tokens; S0, S_final may be
 *                NULL).  Use page-locked (pinned) memory: pageable memory works but does not overlap.
 *   opt          as kda_chunk_fwd_ex (grouped heads, prologue bits incl. bf16 gates), or NULL.
 *   segment_tokens  a positive multiple of 64 (4096 is a good value for 32 heads of 128).
 *   workspace    DEVICE memory, >= kda_chunk_fwd_host_workspace_size(...) bytes, 256-byte aligned:
 *                two input and two output segment buffers, the state and the chunk workspace.
 * Asynchronous on `stream`: the host buffers must stay untouched, and out / S_final are complete,
 * only once `stream` has been synchronised (the call's copy streams are joined into it).  The two
 * copy streams and their events are created by the first call for a (current device, `stream`)
 * pair and reused by every later call on that pair (calls on one pair from several host threads
 * are serialised on the host); kda_host_release() destroys them.  Errors: as kda_chunk_fwd_ex, and
 * KDA_ERR_INVALID_ARG for a segment length that is not a positive multiple of 64, T <= 0 or a NULL
 * input; after KDA_ERR_CUDA the outputs are undefined.
 */
kda_status kda_chunk_fwd_host_workspace_size(int B, int T, int H, int dk, int dv, kda_dtype dt,
                                             const kda_options* opt, int segment_tokens, size_t* bytes);
kda_status kda_chunk_fwd_host(const void* q, const void* k, const void* v, const void* log_alpha,
                              const float* beta, const float* S0, void* out, float* S_final, int B, int T,
                              int H, int dk, int dv, kda_dtype dt, const kda_options* opt, int segment_tokens,
                              void* workspace, size_t workspace_bytes, kda_stream_t stream);

/*
 * kda_host_release -- waits for the copy streams that kda_chunk_fwd_host keeps per (device, caller
 * stream) pair and destroys them and their events, on every device that has some.  Later calls
 * create them again.  Returns KDA_OK, or KDA_ERR_CUDA if a synchronisation or destroy failed.
 */
kda_status kda_host_release(void);

/*
 * kda_chunk_bwd -- the backward pass of kda_chunk_fwd (training): the derivatives of a scalar loss
 * L with respect to every input, given the cotangents of the outputs,
 *
 *     dq = dL/dq, dk = dL/dk, dv = dL/dv, dlog_alpha = dL/dlog_alpha, dbeta = dL/dbeta, dS0 = dL/dS0,
 *
 * for L = sum(dout * out) + sum(dS_final * S_final) with (out, S_final) = kda_chunk_fwd(...).  The
 * pages mention a custom backward only in passing; the derivative is that of the recurrence of the
 * "Kimi Linear" explainer (section "Kimi Delta Attention的技术内核"), taken through the chunk form
 * its section "硬件效率的深度优化" lists: the forward is recomputed chunk-parallel keeping only each
 * chunk's start state, the state cotangent runs backwards over the chunks, and the input
 * derivatives are again chunk-parallel.  Arithmetic is fp32 on CUDA cores; for bf16 inputs with
 * dk = dv = 128 every chunk product and both chains run on the tensor cores with each fp32 operand
 * split into two bf16 parts (hi*hi + hi*lo + lo*hi, about 16 significant bits), which keeps the
 * same fp32-level accuracy.
 *
 *   q, k, v, log_alpha, beta, S0, cu_seqlens, num_seqs, B, T, H, dk, dv, dt:  exactly as given to
 *                kda_chunk_fwd (same layout, same meaning).
 *   dout       [B, T, H, dv] (or packed [T, H, dv]) in dt: dL/dout.
 *   dS_final   [N, H, dk, dv] fp32, or NULL: dL/dS_final = 0.
 *   dq, dk     [B, T, H, dk] in dt;  dv [B, T, H, dv] in dt;  dlog_alpha [B, T, H, dk] fp32;
 *   dbeta      [B, T, H] fp32;  dS0 [N, H, dk, dv] fp32 or NULL (not wanted).  All written whole.
 *   opt        NULL, or the options of the forward call: grouped q/k heads (num_qk_heads = Hk: q, k,
 *              dq, dk are [.., Hk, dk]; dq and dk sum the contributions of the H / Hk value heads that
 *              read each q/k head) and any KDA_PROLOGUE_* bits.  With prologue bits the inputs are the
 *              raw ones the forward took and the gradients are those of the raw inputs: through the
 *              q/k norm (its rounding to the input precision passed straight through), the
 *              log-sigmoid of the gate logits and the sigmoid of the beta logits.
 *   workspace  >= kda_chunk_bwd_workspace_size(...) bytes (same opt), 256-byte aligned, owned by
 *              the caller: per (64-token chunk, head) the fp32 chunk intermediates, the chunk's state
 *              and its cotangent; with grouped heads also two fp32 [T, H, dk] buffers.
 * Pointers 16-byte aligned (cu_seqlens 4), device memory, no overlap between outputs and inputs.
 * Errors: as kda_chunk_fwd.  Asynchronous on `stream`; a malformed cu_seqlens sets the device
 * error word (read by kda_check) and computes nothing.
 */
kda_status kda_chunk_bwd_workspace_size(int B, int T, int H, int dk, int dv, int varlen, int num_seqs,
                                        kda_dtype dt, const kda_options* opt, size_t* bytes);
kda_status kda_chunk_bwd(const void* q, const void* k, const void* v, const void* log_alpha, const float* beta,
                         const float* S0, const int32_t* cu_seqlens, int num_seqs, const void* dout,
                         const float* dS_final, void* dq, void* dk, void* dv, float* dlog_alpha, float* dbeta,
                         float* dS0, int B, int T, int H, int dk_dim, int dv_dim, kda_dtype dt,
                         const kda_options* opt, void* workspace, size_t workspace_bytes, kda_stream_t stream);

/*
 * kda_gated_rmsnorm -- the output gate of a KDA layer, one fused streaming pass:
 *
 *     y = o / sqrt(mean_g(o^2) + eps) * weight * act(z)
 *
 * The attention review's GDN/KDA pseudo-code (lanjinlin.com.cn, entry on Qwen3-Next GDN, step
 * "门控归一化") normalises the attention output with an RMS norm and multiplies it by the output gate
 * z; the review's Ring-linear notes take that norm over groups of channels, each group on its own
 * (grouped RMS norm), and fuse the norm, the gate's sigmoid and the product into one kernel.
 *
 *   o, z, y   [rows, d] element type dt, contiguous (e.g. the [B, T, H, dv] output of
 *             kda_chunk_fwd with rows = B*T*H, d = dv, and the gate in the same layout);
 *             y may alias o (in place).
 *   weight    [d] fp32 per-channel scale, or NULL (= ones).
 *   group     channels per norm group: 0 (= d) or a power of two in [8, d] dividing d.
 *   eps       > 0, added to the mean square.
 *   act       KDA_GATE_IDENTITY (z used as given) or KDA_GATE_SIGMOID (sigmoid(z)).
 * Supported: d in {64, 128}.  rows >= 0 (0 is a no-op).  Pointers 16-byte aligned.
 * Errors: KDA_ERR_INVALID_ARG for null/misaligned pointers, a bad group, eps <= 0 or an unknown
 * act; KDA_ERR_UNSUPPORTED for other d.
 */
typedef enum {
    KDA_GATE_IDENTITY = 0,
    KDA_GATE_SIGMOID = 1
} kda_gate_act;
kda_status kda_gated_rmsnorm(const void* o, const void* z, const float* weight, void* y, long long rows, int d,
                             int group, float eps, kda_gate_act act, kda_dtype dt, kda_stream_t stream);

/*
 * kda_chunk_fwd_gated -- the prefill with the output gate applied: `out` receives
 *
 *     y = o / sqrt(mean_g(o^2) + eps) * weight * act(z)
 *
 * (the operation of kda_gated_rmsnorm) where o is the output kda_chunk_fwd_ex would write; o itself
 * is not written anywhere.  On the tensor-core path (bf16, dk = dv = 128) the gate runs in the
 * epilogue that forms o, from its fp32 value before any rounding, so y costs one read of z instead of
 * a write and a read of o; groups of 64 or 128 channels are reduced across the four CTAs that own a
 * head's output columns.  On every other path the prefill writes o to `out` and kda_gated_rmsnorm
 * runs over it in place on the same stream.  The fused epilogue evaluates sigmoid(z) as
 * 0.5 + 0.5 tanh(z / 2) with the hardware's tanh approximation (absolute error about 2^-11, below the
 * bf16 rounding of y).
 *
 *   gate->z        [B, T, H, dv] element type dt (the layout of out), 16-byte aligned; may be NULL
 *                  only when there are no tokens.  Must not alias out.
 *   gate->weight   [dv] fp32, or NULL (= ones); 16-byte aligned.
 *   gate->group    channels per norm group: 0 (= dv) or a power of two in [8, dv].
 *   gate->eps      > 0.
 *   gate->act      KDA_GATE_IDENTITY or KDA_GATE_SIGMOID.
 *   gate->reserved must be zero.
 * gate = NULL is exactly kda_chunk_fwd_ex.  All other arguments, the workspace, the errors and the
 * asynchrony are those of kda_chunk_fwd_ex; a bad gate field returns KDA_ERR_INVALID_ARG before
 * anything is launched.
 */
typedef struct {
    const void* z;
    const float* weight;
    int group;
    float eps;
    kda_gate_act act;
    int reserved[3];
} kda_output_gate;
kda_status kda_chunk_fwd_gated(const void* q, const void* k, const void* v, const void* log_alpha, const float* beta,
                               const float* S0, const int32_t* cu_seqlens, int num_seqs, void* out, float* S_final,
                               int B, int T, int H, int dk, int dv, kda_dtype dt, const kda_options* opt,
                               const kda_output_gate* gate, void* workspace, size_t workspace_bytes,
                               kda_stream_t stream);

/*
 * kda_check -- synchronise `stream`, then read and clear the device error word of the current
 * device.  Returns KDA_OK, KDA_ERR_CUDA (a sticky CUDA error), KDA_ERR_BAD_SEQLENS or
 * KDA_ERR_TIMEOUT.
 */
kda_status kda_check(kda_stream_t stream);

/*
 * kda_selftest_timeout -- exercises the failure path of the library's bounded device waits (no
 * operator work): launches one small kernel that waits, with the same bounded wait the tensor-core
 * kernels use, on a barrier nothing ever completes.  The wait gives up after ~0.2 s, records
 * KDA_ERR_TIMEOUT in the device error word and the kernel exits normally; the next kda_check()
 * returns KDA_ERR_TIMEOUT and clears the word.  The context stays usable.
 */
kda_status kda_selftest_timeout(kda_stream_t stream);

/*
 * kda_chunk_fwd_noalloc -- kda_chunk_fwd for callers that cannot allocate device memory.
 *
 * The pages describe no counterpart: this is a deployment convenience of this library.  Some
 * hosts of this operator cannot hand it a workspace: an engine whose device memory is fully
 * reserved up front by its own pool, a plugin whose enqueue hook may not call cudaMalloc, or a
 * runtime with a fixed, audited memory budget.  This entry point takes the same arguments as
 * kda_chunk_fwd minus the workspace and uses instead a scratch array compiled into the library:
 * KDA_NOALLOC_SCRATCH_BYTES bytes of static device memory on every GPU that loads the library,
 * held until the process exits.  It calls no cudaMalloc, cudaFree or allocating library routine.
 *   - Limit: a problem whose kda_chunk_fwd_workspace_size() exceeds KDA_NOALLOC_SCRATCH_BYTES is
 *     rejected with KDA_ERR_WORKSPACE before anything is launched.  For bf16 with dk = dv = 128 the
 *     workspace is 512 B (more past 31 sequences) plus 82,432 B per (chunk, head), with
 *     ceil(T / 64) chunks per sequence for regular batches and T / 64 + num_seqs for packed input:
 *     at H = 32, 25 chunks, i.e. 1,600 tokens of one sequence.  Longer inputs can be fed in
 *     pieces, passing S_final of one call as S0 of the next.
 *   - Every call looks up the array's device address on the device current at the call (make
 *     the device of the tensors current); make the first call on a device before any stream
 *     capture, since it may load the library's device code on that device.
 *   - All calls on a device share the one array: calls that overlap on the GPU (e.g. on two
 *     streams at once) race and corrupt each other's results.  Serialise them.  The kernels
 *     rewrite every scratch byte they read within the same call, so nothing has to start zeroed
 *     and stale contents from an earlier call are harmless.
 * Returns the same codes as kda_chunk_fwd.
 */
#define KDA_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
kda_status kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const float* log_alpha,
                                 const float* beta, const float* S0, const int32_t* cu_seqlens, int num_seqs,
                                 void* out, float* S_final, int B, int T, int H, int dk, int dv, kda_dtype dt,
                                 kda_stream_t stream);

/*
 * Per-launch timing, for benchmarks and profiles (not part of the operator).  Between
 * kda_profile_begin() and kda_profile_end() every kernel the library launches is bracketed by two
 * CUDA events recorded on the launch's own stream.  kda_profile_kernels() waits for the recorded
 * events and fills, for up to `max_kernels` distinct kernels, a static name (valid for the life of
 * the library), the number of launches and their summed device time in milliseconds; it returns
 * the number of distinct kernels, or -1 if a buffer is too small or an event query failed.
 * Recording is off by default and costs two event records per launch when on.
 */
kda_status kda_profile_begin(void);
kda_status kda_profile_end(void);
int kda_profile_kernels(int max_kernels, const char** names, int* launches, double* total_ms);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H */
