// chunks.cuh -- per-sequence chunk table for the chunked prefill (regular batches and varlen).
//
// Besides the chunk offsets the kernel writes order[N]: the sequences sorted by length, longest
// first (stable; identity for regular batches and for more than kOrderMax sequences).  The
// sequential phase launches its CTAs in this order, so the longest chains start first and short
// ones fill in behind them.
//
// Chunks never straddle a sequence boundary: sequence n of length len_n owns ceil(len_n / 64)
// chunks, the last one possibly partial.  The table is off[n] = sum_{m<n} ceil(len_m / 64)
// (off[N] = total) plus a header with the total and a "bad input" flag.  One CTA computes it
// with a block-wide scan; cu_seqlens is validated here (c0 = 0, non-decreasing, cN = T), and a
// malformed array sets the flag (every later kernel of the call then does nothing) and the
// device error word.
#pragma once

#include "common.cuh"

namespace kda {

constexpr int kTableThreads = 1024;
constexpr int kOrderMax = 1024;

__global__ void __launch_bounds__(kTableThreads)
chunk_table_kernel(const int32_t* __restrict__ cu, int N, int Tseq, long long Ttot, WsHeader* hdr, int* off,
                   int* order)
{
    __shared__ int s_len[kOrderMax];
    __shared__ int s_warp[32];
    __shared__ int s_carry;
    __shared__ int s_bad;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    if (tid == 0) { s_carry = 0; s_bad = 0; }
    __syncthreads();
    if (cu) {
        if (tid == 0 && (cu[0] != 0 || (long long)cu[N] != Ttot)) s_bad = 1;
        for (int n = tid; n < N; n += kTableThreads)
            if (cu[n + 1] < cu[n]) s_bad = 1;
    }
    __syncthreads();
    const int bad = s_bad;
    for (int base = 0; base < N; base += kTableThreads) {
        const int n = base + tid;
        int cnt = 0;
        if (!bad && n < N) {
            const long long len = cu ? (long long)cu[n + 1] - cu[n] : (long long)Tseq;
            cnt = (int)((len + kChunk - 1) / kChunk);
        }
        // inclusive warp scan
        int x = cnt;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, d);
            if (lane >= d) x += y;
        }
        if (lane == 31) s_warp[wid] = x;
        __syncthreads();
        if (wid == 0) {
            int s = s_warp[lane];
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, s, d);
                if (lane >= d) s += y;
            }
            s_warp[lane] = s;  // inclusive prefix of warp totals
        }
        __syncthreads();
        const int excl = s_carry + (wid > 0 ? s_warp[wid - 1] : 0) + x - cnt;
        if (n < N) off[n] = excl;
        __syncthreads();
        if (tid == kTableThreads - 1) s_carry = excl + cnt;
        __syncthreads();
    }
    // longest-first order of the sequences
    if (cu && !bad && N <= kOrderMax) {
        for (int n = tid; n < N; n += kTableThreads) s_len[n] = cu[n + 1] - cu[n];
        __syncthreads();
        for (int i = tid; i < N; i += kTableThreads) {
            const int li = s_len[i];
            int rank = 0;
            for (int jj = 0; jj < N; ++jj) {
                const int lj = s_len[jj];
                rank += (lj > li) || (lj == li && jj < i);
            }
            order[rank] = i;
        }
    } else {
        for (int n = tid; n < N; n += kTableThreads) order[n] = n;
    }
    if (tid == 0) {
        off[N] = s_carry;
        hdr->total_chunks = s_carry;
        hdr->bad = bad;
        hdr->next_unit = 0;
        if (bad) set_error(KDA_ERR_BAD_SEQLENS);
    }
}

}  // namespace kda
