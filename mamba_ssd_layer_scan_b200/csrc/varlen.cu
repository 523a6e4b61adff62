// Packed variable-length sequences: the chunk table.
//
// Several sequences packed back to back along the token axis each carry their own state: the
// recurrence restarts at every sequence boundary (mohakchugh.is-a.dev "Mamba-2", the state
// passing between blocks; the pages' remark that the scan needs no padding).  The chunked scan
// handles this without masks inside a chunk by never letting a chunk span two sequences: every
// sequence is cut into its own chunks of Q tokens, its last chunk possibly partial, and the table
// lists each chunk's first token and length.  Every kernel then treats a table chunk exactly as
// it treats the partial last chunk of a fixed-length sequence (dt = 0 past the chunk's end, rows
// past it neither contribute nor are stored), and state passing walks the chunks of each
// sequence from that sequence's own initial state.
//
// One CTA builds the table: per sequence its chunk count, an exclusive prefix sum over the
// sequences (1024 at a time, warp shuffles plus one pass over the warp totals), then each thread
// writes its sequence's entries.  Slots past the total keep length 0; the kernels launched over
// the upper bound of slots skip them.
#include "common.cuh"

namespace ssd {
namespace {

constexpr int kTableThreads = 1024;

__global__ void __launch_bounds__(kTableThreads)
build_chunk_table_kernel(const int32_t *__restrict__ cu, int nseq, int64_t seqlen, int Q,
                         int64_t nslots, int2 *__restrict__ tab, int32_t *__restrict__ cstart,
                         int *__restrict__ status)
{
    __shared__ int warp_tot[kTableThreads / 32];
    __shared__ int carry;
    __shared__ int bad;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    if (tid == 0) {
        carry = 0;
        bad = 0;
        *status = 0;   // first kernel of the call: start from a clean status word
    }
    __syncthreads();
    // cu_seqlens must start at 0, end at the token count and never decrease
    for (int s = tid; s <= nseq; s += kTableThreads) {
        const int64_t v = cu[s];
        bool wrong = v < 0 || v > seqlen || (s == 0 && v != 0) || (s == nseq && v != seqlen);
        if (s > 0 && cu[s - 1] > v) wrong = true;
        if (wrong) atomicOr(&bad, 1);
    }
    __syncthreads();
    const bool ok = bad == 0;
    for (int base = 0; base < nseq; base += kTableThreads) {
        const int s = base + tid;
        const int n = (ok && s < nseq) ? (cu[s + 1] - cu[s] + Q - 1) / Q : 0;
        int incl = n;   // inclusive scan within the warp
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += u;
        }
        if (lane == 31) warp_tot[w] = incl;
        __syncthreads();
        if (w == 0) {   // inclusive scan of the 32 warp totals
            int t = warp_tot[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, t, o);
                if (lane >= o) t += u;
            }
            warp_tot[lane] = t;
        }
        __syncthreads();
        const int first = carry + (w > 0 ? warp_tot[w - 1] : 0) + incl - n;
        if (s < nseq) {
            cstart[s] = first;
            const int t0 = ok ? cu[s] : 0;
            const int len = ok ? cu[s + 1] - cu[s] : 0;
            for (int i = 0; i < n; ++i)
                tab[first + i] = make_int2(t0 + i * Q, min(Q, len - i * Q));
        }
        __syncthreads();
        if (tid == kTableThreads - 1) carry = first + n;
        __syncthreads();
    }
    const int total = carry;
    if (tid == 0) {
        cstart[nseq] = total;
        if (!ok) atomicOr(status, kStatusBadSeqlens);
    }
    for (int64_t k = total + tid; k < nslots; k += kTableThreads) tab[k] = make_int2(0, 0);
}

}  // namespace

cudaError_t launch_build_chunk_table(const int32_t *cu_seqlens, int nseq, int64_t seqlen, int Q,
                                     int64_t nchunks, int2 *tab, int32_t *cstart, int *status,
                                     cudaStream_t st)
{
    build_chunk_table_kernel<<<1, kTableThreads, 0, st>>>(cu_seqlens, nseq, seqlen, Q, nchunks,
                                                          tab, cstart, status);
    return cudaGetLastError();
}

}  // namespace ssd
