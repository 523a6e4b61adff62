// dA cumsum: the chunk-local log-decay prefix of every (batch, chunk, head).
//
// cs[b][k][h][tau] = sum_{s <= tau} dt[b][kQ+s][h] * A_h over the tokens of chunk k, so that
// the decay from token i to token t of the same chunk is exp(cs_t - cs_i) = prod_{j=i+1..t} a_j
// with a_j = exp(dt_j A_h) (eightmm.github.io "Mamba-2", Matrix Mixer View: the product of the
// A_j between two positions; mohakchugh.is-a.dev "Mamba-2", Block Decomposition: the sequence
// is cut into chunks of Q tokens).  Positions past the end of the sequence (a partial last
// chunk) contribute dt = 0, so cs stays flat there and the chunk's total log-decay is always
// cs[..][Q-1].  Resetting the sum at every chunk keeps its magnitude bounded by Q*max|dt*A|.
//
// One CTA per (8-head tile, chunk, batch): the chunk's dt rows for the 8 heads are staged in
// shared memory, then one warp per head scans its Q values with shuffles.  When
// dtc is given, dt is also written in the same (b, c, H, Q) layout as cs (0 past the end of the
// sequence), so that the tensor-core kernels can fetch both per-head rows with one bulk copy.
#include "common.cuh"

namespace ssd {
namespace {

constexpr int kHeadTile = 8;     // heads per CTA, one warp each
constexpr int kThreads = 32 * kHeadTile;
constexpr int kMaxSeg = 8;       // Q <= 256 = 8 segments of 32 tokens

__global__ void __launch_bounds__(kThreads)
chunk_cumsum_kernel(const float *__restrict__ dt, const float *__restrict__ A,
                    float *__restrict__ cs, float *__restrict__ dtc, int *__restrict__ status,
                    int64_t seqlen, int H, int Q, int64_t nchunks, const int2 *__restrict__ tab,
                    bool unit_weights)
{
    griddep_wait();               // nothing of an earlier kernel is touched before this
    griddep_launch_dependents();
    // First kernel of every scan: clears the workspace status word the later kernels may set.
    if (status && blockIdx.x == 0 && threadIdx.x == 0) *status = 0;
    extern __shared__ float tile[];  // [Q][kHeadTile + 1]
    const int nht = (H + kHeadTile - 1) / kHeadTile;
    const int h0 = (int)(blockIdx.x % nht) * kHeadTile;
    const int64_t k = (blockIdx.x / nht) % nchunks;
    const int64_t b = blockIdx.x / nht / nchunks;
    const int nh = min(kHeadTile, H - h0);
    int64_t t0;
    int len;
    chunk_span(tab, k, Q, seqlen, t0, len);
    if (len <= 0) return;   // unused slot of a chunk table

    for (int idx = threadIdx.x; idx < Q * kHeadTile; idx += kThreads) {
        const int tau = idx / kHeadTile, j = idx % kHeadTile;
        float v = 0.f;
        if (tau < len && j < nh)
            v = dt[(b * seqlen + t0 + tau) * H + h0 + j];
        tile[tau * (kHeadTile + 1) + j] = v;
    }
    __syncthreads();

    const int j = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (j >= nh) return;
    const int64_t row = ((b * nchunks + k) * H + h0 + j) * (int64_t)Q;
    const float Ah = A[h0 + j];
    const int nseg = (Q + 31) / 32;
    // Independent inclusive scans of every 32-token segment (interleaved for ILP), then the
    // segment totals are carried forward.
    float v[kMaxSeg];
#pragma unroll
    for (int sg = 0; sg < kMaxSeg; ++sg) {
        const int tau = sg * 32 + lane;
        const float d = (sg < nseg && tau < Q) ? tile[tau * (kHeadTile + 1) + j] : 0.f;
        // unit_weights: the input weight of every token is 1 (decay still from dt); 0 past the end
        if (dtc && sg < nseg && tau < Q) dtc[row + tau] = unit_weights ? (tau < len ? 1.f : 0.f) : d;
        v[sg] = d * Ah;
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
        for (int sg = 0; sg < kMaxSeg; ++sg) {
            const float n = __shfl_up_sync(0xffffffffu, v[sg], o);
            if (lane >= o) v[sg] += n;
        }
    }
    float carry = 0.f;
#pragma unroll
    for (int sg = 0; sg < kMaxSeg; ++sg) {
        const float total = __shfl_sync(0xffffffffu, v[sg], 31);
        const int tau = sg * 32 + lane;
        if (sg < nseg && tau < Q) cs[row + tau] = v[sg] + carry;
        carry += total;
    }
}

__global__ void fill_final_kernel(const float *__restrict__ init, float *__restrict__ out,
                                  int64_t n)
{
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i < n) out[i] = init ? init[i] : 0.f;
}

}  // namespace

cudaError_t launch_chunk_cumsum(const float *dt, const float *A, float *cs, float *dtc,
                                int *status, int64_t batch, int64_t seqlen, int nheads, int Q,
                                int64_t nchunks, cudaStream_t st, const int2 *tab,
                                bool unit_weights)
{
    const unsigned grid = (unsigned)(((nheads + kHeadTile - 1) / kHeadTile) * nchunks * batch);
    const size_t smem = (size_t)Q * (kHeadTile + 1) * sizeof(float);
    return launch_pdl(chunk_cumsum_kernel, grid, kThreads, smem, st, dt, A, cs, dtc, status,
                      seqlen, nheads, Q, nchunks, tab, unit_weights);
}

cudaError_t launch_fill_final(const float *init, float *final_state, int64_t n,
                              cudaStream_t st)
{
    if (n == 0) return cudaSuccess;
    fill_final_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(init, final_state, n);
    return cudaGetLastError();
}

}  // namespace ssd
