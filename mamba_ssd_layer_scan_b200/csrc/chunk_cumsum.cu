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
// One CTA per (32-head tile, chunk, batch): a coalesced load of the chunk's dt rows for the
// 32 heads into shared memory, then one warp per head scans the Q values with shuffles.
#include "common.cuh"

namespace ssd {
namespace {

constexpr int kHeadTile = 32;
constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
chunk_cumsum_kernel(const float *__restrict__ dt, const float *__restrict__ A,
                    float *__restrict__ cs, int *__restrict__ status, int64_t seqlen, int H,
                    int Q, int64_t nchunks)
{
    // First kernel of every scan: clears the workspace status word the later kernels may set.
    if (status && blockIdx.x == 0 && threadIdx.x == 0) *status = 0;
    extern __shared__ float tile[];  // [Q][kHeadTile + 1]
    const int nht = (H + kHeadTile - 1) / kHeadTile;
    const int h0 = (int)(blockIdx.x % nht) * kHeadTile;
    const int64_t k = (blockIdx.x / nht) % nchunks;
    const int64_t b = blockIdx.x / nht / nchunks;
    const int nh = min(kHeadTile, H - h0);
    const int64_t t0 = k * Q;
    const int len = (int)min((int64_t)Q, seqlen - t0);

    for (int idx = threadIdx.x; idx < Q * kHeadTile; idx += kThreads) {
        const int tau = idx / kHeadTile, j = idx % kHeadTile;
        float v = 0.f;
        if (tau < len && j < nh)
            v = dt[(b * seqlen + t0 + tau) * H + h0 + j] * A[h0 + j];
        tile[tau * (kHeadTile + 1) + j] = v;
    }
    __syncthreads();

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    for (int j = warp; j < nh; j += kThreads / 32) {
        float *out = cs + ((b * nchunks + k) * H + h0 + j) * (int64_t)Q;
        float carry = 0.f;
        for (int s = 0; s < Q; s += 32) {
            float v = (s + lane < Q) ? tile[(s + lane) * (kHeadTile + 1) + j] : 0.f;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float n = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += n;
            }
            v += carry;
            if (s + lane < Q) out[s + lane] = v;
            carry = __shfl_sync(0xffffffffu, v, 31);
        }
    }
}

__global__ void fill_final_kernel(const float *__restrict__ init, float *__restrict__ out,
                                  int64_t n)
{
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i < n) out[i] = init ? init[i] : 0.f;
}

}  // namespace

cudaError_t launch_chunk_cumsum(const float *dt, const float *A, float *cs, int *status,
                                int64_t batch, int64_t seqlen, int nheads, int Q,
                                int64_t nchunks, cudaStream_t st)
{
    const unsigned grid = (unsigned)(((nheads + kHeadTile - 1) / kHeadTile) * nchunks * batch);
    const size_t smem = (size_t)Q * (kHeadTile + 1) * sizeof(float);
    chunk_cumsum_kernel<<<grid, kThreads, smem, st>>>(dt, A, cs, status, seqlen, nheads, Q,
                                                      nchunks);
    return cudaGetLastError();
}

cudaError_t launch_fill_final(const float *init, float *final_state, int64_t n,
                              cudaStream_t st)
{
    if (n == 0) return cudaSuccess;
    fill_final_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(init, final_state, n);
    return cudaGetLastError();
}

}  // namespace ssd
