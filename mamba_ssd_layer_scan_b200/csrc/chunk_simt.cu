// CUDA-core (float32 arithmetic) chunk-state and intra-chunk kernels.
//
// They serve float32 inputs, whose 1e-4 parity bound bf16 tensor cores cannot meet, and the
// bf16 shapes the tensor-core kernels do not cover.  Same math as the tcgen05 kernels:
//
//   chunk state   S_k[p][n] = sum_{tau in k} exp(cs_last - cs_tau) dt_tau x_tau[p] B_tau[n]
//   chunk output  y_t[p]    = sum_{i <= t, i in k} (C_t . B_i) exp(cs_t - cs_i) dt_i x_i[p]
//                           + exp(cs_t) sum_n C_t[n] h_in[p][n]  +  D_h x_t[p]
//
// i.e. the within-block quadratic (attention-like) form plus the contribution of the state
// carried in from earlier blocks (mohakchugh.is-a.dev "Mamba-2", Block Decomposition and The
// Duality; the decay inside the off-chunk term is exp(cs_t), the product of a_j from the
// chunk start to t, which the page's sketch leaves out).
#include "common.cuh"

namespace ssd {
namespace {

constexpr int kThreads = 256;
constexpr int kRows = 32;      // tokens per shared-memory tile
constexpr int kMaxAcc = 64;    // outputs per thread: P*N <= 16384 = 256 * 64

// One CTA per (head, chunk, batch).
template <typename T>
__global__ void __launch_bounds__(kThreads)
chunk_state_simt_kernel(const T *__restrict__ x, const float *__restrict__ dt,
                        const T *__restrict__ B, const float *__restrict__ cs,
                        float *__restrict__ states, int64_t seqlen, int H, int G, int P, int N,
                        int Q, int64_t nchunks)
{
    extern __shared__ float sm[];
    float *xs = sm;                    // [kRows][P], rows already scaled by w
    float *bs = xs + kRows * P;        // [kRows][N]
    float *w = bs + kRows * N;         // [kRows]
    const int h = (int)(blockIdx.x % H);
    const int64_t k = (blockIdx.x / H) % nchunks, b = blockIdx.x / H / nchunks;
    const int g = h / (H / G);
    const int64_t t0 = k * Q;
    const int len = (int)min((int64_t)Q, seqlen - t0);
    const float *csk = cs + ((b * nchunks + k) * H + h) * (int64_t)Q;
    const float cs_last = csk[Q - 1];
    const int PN = P * N;

    float acc[kMaxAcc];
#pragma unroll
    for (int j = 0; j < kMaxAcc; ++j) acc[j] = 0.f;

    for (int s = 0; s < len; s += kRows) {
        const int rows = min(kRows, len - s);
        __syncthreads();
        if (threadIdx.x < kRows) {
            const int r = threadIdx.x;
            float wr = 0.f;
            if (r < rows)
                wr = __expf(cs_last - csk[s + r]) * dt[(b * seqlen + t0 + s + r) * H + h];
            w[r] = wr;
        }
        __syncthreads();
        for (int idx = threadIdx.x; idx < kRows * P; idx += kThreads) {
            const int r = idx / P, p = idx % P;
            float v = 0.f;
            if (r < rows) v = w[r] * to_f32(x[((b * seqlen + t0 + s + r) * H + h) * P + p]);
            xs[idx] = v;
        }
        for (int idx = threadIdx.x; idx < kRows * N; idx += kThreads) {
            const int r = idx / N, n = idx % N;
            float v = 0.f;
            if (r < rows) v = to_f32(B[((b * seqlen + t0 + s + r) * G + g) * N + n]);
            bs[idx] = v;
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < kMaxAcc; ++j) {
            const int o = threadIdx.x + j * kThreads;
            if (o < PN) {
                const int p = o / N, n = o % N;
                float a = acc[j];
                for (int r = 0; r < rows; ++r) a = fmaf(xs[r * P + p], bs[r * N + n], a);
                acc[j] = a;
            }
        }
    }
    float *out = states + ((b * nchunks + k) * H + h) * (int64_t)PN;
#pragma unroll
    for (int j = 0; j < kMaxAcc; ++j) {
        const int o = threadIdx.x + j * kThreads;
        if (o < PN) out[o] = acc[j];
    }
}

// One CTA per (32-token tile, head, batch*chunk).  Thread owns outputs (t, p) of the tile.
constexpr int kMaxOut = 16;    // kRows * P / kThreads with P <= 128

template <typename T>
__global__ void __launch_bounds__(kThreads)
chunk_scan_simt_kernel(const T *__restrict__ x, const float *__restrict__ dt,
                       const T *__restrict__ B, const T *__restrict__ C,
                       const float *__restrict__ cs, const float *__restrict__ hin,
                       const float *__restrict__ D, T *__restrict__ y, int64_t seqlen, int H,
                       int G, int P, int N, int Q, int64_t nchunks, const T *__restrict__ z)
{
    extern __shared__ float sm[];
    float *cts = sm;                   // [kRows][N]   C rows of this tile
    float *bts = cts + kRows * N;      // [kRows][N]   B rows of a source tile
    float *xts = bts + kRows * N;      // [kRows][P]   x rows of a source tile
    float *gts = xts + kRows * P;      // [kRows][kRows + 1] masked C.B^T block
    float *hts = gts + kRows * (kRows + 1);  // [P][kRows + 1] slice of h_in over n
    const int ntiles = (Q + kRows - 1) / kRows;
    const int tt = (int)(blockIdx.x % ntiles);
    const int h = (int)((blockIdx.x / ntiles) % H);
    const int64_t bk = blockIdx.x / ntiles / H;
    const int64_t b = bk / nchunks, k = bk % nchunks;
    const int g = h / (H / G);
    const int64_t t0 = k * Q;
    const int len = (int)min((int64_t)Q, seqlen - t0);
    const int r0 = tt * kRows;  // first row of this tile within the chunk
    if (r0 >= len) return;
    const int rows = min(kRows, len - r0);
    const float *csk = cs + ((b * nchunks + k) * H + h) * (int64_t)Q;
    const float *hk = hin + ((b * nchunks + k) * H + h) * (int64_t)P * N;
    const int nout = kRows * P;

    for (int idx = threadIdx.x; idx < kRows * N; idx += kThreads) {
        const int r = idx / N, n = idx % N;
        cts[idx] = r < rows ? to_f32(C[((b * seqlen + t0 + r0 + r) * G + g) * N + n]) : 0.f;
    }

    // Off-chunk term: exp(cs_t) * sum_n C_t[n] h_in[p][n], accumulated over n-slices of h_in.
    float acc[kMaxOut];
#pragma unroll
    for (int j = 0; j < kMaxOut; ++j) acc[j] = 0.f;
    for (int n0 = 0; n0 < N; n0 += kRows) {
        __syncthreads();
        for (int idx = threadIdx.x; idx < P * kRows; idx += kThreads) {
            const int p = idx / kRows, n = idx % kRows;
            hts[p * (kRows + 1) + n] = hk[(int64_t)p * N + n0 + n];
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < kMaxOut; ++j) {
            const int o = threadIdx.x + j * kThreads;
            if (o < nout) {
                const int t = o / P, p = o % P;
                float a = acc[j];
                for (int n = 0; n < kRows; ++n)
                    a = fmaf(cts[t * N + n0 + n], hts[p * (kRows + 1) + n], a);
                acc[j] = a;
            }
        }
    }
#pragma unroll
    for (int j = 0; j < kMaxOut; ++j) {
        const int o = threadIdx.x + j * kThreads;
        if (o < nout) acc[j] *= __expf(csk[min(r0 + o / P, Q - 1)]);
    }

    // Within-chunk quadratic term over source tiles s <= tt.
    for (int st = 0; st <= tt; ++st) {
        const int s0 = st * kRows;
        __syncthreads();
        for (int idx = threadIdx.x; idx < kRows * N; idx += kThreads) {
            const int r = idx / N, n = idx % N;
            bts[idx] = (s0 + r < len) ? to_f32(B[((b * seqlen + t0 + s0 + r) * G + g) * N + n])
                                      : 0.f;
        }
        for (int idx = threadIdx.x; idx < kRows * P; idx += kThreads) {
            const int r = idx / P, p = idx % P;
            xts[idx] = (s0 + r < len) ? to_f32(x[((b * seqlen + t0 + s0 + r) * H + h) * P + p])
                                      : 0.f;
        }
        __syncthreads();
        for (int idx = threadIdx.x; idx < kRows * kRows; idx += kThreads) {
            const int t = idx / kRows, i = idx % kRows;
            const int tg = r0 + t, ig = s0 + i;  // rows within the chunk
            float v = 0.f;
            if (ig <= tg && ig < len && tg < len) {
                float dot = 0.f;
                for (int n = 0; n < N; ++n) dot = fmaf(cts[t * N + n], bts[i * N + n], dot);
                v = dot * __expf(csk[tg] - csk[ig]) * dt[(b * seqlen + t0 + ig) * H + h];
            }
            gts[t * (kRows + 1) + i] = v;
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < kMaxOut; ++j) {
            const int o = threadIdx.x + j * kThreads;
            if (o < nout) {
                const int t = o / P, p = o % P;
                float a = acc[j];
                for (int i = 0; i < kRows; ++i)
                    a = fmaf(gts[t * (kRows + 1) + i], xts[i * P + p], a);
                acc[j] = a;
            }
        }
    }

    const float Dh = D[h];
#pragma unroll
    for (int j = 0; j < kMaxOut; ++j) {
        const int o = threadIdx.x + j * kThreads;
        if (o < nout) {
            const int t = o / P, p = o % P;
            if (t < rows) {
                const int64_t off = ((b * seqlen + t0 + r0 + t) * H + h) * P + p;
                const float v = acc[j] + Dh * to_f32(x[off]);
                y[off] = from_f32<T>(z ? v * silu(to_f32(z[off])) : v);
            }
        }
    }
}

}  // namespace

cudaError_t launch_chunk_state_simt(bool is_bf16, const void *x, const float *dt,
                                    const void *B, const float *cs, float *states,
                                    int64_t batch, int64_t seqlen, int H, int G, int P, int N,
                                    int Q, int64_t nchunks, cudaStream_t st)
{
    const unsigned grid = (unsigned)(H * nchunks * batch);
    const size_t smem = (size_t)(kRows * P + kRows * N + kRows) * sizeof(float);
    cudaError_t e;
    if (is_bf16) {
        auto kern = chunk_state_simt_kernel<bf16>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<grid, kThreads, smem, st>>>((const bf16 *)x, dt, (const bf16 *)B, cs, states,
                                           seqlen, H, G, P, N, Q, nchunks);
    } else {
        auto kern = chunk_state_simt_kernel<float>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<grid, kThreads, smem, st>>>((const float *)x, dt, (const float *)B, cs, states,
                                           seqlen, H, G, P, N, Q, nchunks);
    }
    return cudaGetLastError();
}

cudaError_t launch_chunk_scan_simt(bool is_bf16, const void *x, const float *dt,
                                   const void *B, const void *C, const float *cs,
                                   const float *hin, const float *D, void *y, int64_t batch,
                                   int64_t seqlen, int H, int G, int P, int N, int Q,
                                   int64_t nchunks, cudaStream_t st, const void *z)
{
    const unsigned grid = (unsigned)(((Q + kRows - 1) / kRows) * H * batch * nchunks);
    const size_t smem = (size_t)(2 * kRows * N + kRows * P + kRows * (kRows + 1) +
                                 P * (kRows + 1)) * sizeof(float);
    cudaError_t e = cudaSuccess;
    if (is_bf16) {
        auto kern = chunk_scan_simt_kernel<bf16>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<grid, kThreads, smem, st>>>((const bf16 *)x, dt, (const bf16 *)B,
                                           (const bf16 *)C, cs, hin, D, (bf16 *)y, seqlen, H, G,
                                           P, N, Q, nchunks, (const bf16 *)z);
    } else {
        auto kern = chunk_scan_simt_kernel<float>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<grid, kThreads, smem, st>>>((const float *)x, dt, (const float *)B,
                                           (const float *)C, cs, hin, D, (float *)y, seqlen, H,
                                           G, P, N, Q, nchunks, (const float *)z);
    }
    return cudaGetLastError();
}

}  // namespace ssd
