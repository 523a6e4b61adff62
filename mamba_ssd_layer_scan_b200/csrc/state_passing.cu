// Inter-chunk state passing: the linear recurrence across chunks.
//
//     h_in[0] = h0 (or 0);   h_in[k+1] = exp(cs_k[Q-1]) * h_in[k] + S_k
//
// S_k is chunk k's own contribution to the state at its end (from the chunk-state kernel) and
// exp(cs_k[Q-1]) the chunk's total decay; h_in[k] is the state entering chunk k, which the
// intra-chunk kernel turns into the off-chunk output term, and h_in[c] is the final state
// (mohakchugh.is-a.dev "Mamba-2", Block Decomposition: across blocks the state is propagated
// sequentially; ql.gl, The Core of SSD: a summarized recurrent state is passed between blocks).
//
// HBM-bound: every element of S is read once and every h_in written once.  Each thread owns
// four consecutive state elements (one 16-byte vector) of one (batch, head) and walks the
// chunks in order, issuing the loads of a group of chunks before consuming them so that
// several 16-byte loads per thread are in flight.
#include "common.cuh"

namespace ssd {
namespace {

constexpr int kThreads = 128;
constexpr int kGroup = 8;  // chunks whose loads are issued together

// kBf16Out (tensor-core path): the chunk states are [N][P] per (batch, chunk, head) and the
// entering states go to hin in the chunk scan's operand layout; otherwise the states are [P][N]
// and are overwritten in place by the entering states.  init and final_state are [P][N].
template <bool kBf16Out>
__global__ void __launch_bounds__(kThreads)
state_passing_kernel(float *__restrict__ states, const float *__restrict__ cs,
                     const float *__restrict__ init, float *__restrict__ final_state,
                     bf16 *__restrict__ hin, int H, int P, int N, int Q, int64_t nchunks,
                     const int32_t *__restrict__ cstart)
{
    griddep_wait();   // the chunk states come from the previous kernel
    griddep_launch_dependents();
    const int PN = P * N;
    const int nblk = (PN / 4 + kThreads - 1) / kThreads;
    const int64_t v = (blockIdx.x % nblk) * (int64_t)kThreads + threadIdx.x;  // float4 index
    // b: batch row, or the packed sequence when cstart is given (its chunks are
    // [cstart[b], cstart[b + 1]) of the single workspace row)
    const int64_t h = (blockIdx.x / nblk) % H, b = blockIdx.x / nblk / H;
    if (v * 4 >= PN) return;
    const int64_t kbeg = cstart ? cstart[b] : 0;
    const int64_t kend = cstart ? cstart[b + 1] : nchunks;
    const int64_t rb = cstart ? 0 : b;   // workspace batch row
    // the four elements of this thread in the caller's [P][N] layout: (p0 + i, n) for the
    // transposed tensor-core states, (p0, n + i) otherwise
    const int e = (int)(v * 4);
    const int n_t = e / P, p_t = e % P;
    const int64_t ubase = (b * H + h) * (int64_t)PN;

    float4 hs = make_float4(0.f, 0.f, 0.f, 0.f);
    if (init) {
        if (kBf16Out) {
            const float *ip = init + ubase + (int64_t)p_t * N + n_t;
            hs = make_float4(ip[0], ip[N], ip[2 * N], ip[3 * N]);
        } else {
            hs = *reinterpret_cast<const float4 *>(init + ubase + e);
        }
    }

    for (int64_t k0 = kbeg; k0 < kend; k0 += kGroup) {
        float4 s[kGroup];
        float decay[kGroup];
#pragma unroll
        for (int j = 0; j < kGroup; ++j) {
            const int64_t k = k0 + j;
            if (k < kend) {
                const int64_t row = (rb * nchunks + k) * H + h;
                s[j] = __ldcs(reinterpret_cast<const float4 *>(states + row * PN + e));
                decay[j] = cs[row * Q + Q - 1];
            }
        }
#pragma unroll
        for (int j = 0; j < kGroup; ++j) {
            const int64_t k = k0 + j;
            if (k < kend) {
                const int64_t off = ((rb * nchunks + k) * H + h) * PN;
                if (kBf16Out) {
                    // tensor-core path (P = 64, N = 128): four consecutive p of row n of the
                    // swizzled operand block, one 8-byte store
                    __nv_bfloat162 lo = __floats2bfloat162_rn(hs.x, hs.y);
                    __nv_bfloat162 hi = __floats2bfloat162_rn(hs.z, hs.w);
                    uint2 packed;
                    packed.x = *reinterpret_cast<uint32_t *>(&lo);
                    packed.y = *reinterpret_cast<uint32_t *>(&hi);
                    __stcs(reinterpret_cast<uint2 *>(hin + off + hin_swizzled_offset(p_t, n_t)),
                           packed);
                } else {
                    __stcs(reinterpret_cast<float4 *>(states + off + e), hs);
                }
                const float a = __expf(decay[j]);
                hs.x = fmaf(a, hs.x, s[j].x);
                hs.y = fmaf(a, hs.y, s[j].y);
                hs.z = fmaf(a, hs.z, s[j].z);
                hs.w = fmaf(a, hs.w, s[j].w);
            }
        }
    }
    if (final_state) {
        if (kBf16Out) {
            float *fp = final_state + ubase + (int64_t)p_t * N + n_t;
            fp[0] = hs.x;
            fp[N] = hs.y;
            fp[2 * N] = hs.z;
            fp[3 * N] = hs.w;
        } else {
            *reinterpret_cast<float4 *>(final_state + ubase + e) = hs;
        }
    }
}

}  // namespace

cudaError_t launch_state_passing(float *states, const float *cs, const float *init,
                                 float *final_state, bf16 *hin_bf16, int64_t batch, int H,
                                 int P, int N, int Q, int64_t nchunks, cudaStream_t st)
{
    const int PN = P * N;  // multiple of 32 (N is)
    const unsigned grid = (unsigned)(((PN / 4 + kThreads - 1) / kThreads) * H * batch);
    const int32_t *none = nullptr;
    return launch_pdl(hin_bf16 ? state_passing_kernel<true> : state_passing_kernel<false>, grid,
                      kThreads, 0, st, states, cs, init, final_state, hin_bf16, H, P, N, Q, nchunks,
                      none);
}

cudaError_t launch_state_passing_varlen(float *states, const float *cs, const float *init,
                                        float *final_state, bf16 *hin_bf16,
                                        const int32_t *cstart, int nseq, int H, int P, int N,
                                        int Q, int64_t nchunks, cudaStream_t st)
{
    const int PN = P * N;
    const unsigned grid = (unsigned)(((PN / 4 + kThreads - 1) / kThreads) * H * (int64_t)nseq);
    return launch_pdl(hin_bf16 ? state_passing_kernel<true> : state_passing_kernel<false>, grid,
                      kThreads, 0, st, states, cs, init, final_state, hin_bf16, H, P, N, Q, nchunks,
                      cstart);
}

}  // namespace ssd
