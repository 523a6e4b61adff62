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
// Programmatic dependent launch: over chains of at most this many chunks the kernel lets the
// chunk scan launch at its start, so that the scan's set-up (barriers, TMEM, its first C and B
// tiles and C B^T) overlaps the recurrence; over longer chains only at its end, because the
// scan's early CTAs then slowed the recurrence itself (256 chunks at L = 65536: 25 us).
constexpr int64_t kEarlyTriggerChunks = 64;

template <bool kBf16Out>
__global__ void __launch_bounds__(kThreads)
state_passing_kernel(float *__restrict__ states, const float *__restrict__ cs,
                     const float *__restrict__ init, float *__restrict__ final_state,
                     bf16 *__restrict__ hin, int H, int PN, int Q, int64_t nchunks,
                     const int32_t *__restrict__ cstart, bool trigger_early)
{
    griddep_wait();   // the chunk states come from the previous kernel
    if (trigger_early) griddep_launch_dependents();
    const int nblk = (PN / 4 + kThreads - 1) / kThreads;
    const int64_t v = (blockIdx.x % nblk) * (int64_t)kThreads + threadIdx.x;  // float4 index
    // b: batch row, or the packed sequence when cstart is given (its chunks are
    // [cstart[b], cstart[b + 1]) of the single workspace row)
    const int64_t h = (blockIdx.x / nblk) % H, b = blockIdx.x / nblk / H;
    if (v * 4 >= PN) return;
    const int64_t kbeg = cstart ? cstart[b] : 0;
    const int64_t kend = cstart ? cstart[b + 1] : nchunks;
    const int64_t rb = cstart ? 0 : b;   // workspace batch row

    float4 hs = make_float4(0.f, 0.f, 0.f, 0.f);
    if (init) hs = *reinterpret_cast<const float4 *>(init + (b * H + h) * PN + v * 4);

    for (int64_t k0 = kbeg; k0 < kend; k0 += kGroup) {
        float4 s[kGroup];
        float decay[kGroup];
#pragma unroll
        for (int j = 0; j < kGroup; ++j) {
            const int64_t k = k0 + j;
            if (k < kend) {
                const int64_t row = (rb * nchunks + k) * H + h;
                s[j] = __ldcs(reinterpret_cast<const float4 *>(states + row * PN + v * 4));
                decay[j] = cs[row * Q + Q - 1];
            }
        }
#pragma unroll
        for (int j = 0; j < kGroup; ++j) {
            const int64_t k = k0 + j;
            if (k < kend) {
                const int64_t off = ((rb * nchunks + k) * H + h) * PN + v * 4;
                if (kBf16Out) {
                    // tensor-core path (P = 64, N = 128): the swizzled block layout
                    const int e = (int)(v * 4);
                    const int64_t hoff =
                        ((rb * nchunks + k) * H + h) * PN + hin_swizzled_offset(e >> 7, e & 127);
                    __nv_bfloat162 lo = __floats2bfloat162_rn(hs.x, hs.y);
                    __nv_bfloat162 hi = __floats2bfloat162_rn(hs.z, hs.w);
                    uint2 packed;
                    packed.x = *reinterpret_cast<uint32_t *>(&lo);
                    packed.y = *reinterpret_cast<uint32_t *>(&hi);
                    __stcs(reinterpret_cast<uint2 *>(hin + hoff), packed);
                } else {
                    __stcs(reinterpret_cast<float4 *>(states + off), hs);
                }
                const float a = __expf(decay[j]);
                hs.x = fmaf(a, hs.x, s[j].x);
                hs.y = fmaf(a, hs.y, s[j].y);
                hs.z = fmaf(a, hs.z, s[j].z);
                hs.w = fmaf(a, hs.w, s[j].w);
            }
        }
    }
    if (final_state)
        *reinterpret_cast<float4 *>(final_state + (b * H + h) * PN + v * 4) = hs;
    if (!trigger_early) griddep_launch_dependents();
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
                      kThreads, 0, st, states, cs, init, final_state, hin_bf16, H, PN, Q, nchunks,
                      none, nchunks <= kEarlyTriggerChunks);
}

cudaError_t launch_state_passing_varlen(float *states, const float *cs, const float *init,
                                        float *final_state, bf16 *hin_bf16,
                                        const int32_t *cstart, int nseq, int H, int P, int N,
                                        int Q, int64_t nchunks, cudaStream_t st)
{
    const int PN = P * N;
    const unsigned grid = (unsigned)(((PN / 4 + kThreads - 1) / kThreads) * H * (int64_t)nseq);
    // packed sequences: chains of one sequence each, short next to the packed total
    return launch_pdl(hin_bf16 ? state_passing_kernel<true> : state_passing_kernel<false>, grid,
                      kThreads, 0, st, states, cs, init, final_state, hin_bf16, H, PN, Q, nchunks,
                      cstart, true);
}

}  // namespace ssd
