// Sequence parallelism: a long sequence split into contiguous segments, one per GPU.
//
// The state is carried across segments exactly as across chunks (mohakchugh.is-a.dev
// "Mamba-2", Block Decomposition: across blocks the state is propagated sequentially; the same
// page's note that the recurrence splits over devices with one exchange of states).  Every
// segment first runs its chunk states and a state passing from a zero initial state, which gives
// its local final state h_loc and its total log-decay (the sum of dt A_h over its tokens).  After
// the caller has exchanged those (an all-gather over the ranks), segment r's true initial state
// is
//     h_in(r) = sum_{q < r} exp(sum_{q < s < r} logdec_s) h_loc(q) + exp(sum_{s < r} logdec_s) h0
// (h0 the sequence's initial state), because the recurrence is linear in its initial state and
// the decay over a segment is the product of its per-token decays.  The segment then reruns
// state passing from h_in(r) and its chunk scan.
//
// Two small kernels live here: the per-(batch, head) segment log-decay (a sum over the chunks'
// last cumsum entries) and the combine above (elementwise over the state, a loop over ranks).
#include "common.cuh"

namespace ssd {
namespace {

__global__ void segment_log_decay_kernel(const float *__restrict__ cs, float *__restrict__ out,
                                         int64_t batch, int H, int Q, int64_t nchunks)
{
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;   // b * H + h
    if (i >= batch * H) return;
    const int64_t b = i / H, h = i % H;
    float s = 0.f;
    for (int64_t k = 0; k < nchunks; ++k) s += cs[((b * nchunks + k) * H + h) * Q + Q - 1];
    out[i] = s;
}

// One thread per float4 of the (batch, head, P, N) state.
__global__ void seqpar_combine_kernel(const float *__restrict__ h_loc_all,
                                      const float *__restrict__ logdec_all,
                                      const float *__restrict__ init, float *__restrict__ h_in,
                                      int nranks, int rank, int64_t BH, int PN)
{
    const int64_t v = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;   // float4 index
    const int64_t n4 = BH * PN / 4;
    if (v >= n4) return;
    const int64_t bh = v * 4 / PN;
    // walk the earlier segments from the first: acc <- exp(logdec_q) acc + h_loc(q)
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (init) acc = reinterpret_cast<const float4 *>(init)[v];
    for (int q = 0; q < rank; ++q) {
        const float a = __expf(logdec_all[q * BH + bh]);
        const float4 hl = reinterpret_cast<const float4 *>(h_loc_all + q * BH * PN)[v];
        acc.x = fmaf(a, acc.x, hl.x);
        acc.y = fmaf(a, acc.y, hl.y);
        acc.z = fmaf(a, acc.z, hl.z);
        acc.w = fmaf(a, acc.w, hl.w);
    }
    reinterpret_cast<float4 *>(h_in)[v] = acc;
}

}  // namespace

cudaError_t launch_segment_log_decay(const float *cs, float *out, int64_t batch, int H, int Q,
                                     int64_t nchunks, cudaStream_t st)
{
    const int64_t n = batch * H;
    if (n == 0) return cudaSuccess;
    segment_log_decay_kernel<<<(unsigned)((n + 127) / 128), 128, 0, st>>>(cs, out, batch, H, Q,
                                                                         nchunks);
    return cudaGetLastError();
}

cudaError_t launch_seqpar_combine(const float *h_loc_all, const float *logdec_all,
                                  const float *init, float *h_in, int nranks, int rank,
                                  int64_t BH, int PN, cudaStream_t st)
{
    const int64_t n4 = BH * PN / 4;
    if (n4 == 0) return cudaSuccess;
    seqpar_combine_kernel<<<(unsigned)((n4 + 255) / 256), 256, 0, st>>>(
        h_loc_all, logdec_all, init, h_in, nranks, rank, BH, PN);
    return cudaGetLastError();
}

}  // namespace ssd
