// Backward pass of the scan: the elementwise and reduction kernels around its three scans.
//
// Reverse-mode differentiation of the recurrence h_t = a_t h_{t-1} + dt_t x_t B_t^T,
// y_t = h_t C_t + D x_t (a_t = exp(dt_t A_h)) gives an adjoint state g_t = dy_t C_t^T +
// a_{t+1} g_{t+1} that runs backwards in time (mohakchugh.is-a.dev "Mamba-2", The Duality: the
// mixing matrix is semiseparable, and so is its transpose, which propagates the gradients).  All
// three contractions of the backward are therefore scans of the same form as the forward one:
//
//   g_t B_t          = the forward scan of the time-reversed sequence with x' = dy, B' = C,
//                      C' = B, unit input weights and each decay shifted by one token, started
//                      from dfinal (tensor cores);  dx_t = D dy_t + dt_t g_t B_t
//   dB_t (per head)  = dt_t times the output of the reversed scan with x' = C, B' = dy, C' = x,
//                      unit weights, started from dfinal^T
//   dC_t (per head)  = the output of the forward scan with x' = B, B' = x, C' = dy, weights dt,
//                      started from h0^T
//
// (the last two have head dimension N and state dimension P, run on CUDA cores in float32 --
// bwd_scan.cu -- and are summed over the heads of a group).  The decay gradient uses the identity, for the global
// log-decay cumsum Lcs_k,
//     dL/dLcs_k = <dy_k, y_k - D x_k> - dt_k <x_k, g_k B_k>  (+ <dfinal, final> at k = L-1)
// followed by a reverse cumsum: dL/d(dt_k A_h) = sum_{j >= k} dL/dLcs_j (which equals
// exp(dt_k A_h) <g_k, h_{k-1}>, a quantity of the size of one term); then
// ddt_k = <x_k, g_k B_k> + A_h dL/d(dt_k A_h), dA_h = sum_k dt_k dL/d(dt_k A_h).  The reverse
// cumsum telescopes, so its terms must be accurate to well below the result: both dot products
// are taken from the float32 scans, <dy_k, y_k - D x_k> = <h_k^T dy_k, C_k> from the dC scan's
// per-head output and <x_k, g_k B_k> = <g_k^T x_k, B_k> from the dB scan's (a bf16 y or g B
// would leave errors of 1e-2 relative in ddt and 1e-1 in dA after the cumsum).
#include "common.cuh"

namespace ssd {
namespace {

// out[b][t][r][:] = in[b][src][r / (rows_out / rows_in)][:] (src = L-1-t when `reverse`), rows of
// E8 16-byte vectors, one vector per thread.
__global__ void gather8_kernel(const uint4 *__restrict__ in, uint4 *__restrict__ out,
                               int64_t batch, int64_t L, int rows_in, int rows_out, int E8,
                               bool reverse)
{
    const int64_t n = batch * L * rows_out * E8;
    const int rep = rows_out / rows_in;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int e = (int)(i % E8);
        int64_t r = i / E8;
        const int ro = (int)(r % rows_out);
        r /= rows_out;
        const int64_t t = r % L, b = r / L;
        const int64_t src = reverse ? L - 1 - t : t;
        out[i] = in[((b * L + src) * rows_in + ro / rep) * E8 + e];
    }
}

__global__ void reverse_shift_dt_kernel(const float *__restrict__ dt, float *__restrict__ out,
                                        int64_t batch, int64_t L, int H)
{
    const int64_t n = batch * L * H;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int h = (int)(i % H);
        const int64_t t = (i / H) % L, b = i / H / L;
        out[i] = t == 0 ? 0.f : dt[(b * L + (L - t)) * H + h];
    }
}

__global__ void fill_kernel(float *__restrict__ out, float v, int64_t n)
{
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        out[i] = v;
}

// Eight lanes per (b, t, h) row of P = 64 channels, 16 bytes of each bf16 input per lane: dx,
// <x, dy>, and the decay-gradient term q.
constexpr int kTokLanes = 8;

__global__ void bwd_tokens_kernel(const bf16 *__restrict__ x, const bf16 *__restrict__ dy,
                                  const float *__restrict__ dt, const float *__restrict__ D,
                                  const bf16 *__restrict__ gb_rev,
                                  const float *__restrict__ ydot,
                                  const float *__restrict__ ddt_in,
                                  const float *__restrict__ fdot, float *__restrict__ dx,
                                  float *__restrict__ q, float *__restrict__ xdy, int64_t batch,
                                  int64_t L, int H)
{
    constexpr int P = kTokLanes * 8;
    const int64_t gid = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    const int64_t w = gid / kTokLanes;   // (b, t, h) row
    const int part = (int)(gid % kTokLanes);
    const bool ok = w < batch * L * H;
    const int h = (int)(w % H);
    const int64_t t = (w / H) % L, b = w / H / L;
    float sd = 0.f, sf = 0.f, dth = 0.f;
    if (ok) {
        dth = dt[w];
        const int64_t row = w * P + part * 8;
        const int64_t rrow = ((b * L + (L - 1 - t)) * H + h) * P + part * 8;
        float xv[8], dyv[8], gv[8];
        const uint4 rx = *reinterpret_cast<const uint4 *>(x + row);
        const uint4 rd = *reinterpret_cast<const uint4 *>(dy + row);
        const uint4 rg = *reinterpret_cast<const uint4 *>(gb_rev + rrow);
        const bf16 *px = reinterpret_cast<const bf16 *>(&rx);
        const bf16 *pd = reinterpret_cast<const bf16 *>(&rd);
        const bf16 *pg = reinterpret_cast<const bf16 *>(&rg);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            xv[i] = __bfloat162float(px[i]);
            dyv[i] = __bfloat162float(pd[i]);
            gv[i] = __bfloat162float(pg[i]);
            sd = fmaf(dyv[i], xv[i], sd);
        }
        const float Dh = D[h];
        float o[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = fmaf(Dh, dyv[i], dth * gv[i]);
        *reinterpret_cast<float4 *>(dx + row) = make_float4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<float4 *>(dx + row + 4) = make_float4(o[4], o[5], o[6], o[7]);
        // the final state also depends on the last log-decay cumsum: + <dfinal, final>
        if (fdot && t == L - 1) sf = fdot[b * H + h];
    }
#pragma unroll
    for (int o = 1; o < kTokLanes; o <<= 1) sd += __shfl_xor_sync(0xffffffffu, sd, o);
    if (ok && part == 0) {
        q[w] = ydot[w] - dth * ddt_in[w] + sf;
        xdy[w] = sd;
    }
}

// One block per (b, h): out[b][h] = <a, c> over the (b, h) state, both in the same layout.
__global__ void __launch_bounds__(256)
state_dot_kernel(const float *__restrict__ a, const float *__restrict__ c, float *__restrict__ out,
                 int PN)
{
    __shared__ float red[8];
    const float4 *a4 = reinterpret_cast<const float4 *>(a + blockIdx.x * (int64_t)PN);
    const float4 *c4 = reinterpret_cast<const float4 *>(c + blockIdx.x * (int64_t)PN);
    float s = 0.f;
    for (int i = threadIdx.x; i < PN / 4; i += 256) {
        const float4 u = a4[i], v = c4[i];
        s = fmaf(u.x, v.x, fmaf(u.y, v.y, fmaf(u.z, v.z, fmaf(u.w, v.w, s))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = 0.f;
        for (int j = 0; j < 8; ++j) t += red[j];
        out[blockIdx.x] = t;
    }
}

// One block per (b, h): the reverse cumsum of q over t (each thread a contiguous segment, the
// segments' totals combined by a block-wide suffix scan), ddt, and the (b, h) partial sums of dA
// and dD, written to part[0][b][h] and part[1][b][h] (summed over the batch in a fixed order by
// batch_sum_kernel, so the result does not depend on the order the blocks run in).
constexpr int kDecayThreads = 256;

__global__ void __launch_bounds__(kDecayThreads)
bwd_decay_kernel(const float *__restrict__ q, const float *__restrict__ ddt_in,
                 const float *__restrict__ dt, const float *__restrict__ A,
                 const float *__restrict__ xdy, float *__restrict__ ddt, float *__restrict__ part,
                 int64_t batch, int64_t L, int H)
{
    __shared__ float wsum[kDecayThreads / 32];
    __shared__ float red[2][kDecayThreads / 32];
    const int h = (int)(blockIdx.x % H);
    const int64_t b = blockIdx.x / H;
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
    const int64_t per = (L + kDecayThreads - 1) / kDecayThreads;
    const int64_t ta = min(L, threadIdx.x * per), te = min(L, ta + per);
    const int64_t base = b * L * H + h;
    float tot = 0.f;
    for (int64_t t = ta; t < te; ++t) tot += q[base + t * H];
    // exclusive suffix sum of the threads' totals: within the warp, then over the warps
    float v = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_down_sync(0xffffffffu, v, o);
        if (lane + o < 32) v += u;
    }
    if (lane == 0) wsum[warp] = v;   // the warp's total
    __syncthreads();
    float carry = v - tot;           // later threads of this warp
    for (int j = warp + 1; j < kDecayThreads / 32; ++j) carry += wsum[j];
    const float Ah = A[h];
    float sa = 0.f, sd = 0.f;
    for (int64_t t = te - 1; t >= ta; --t) {
        const int64_t i = base + t * H;
        carry += q[i];
        ddt[i] = ddt_in[i] + Ah * carry;
        sa = fmaf(dt[i], carry, sa);
        sd += xdy[i];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        sa += __shfl_xor_sync(0xffffffffu, sa, o);
        sd += __shfl_xor_sync(0xffffffffu, sd, o);
    }
    if (lane == 0) {
        red[0][warp] = sa;
        red[1][warp] = sd;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float a = 0.f, d = 0.f;
        for (int j = 0; j < kDecayThreads / 32; ++j) {
            a += red[0][j];
            d += red[1][j];
        }
        part[b * H + h] = a;
        part[(batch + b) * H + h] = d;
    }
}

// dA[h] = sum_b part[0][b][h], dD[h] = sum_b part[1][b][h], in batch order.
__global__ void batch_sum_kernel(const float *__restrict__ part, float *__restrict__ dA,
                                 float *__restrict__ dD, int64_t batch, int H)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= 2 * H) return;
    const int h = i % H, which = i / H;
    float s = 0.f;
    for (int64_t b = 0; b < batch; ++b) s += part[(which * batch + b) * H + h];
    (which ? dD : dA)[h] = s;
}

__global__ void group_sum_kernel(const float *__restrict__ in, const float *__restrict__ w,
                                 float *__restrict__ out, int64_t batch, int64_t L, int H, int G,
                                 int N, bool reverse)
{
    const int64_t n = batch * L * G * N;
    const int hpg = H / G;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int e = (int)(i % N);
        const int g = (int)((i / N) % G);
        const int64_t t = (i / N / G) % L, b = i / N / G / L;
        const int64_t src = reverse ? L - 1 - t : t;
        float s = 0.f;
        for (int j = 0; j < hpg; ++j) {
            const int h = g * hpg + j;
            const float wv = w ? w[(b * L + t) * H + h] : 1.f;
            s = fmaf(wv, in[((b * L + src) * H + h) * N + e], s);
        }
        out[i] = s;
    }
}

__global__ void scale_init_grad_kernel(const float *__restrict__ F, const float *__restrict__ dt,
                                       const float *__restrict__ A, float *__restrict__ out,
                                       int64_t batch, int64_t L, int H, int PN)
{
    const int64_t n = batch * H * PN;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t bh = i / PN;
        const int h = (int)(bh % H);
        const int64_t b = bh / H;
        out[i] = __expf(dt[(b * L) * H + h] * A[h]) * F[i];
    }
}

unsigned grid_for(int64_t n) { return (unsigned)std::min<int64_t>((n + 255) / 256, 148 * 32); }

}  // namespace

cudaError_t launch_gather(const bf16 *in, bf16 *out, int64_t batch, int64_t L, int rows_in,
                          int rows_out, int E, bool reverse, cudaStream_t st)
{
    if (E % 8 != 0 || rows_in <= 0 || rows_out % rows_in != 0) return cudaErrorInvalidValue;
    const int64_t n = batch * L * rows_out * (E / 8);
    if (n == 0) return cudaSuccess;
    gather8_kernel<<<grid_for(n), 256, 0, st>>>(reinterpret_cast<const uint4 *>(in),
                                               reinterpret_cast<uint4 *>(out), batch, L, rows_in,
                                               rows_out, E / 8, reverse);
    return cudaGetLastError();
}

cudaError_t launch_reverse_shift_dt(const float *dt, float *out, int64_t batch, int64_t L, int H,
                                   cudaStream_t st)
{
    const int64_t n = batch * L * H;
    if (n == 0) return cudaSuccess;
    reverse_shift_dt_kernel<<<grid_for(n), 256, 0, st>>>(dt, out, batch, L, H);
    return cudaGetLastError();
}

cudaError_t launch_fill(float *out, float value, int64_t n, cudaStream_t st)
{
    if (n == 0) return cudaSuccess;
    fill_kernel<<<grid_for(n), 256, 0, st>>>(out, value, n);
    return cudaGetLastError();
}

cudaError_t launch_state_dot(const float *a, const float *c, float *out, int64_t mats, int PN,
                             cudaStream_t st)
{
    if (PN % 4 != 0) return cudaErrorInvalidValue;
    if (mats == 0) return cudaSuccess;
    state_dot_kernel<<<(unsigned)mats, 256, 0, st>>>(a, c, out, PN);
    return cudaGetLastError();
}

cudaError_t launch_bwd_tokens(const bf16 *x, const bf16 *dy, const float *dt, const float *D,
                              const bf16 *gb_rev, const float *ydot, const float *ddt_in,
                              const float *fdot, float *dx, float *q, float *xdy, int64_t batch,
                              int64_t L, int H, int P, cudaStream_t st)
{
    if (P != kTokLanes * 8) return cudaErrorInvalidValue;
    const int64_t threads = batch * L * H * kTokLanes;
    if (threads == 0) return cudaSuccess;
    bwd_tokens_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(
        x, dy, dt, D, gb_rev, ydot, ddt_in, fdot, dx, q, xdy, batch, L, H);
    return cudaGetLastError();
}

cudaError_t launch_bwd_decay(const float *q, const float *ddt_in, const float *dt,
                             const float *A, const float *xdy, float *ddt, float *dA, float *dD,
                             float *part, int64_t batch, int64_t L, int H, cudaStream_t st)
{
    const int64_t n = batch * H;
    if (n == 0 || L == 0) {
        cudaError_t e = cudaMemsetAsync(dA, 0, H * sizeof(float), st);
        if (e == cudaSuccess) e = cudaMemsetAsync(dD, 0, H * sizeof(float), st);
        return e;
    }
    bwd_decay_kernel<<<(unsigned)n, kDecayThreads, 0, st>>>(q, ddt_in, dt, A, xdy, ddt, part,
                                                           batch, L, H);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    batch_sum_kernel<<<(2 * H + 127) / 128, 128, 0, st>>>(part, dA, dD, batch, H);
    return cudaGetLastError();
}

cudaError_t launch_group_sum(const float *in, const float *w, float *out, int64_t batch,
                             int64_t L, int H, int G, int N, bool reverse, cudaStream_t st)
{
    const int64_t n = batch * L * G * N;
    if (n == 0) return cudaSuccess;
    group_sum_kernel<<<grid_for(n), 256, 0, st>>>(in, w, out, batch, L, H, G, N, reverse);
    return cudaGetLastError();
}

cudaError_t launch_scale_init_grad(const float *F, const float *dt, const float *A, float *out,
                                   int64_t batch, int64_t L, int H, int PN, cudaStream_t st)
{
    const int64_t n = batch * H * PN;
    if (n == 0) return cudaSuccess;
    scale_init_grad_kernel<<<grid_for(n), 256, 0, st>>>(F, dt, A, out, batch, L, H, PN);
    return cudaGetLastError();
}

}  // namespace ssd
