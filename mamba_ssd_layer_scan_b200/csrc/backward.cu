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
//   dB_t (per head)  = dt_t x (reversed scan with x' = C, B' = dy, C' = x, from dfinal^T)
//   dC_t (per head)  = the forward scan with x' = B, B' = x, C' = dy, weights dt, from h0^T
//
// (the last two have head dimension N and state dimension P, run on CUDA cores in float32, and
// are summed over the heads of a group).  The decay gradient uses the identity, for the global
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

template <typename TI, typename TO>
__global__ void gather_kernel(const TI *__restrict__ in, TO *__restrict__ out, int64_t batch,
                              int64_t L, int rows_in, int rows_out, int E, bool reverse)
{
    const int64_t n = batch * L * rows_out * E;
    const int rep = rows_out / rows_in;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int e = (int)(i % E);
        int64_t r = i / E;
        const int ro = (int)(r % rows_out);
        r /= rows_out;
        const int64_t t = r % L, b = r / L;
        const int64_t src = reverse ? L - 1 - t : t;
        out[i] = from_f32<TO>(to_f32(in[((b * L + src) * rows_in + ro / rep) * E + e]));
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

__global__ void transpose_kernel(const float *__restrict__ in, float *__restrict__ out,
                                 int64_t mats, int rows, int cols)
{
    const int64_t n = mats * rows * cols;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int c = (int)(i % cols);
        const int r = (int)((i / cols) % rows);
        const int64_t m = i / cols / rows;
        out[(m * cols + c) * rows + r] = in[i];
    }
}

// One warp per (b, t, h): dx over the P channels, and the decay-gradient term q.
__global__ void bwd_tokens_kernel(const bf16 *__restrict__ dy, const float *__restrict__ dt,
                                  const float *__restrict__ D, const bf16 *__restrict__ gb_rev,
                                  const float *__restrict__ ydot,
                                  const float *__restrict__ ddt_in,
                                  const float *__restrict__ dfinal,
                                  const float *__restrict__ fin_t, float *__restrict__ dx,
                                  float *__restrict__ q, int64_t batch, int64_t L, int H, int P,
                                  int N)
{
    const int lane = threadIdx.x % 32;
    const int64_t w = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) / 32;
    if (w >= batch * L * H) return;
    const int h = (int)(w % H);
    const int64_t t = (w / H) % L, b = w / H / L;
    const int64_t row = w * P;                                   // (b, t, h) row of dy / dx
    const int64_t rrow = ((b * L + (L - 1 - t)) * H + h) * P;    // reversed row of gb
    const float dth = dt[w];
    for (int p = lane; p < P; p += 32)
        dx[row + p] = D[h] * to_f32(dy[row + p]) + dth * to_f32(gb_rev[rrow + p]);
    float sf = 0.f;
    if (dfinal && t == L - 1) {   // the final state also depends on the last log-decay cumsum
        // fin_t is the final state transposed, (n, p)
        const int64_t base = (b * H + h) * (int64_t)P * N;
        for (int i = lane; i < P * N; i += 32)
            sf = fmaf(dfinal[base + i], fin_t[base + (int64_t)(i % N) * P + i / N], sf);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sf += __shfl_xor_sync(0xffffffffu, sf, o);
    }
    if (lane == 0) q[w] = ydot[w] - dth * ddt_in[w] + sf;
}

// One warp per (b, t, h): out = <in[b][src(t)][h][:], v[b][t][g(h)][:]> over N (src = L-1-t
// when `reverse`).
__global__ void head_dot_kernel(const float *__restrict__ in, const bf16 *__restrict__ v,
                                float *__restrict__ out, int64_t batch, int64_t L, int H, int G,
                                int N, bool reverse)
{
    const int lane = threadIdx.x % 32;
    const int64_t w = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) / 32;
    if (w >= batch * L * H) return;
    const int h = (int)(w % H);
    const int64_t t = (w / H) % L, b = w / H / L;
    const int64_t src = reverse ? L - 1 - t : t;
    const float *a = in + ((b * L + src) * H + h) * (int64_t)N;
    const bf16 *c = v + ((b * L + t) * G + h / (H / G)) * (int64_t)N;
    float s = 0.f;
    for (int n = lane; n < N; n += 32) s = fmaf(a[n], to_f32(c[n]), s);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) out[w] = s;
}

// One warp per (b, h): reverse cumsum of q over t in tiles of 32; ddt and the per-(b, h)
// partial sums of dA and dD (atomically added per head).
__global__ void bwd_decay_kernel(const float *__restrict__ q, const float *__restrict__ ddt_in,
                                 const float *__restrict__ dt, const float *__restrict__ A,
                                 const bf16 *__restrict__ x, const bf16 *__restrict__ dy,
                                 float *__restrict__ ddt, float *__restrict__ dA,
                                 float *__restrict__ dD, int64_t batch, int64_t L, int H, int P)
{
    const int lane = threadIdx.x % 32;
    const int64_t w = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) / 32;
    if (w >= batch * H) return;
    const int h = (int)(w % H);
    const int64_t b = w / H;
    const float Ah = A[h];
    float carry = 0.f, sa = 0.f, sd = 0.f;
    for (int64_t t0 = ((L - 1) / 32) * 32; t0 >= 0; t0 -= 32) {
        const int64_t t = t0 + lane;
        const int64_t i = (b * L + t) * H + h;
        const float qv = t < L ? q[i] : 0.f;
        // inclusive suffix sum within the tile (lane l sums lanes l..31), then the carry
        float v = qv;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float u = __shfl_down_sync(0xffffffffu, v, o);
            if (lane + o < 32) v += u;
        }
        const float dl = v + carry;
        carry += __shfl_sync(0xffffffffu, v, 0);
        if (t < L) {
            ddt[i] = ddt_in[i] + Ah * dl;
            sa = fmaf(dt[i], dl, sa);
        }
    }
    for (int64_t i = lane; i < L * P; i += 32) {   // dD_h = sum_t <dy_t, x_t>
        const int64_t t = i / P, p = i % P;
        const int64_t off = ((b * L + t) * H + h) * P + p;
        sd = fmaf(to_f32(dy[off]), to_f32(x[off]), sd);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        sa += __shfl_xor_sync(0xffffffffu, sa, o);
        sd += __shfl_xor_sync(0xffffffffu, sd, o);
    }
    if (lane == 0) {
        atomicAdd(&dA[h], sa);
        atomicAdd(&dD[h], sd);
    }
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

cudaError_t launch_gather(const void *in, bool in_bf16, void *out, bool out_bf16, int64_t batch,
                          int64_t L, int rows_in, int rows_out, int E, bool reverse,
                          cudaStream_t st)
{
    const int64_t n = batch * L * rows_out * E;
    if (n == 0) return cudaSuccess;
    const unsigned g = grid_for(n);
    if (in_bf16 && out_bf16)
        gather_kernel<bf16, bf16><<<g, 256, 0, st>>>((const bf16 *)in, (bf16 *)out, batch, L,
                                                     rows_in, rows_out, E, reverse);
    else if (in_bf16)
        gather_kernel<bf16, float><<<g, 256, 0, st>>>((const bf16 *)in, (float *)out, batch, L,
                                                      rows_in, rows_out, E, reverse);
    else if (out_bf16)
        gather_kernel<float, bf16><<<g, 256, 0, st>>>((const float *)in, (bf16 *)out, batch, L,
                                                      rows_in, rows_out, E, reverse);
    else
        gather_kernel<float, float><<<g, 256, 0, st>>>((const float *)in, (float *)out, batch, L,
                                                       rows_in, rows_out, E, reverse);
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

cudaError_t launch_transpose(const float *in, float *out, int64_t mats, int rows, int cols,
                             cudaStream_t st)
{
    const int64_t n = mats * rows * cols;
    if (n == 0) return cudaSuccess;
    transpose_kernel<<<grid_for(n), 256, 0, st>>>(in, out, mats, rows, cols);
    return cudaGetLastError();
}

cudaError_t launch_bwd_tokens(const bf16 *dy, const float *dt, const float *D,
                              const bf16 *gb_rev, const float *ydot, const float *ddt_in,
                              const float *dfinal, const float *fin_t, float *dx, float *q,
                              int64_t batch, int64_t L, int H, int P, int N, cudaStream_t st)
{
    const int64_t warps = batch * L * H;
    if (warps == 0) return cudaSuccess;
    bwd_tokens_kernel<<<(unsigned)((warps * 32 + 255) / 256), 256, 0, st>>>(
        dy, dt, D, gb_rev, ydot, ddt_in, dfinal, fin_t, dx, q, batch, L, H, P, N);
    return cudaGetLastError();
}

cudaError_t launch_head_dot(const float *in, const bf16 *v, float *out, int64_t batch, int64_t L,
                            int H, int G, int N, bool reverse, cudaStream_t st)
{
    const int64_t warps = batch * L * H;
    if (warps == 0) return cudaSuccess;
    head_dot_kernel<<<(unsigned)((warps * 32 + 255) / 256), 256, 0, st>>>(in, v, out, batch, L,
                                                                       H, G, N, reverse);
    return cudaGetLastError();
}

cudaError_t launch_bwd_decay(const float *q, const float *ddt_in, const float *dt,
                             const float *A, const bf16 *x, const bf16 *dy, float *ddt,
                             float *dA, float *dD, int64_t batch, int64_t L, int H, int P,
                             cudaStream_t st)
{
    cudaError_t e = cudaMemsetAsync(dA, 0, H * sizeof(float), st);
    if (e == cudaSuccess) e = cudaMemsetAsync(dD, 0, H * sizeof(float), st);
    if (e != cudaSuccess) return e;
    const int64_t warps = batch * H;
    if (warps == 0) return cudaSuccess;
    bwd_decay_kernel<<<(unsigned)((warps * 32 + 127) / 128), 128, 0, st>>>(
        q, ddt_in, dt, A, x, dy, ddt, dA, dD, batch, L, H, P);
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
