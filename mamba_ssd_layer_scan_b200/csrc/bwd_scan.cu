// The chunk-output kernel of the backward pass's two scans (dB and dC), in float32,
// specialised for their shape.
//
// Both scans are of the forward's kind with the head and state dimensions swapped: the state
// is K x E = P x N (64 x 128) per (batch, head), stored [j][e] like the forward's [p][n]; the
// "x" operand x'' has E = N = 128 channels and is shared by the heads of a group (it is B or C),
// the "B" and "C" operands B'', C'' have K = P = 64 channels per head (x or dy):
//
//   chunk state   S_k[j][e] = sum_{r in k} exp(cs_last - cs_r) w_r B''_r[j] x''_r[e]
//   chunk output  y_t[e]    = sum_{s <= t, s in k} exp(cs_t - cs_s) w_s (C''_t . B''_s) x''_s[e]
//                           + exp(cs_t) sum_j S_in[j][e] C''_t[j]
//
// (the same chunked form as the forward: mohakchugh.is-a.dev "Mamba-2", Block Decomposition).
// dB runs it on the time-reversed sequence (x'' = C, B'' = dy, C'' = x, unit weights, decays
// shifted by one token), dC forward (x'' = B, B'' = x, C'' = dy, weights dt).  The chunk states
// come from the tensor-core chunk-state kernel (chunk_tc.cu) with split bf16 operands; this
// kernel forms the chunk outputs.  It reads the operands in place from the bf16 inputs
// (reversed rows, the group's row for x''); everything is float32 from there on, because the
// decay gradient needs the outputs' dot products with B and C to float32 accuracy (see
// backward.cu).  Each output row's dot product with the group's B or C row is formed in the
// epilogue.
//
// Register tiling: each thread holds 4 rows x 8 channels of the 64 x 128 output tile, and 4 x 4
// of the 64 x 64 masked Gram matrix before that.  The channels of a thread are two runs of 4 at
// e0 and 64 + e0, so that each 16-byte shared-memory load of a half warp reads 256 contiguous
// bytes (two wavefronts, no bank conflict).
#include "common.cuh"

namespace ssd {
namespace {

constexpr int kQs = 64;     // chunk
constexpr int kE = 128;     // x'' channels (dstate of the forward)
constexpr int kK = 64;      // B'' / C'' channels (headdim of the forward)
constexpr int kThreads = 256;
constexpr int kTS = kQs + 4;   // row stride of the transposed [channel][token] tiles

__device__ __forceinline__ void unpack8(const uint4 raw, float *v)
{
    const bf16 *p = reinterpret_cast<const bf16 *>(&raw);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __bfloat162float(p[i]);
}

__device__ __forceinline__ int64_t src_row(int64_t tau, int64_t L, bool rev)
{
    return rev ? L - 1 - tau : tau;
}

// x'' and C'' are bf16 inputs and stay bf16 here (exact); B'' * w, the Gram matrix and the
// entering state are float32.  74 KB: three CTAs per SM.
struct ScanSmem {
    bf16 xs[kQs][kE];         // x'' rows
    union {
        float bT[kK][kTS];    // B'' * w transposed: bT[j][s] (until the Gram matrix is formed)
        float pT[kQs][kTS];   // masked, decayed Gram matrix, transposed: pT[s][t]
    };
    bf16 cT[kK][kTS];         // C'' transposed: cT[j][t]
    float hT[kK][kE];         // entering state transposed: hT[j][e]
    float css[kQs];           // chunk-local cumsum
};

// four bf16 (8 bytes) -> float32, exactly: the bf16 bits are the float's upper half
__device__ __forceinline__ void bf16x4_to_f32(const uint2 r, float *v)
{
    v[0] = __uint_as_float(r.x << 16);
    v[1] = __uint_as_float(r.x & 0xffff0000u);
    v[2] = __uint_as_float(r.y << 16);
    v[3] = __uint_as_float(r.y & 0xffff0000u);
}
static_assert(kK == kQs, "bT and pT share their storage");

// One CTA per (batch, chunk, run of kHPC heads of one group): the group's x'' rows are loaded
// once, the heads are taken in turn, and their output rows -- weighted by ow (dt for dB, 1 for
// dC) -- are summed in registers, so the CTA writes one partial sum of the group's output per
// run of heads (the group sum then adds H / G / kHPC partials instead of H / G outputs).
template <int kHPC>
__global__ void __launch_bounds__(kThreads, kHPC > 1 ? 2 : 3)
bwd_chunk_scan_kernel(const bf16 *__restrict__ xg, const bf16 *__restrict__ bh,
                      const bf16 *__restrict__ ch, const float *__restrict__ w,
                      const float *__restrict__ cs, const float *__restrict__ hin,
                      const bf16 *__restrict__ vg, const float *__restrict__ ow,
                      float *__restrict__ ys, float *__restrict__ dot, int64_t L, int H, int G,
                      int64_t nch, bool rev)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    ScanSmem &sm = *reinterpret_cast<ScanSmem *>(smem_raw);
    const int nhb = H / kHPC;                      // runs of heads
    const int hb = (int)(blockIdx.x % nhb);
    const int64_t k = (blockIdx.x / nhb) % nch, b = blockIdx.x / nhb / nch;
    const int g = hb * kHPC / (H / G);
    const int64_t t0 = k * kQs;
    const int len = (int)min((int64_t)kQs, L - t0);

    for (int i = threadIdx.x; i < kQs * kE / 8; i += kThreads) {
        const int r = i / (kE / 8), c8 = i % (kE / 8);
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (r < len) {
            const int64_t s = src_row(t0 + r, L, rev);
            v = *reinterpret_cast<const uint4 *>(xg + ((b * L + s) * G + g) * kE + c8 * 8);
        }
        *reinterpret_cast<uint4 *>(&sm.xs[r][c8 * 8]) = v;
    }

    // output rows tg..tg+3, channels e0..e0+3 and 64+e0..64+e0+3 (each 16-byte shared-memory load
    // of a half warp covers 256 contiguous bytes)
    const int tg = (threadIdx.x / 16) * 4, e0 = (threadIdx.x % 16) * 4;
    float tot[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int m = 0; m < 8; ++m) tot[i][m] = 0.f;

    for (int hh = 0; hh < kHPC; ++hh) {
        const int h = hb * kHPC + hh;
        const float *csk = cs + ((b * nch + k) * H + h) * (int64_t)kQs;
        const float *hk = hin + ((b * nch + k) * H + h) * (int64_t)(kE * kK);
        if (hh > 0) __syncthreads();   // the previous head is done with css, bT / pT, cT, hT
        if (threadIdx.x < kQs) sm.css[threadIdx.x] = threadIdx.x < len ? csk[threadIdx.x] : 0.f;
        for (int i = threadIdx.x; i < kQs * kK / 8; i += kThreads) {
            const int r = i % kQs, c8 = i / kQs;   // consecutive threads: consecutive tokens, so
                                                   // the transposed stores below hit distinct banks
            float vb[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            uint4 rc = make_uint4(0u, 0u, 0u, 0u);
            if (r < len) {
                const int64_t tau = t0 + r, s = src_row(tau, L, rev);
                const int64_t off = ((b * L + s) * H + h) * kK + c8 * 8;
                unpack8(*reinterpret_cast<const uint4 *>(bh + off), vb);
                rc = *reinterpret_cast<const uint4 *>(ch + off);
                const float f = w ? w[(b * L + tau) * H + h] : 1.f;
#pragma unroll
                for (int j = 0; j < 8; ++j) vb[j] *= f;
            }
            const bf16 *pc = reinterpret_cast<const bf16 *>(&rc);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                sm.bT[c8 * 8 + j][r] = vb[j];
                sm.cT[c8 * 8 + j][r] = pc[j];
            }
        }
        for (int i = threadIdx.x; i < kE * kK / 4; i += kThreads) {   // [j][e]: a plain copy
            const int j = i / (kE / 4), e4 = i % (kE / 4);
            *reinterpret_cast<float4 *>(&sm.hT[j][e4 * 4]) =
                *reinterpret_cast<const float4 *>(hk + j * kE + e4 * 4);
        }
        __syncthreads();

        // masked, decayed Gram matrix P[t][s] = (C''_t . w_s B''_s) exp(cs_t - cs_s), s <= t < len
        {
            const int ta = (threadIdx.x / 16) * 4, sa = (threadIdx.x % 16) * 4;
            float gm[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) gm[i][j] = 0.f;
            if (sa <= ta + 3) {
                for (int j = 0; j < kK; ++j) {
                    float ca[4];
                    bf16x4_to_f32(*reinterpret_cast<const uint2 *>(&sm.cT[j][ta]), ca);
                    const float4 bb = *reinterpret_cast<const float4 *>(&sm.bT[j][sa]);
                    const float ba[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i)
#pragma unroll
                        for (int q = 0; q < 4; ++q) gm[i][q] = fmaf(ca[i], ba[q], gm[i][q]);
                }
            }
            __syncthreads();   // every read of bT is done before pT overwrites it
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int s = sa + q;
                float o[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int t = ta + i;
                    o[i] = (s <= t && t < len) ? gm[i][q] * __expf(sm.css[t] - sm.css[s]) : 0.f;
                }
                *reinterpret_cast<float4 *>(&sm.pT[s][ta]) = make_float4(o[0], o[1], o[2], o[3]);
            }
        }
        __syncthreads();

        // first the entering state's term exp(cs_t) sum_j C''_t[j] S_in[j][e], scaled in
        // registers, then the masked P X on top
        float acc[4][8];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int m = 0; m < 8; ++m) acc[i][m] = 0.f;
        for (int j = 0; j < kK; ++j) {
            float ca[4];
            bf16x4_to_f32(*reinterpret_cast<const uint2 *>(&sm.cT[j][tg]), ca);
            const float4 h0 = *reinterpret_cast<const float4 *>(&sm.hT[j][e0]);
            const float4 h1 = *reinterpret_cast<const float4 *>(&sm.hT[j][64 + e0]);
            const float hv[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int m = 0; m < 8; ++m) acc[i][m] = fmaf(ca[i], hv[m], acc[i][m]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float dec = __expf(sm.css[tg + i]);
#pragma unroll
            for (int m = 0; m < 8; ++m) acc[i][m] *= dec;
        }
        const int smax = min(len, tg + 4);
        for (int s = 0; s < smax; ++s) {
            const float4 p = *reinterpret_cast<const float4 *>(&sm.pT[s][tg]);
            const float pa[4] = {p.x, p.y, p.z, p.w};
            float xv[8];
            bf16x4_to_f32(*reinterpret_cast<const uint2 *>(&sm.xs[s][e0]), xv);
            bf16x4_to_f32(*reinterpret_cast<const uint2 *>(&sm.xs[s][64 + e0]), xv + 4);
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int m = 0; m < 8; ++m) acc[i][m] = fmaf(pa[i], xv[m], acc[i][m]);
        }

        // this head's rows: the dot with the group's V row (at the row's source token), and
        // the weighted sum over the run of heads
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int t = tg + i;
            const bool valid = t < len;
            const int64_t s = valid ? src_row(t0 + t, L, rev) : 0;
            float d = 0.f;
            if (valid) {
                const bf16 *vrow = vg + ((b * L + s) * G + g) * (int64_t)kE + e0;
                const uint2 r0 = *reinterpret_cast<const uint2 *>(vrow);
                const uint2 r1 = *reinterpret_cast<const uint2 *>(vrow + 64);
                float v[8];
                bf16x4_to_f32(r0, v);
                bf16x4_to_f32(r1, v + 4);
#pragma unroll
                for (int m = 0; m < 8; ++m) d = fmaf(acc[i][m], v[m], d);
                const float wo = ow ? ow[(b * L + s) * H + h] : 1.f;
#pragma unroll
                for (int m = 0; m < 8; ++m) tot[i][m] = fmaf(wo, acc[i][m], tot[i][m]);
            }
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
            if (valid && e0 == 0) dot[(b * L + s) * H + h] = d;
        }
    }

    // the run's partial sum of the group's output, at the rows' source tokens (forward time)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int t = tg + i;
        if (t >= len) continue;
        const int64_t s = src_row(t0 + t, L, rev);
        float *yrow = ys + ((b * L + s) * nhb + hb) * (int64_t)kE + e0;
        *reinterpret_cast<float4 *>(yrow) =
            make_float4(tot[i][0], tot[i][1], tot[i][2], tot[i][3]);
        *reinterpret_cast<float4 *>(yrow + 64) =
            make_float4(tot[i][4], tot[i][5], tot[i][6], tot[i][7]);
    }
}

}  // namespace

bool bwd_scan_supported(int P, int N) { return P == kK && N == kE; }

int bwd_scan_heads_per_cta(int H, int G)
{
    const int hpg = H / G;
    return hpg % 4 == 0 ? 4 : (hpg % 2 == 0 ? 2 : 1);
}

cudaError_t launch_bwd_chunk_scan(const bf16 *xg, const bf16 *bh, const bf16 *ch, const float *w,
                                  const float *cs, const float *hin, const bf16 *vg,
                                  const float *ow, float *ys, float *dot, int64_t batch,
                                  int64_t L, int H, int G, int64_t nch, bool rev, cudaStream_t st)
{
    const int hpc = bwd_scan_heads_per_cta(H, G);
    const int64_t n = batch * nch * (H / hpc);
    if (n == 0) return cudaSuccess;
    const int smem = (int)sizeof(ScanSmem);
    auto kern = hpc == 4 ? bwd_chunk_scan_kernel<4>
                         : (hpc == 2 ? bwd_chunk_scan_kernel<2> : bwd_chunk_scan_kernel<1>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)n, kThreads, smem, st>>>(xg, bh, ch, w, cs, hin, vg, ow, ys, dot, L, H, G,
                                               nch, rev);
    return cudaGetLastError();
}

}  // namespace ssd
