// The chunk-output kernel of the backward pass's two scans (dB and dC), specialised for their
// shape.
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
// kernel forms the chunk outputs, reading the operands in place from the bf16 inputs (reversed
// rows, the group's row for x'').  The decay gradient needs the outputs' dot products with B
// and C to float32 accuracy (see backward.cu), so every operand that is not bf16 already is
// split into two bf16 parts, and every product accumulates in float32.  Each output row's dot
// product with the group's B or C row is formed in the epilogue.
#include "common.cuh"

namespace ssd {
namespace {

constexpr int kQs = 64;     // chunk
constexpr int kE = 128;     // x'' channels (dstate of the forward)
constexpr int kK = 64;      // B'' / C'' channels (headdim of the forward)
constexpr int kThreads = 256;

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

// The chunk outputs on warp-level bf16 tensor-core products (mma.sync m16n8k16, float32
// accumulate).  The operands that are not bf16 already -- w B'' (the Gram matrix's right
// factor), the masked Gram matrix P and the entering state S -- are split into their bf16
// rounding and the bf16 rounding of the remainder, and each product with them runs as two
// chains into the same float32 accumulator, which keeps the outputs to about float32 accuracy.
// Per head, with 8 warps:
//   G = C'' (w B'')^T       64 x 64, K = 64: warp (mt, nh) the rows 16 mt.., columns 32 nh..
//   P = G o decay o causal  masked in registers, split, stored [t][s]
//   Y = exp(cs_t) C'' S + P x''   64 x 128: warp (mt, nh) the rows 16 mt.., columns 64 nh..
// One CTA per (batch, chunk, run of kHPC heads of one group): the group's x'' rows are loaded
// once, the heads are taken in turn (the next head's entering state fetched with cp.async while
// the current one computes), and their output rows, weighted by ow (dt for dB, 1 for dC), are
// summed in registers, so the CTA writes one partial sum of the group's output per run (the
// group sum then adds H / G / kHPC partials).
// Fragment layouts are those of the PTX ISA for mma.m16n8k16 (row-major A, column-major B);
// ldmatrix loads them from shared-memory tiles whose row pitches (144 and 272 bytes) put the 8
// rows of each 8 x 8 matrix in distinct bank groups.
constexpr int kPA = 72;    // row pitch (elements) of the 64-column bf16 tiles
constexpr int kPB = 136;   // row pitch of the 128-column bf16 tiles
struct MmaSmem {
    bf16 xm[kQs][kPB];        // x'' rows [s][e], the group's (once per CTA)
    bf16 cm[kQs][kPA];        // C'' rows [t][j]
    bf16 bw[2][kQs][kPA];     // w B'' rows [s][j], split; then P [t][s], split
    bf16 st[2][kK][kPB];      // entering state [j][e], split
    float sf[kK][kE];         // the entering state as loaded (float32), fetched one head ahead
    float css[kQs];           // chunk-local cumsum
    float dotp[2][kQs];       // per column half: the rows' partial dot products with V
};

__device__ __forceinline__ uint32_t sh_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void *p)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(sh_addr(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void *p)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(sh_addr(p)));
}
// 16-byte global -> shared copies that complete asynchronously (cp.async), in one group
__device__ __forceinline__ void cp_async16(void *dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sh_addr(dst)), "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
                 "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// two floats -> their bf16 roundings (hi) and the bf16 roundings of the remainders (lo), each
// pair packed with the first value in the low half
__device__ __forceinline__ void split2(float x, float y, uint32_t &hi, uint32_t &lo)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(x - hf.x, y - hf.y);
    hi = *reinterpret_cast<const uint32_t *>(&h);
    lo = *reinterpret_cast<const uint32_t *>(&l);
}

template <int kHPC>
__global__ void __launch_bounds__(kThreads, 2)
bwd_chunk_scan_mma_kernel(const bf16 *__restrict__ xg, const bf16 *__restrict__ bh,
                          const bf16 *__restrict__ ch, const float *__restrict__ w,
                          const float *__restrict__ cs, const float *__restrict__ hin,
                          const bf16 *__restrict__ vg, const float *__restrict__ ow,
                          float *__restrict__ ys, float *__restrict__ dot, int64_t L, int H,
                          int G, int64_t nch, bool rev)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    MmaSmem &sm = *reinterpret_cast<MmaSmem *>(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g8 = lane >> 2, c4 = lane & 3;   // fragment row and column pair
    const int mt = warp & 3, nh = warp >> 2;   // this warp's row tile and column half
    const int nhb = H / kHPC;
    const int hb = (int)(blockIdx.x % nhb);
    const int64_t k = (blockIdx.x / nhb) % nch, b = blockIdx.x / nhb / nch;
    const int g = hb * kHPC / (H / G);
    const int64_t t0 = k * kQs;
    const int len = (int)min((int64_t)kQs, L - t0);
    // the entering state of the run's head hh into sf, asynchronously
    auto fetch_state = [&](int hh) {
        const float *hk =
            hin + ((b * nch + k) * H + hb * kHPC + hh) * (int64_t)(kE * kK);
        for (int i = threadIdx.x; i < kK * kE / 4; i += kThreads)
            cp_async16(&sm.sf[0][0] + 4 * i, hk + 4 * i);
        cp_async_commit();
    };
    fetch_state(0);

    for (int i = threadIdx.x; i < kQs * kE / 8; i += kThreads) {   // x'' rows, once
        const int r = i / (kE / 8), c8 = i % (kE / 8);
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (r < len) {
            const int64_t s = src_row(t0 + r, L, rev);
            v = *reinterpret_cast<const uint4 *>(xg + ((b * L + s) * G + g) * kE + c8 * 8);
        }
        *reinterpret_cast<uint4 *>(&sm.xm[r][c8 * 8]) = v;
    }

    float tot[8][4];   // the run's weighted sum of output fragments (8 column tiles of 8)
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
        for (int q = 0; q < 4; ++q) tot[n][q] = 0.f;

    for (int hh = 0; hh < kHPC; ++hh) {
        const int h = hb * kHPC + hh;
        const float *csk = cs + ((b * nch + k) * H + h) * (int64_t)kQs;
        if (hh > 0) __syncthreads();   // the previous head is done with css, cm, bw, st, dotp
        cp_async_wait_all();           // this head's entering state (every thread's part) ...
        __syncthreads();               // ... is in sf
        if (threadIdx.x < kQs) sm.css[threadIdx.x] = threadIdx.x < len ? csk[threadIdx.x] : 0.f;
        for (int i = threadIdx.x; i < kQs * kK / 8; i += kThreads) {   // C'' and w B'' rows
            const int r = i / (kK / 8), c8 = i % (kK / 8);
            uint4 cv = make_uint4(0u, 0u, 0u, 0u), bhi = cv, blo = cv;
            if (r < len) {
                const int64_t tau = t0 + r, s = src_row(tau, L, rev);
                const int64_t off = ((b * L + s) * H + h) * kK + c8 * 8;
                cv = *reinterpret_cast<const uint4 *>(ch + off);
                float vb[8];
                unpack8(*reinterpret_cast<const uint4 *>(bh + off), vb);
                const float f = w ? w[(b * L + tau) * H + h] : 1.f;
                split2(vb[0] * f, vb[1] * f, bhi.x, blo.x);
                split2(vb[2] * f, vb[3] * f, bhi.y, blo.y);
                split2(vb[4] * f, vb[5] * f, bhi.z, blo.z);
                split2(vb[6] * f, vb[7] * f, bhi.w, blo.w);
            }
            *reinterpret_cast<uint4 *>(&sm.cm[r][c8 * 8]) = cv;
            *reinterpret_cast<uint4 *>(&sm.bw[0][r][c8 * 8]) = bhi;
            *reinterpret_cast<uint4 *>(&sm.bw[1][r][c8 * 8]) = blo;
        }
        for (int i = threadIdx.x; i < kK * kE / 4; i += kThreads) {   // entering state, split
            const int j = i / (kE / 4), e4 = i % (kE / 4);
            const float4 v = *reinterpret_cast<const float4 *>(&sm.sf[j][e4 * 4]);
            uint2 hi, lo;
            split2(v.x, v.y, hi.x, lo.x);
            split2(v.z, v.w, hi.y, lo.y);
            *reinterpret_cast<uint2 *>(&sm.st[0][j][e4 * 4]) = hi;
            *reinterpret_cast<uint2 *>(&sm.st[1][j][e4 * 4]) = lo;
        }
        __syncthreads();
        if (hh + 1 < kHPC) fetch_state(hh + 1);   // sf is free: lands while this head computes

        // G = C'' (w B'')^T for rows 16 mt.., columns 32 nh.. (none above the diagonal)
        const bool gram_on = 16 * mt + 15 >= 32 * nh;
        float gacc[4][4];
#pragma unroll
        for (int n = 0; n < 4; ++n)
#pragma unroll
            for (int q = 0; q < 4; ++q) gacc[n][q] = 0.f;
        if (gram_on) {
#pragma unroll
            for (int kk = 0; kk < kK / 16; ++kk) {
                uint32_t a[4];
                ldsm_x4(a, &sm.cm[16 * mt + (lane & 15)][16 * kk + (lane >> 4) * 8]);
#pragma unroll
                for (int part = 0; part < 2; ++part)
#pragma unroll
                    for (int np = 0; np < 2; ++np) {
                        uint32_t bb[4];
                        const int n0 = 32 * nh + 16 * np;
                        ldsm_x4(bb, &sm.bw[part][n0 + (lane & 7) + ((lane >> 4) << 3)]
                                              [16 * kk + ((lane >> 3) & 1) * 8]);
                        mma16816(gacc[2 * np], a, bb[0], bb[1]);
                        mma16816(gacc[2 * np + 1], a, bb[2], bb[3]);
                    }
            }
        }
        __syncthreads();   // every read of w B'' is done before P overwrites it
        if (gram_on) {     // P = G exp(cs_t - cs_s) for s <= t < len, else 0; split, [t][s]
#pragma unroll
            for (int n = 0; n < 4; ++n)
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int t = 16 * mt + g8 + 8 * half;
                    const int s0 = 32 * nh + 8 * n + 2 * c4;
                    const float ct = sm.css[t];
                    const float p0 = (s0 <= t && t < len)
                                         ? gacc[n][2 * half] * __expf(ct - sm.css[s0]) : 0.f;
                    const float p1 = (s0 + 1 <= t && t < len)
                                         ? gacc[n][2 * half + 1] * __expf(ct - sm.css[s0 + 1])
                                         : 0.f;
                    uint32_t hi, lo;
                    split2(p0, p1, hi, lo);
                    *reinterpret_cast<uint32_t *>(&sm.bw[0][t][s0]) = hi;
                    *reinterpret_cast<uint32_t *>(&sm.bw[1][t][s0]) = lo;
                }
        }
        __syncthreads();

        // Y for rows 16 mt.., columns 64 nh..: the entering state's term, scaled by exp(cs_t),
        // then P x'' (source columns s <= 16 mt + 15 only)
        float acc[8][4];
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[n][q] = 0.f;
#pragma unroll
        for (int kk = 0; kk < kK / 16; ++kk) {
            uint32_t a[4];
            ldsm_x4(a, &sm.cm[16 * mt + (lane & 15)][16 * kk + (lane >> 4) * 8]);
#pragma unroll
            for (int part = 0; part < 2; ++part)
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    uint32_t bb[4];
                    const int n0 = 64 * nh + 16 * np;
                    ldsm_x4_t(bb, &sm.st[part][16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8]
                                             [n0 + (lane >> 4) * 8]);
                    mma16816(acc[2 * np], a, bb[0], bb[1]);
                    mma16816(acc[2 * np + 1], a, bb[2], bb[3]);
                }
        }
        {
            const float d0 = __expf(sm.css[16 * mt + g8]), d1 = __expf(sm.css[16 * mt + g8 + 8]);
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                acc[n][0] *= d0;
                acc[n][1] *= d0;
                acc[n][2] *= d1;
                acc[n][3] *= d1;
            }
        }
        for (int kk = 0; kk <= mt; ++kk) {
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                uint32_t a[4];
                ldsm_x4(a, &sm.bw[part][16 * mt + (lane & 15)][16 * kk + (lane >> 4) * 8]);
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    uint32_t bb[4];
                    const int n0 = 64 * nh + 16 * np;
                    ldsm_x4_t(bb, &sm.xm[16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8]
                                        [n0 + (lane >> 4) * 8]);
                    mma16816(acc[2 * np], a, bb[0], bb[1]);
                    mma16816(acc[2 * np + 1], a, bb[2], bb[3]);
                }
            }
        }

        // this head's rows: the dot with the group's V row (at the row's source token), and the
        // weighted sum over the run of heads
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int t = 16 * mt + g8 + 8 * half;
            const bool valid = t < len;
            const int64_t s = valid ? src_row(t0 + t, L, rev) : 0;
            float d = 0.f;
            if (valid) {
                const bf16 *vrow = vg + ((b * L + s) * G + g) * (int64_t)kE + 64 * nh + 2 * c4;
                const float wo = ow ? ow[(b * L + s) * H + h] : 1.f;
#pragma unroll
                for (int n = 0; n < 8; ++n) {
                    const float2 v = __bfloat1622float2(
                        *reinterpret_cast<const __nv_bfloat162 *>(vrow + 8 * n));
                    d = fmaf(acc[n][2 * half], v.x, d);
                    d = fmaf(acc[n][2 * half + 1], v.y, d);
                    tot[n][2 * half] = fmaf(wo, acc[n][2 * half], tot[n][2 * half]);
                    tot[n][2 * half + 1] = fmaf(wo, acc[n][2 * half + 1], tot[n][2 * half + 1]);
                }
            }
            d += __shfl_xor_sync(0xffffffffu, d, 1);
            d += __shfl_xor_sync(0xffffffffu, d, 2);
            if (c4 == 0) sm.dotp[nh][t] = d;
        }
        __syncthreads();
        if (threadIdx.x < len)
            dot[(b * L + src_row(t0 + threadIdx.x, L, rev)) * H + h] =
                sm.dotp[0][threadIdx.x] + sm.dotp[1][threadIdx.x];
    }

    // the run's partial sum of the group's output, at the rows' source tokens (forward time)
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int t = 16 * mt + g8 + 8 * half;
        if (t >= len) continue;
        const int64_t s = src_row(t0 + t, L, rev);
        float *yrow = ys + ((b * L + s) * nhb + hb) * (int64_t)kE + 64 * nh + 2 * c4;
#pragma unroll
        for (int n = 0; n < 8; ++n)
            *reinterpret_cast<float2 *>(yrow + 8 * n) =
                make_float2(tot[n][2 * half], tot[n][2 * half + 1]);
    }
}

}  // namespace

bool bwd_scan_supported(int P, int N) { return P == kK && N == kE; }

int bwd_scan_heads_per_cta(int H, int G)
{
    const int hpg = H / G;
    return hpg % 8 == 0 ? 8 : (hpg % 4 == 0 ? 4 : (hpg % 2 == 0 ? 2 : 1));
}

cudaError_t launch_bwd_chunk_scan(const bf16 *xg, const bf16 *bh, const bf16 *ch, const float *w,
                                  const float *cs, const float *hin, const bf16 *vg,
                                  const float *ow, float *ys, float *dot, int64_t batch,
                                  int64_t L, int H, int G, int64_t nch, bool rev, cudaStream_t st)
{
    const int hpc = bwd_scan_heads_per_cta(H, G);
    const int64_t n = batch * nch * (H / hpc);
    if (n == 0) return cudaSuccess;
    const int smem = (int)sizeof(MmaSmem);
    auto kern = hpc == 8 ? bwd_chunk_scan_mma_kernel<8>
                : hpc == 4 ? bwd_chunk_scan_mma_kernel<4>
                         : (hpc == 2 ? bwd_chunk_scan_mma_kernel<2> : bwd_chunk_scan_mma_kernel<1>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)n, kThreads, smem, st>>>(xg, bh, ch, w, cs, hin, vg, ow, ys, dot, L, H, G,
                                               nch, rev);
    return cudaGetLastError();
}

}  // namespace ssd
