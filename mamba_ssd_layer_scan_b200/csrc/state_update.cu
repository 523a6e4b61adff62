// Recurrent decode: one token per sequence, O(1) in the length of the past.
//
//     state[b][h] <- exp(dt A_h) state[b][h] + dt x (outer) B_g,     y[p] = state[p] . C_g + D_h x[p]
//
// (crackai.dev "Transformers are SSMs", Why It Matters: each new token costs O(1) time and
// constant memory; mohakchugh.is-a.dev "Mamba-2", Why This Matters for Hardware: the linear,
// recurrent mode used for autoregressive generation.)
//
// HBM-bound: the float32 state is read and written once per call and everything else is tiny.
// A warp owns whole rows p of one (batch, head) state: lane l holds the dstate/32 consecutive
// elements [l*V, l*V+V) of the row (16-byte vectors for dstate = 128), so every row is one fully
// coalesced 512-byte access; a warp issues the loads of kRowsInFlight rows before it uses them,
// and reduces each row's dot product with C by warp shuffles.  Loads and stores of the state
// are marked streaming (evict first): the state is much larger than L2 and is not reused
// within a call.
#include "common.cuh"

namespace ssd {
namespace {

constexpr int kWarps = 4;
constexpr int kRowsPerWarp = 16;
constexpr int kRowsInFlight = 8;
constexpr int kRowsPerCta = kWarps * kRowsPerWarp;

template <int V> struct Vec;
template <> struct Vec<1> {
    static __device__ __forceinline__ void ld(const float *p, float *r) { r[0] = __ldcs(p); }
    static __device__ __forceinline__ void st(float *p, const float *r) { __stcs(p, r[0]); }
};
template <> struct Vec<2> {
    static __device__ __forceinline__ void ld(const float *p, float *r) {
        const float2 v = __ldcs(reinterpret_cast<const float2 *>(p));
        r[0] = v.x; r[1] = v.y;
    }
    static __device__ __forceinline__ void st(float *p, const float *r) {
        __stcs(reinterpret_cast<float2 *>(p), make_float2(r[0], r[1]));
    }
};
template <> struct Vec<4> {
    static __device__ __forceinline__ void ld(const float *p, float *r) {
        const float4 v = __ldcs(reinterpret_cast<const float4 *>(p));
        r[0] = v.x; r[1] = v.y; r[2] = v.z; r[3] = v.w;
    }
    static __device__ __forceinline__ void st(float *p, const float *r) {
        __stcs(reinterpret_cast<float4 *>(p), make_float4(r[0], r[1], r[2], r[3]));
    }
};
template <> struct Vec<8> {
    static __device__ __forceinline__ void ld(const float *p, float *r) {
        Vec<4>::ld(p, r); Vec<4>::ld(p + 4, r + 4);
    }
    static __device__ __forceinline__ void st(float *p, const float *r) {
        Vec<4>::st(p, r); Vec<4>::st(p + 4, r + 4);
    }
};

// grid.x = ceil(P / kRowsPerCta) * H * batch
template <typename T, int V, bool kOpts>   // kOpts: gate and dt prologue (else plain)
__global__ void __launch_bounds__(kWarps * 32)
state_update_kernel(float *__restrict__ state, const T *__restrict__ x,
                    const float *__restrict__ dt, const float *__restrict__ A,
                    const T *__restrict__ B, const T *__restrict__ C,
                    const float *__restrict__ D, T *__restrict__ y, int H, int G, int P,
                    const T *__restrict__ z, const float *__restrict__ dt_bias, bool softplus,
                    bool clamp, float lo, float hi)
{
    constexpr int N = 32 * V;
    const int pblocks = (P + kRowsPerCta - 1) / kRowsPerCta;
    const int pb = (int)(blockIdx.x % pblocks);
    const int h = (int)((blockIdx.x / pblocks) % H);
    const int64_t b = blockIdx.x / pblocks / H;
    const int g = h / (H / G);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int p_begin = pb * kRowsPerCta + warp * kRowsPerWarp;
    const int p_end = min(P, p_begin + kRowsPerWarp);
    if (p_begin >= p_end) return;

    const float dth = kOpts ? dt_transform(dt[b * H + h], dt_bias, h, softplus, clamp, lo, hi)
                            : dt[b * H + h];
    const float a = __expf(dth * A[h]);
    const float Dh = D[h];
    float bv[V], cv[V];
#pragma unroll
    for (int j = 0; j < V; ++j) {
        bv[j] = to_f32(B[(b * G + g) * N + lane * V + j]) * dth;
        cv[j] = to_f32(C[(b * G + g) * N + lane * V + j]);
    }
    float *srow = state + ((b * H + h) * (int64_t)P) * N + lane * V;
    const T *xrow = x + (b * H + h) * (int64_t)P;
    T *yrow = y + (b * H + h) * (int64_t)P;
    const T *zrow = (kOpts && z) ? z + (b * H + h) * (int64_t)P : nullptr;

    for (int p0 = p_begin; p0 < p_end; p0 += kRowsInFlight) {
        float s[kRowsInFlight][V];
        float xv[kRowsInFlight];
#pragma unroll
        for (int r = 0; r < kRowsInFlight; ++r) {
            if (p0 + r < p_end) {
                Vec<V>::ld(srow + (int64_t)(p0 + r) * N, s[r]);
                xv[r] = to_f32(xrow[p0 + r]);
            }
        }
#pragma unroll
        for (int r = 0; r < kRowsInFlight; ++r) {
            float dot = 0.f;
            if (p0 + r < p_end) {
#pragma unroll
                for (int j = 0; j < V; ++j) {
                    s[r][j] = fmaf(a, s[r][j], xv[r] * bv[j]);
                    dot = fmaf(s[r][j], cv[j], dot);
                }
                Vec<V>::st(srow + (int64_t)(p0 + r) * N, s[r]);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
            if (lane == 0 && p0 + r < p_end) {
                const float out = fmaf(Dh, xv[r], dot);
                yrow[p0 + r] =
                    from_f32<T>(kOpts && zrow ? out * silu(to_f32(zrow[p0 + r])) : out);
            }
        }
    }
}

template <typename T>
cudaError_t launch_typed(float *state, const void *x, const float *dt, const float *A,
                         const void *B, const void *C, const float *D, void *y, int64_t batch,
                         int H, int G, int P, int N, cudaStream_t st, const DecodeOptions &o)
{
    const T *zp = (const T *)o.z;
    const unsigned grid = (unsigned)(((P + kRowsPerCta - 1) / kRowsPerCta) * H * batch);
    const T *xp = (const T *)x, *Bp = (const T *)B, *Cp = (const T *)C;
    T *yp = (T *)y;
    const bool opts = o.z || o.dt_bias || o.softplus || o.clamp;
#define SSD_DECODE_LAUNCH(VV)                                                                   \
    (opts ? state_update_kernel<T, VV, true><<<grid, kWarps * 32, 0, st>>>(                      \
                state, xp, dt, A, Bp, Cp, D, yp, H, G, P, zp, o.dt_bias, o.softplus, o.clamp,     \
                o.lo, o.hi)                                                                     \
          : state_update_kernel<T, VV, false><<<grid, kWarps * 32, 0, st>>>(                     \
                state, xp, dt, A, Bp, Cp, D, yp, H, G, P, nullptr, nullptr, false, false, 0.f,   \
                0.f))
    switch (N) {
    case 32: SSD_DECODE_LAUNCH(1); break;
    case 64: SSD_DECODE_LAUNCH(2); break;
    case 128: SSD_DECODE_LAUNCH(4); break;
    case 256: SSD_DECODE_LAUNCH(8); break;
    default: return cudaErrorInvalidValue;
    }
#undef SSD_DECODE_LAUNCH
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_state_update(bool is_bf16, float *state, const void *x, const float *dt,
                                const float *A, const void *B, const void *C, const float *D,
                                void *y, int64_t batch, int H, int G, int P, int N,
                                cudaStream_t st, const DecodeOptions &opt)
{
    if (is_bf16)
        return launch_typed<bf16>(state, x, dt, A, B, C, D, y, batch, H, G, P, N, st, opt);
    return launch_typed<float>(state, x, dt, A, B, C, D, y, batch, H, G, P, N, st, opt);
}

}  // namespace ssd
