// Shared device helpers and the internal launch interface of the SSD kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssd {

using bf16 = __nv_bfloat16;

// Element access for the two storage types of x, B, C and y.
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(bf16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float v) { return __float2bfloat16_rn(v); }

constexpr float kLog2e = 1.4426950408889634f;

// Programmatic dependent launch.  The four kernels of the chunked scan (cumsum, chunk state,
// state passing, chunk scan) are launched so that each may start while its predecessor in the
// stream is still running: a kernel calls griddep_launch_dependents() once its CTAs are resident,
// and its successor calls griddep_wait() before its first access to anything an earlier kernel
// of the stream writes (the wait returns when the predecessor grid has completed and its memory
// is visible; without a programmatic predecessor it returns at once).  The scan's own inputs (x,
// B, C, z, D) are never written by these kernels and may be read before the wait.  Since every
// kernel of the chain waits before it writes anything, completion is transitive: when a wait
// returns, every earlier kernel of the stream has completed.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Launch `kern` on `st` with programmatic stream serialisation (see above).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args &&...args)
{
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// The dt the recurrence uses when the block's raw projection is passed: + bias, then softplus
// log(1 + exp(v)) (equal to v in float32 for v > 20), then the clamp to [lo, hi]; each optional.
__device__ __forceinline__ float dt_transform(float v, const float *bias, int h, bool softplus,
                                              bool clamp, float lo, float hi)
{
    if (bias) v += bias[h];
    if (softplus) v = v > 20.f ? v : log1pf(__expf(v));
    if (clamp) v = fminf(fmaxf(v, lo), hi);
    return v;
}

// The SiLU gate z * sigmoid(z) of the block's output.  Fast exponential and division (about
// 2 ulp; the gated output is stored in bf16 or compared at 1e-4): for z -> -inf the divisor
// overflows to inf and the result is -0, the limit.
__device__ __forceinline__ float silu(float z) { return __fdividef(z, 1.f + __expf(-z)); }

// Workspace regions of one ssd_chunk_scan_fwd call (byte offsets from the workspace base).
struct WsLayout {
    size_t status;      // 256 bytes: device status word (nonzero after an in-kernel timeout)
    size_t cs;          // float [b][c][H][Q]: chunk-local inclusive cumsum of dt*A
    size_t dtc;         // float [b][c][H][Q]: dt per chunk row, 0 past the end (tensor-core path)
    size_t states;      // float [b][c][H][P][N]: per-chunk state, then (in place) state entering
    size_t hin_bf16;    // bf16  [b][c][H] blocks of P x N (hin_swizzled_offset): state entering
                        // each chunk (tensor-core path)
    size_t total;
};

// Where chunk k of the workspace sits in the token sequence.  Without a table (fixed-length
// input) chunk k of batch row b starts at token k Q of that row and holds min(Q, L - k Q)
// tokens.  With a table (packed variable-length input, batch 1) entry k holds the chunk's first
// token and its length, 0 for an unused slot; a chunk never spans two sequences, so every
// kernel treats a table chunk like the partial last chunk of a fixed-length sequence.
__device__ __forceinline__ void chunk_span(const int2 *tab, int64_t k, int Q, int64_t seqlen,
                                           int64_t &t0, int &len)
{
    if (tab) {
        const int2 e = tab[k];
        t0 = e.x;
        len = e.y;
    } else {
        t0 = k * Q;
        len = (int)(seqlen - t0 < Q ? seqlen - t0 : Q);
    }
}

// Workspace status word bits: 1, 2 = a bounded wait timed out (chunk state, chunk scan);
// kStatusBadSeqlens = the cu_seqlens of a variable-length call are inconsistent.
constexpr int kStatusBadSeqlens = 0x10000;

// Sets the calling thread's message returned by ssd_last_error().
void set_last_error(const char *msg);

// Failure injection for the tests of the bounded waits (include/ssd_testing.h): the CTA index of
// the next launch of `kernel` (kTestChunkState or kTestChunkScan) whose TMA producer leaves its
// first head's operand stage unissued, so the consumers' bounded waits on that stage run out;
// -1 (the default) for none.  Reading the setting clears it.
constexpr int kTestChunkState = 1;
constexpr int kTestChunkScan = 2;
int take_test_skip(int kernel);

// ---- launchers (each returns the launch's cudaError_t) ----
// Also zeroes *status (nullable) so each scan starts with a clean status word, and, when dtc is
// non-null, writes dt re-laid out as (b, c, H, Q) with zeros past the end of the sequence.
cudaError_t launch_chunk_cumsum(const float *dt, const float *A, float *cs, float *dtc,
                                int *status, int64_t batch, int64_t seqlen, int nheads, int Q,
                                int64_t nchunks, cudaStream_t st, const int2 *tab = nullptr,
                                bool unit_weights = false);

// Packed variable-length input: the chunk table (tab, nchunks entries) and the first chunk of
// every sequence (cstart, nseq + 1 entries) from cu_seqlens; clears *status and sets
// kStatusBadSeqlens (and an empty table) when cu_seqlens is inconsistent.
cudaError_t launch_build_chunk_table(const int32_t *cu_seqlens, int nseq, int64_t seqlen, int Q,
                                     int64_t nchunks, int2 *tab, int32_t *cstart, int *status,
                                     cudaStream_t st);

cudaError_t launch_chunk_state_simt(bool is_bf16, const void *x, const float *dt,
                                    const void *B, const float *cs, float *states,
                                    int64_t batch, int64_t seqlen, int H, int G, int P, int N,
                                    int Q, int64_t nchunks, cudaStream_t st);

// Carries the state across chunks: states[k] (chunk-local contribution) is replaced in place by
// the state entering chunk k (float32), or that state is written to hin_bf16 when non-null.
cudaError_t launch_state_passing(float *states, const float *cs, const float *init,
                                 float *final_state, bf16 *hin_bf16, int64_t batch, int H,
                                 int P, int N, int Q, int64_t nchunks, cudaStream_t st);
// The same per packed sequence: sequence s owns chunks [cstart[s], cstart[s + 1]) and its own
// initial and final state (init / final_state indexed [s][h][p][n]).
cudaError_t launch_state_passing_varlen(float *states, const float *cs, const float *init,
                                        float *final_state, bf16 *hin_bf16,
                                        const int32_t *cstart, int nseq, int H, int P, int N,
                                        int Q, int64_t nchunks, cudaStream_t st);

// z (nullable, x's element type and layout): the output is gated, y * z * sigmoid(z).
cudaError_t launch_chunk_scan_simt(bool is_bf16, const void *x, const float *dt,
                                   const void *B, const void *C, const float *cs,
                                   const float *hin, const float *D, void *y, int64_t batch,
                                   int64_t seqlen, int H, int G, int P, int N, int Q,
                                   int64_t nchunks, cudaStream_t st, const void *z = nullptr);

// dt_out[r][h] = clamp(softplus(dt[r][h] + bias[h])) over rows r < nrows (bias nullable; the
// softplus and the clamp to [lo, hi] each optional).
cudaError_t launch_dt_prologue(const float *dt, const float *bias, float *dt_out, int64_t nrows,
                               int H, bool softplus, bool clamp, float lo, float hi,
                               cudaStream_t st);

// Options of the decode update (all nullable / off): the gate z (x's type and layout) and the
// dt prologue, as for the fused scan.
struct DecodeOptions {
    const void *z = nullptr;
    const float *dt_bias = nullptr;
    bool softplus = false, clamp = false;
    float lo = 0.f, hi = 0.f;
};
cudaError_t launch_state_update(bool is_bf16, float *state, const void *x, const float *dt,
                                const float *A, const void *B, const void *C, const float *D,
                                void *y, int64_t batch, int H, int G, int P, int N,
                                cudaStream_t st, const DecodeOptions &opt = DecodeOptions());

cudaError_t launch_fill_final(const float *init, float *final_state, int64_t n,
                              cudaStream_t st);

// Tensor-core (tcgen05 + TMA) path: bf16, P = 64, N = 128, Q in {128, 256}.
bool tc_supported(bool is_bf16, int P, int N, int Q);

// split (Q = 64): the scaled rows as rounded bf16 plus their bf16 remainder, two MMA chains
// (float32-accurate states); rev: over the time-reversed sequence (rows read backwards).
cudaError_t launch_chunk_state_tc(const bf16 *x, const float *dtc, const bf16 *B,
                                  const float *cs, float *states, int *status, int64_t batch,
                                  int64_t seqlen, int H, int G, int Q, int64_t nchunks,
                                  cudaStream_t st, const char **why, const int2 *tab = nullptr,
                                  bool split = false, bool rev = false);
// Offset (in elements), inside one (batch, chunk, head) block of the bf16 entering states, of
// state element (p, n) for P = 64, N = 128.  The block is stored exactly as the tensor cores
// read it from shared memory: two halves of 64 n, each 64 rows p of 128 bytes, with the 16-byte
// pieces of row p permuted by p mod 8 (the 128-byte swizzle), so that one contiguous 16 KB copy
// brings a block into shared memory ready for use.
__host__ __device__ __forceinline__ int hin_swizzled_offset(int p, int n)
{
    const int a = n >> 6, nl = n & 63;
    return a * 4096 + p * 64 + ((((nl >> 3) ^ (p & 7)) << 3) | (nl & 7));
}

// Sequence parallelism (one contiguous segment per rank): the segment's total log-decay per
// (batch, head), and the combine of the all-gathered local final states into the segment's
// initial state (h_loc_all [nranks][BH][PN], logdec_all [nranks][BH]; init nullable).
cudaError_t launch_segment_log_decay(const float *cs, float *out, int64_t batch, int H, int Q,
                                     int64_t nchunks, cudaStream_t st);
cudaError_t launch_seqpar_combine(const float *h_loc_all, const float *logdec_all,
                                  const float *init, float *h_in, int nranks, int rank,
                                  int64_t BH, int PN, cudaStream_t st);

// ---- backward helpers (backward.cu)
// bf16 rows of E (a multiple of 8): out[b][t][r][:] = in[b][src][r_in][:], src = L-1-t when
// `reverse`, r_in = r / (rows_out / rows_in) (heads reading their group's row).
cudaError_t launch_gather(const bf16 *in, bf16 *out, int64_t batch, int64_t L, int rows_in,
                          int rows_out, int E, bool reverse, cudaStream_t st);
// dt' for the time-reversed adjoint scan: dt'[b][t][h] = dt[b][L-t][h] for t >= 1, 0 for t = 0.
cudaError_t launch_reverse_shift_dt(const float *dt, float *out, int64_t batch, int64_t L, int H,
                                   cudaStream_t st);
cudaError_t launch_fill(float *out, float value, int64_t n, cudaStream_t st);
// dx[b][t][h][p] = D_h dy + dt[b][t][h] gb[b][L-1-t][h][p];  xdy[b][t][h] = <x, dy>;
// q[b][t][h] = ydot - dt ddt_in (+ fdot[b][h] = <dfinal, final> at t = L-1; fdot nullable)
cudaError_t launch_bwd_tokens(const bf16 *x, const bf16 *dy, const float *dt, const float *D,
                              const bf16 *gb_rev, const float *ydot, const float *ddt_in,
                              const float *fdot, float *dx, float *q, float *xdy, int64_t batch,
                              int64_t L, int H, int P, cudaStream_t st);
// out[m] = <a[m], c[m]> over PN contiguous floats (PN % 4 == 0, 16-byte aligned matrices)
cudaError_t launch_state_dot(const float *a, const float *c, float *out, int64_t mats, int PN,
                             cudaStream_t st);
// dl = reverse cumsum of q over t per (b, h); ddt = ddt_in + A_h dl; dA_h = sum dt dl;
// dD_h = sum xdy (both summed over the batch in batch order, through the 2 * batch * H floats of
// `part`, so repeated calls give bit-identical results)
cudaError_t launch_bwd_decay(const float *q, const float *ddt_in, const float *dt,
                             const float *A, const float *xdy, float *ddt, float *dA, float *dD,
                             float *part, int64_t batch, int64_t L, int H, cudaStream_t st);
// The backward's float32 chunk-output kernel for P = 64, N = 128 (bwd_scan.cu): x''
// (batch, L, G, 128) bf16, B'' and C'' (batch, L, H, 64) bf16, all read at row L-1-tau for scan
// step tau when `rev`; w (batch, L, H) in scan order, null = 1; cs (batch, nch, H, 64)
// chunk-local cumsum in scan order; hin (batch, nch, H, 64, 128), the entering states [p][n].
// It writes each head's output row tau's dot product with vg[b][src(tau)][g(h)][:] at
// dot[b][src(tau)][h].
// Each CTA takes a run of bwd_scan_heads_per_cta(H, G) (8, 4, 2 or 1) heads of one group and
// writes the sum of their output rows, each weighted by ow[b][src][h] (null = 1), to
// ys[b][src][run][:] (batch, L, H / heads_per_cta, 128).
bool bwd_scan_supported(int P, int N);
int bwd_scan_heads_per_cta(int H, int G);
cudaError_t launch_bwd_chunk_scan(const bf16 *xg, const bf16 *bh, const bf16 *ch, const float *w,
                                  const float *cs, const float *hin, const bf16 *vg,
                                  const float *ow, float *ys, float *dot, int64_t batch,
                                  int64_t L, int H, int G, int64_t nch, bool rev, cudaStream_t st);
// out[b][t][g][n] = sum_{h in g} w[b][t][h] in[b][src(t)][h][n] (w = dt, or 1 when null)
cudaError_t launch_group_sum(const float *in, const float *w, float *out, int64_t batch,
                             int64_t L, int H, int G, int N, bool reverse, cudaStream_t st);
// dinit[b][h] = exp(dt[b][0][h] A_h) F[b][h]
cudaError_t launch_scale_init_grad(const float *F, const float *dt, const float *A, float *out,
                                   int64_t batch, int64_t L, int H, int PN, cudaStream_t st);

cudaError_t launch_chunk_scan_tc(const bf16 *x, const float *dtc, const bf16 *B, const bf16 *C,
                                 const float *cs, const bf16 *hin, const float *D, bf16 *y,
                                 int *status, int64_t batch, int64_t seqlen, int H, int G,
                                 int Q, int64_t nchunks, cudaStream_t st, const char **why,
                                 const int2 *tab = nullptr, const bf16 *z = nullptr);

}  // namespace ssd
