// Tensor-core (tcgen05 + TMEM, fed by TMA) kernels of the chunked scan: bf16 operands, f32
// accumulation, headdim P = 64, dstate N = 128, chunk Q in {128, 256}.
//
// Within a chunk the SSD output is a dense, masked matrix product -- the semiseparable block
// (C B^T o L) applied to dt*x -- which is what makes the layer run on tensor cores
// (mohakchugh.is-a.dev "Mamba-2", The Tensor Core Connection: the structured mask inside a
// chunk is materialised as a dense Q x Q matrix and multiplied against the chunk's values;
// chipfoundryservices.com "hybrid attention-SSM": the SSD algorithm exposes the computation as
// block matrix multiplications).  Two kernels:
//
// chunk_state_tc_kernel   S_k^T = B_k^T (w o X_k),  w_tau = exp(cs_last - cs_tau) dt_tau
//     One CTA per SM, each taking an equal run of the flat list of (batch, chunk, group, head)
//     items.  A chunk's B rows are loaded once per run of its heads and shared by them; per
//     head, the x tile and the head's cs / dt rows arrive by TMA (4 stages), 8 warps scale the x
//     rows by w in shared memory, one M=128 (n) x N=64 (p) x K=Q MMA chain accumulates S^T in
//     TMEM (double-buffered), and 4 epilogue warps move it to global memory while the next
//     head's MMAs run.
//
// chunk_scan_tc_kernel    y = (C B^T o L o dt + diag(D)) X  +  exp(cs) o (C h_in^T)
//     One CTA per SM per 128-row tile class of the chunks, each taking an equal run of the flat
//     (batch, chunk, group, head) list, and for 256-token chunks a third group of CTAs that takes
//     the tails of the second-tile runs (see scan_work).  C B^T is computed once per segment (a
//     run of one chunk's heads of a group, which see the same B and C) and shared by its heads.
//     The diagonal 128 x 128 block of the masked matrix is built per head by 8 worker warps from
//     TMEM and written back to TMEM as bf16 (a ring of 64-column blocks), where the MMAs read it
//     as their A operand; for the second tile of a 256-token chunk the off-diagonal block is
//     rank-1 in its decay and runs as a plain product with C B_off^T converted to bf16 once per
//     segment (see the section comment below).  The decay is factorised so that no element
//     needs an exponential of its own.  The same worker warps then run the previous head's
//     epilogue.
//
// Roles (warp-specialised; every wait is on an mbarrier and bounded, see sm100.cuh):
//   state kernel: warp 0 TMA, warp 1 MMA, warp 2 TMEM owner, warps 4-11 scale, 12-15 epilogue
//   scan  kernel: warp 0 TMA, warp 1 MMA and TMEM owner, warps 2-9 mask + epilogue, and for a
//                 gated output warp 10, which stages each head's gate rows by TMA
// A buffer that a TMA or bulk copy fills and that threads then read (or write) with plain
// loads is released to the next copy only after those threads' fence.proxy.async: the copy
// runs in the async proxy, which the generic proxy's release and acquire alone do not order.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <mutex>

#include "common.cuh"
#include "sm100.cuh"

namespace ssd {
namespace {

using namespace sm100;

constexpr int kP = 64;
constexpr int kN = 128;
constexpr int kRowBytes = 128;                  // one swizzled smem row: 64 bf16
constexpr int kTileRows = 128;                  // rows of one TMA box / one MMA M tile
constexpr int kBoxBytes = kTileRows * kRowBytes;  // 16 KB

// Warp-uniform bounded wait: lane 0 polls, the verdict is broadcast.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort)
{
    bool ok = true;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort);
    return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}
// The same with every lane observing the phase itself: for data that a TMA copy writes just
// before the lanes read it (one lane's observation does not make the copy's bytes visible to
// the others).  The result is the same for the whole warp.
__device__ __forceinline__ bool warp_wait_each(uint64_t *bar, uint32_t parity,
                                               volatile int *abort)
{
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort) ? 1 : 0) != 0;
}

// z * sigmoid(z) = z (1 + tanh(z / 2)) / 2 with the hardware tanh approximation: one
// special-function operation per element instead of an exponential and a reciprocal (relative
// error about 2^-11, below the bf16 rounding of the gated output it feeds).
__device__ __forceinline__ float silu_approx(float z)
{
    const float hz = 0.5f * z;
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(hz));
    return fmaf(hz, t, hz);
}

// ============================================================ chunk state
//
// Work is the flat list of (batch, chunk, group, head) items, the heads of a group consecutive;
// CTA c of a grid of one CTA per SM takes items [c n / grid, (c + 1) n / grid), so every SM gets
// the same number of heads to within one.  A run of items of the same (batch, chunk, group) is a
// segment: its heads share the chunk's B tile, which the CTA loads once per segment.
constexpr int kStateStages = 4;
struct alignas(1024) StateSmem {
    bf16 Bs[2][256 * 64];                 // MN-major A operand: [n atom][Q rows tau][64 n]
    bf16 Xs[kStateStages][256 * 64];      // MN-major B operand per stage: [Q rows tau][64 p]
    float cs_v[kStateStages][256];        // per stage: the head's chunk-local cumsum row
    float dt_v[kStateStages][256];        // per stage: the head's dt row (0 past the end)
    uint64_t bar_b, bar_b_free;
    uint64_t bar_x_full[kStateStages], bar_x_ready[kStateStages], bar_x_free[kStateStages];
    uint64_t bar_acc_full[2], bar_acc_free[2];
    uint64_t bar_drain;
    uint32_t tmem_base;
    int abort;
};
// warp 0 TMA, warp 1 MMA, warp 2 TMEM owner, warps 4-11 scale x, warps 12-15 epilogue
constexpr int kStateThreads = 512;
constexpr int kStateScaleThreads = 256;
constexpr uint32_t kStateTmemCols = 128;   // two accumulator buffers of 64 p

// Item f of the flat list: its batch row, chunk, group and head.
struct StateItem {
    int64_t b, k;
    int g, h;
    bool seg_start;   // first item of its (batch, chunk, group) within the CTA
};
__device__ __forceinline__ StateItem state_item(int64_t f, int64_t f0, int hpg, int G,
                                                int64_t nchunks)
{
    StateItem it;
    const int hl = (int)(f % hpg);
    const int64_t seg = f / hpg;
    it.g = (int)(seg % G);
    const int64_t bk = seg / G;
    it.k = bk % nchunks;
    it.b = bk / nchunks;
    it.h = it.g * hpg + hl;
    it.seg_start = f == f0 || hl == 0;
    return it;
}

// kSplit (Q = 64 only): the scaled rows w_tau x_tau go to the MMA as two bf16 tiles, the rounded
// value and the rounding remainder (the second in the upper part of the stage), accumulated by
// two MMA chains: the state to about float32 accuracy (the backward's decay gradient needs it).
// kRev: the chunks run over the time-reversed sequence: chunk k covers the reversed tokens
// [kQ, kQ + Q), i.e. the memory rows [L - kQ - Q, L - kQ) in descending order; the rows are
// loaded in memory order and row i of the tile is reversed token Q - 1 - i.
template <bool kSplit, bool kRev>
__global__ void __launch_bounds__(kStateThreads, 1)
chunk_state_tc_kernel(const __grid_constant__ CUtensorMap tm_x,
                      const __grid_constant__ CUtensorMap tm_b, const float *__restrict__ dtc,
                      const float *__restrict__ cs, float *__restrict__ states,
                      int *__restrict__ status, int H, int G, int Q, int64_t nchunks,
                      int64_t nitems, int64_t seqlen, const int2 *__restrict__ tab, int skip_cta)
{
    extern __shared__ uint8_t smem_raw[];
    StateSmem &sm = *reinterpret_cast<StateSmem *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int hpg = H / G;
    const int64_t f0 = (int64_t)blockIdx.x * nitems / gridDim.x;
    const int64_t f1 = ((int64_t)blockIdx.x + 1) * nitems / gridDim.x;
    const int nh = (int)(f1 - f0);
    if (nh <= 0) return;
    // first memory row of the tile of the chunk that starts at (reversed) token t0
    auto row0 = [&](int64_t t0) { return (int)(kRev ? seqlen - t0 - Q : t0); };
    // L2 prefetches are hints: a tile that starts before row 0 is not prefetched
    auto pf_row = [&](int64_t t0) { return row0(t0) < 0 ? 0 : row0(t0); };

    if (threadIdx.x == 0) {
        mbar_init(&sm.bar_b, 1);
        mbar_init(&sm.bar_b_free, 1);
        for (int s = 0; s < kStateStages; ++s) {
            mbar_init(&sm.bar_x_full[s], 1);
            mbar_init(&sm.bar_x_ready[s], kStateScaleThreads);
            mbar_init(&sm.bar_x_free[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sm.bar_acc_full[s], 1);
            mbar_init(&sm.bar_acc_free[s], 128);
        }
        mbar_init(&sm.bar_drain, 1);
        sm.abort = 0;
        fence_mbar_init();
    }
    if (warp == 2) {
        tmem_alloc(&sm.tmem_base, kStateTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (threadIdx.x == 0) griddep_launch_dependents();
    const uint32_t tmem = sm.tmem_base;
    volatile int *abort = &sm.abort;

    if (warp == 0) {
        // ---------------- TMA producer (lane 0 alone): per segment the B tile, per head its x
        // tile and cs / dt rows
        if (lane == 0) {
            tma_prefetch_desc(&tm_x);
            tma_prefetch_desc(&tm_b);
            // x and B are inputs of the scan: start streaming the first heads' tiles into L2
            // while the cumsum kernel finishes
            for (int j = 0; j < nh && j < kStateStages; ++j) {
                const StateItem it = state_item(f0 + j, f0, hpg, G, nchunks);
                int64_t t0;
                int len;
                chunk_span(tab, it.k, Q, seqlen, t0, len);
                tma_prefetch_l2_4d(&tm_x, 0, it.h, pf_row(t0), (int)it.b);
            }
            griddep_wait();   // cs / dt (and a chunk table) come from earlier kernels
            int seg = -1;
            for (int j = 0; j < nh; ++j) {
                const StateItem it = state_item(f0 + j, f0, hpg, G, nchunks);
                int64_t t0;
                int len;
                chunk_span(tab, it.k, Q, seqlen, t0, len);
                if (it.seg_start) {
                    ++seg;
                    // the previous segment's MMAs must be done with the B tile
                    if (seg > 0 && !mbar_wait(&sm.bar_b_free, (seg - 1) & 1, abort)) break;
                    mbar_arrive_expect_tx(&sm.bar_b, 2u * Q * kRowBytes);
                    for (int a = 0; a < 2; ++a)   // boxes of Q rows
                        tma_load_4d(&sm.Bs[a][0], &tm_b, &sm.bar_b, 64 * a, it.g, row0(t0),
                                    (int)it.b);
                    // the next segment's B tile into L2 now, so that its load after this
                    // segment's last MMA is short
                    const int64_t fn = (f0 + j) - (f0 + j) % hpg + hpg;
                    if (fn < f1) {
                        const StateItem nx = state_item(fn, f0, hpg, G, nchunks);
                        int64_t nt0;
                        int nlen;
                        chunk_span(tab, nx.k, Q, seqlen, nt0, nlen);
                        for (int a = 0; a < 2; ++a)
                            tma_prefetch_l2_4d(&tm_b, 64 * a, nx.g, pf_row(nt0), (int)nx.b);
                    }
                }
                const int s = j % kStateStages;
                const uint32_t use = j / kStateStages;
                if (j >= kStateStages && !mbar_wait(&sm.bar_x_free[s], (use - 1) & 1, abort))
                    break;
                // failure injection (tests only): this stage is left unissued
                if (j == 0 && (int)blockIdx.x == skip_cta) continue;
                const int64_t vrow = ((it.b * nchunks + it.k) * H + it.h) * (int64_t)Q;
                mbar_arrive_expect_tx(&sm.bar_x_full[s], (uint32_t)Q * (kRowBytes + 8));
                tma_load_4d(&sm.Xs[s][0], &tm_x, &sm.bar_x_full[s], 0, it.h, row0(t0), (int)it.b);
                bulk_load(sm.cs_v[s], cs + vrow, Q * 4, &sm.bar_x_full[s]);
                bulk_load(sm.dt_v[s], dtc + vrow, Q * 4, &sm.bar_x_full[s]);
                // the tile this stage will hold next: into L2 now, so its load is an L2 hit
                if (j + kStateStages < nh) {
                    const StateItem nx = state_item(f0 + j + kStateStages, f0, hpg, G, nchunks);
                    int64_t nt0;
                    int nlen;
                    chunk_span(tab, nx.k, Q, seqlen, nt0, nlen);
                    tma_prefetch_l2_4d(&tm_x, 0, nx.h, pf_row(nt0), (int)nx.b);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer: D[n][p] += sum_tau B[tau][n] * Xw[tau][p].  Lane 0 alone
        // runs the whole loop, waits included: a lane that issued tcgen05.mma and then rejoins
        // its warp stalls for the MMAs' issue latency (hundreds of cycles) at every rejoin.
        const uint32_t idesc = idesc_bf16_f32(128, kP, true, true);
        const uint32_t atom_bytes = 256 * kRowBytes;  // distance between the two n atoms of Bs
        if (lane == 0) {
            int seg = -1;
            for (int j = 0; j < nh; ++j) {
                const StateItem it = state_item(f0 + j, f0, hpg, G, nchunks);
                const bool seg_end = j + 1 == nh || (f0 + j + 1) % hpg == 0;
                if (it.seg_start) {
                    ++seg;
                    if (!mbar_wait(&sm.bar_b, seg & 1, abort)) break;
                }
                const int s = j % kStateStages;
                const uint32_t use = j / kStateStages;
                const int a = j & 1;
                if (!mbar_wait(&sm.bar_x_ready[s], use & 1, abort)) break;
                if (j >= 2 && !mbar_wait(&sm.bar_acc_free[a], ((j >> 1) - 1) & 1, abort)) break;
                tc_fence_after();
                const uint32_t d = tmem + a * kP;
                // base descriptors + constant K steps (16 rows = 2048 bytes) in fully unrolled
                // loops: the issuing thread's own instruction chain sets the MMA issue rate
                const uint64_t ad = smem_desc_sw128(smem_u32(&sm.Bs[0][0]), atom_bytes, 1024);
                const uint64_t bd = smem_desc_sw128(smem_u32(&sm.Xs[s][0]), atom_bytes, 1024);
                if (kSplit) {   // Q = 64: the rounded rows, then their remainders (8 KB on)
                    const uint64_t bl = bd + ((64 * kRowBytes) >> 4);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(d, ad + kk * 128, bd + kk * 128, idesc, kk > 0 ? 1u : 0u);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(d, ad + kk * 128, bl + kk * 128, idesc, 1u);
                } else if (Q == 256) {
#pragma unroll
                    for (int kk = 0; kk < 16; ++kk)
                        mma_bf16(d, ad + kk * 128, bd + kk * 128, idesc, kk > 0 ? 1u : 0u);
                } else {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16(d, ad + kk * 128, bd + kk * 128, idesc, kk > 0 ? 1u : 0u);
                }
                mma_commit(&sm.bar_x_free[s]);
                mma_commit(&sm.bar_acc_full[a]);
                if (seg_end) mma_commit(&sm.bar_b_free);
            }
        }
    } else if (warp >= 4 && warp < 12) {
        // ---------------- scale x rows by w_tau = exp(cs_last - cs_tau) dt_tau (in place)
        const int st = threadIdx.x - 128;             // 0..255
        const int chunks = Q * 8;                     // 16-byte pieces of the tile
        for (int j = 0; j < nh; ++j) {
            const int s = j % kStateStages;
            const uint32_t use = j / kStateStages;
            if (!warp_wait(&sm.bar_x_full[s], use & 1, abort)) break;
            const float cs_last = sm.cs_v[s][Q - 1];
            for (int c = st; c < chunks; c += kStateScaleThreads) {
                const int tau = kRev ? Q - 1 - (c >> 3) : c >> 3;   // (reversed) token of the row
                const float w = __expf(cs_last - sm.cs_v[s][tau]) * sm.dt_v[s][tau];
                uint4 *ptr = reinterpret_cast<uint4 *>(&sm.Xs[s][0]) + c;
                uint4 v = *ptr;
                uint32_t *wv = &v.x;
                uint4 lo = make_uint4(0u, 0u, 0u, 0u);
                uint32_t *lv = &lo.x;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __bfloat1622float2(
                        *reinterpret_cast<const __nv_bfloat162 *>(&wv[e]));
                    const float2 sc = fmul2(f, make_float2(w, w));
                    wv[e] = pack_bf16x2(sc.x, sc.y);
                    if (kSplit) {   // the remainder sc - bf16(sc), rounded to bf16 in turn
                        const float2 hi = __bfloat1622float2(
                            *reinterpret_cast<const __nv_bfloat162 *>(&wv[e]));
                        lv[e] = pack_bf16x2(sc.x - hi.x, sc.y - hi.y);
                    }
                }
                *ptr = v;
                if (kSplit) ptr[64 * 8] = lo;   // Q = 64: the remainder tile 8 KB on
            }
            fence_async_smem();
            mbar_arrive(&sm.bar_x_ready[s]);
        }
    } else if (warp >= 12) {
        // ---------------- epilogue: TMEM (lane n, column p) -> states[b][k][h][p][n]
        const int q = warp & 3;
        const int n = q * 32 + lane;
        for (int j = 0; j < nh; ++j) {
            const StateItem it = state_item(f0 + j, f0, hpg, G, nchunks);
            const int a = j & 1;
            if (!warp_wait(&sm.bar_acc_full[a], (j >> 1) & 1, abort)) break;
            tc_fence_after();
            uint32_t r0[32], r1[32];
            const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + a * kP;
            tmem_ld32(taddr, r0);
            tmem_ld32(taddr + 32, r1);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(&sm.bar_acc_free[a]);
            // lane n writes column n of every row p: each store of the warp is 128 contiguous
            // bytes
            float *out = states + ((it.b * nchunks + it.k) * H + it.h) * (int64_t)(kP * kN) + n;
#pragma unroll
            for (int p = 0; p < 32; ++p) out[p * kN] = __uint_as_float(r0[p]);
#pragma unroll
            for (int p = 0; p < 32; ++p) out[(32 + p) * kN] = __uint_as_float(r1[p]);
        }
    }

    __syncthreads();
    if (sm.abort) {
        // Let this CTA's own MMAs and TMA copies finish before TMEM and smem are released.
        if (warp == 1 && lane == 0) {
            mma_commit(&sm.bar_drain);
            mbar_wait_drain(&sm.bar_drain, 0);
        }
        if (threadIdx.x == 0) {
            drain_sleep();
            atomicOr(status, 1);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, kStateTmemCols);
    }
}

// ============================================================ chunk scan (intra-chunk + off-chunk)
//
// Tile T of a chunk holds rows [128 T, 128 T + 128).  Its output splits into
//   - the diagonal 128 x 128 block (source columns of the same tile): P = C B^T o L o dt (+ D on
//     the diagonal), built elementwise by the mask warps and multiplied by x from TMEM;
//   - for T = 1, the off-diagonal block (source columns [0, 128)): every source precedes every
//     target, so with the reference row r = 127, exp(cs_t - cs_i) = u_t v_i, u_t = exp(cs_t -
//     cs_127), v_i = exp(cs_127 - cs_i) (both <= 1), and the block's contribution is
//     diag(u) (C B_off^T) diag(v dt) X_off: C B_off^T is converted to bf16 once per CTA and
//     shared by all heads, X_off is scaled row-wise per head, and u is applied in the epilogue;
//   - the off-chunk term exp(cs_t) C h_in^T = u_t C (exp(cs_127) h_in)^T, which (scaled h_in)
//     accumulates into the same TMEM accumulator as the off-diagonal block.
// So y = Y_diag + f_t Y_A with f_t = exp(cs_t) (T = 0) or u_t (T = 1).  Where the whole chunk
// decays by at most exp(kRef0Floor) (cs_{Q-1} >= kRef0Floor), T = 1 instead takes the reference
// "row -1" (cs = 0): x_off scaled by exp(-cs_i) dt_i <= exp(-kRef0Floor) dt_i, h_in unscaled,
// f_t = exp(cs_t) >= exp(kRef0Floor), which saves scaling h_in; the factors stay well inside the
// float32 and bf16 range (e^60 ~ 1e26).
constexpr float kRef0Floor = -60.f;
__device__ __forceinline__ bool scan_ref0(float cs_last) { return cs_last >= kRef0Floor; }
constexpr int kXStagesMax = 5;   // x / h_in stages: tiles without an off-diagonal block use 5
                                 // of 32 KB (three in S01, two in the B tile's space once C B^T
                                 // is done); the second tile of a chunk with one uses 2 of 48 KB
                                 // (S01; the B tile's space then holds the bf16 block)
constexpr int kScanVecStages = 6; // cs / dt row stages (one head each)
constexpr int kRing = 4;         // 64-column blocks of P in TMEM (two heads)
constexpr int kStageBytes = 256 * kRowBytes + 2 * kP * kRowBytes;  // 48 KB: 256 x rows + h_in
constexpr int kStage32 = 128 * kRowBytes + 2 * kP * kRowBytes;     // 32 KB: 128 x rows + h_in
struct alignas(1024) ScanSmem {
    bf16 Cs[2][kTileRows * 64];     // K-major A (C tile): [n atom][128 rows t][64 n]
    uint8_t R[kStageBytes + 16384]; // B rows for C B^T (K-major [n atom][KI rows][64]); after
                                    // that, T = 0: x / h_in stage 2; T = 1: bf16 C B_off^T
                                    // (K-major [i atom][128 rows t][64 i])
    uint8_t S01[2 * kStageBytes];   // x / h_in stages: [KI rows i][64 p] then h_in
                                    // [n atom][64 rows p][64 n]
    float cs_v[kScanVecStages][256];  // per stage: one head's chunk-local cumsum row
    float dt_v[kScanVecStages][256];  // per stage: its dt row (0 past the end)
    float vt[8][64];                // per worker warp: column factors of its two slices
    uint64_t bar_cb, bar_g, bar_goff, bar_seg_done;
    uint64_t bar_xh_full[kXStagesMax], bar_xh_free[kXStagesMax], bar_xv_ready[kXStagesMax];
    uint64_t bar_vec_full[kScanVecStages], bar_vec_free[kScanVecStages];
    uint64_t bar_slot_full[kRing], bar_slot_free[kRing];
    uint64_t bar_acc_full[2], bar_acc_free[2];
    uint64_t bar_z_full, bar_z_free;   // the gate rows' stage (gated output only)
    uint64_t bar_drain;
    uint32_t tmem_base;
    int abort;
};
// Gated output: one head's gate rows (128 rows x 64 columns bf16, 128-byte swizzle) in a stage
// after ScanSmem, loaded by TMA one P build ahead of the epilogue that reads them.
constexpr int kZStageBytes = kTileRows * kRowBytes;
// warp 0 TMA, warp 1 MMA and TMEM owner, warps 2-9 workers: two per TMEM
// lane quarter, each owning a 32-column slice of every 64-column block; per head they build
// their slice of P (mask) and then run the epilogue of the previous head for their slice of y
constexpr int kScanWorkers = 256;
constexpr int kScanThreads = 64 + kScanWorkers;   // 320 threads
constexpr int kZWarp = kScanThreads / 32;          // gated output: warp 10 loads the gate rows
constexpr uint32_t kScanTmemCols = 512;
constexpr uint32_t kAccCol = 256;   // accumulator buffer a: Y_diag at 256 + 128 a, Y_A at +64

static_assert(sizeof(StateSmem) + 1024 <= 232448, "chunk state smem exceeds 227 KB");
static_assert(sizeof(ScanSmem) + 1024 + kZStageBytes <= 232448, "chunk scan smem exceeds 227 KB");

// Stage s: with an off-diagonal block (48 KB stages) s in {0, 1} in S01; otherwise (32 KB
// stages) s in 0..2 in S01 and 3..4 in the B tile's space.  h_in follows the x rows.
__device__ __forceinline__ uint8_t *scan_stage(ScanSmem &sm, int s, bool offd)
{
    if (offd) return sm.S01 + s * kStageBytes;
    return s < 3 ? sm.S01 + s * kStage32 : sm.R + (s - 3) * kStage32;
}
__device__ __forceinline__ int scan_hoff(bool offd) { return (offd ? 256 : 128) * kRowBytes; }

// Scale the 16-byte pieces [first, first + count * stride) of a bf16 smem tile in place; the
// factor of piece c is f(c).  Works on any swizzled layout whose rows are whole 128-byte lines.
template <int kCount, typename F>
__device__ __forceinline__ void scale_pieces(uint8_t *base, int first, int stride, F f)
{
    float wf[kCount];
#pragma unroll
    for (int m = 0; m < kCount; ++m) wf[m] = f(first + m * stride);   // independent: overlap
#pragma unroll
    for (int m = 0; m < kCount; ++m) {
        const int c = first + m * stride;
        const float w = wf[m];
        uint4 *ptr = reinterpret_cast<uint4 *>(base) + c;
        uint4 v = *ptr;
        uint32_t *wv = &v.x;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&wv[e]));
            const float2 sc = fmul2(x, make_float2(w, w));
            wv[e] = pack_bf16x2(sc.x, sc.y);
        }
        *ptr = v;
    }
}

// Work of one launch: for each 128-row tile class T of the chunks (T = 1, the tiles with an
// off-diagonal block, exists for Q = 256), the flat list of (batch, chunk, group, head) items,
// heads of a group consecutive.  One CTA per SM: CTAs [0, ncta1) take the T = 1 items, the next
// ones the T = 0 items, each an equal run of its class's list.  For Q = 256 the two classes get
// the same number of CTAs and the same runs, so CTA i of each class walks the same heads in the
// same order at about the same time: both tiles of a head read x rows 0-127 and the head's
// entering state, and the second read is then an L2 hit (with the classes split unevenly it was
// not: 415 MB of DRAM reads per launch at the 2.7B shape instead of 271 MB).  A second tile
// costs more than a first (twice the mask and P x work, and the scaling of x_off), so the last
// tail_q / 1024 of each second-tile run goes to a third group of CTAs, [2 ncta1, 3 ncta1).
// With one CTA per SM these start only as SMs free up, which the first-tile CTAs do first, when
// the second-tile CTAs are nearly at their tails: both classes then end together, and the
// tails' x rows are still in L2.  No CTA waits for another, so the order in which the CTAs
// start matters for time only.  A run of items of the same (batch, chunk, group) is a segment: its heads share the C and B tiles and C B^T, which
// the CTA computes once per segment; the per-head pipeline runs on across segments, its barrier
// phases counted by a head counter that does not restart.
struct ScanWork {
    int T;               // tile class of this CTA
    int64_t f0, f1;      // its run of items
};
__device__ __forceinline__ ScanWork scan_work(int nT, int ncta1, int64_t nitems, int tail_q)
{
    ScanWork w;
    int idx = blockIdx.x, m = gridDim.x;
    if (nT == 2 && (int)blockIdx.x < ncta1) {
        w.T = 1;
        m = ncta1;
    } else {
        w.T = 0;
        if (nT == 2) {
            idx -= ncta1;
            m = ncta1;
        }
    }
    const int tail = nT == 2 && idx >= m;   // the tails of the second-tile runs
    if (tail) {
        w.T = 1;
        idx -= m;
    }
    const int64_t f0 = (int64_t)idx * nitems / m, f1 = ((int64_t)idx + 1) * nitems / m;
    const int64_t nt = w.T ? (f1 - f0) * tail_q / 1024 : 0;
    w.f0 = tail ? f1 - nt : f0;
    w.f1 = tail ? f1 : f1 - nt;
    return w;
}

// The segment that starts at item f of a CTA's run [.., f1): its (batch, chunk, group), first
// head and head count, and its chunk's span.  A segment whose tile lies past the end of its
// chunk (a short last chunk, an unused slot of a chunk table) is skipped by every role alike.
struct Seg {
    int64_t b, k, t0;
    int g, h0, nh, len;
    bool skip;
};
__device__ __forceinline__ Seg scan_segment(int64_t f, int64_t f1, int hpg, int G,
                                            int64_t nchunks, int Q, int64_t seqlen, int T,
                                            const int2 *tab)
{
    Seg sg;
    const int64_t id = f / hpg;
    const int64_t hi = min(f1, (id + 1) * hpg);
    sg.g = (int)(id % G);
    const int64_t bk = id / G;
    sg.k = bk % nchunks;
    sg.b = bk / nchunks;
    sg.h0 = sg.g * hpg + (int)(f % hpg);
    sg.nh = (int)(hi - f);
    chunk_span(tab, sg.k, Q, seqlen, sg.t0, sg.len);
    sg.skip = T * kTileRows >= sg.len;
    return sg;
}

template <bool kGate>   // kGate: the output is y * z * sigmoid(z)
__global__ void __launch_bounds__(kGate ? kScanThreads + 32 : kScanThreads, 1)
chunk_scan_tc_kernel(const __grid_constant__ CUtensorMap tm_x,
                     const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_c,
                     const __grid_constant__ CUtensorMap tm_x2,
                     const __grid_constant__ CUtensorMap tm_z, const bf16 *__restrict__ hin,
                     const float *__restrict__ dtc,
                     const float *__restrict__ cs, const float *__restrict__ D,
                     bf16 *__restrict__ y, int *__restrict__ status, int64_t seqlen, int H,
                     int G, int Q, int64_t nchunks, int64_t nitems, int ncta1,
                     const int2 *__restrict__ tab, const bf16 *__restrict__ z, int tail_q,
                     int skip_cta)
{
    extern __shared__ uint8_t smem_raw[];
    ScanSmem &sm = *reinterpret_cast<ScanSmem *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *zst = reinterpret_cast<uint8_t *>(&sm) + sizeof(ScanSmem);   // gate rows (kGate)
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    const int nT = Q / kTileRows;
    const ScanWork wk = scan_work(nT, ncta1, nitems, tail_q);
    const int T = wk.T;
    const int hpg = H / G;
    if (wk.f1 <= wk.f0) return;
    const bool offd = T != 0;            // the second tile has an off-diagonal block
    const int KI = offd ? 2 * kTileRows : kTileRows;  // source columns (x rows) of the tile
    const int nst = offd ? 2 : kXStagesMax;   // x / h_in stages
    const uint32_t gdiag = offd ? 128u : 0u;  // TMEM column of the diagonal block of C B^T
    const uint32_t pcol = offd ? 0u : 128u;   // TMEM columns of the P ring (over C B_off^T)
    const int xdiag = offd ? kTileRows : 0;   // first x row of the diagonal block in the stage

#define segment(f) scan_segment((f), wk.f1, hpg, G, nchunks, Q, seqlen, T, tab)

    if (threadIdx.x == 0) {
        mbar_init(&sm.bar_cb, 1);
        mbar_init(&sm.bar_g, 1);
        mbar_init(&sm.bar_goff, kScanWorkers);
        mbar_init(&sm.bar_seg_done, 1);
        for (int s = 0; s < kXStagesMax; ++s) {
            mbar_init(&sm.bar_xh_full[s], 1);
            mbar_init(&sm.bar_xh_free[s], 1);
            mbar_init(&sm.bar_xv_ready[s], kScanWorkers);
        }
        for (int s = 0; s < kScanVecStages; ++s) {
            mbar_init(&sm.bar_vec_full[s], 1);
            mbar_init(&sm.bar_vec_free[s], kScanWorkers);
        }
        for (int s = 0; s < kRing; ++s) {
            mbar_init(&sm.bar_slot_full[s], kScanWorkers);
            mbar_init(&sm.bar_slot_free[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&sm.bar_acc_full[a], 1);
            mbar_init(&sm.bar_acc_free[a], kScanWorkers);
        }
        mbar_init(&sm.bar_z_full, 1);
        mbar_init(&sm.bar_z_free, kScanWorkers);
        mbar_init(&sm.bar_drain, 1);
        sm.abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, kScanTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (threadIdx.x == 0) griddep_launch_dependents();
    const uint32_t tmem = sm.tmem_base;
    volatile int *abort = &sm.abort;

    if (warp == 0) {
        // ---------------- TMA producer (lane 0 alone): per segment the C and B tiles, per
        // head its cs / dt rows and its x / h_in stage
        if (lane == 0) {
            tma_prefetch_desc(&tm_x);
            tma_prefetch_desc(&tm_b);
            tma_prefetch_desc(&tm_c);
            tma_prefetch_desc(&tm_x2);
            if (kGate) tma_prefetch_desc(&tm_z);
            uint32_t J = 0;   // heads issued so far (all segments)
            int si = 0;       // segments whose tiles were loaded
            bool ok = true;
            for (int64_t f = wk.f0; ok && f < wk.f1;) {
                const Seg sg = segment(f);
                f += sg.nh;
                if (sg.skip) continue;
                // the previous segment's MMAs must be done with the C tile and the B space
                if (si > 0 && !mbar_wait(&sm.bar_seg_done, (si - 1) & 1, abort)) break;
                mbar_arrive_expect_tx(&sm.bar_cb, (uint32_t)(2 * kBoxBytes + 2 * KI * kRowBytes));
                for (int a = 0; a < 2; ++a)
                    tma_load_4d(&sm.Cs[a][0], &tm_c, &sm.bar_cb, 64 * a, sg.g,
                                (int)(sg.t0 + kTileRows * T), (int)sg.b);
                for (int a = 0; a < 2; ++a)
                    for (int r = 0; r < KI / kTileRows; ++r)
                        tma_load_4d(sm.R + a * KI * kRowBytes + r * kBoxBytes, &tm_b, &sm.bar_cb,
                                    64 * a, sg.g, (int)(sg.t0 + kTileRows * r), (int)sg.b);
                // the next segment's C and B tiles into L2 now, so that their loads after this
                // segment's last MMA are short
                if (f < wk.f1) {
                    const Seg nx = segment(f);
                    if (!nx.skip)
                        for (int a = 0; a < 2; ++a) {
                            tma_prefetch_l2_4d(&tm_c, 64 * a, nx.g,
                                               (int)(nx.t0 + kTileRows * T), (int)nx.b);
                            for (int r = 0; r < KI / kTileRows; ++r)
                                tma_prefetch_l2_4d(&tm_b, 64 * a, nx.g,
                                                   (int)(nx.t0 + kTileRows * r), (int)nx.b);
                        }
                }
                if (si == 0) {
                    // x is an input of the scan: start streaming the first heads' tiles into
                    // L2 while the state-passing kernel finishes
                    for (int j = 0; j < sg.nh && j < nst; ++j)
                        tma_prefetch_l2_4d(offd ? &tm_x2 : &tm_x, 0, sg.h0 + j, (int)sg.t0,
                                           (int)sg.b);
                    griddep_wait();   // cs / dt and the entering states come from earlier kernels
                }
                const bf16 *hblk = hin + (sg.b * nchunks + sg.k) * (int64_t)H * (kP * kN);
                bool waited_g = false;
                for (int j = 0; j < sg.nh; ++j, ++J) {
                    const int h = sg.h0 + j;
                    const int vs = J % kScanVecStages;
                    const uint32_t vu = J / kScanVecStages;
                    if (J >= kScanVecStages &&
                        !mbar_wait(&sm.bar_vec_free[vs], (vu - 1) & 1, abort)) {
                        ok = false;
                        break;
                    }
                    const int64_t vrow = ((sg.b * nchunks + sg.k) * H + h) * (int64_t)Q;
                    mbar_arrive_expect_tx(&sm.bar_vec_full[vs], (uint32_t)(8 * Q));
                    bulk_load(sm.cs_v[vs], cs + vrow, Q * 4, &sm.bar_vec_full[vs]);
                    bulk_load(sm.dt_v[vs], dtc + vrow, Q * 4, &sm.bar_vec_full[vs]);
                    const int xs = J % nst;
                    const uint32_t xu = J / nst;
                    if (J >= (uint32_t)nst &&
                        !mbar_wait(&sm.bar_xh_free[xs], (xu - 1) & 1, abort)) {
                        ok = false;
                        break;
                    }
                    if (!offd && xs >= 3 && !waited_g) {
                        // the B tile's space is in use until this segment's C B^T is done
                        if (!mbar_wait(&sm.bar_g, si & 1, abort)) {
                            ok = false;
                            break;
                        }
                        waited_g = true;
                    }
                    // failure injection (tests only): this stage is left unissued
                    if (J == 0 && (int)blockIdx.x == skip_cta) continue;
                    uint8_t *stg = scan_stage(sm, xs, offd);
                    mbar_arrive_expect_tx(&sm.bar_xh_full[xs],
                                          (uint32_t)(KI * kRowBytes + 2 * kP * kRowBytes));
                    // x rows [0, KI) of the chunk as one box (fewer, larger TMA boxes stream
                    // faster); h_in is stored in its shared-memory layout, so one contiguous copy
                    tma_load_4d(stg, offd ? &tm_x2 : &tm_x, &sm.bar_xh_full[xs], 0, h,
                                (int)sg.t0, (int)sg.b);
                    bulk_load(stg + scan_hoff(offd), hblk + (int64_t)h * (kP * kN), kP * kN * 2,
                              &sm.bar_xh_full[xs]);
                    // the operands this stage will hold next: into L2 now (the same segment's
                    // heads only), so their loads are L2 hits
                    if (j + nst < sg.nh) {
                        tma_prefetch_l2_4d(offd ? &tm_x2 : &tm_x, 0, h + nst, (int)sg.t0,
                                           (int)sg.b);
                        bulk_prefetch_l2(hblk + (int64_t)(h + nst) * (kP * kN), kP * kN * 2);
                    }
                    // the gate rows this tile's epilogue will read: into L2 now
                    if (kGate)
                        tma_prefetch_l2_4d(&tm_z, 0, h, (int)(sg.t0 + kTileRows * T), (int)sg.b);
                }
                ++si;
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (lane 0 alone runs the loop: a lane that issued
        // tcgen05.mma and then rejoins its warp stalls for the MMAs' issue latency)
        const uint32_t id_g = idesc_bf16_f32(128, KI, false, false);
        const uint32_t id_kk = idesc_bf16_f32(128, kP, false, false);   // K-major A and B
        const uint32_t id_kmn = idesc_bf16_f32(128, kP, false, true);   // B (x) MN-major
        // base descriptors; K steps are constant offsets added in fully unrolled loops (the
        // issuing thread's own instruction chain sets the MMA issue rate)
        const uint64_t cd = smem_desc_sw128(smem_u32(&sm.Cs[0][0]), 16, 1024);
        const uint64_t rd = smem_desc_sw128(smem_u32(sm.R), 16, 1024);
        bool ok = lane == 0;
        uint32_t J = 0;
        int si = 0;
        for (int64_t f = wk.f0; ok && f < wk.f1;) {
            const Seg sg = segment(f);
            f += sg.nh;
            if (sg.skip) continue;
            if (!mbar_wait(&sm.bar_cb, si & 1, abort)) break;
            tc_fence_after();
            // G = C B^T: M = 128 rows t, N = KI columns i, K = 128 (n).  It overwrites the P
            // ring and C B_off^T of the previous segment only after this thread's earlier MMAs,
            // which read them, were issued (in order).
#pragma unroll
            for (int kk = 0; kk < kN / 16; ++kk) {
                const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
                const uint32_t boff = (kk >> 2) * KI * kRowBytes + (kk & 3) * 32;
                mma_bf16(tmem, cd + (off >> 4), rd + (boff >> 4), id_g, kk > 0 ? 1u : 0u);
            }
            mma_commit(&sm.bar_g);
            if (offd && !mbar_wait(&sm.bar_goff, si & 1, abort)) break;   // bf16 C B_off^T
            for (int j = 0; ok && j < sg.nh; ++j, ++J) {
                const int xs = J % nst;
                const uint32_t xu = J / nst;
                const int a = J & 1;
                if (!mbar_wait(&sm.bar_xh_full[xs], xu & 1, abort)) { ok = false; break; }
                if (offd && !mbar_wait(&sm.bar_xv_ready[xs], xu & 1, abort)) { ok = false; break; }
                if (J >= 2 && !mbar_wait(&sm.bar_acc_free[a], ((J >> 1) - 1) & 1, abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t stg = smem_u32(scan_stage(sm, xs, offd));
                const uint32_t dD = tmem + kAccCol + 128 * a, dA = dD + 64;
                const uint64_t xd = smem_desc_sw128(stg, 256 * kRowBytes, 1024);   // x, MN-major
                const uint64_t hd = smem_desc_sw128(stg + scan_hoff(offd), 16, 1024);  // h_in
                if (offd) {
                    // Y_A = (C B_off^T) (v dt o X_off): A = bf16 block in R, K = 128 (i)
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t aoff = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
                        mma_bf16(dA, rd + (aoff >> 4), xd + kk * 128, id_kmn, kk > 0 ? 1u : 0u);
                    }
                }
                // Y_A (+)= C h^T: K = 128 (n), h K-major (rows p, two halves of 64 n);
                // h = h_in (T = 0) or exp(cs_127) h_in (T = 1)
#pragma unroll
                for (int kk = 0; kk < kN / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
                    const uint32_t hoff = (kk >> 2) * (kP * kRowBytes) + (kk & 3) * 32;
                    mma_bf16(dA, cd + (off >> 4), hd + (hoff >> 4), id_kk,
                             (offd || kk > 0) ? 1u : 0u);
                }
                for (int qb = 0; qb < 2; ++qb) {
                    const uint32_t blk = 2 * J + qb;           // P blocks are numbered per head
                    const uint32_t slot = blk % kRing, su = blk / kRing;
                    if (!mbar_wait(&sm.bar_slot_full[slot], su & 1, abort)) { ok = false; break; }
                    tc_fence_after();
                    // Y_diag += P[:, 64qb : +64] X[xdiag + 64qb : +64, :], P read from TMEM
                    const uint32_t pa = tmem + pcol + 32 * slot;
                    const uint64_t bd = xd + (uint64_t)((xdiag / 16 + qb * 4) * 128);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16_ts(dD, pa + 8 * kk, bd + kk * 128, id_kmn,
                                    (qb | kk) != 0 ? 1u : 0u);
                    mma_commit(&sm.bar_slot_free[slot]);
                }
                if (!ok) break;
                mma_commit(&sm.bar_acc_full[a]);
                mma_commit(&sm.bar_xh_free[xs]);
            }
            if (!ok) break;
            mma_commit(&sm.bar_seg_done);   // this segment's MMAs are done with C and R
            ++si;
        }
    } else if (kGate && warp == kZWarp) {
        // ---------------- gate rows (lane 0 alone): each head's into the z stage, in the
        // workers' order, as soon as the epilogue of the previous head has read the stage
        if (lane == 0) {
            uint32_t Jz = 0;
            bool ok = true;
            for (int64_t f = wk.f0; ok && f < wk.f1;) {
                const Seg sg = segment(f);
                f += sg.nh;
                if (sg.skip) continue;
                for (int j = 0; j < sg.nh; ++j, ++Jz) {
                    if (Jz >= 1 && !mbar_wait(&sm.bar_z_free, (Jz - 1) & 1, abort)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&sm.bar_z_full, (uint32_t)kZStageBytes);
                    tma_load_4d(zst, &tm_z, &sm.bar_z_full, 0, sg.h0 + j,
                                (int)(sg.t0 + kTileRows * T), (int)sg.b);
                }
            }
        }
    } else if (warp >= 2) {
        // ---------------- workers, two per TMEM lane quarter.  Warp (qd, cq) owns rows
        // t = 32 qd + lane of the tile and the 32-column slice [32 cq, 32 cq + 32) of every
        // 64-column block: per head it builds that slice of both P blocks (mask; for T = 1 after
        // its share of scaling x_off and h_in), then the epilogue y = Y_diag + f_t Y_A of the
        // previous head for output columns [32 cq, 32 cq + 32).
        const int wt = threadIdx.x - 64;           // 0 .. kScanWorkers - 1
        const int qd = warp & 3;
        const int cq = (warp - 2) >> 2;
        const int t = qd * 32 + lane;             // row within the tile = TMEM lane
        const int tau = kTileRows * T + t;        // row within the chunk
        const int r = kTileRows * T + qd * 32 - 1;  // last row above this warp's 32-row slice
        const uint32_t lane_base = tmem + ((uint32_t)(qd * 32) << 16);
        float *vt = sm.vt[warp - 2];
        // The slice of block qb is the 32-column unit u = 2 qb + cq of the diagonal block; its
        // class relative to this row quarter: 0 below the 32 x 32 diagonal sub-block, 1 the
        // sub-block itself, 2 above it (all zero).
        const int u0 = cq, u1 = 2 + cq;
        const int cls0 = u0 < qd ? 0 : (u0 == qd ? 1 : 2);
        const int cls1 = u1 < qd ? 0 : (u1 == qd ? 1 : 2);
        bool ok = true;
        uint32_t J = 0;
        int si = 0;
        for (int64_t f = wk.f0; ok && f < wk.f1;) {
            const Seg sg = segment(f);
            f += sg.nh;
            if (sg.skip) continue;
            ok = warp_wait(&sm.bar_g, si & 1, abort);
            if (!ok) break;
            tc_fence_after();
            if (offd) {
                // C B_off^T (TMEM columns [0, 128)) -> bf16, K-major swizzled tile in R; this
                // warp converts its 32 rows x columns [64 cq, 64 cq + 64) (one 64-column atom)
                uint8_t *dst = sm.R + cq * kBoxBytes + t * kRowBytes;
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    uint32_t gv[32];
                    tmem_ld32(lane_base + 64 * cq + 32 * e, gv);
                    tmem_ld_wait();
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const int pos = (e * 4 + m) ^ (t & 7);
                        *reinterpret_cast<uint4 *>(dst + pos * 16) = make_uint4(
                            pack_bf16x2(__uint_as_float(gv[8 * m]), __uint_as_float(gv[8 * m + 1])),
                            pack_bf16x2(__uint_as_float(gv[8 * m + 2]), __uint_as_float(gv[8 * m + 3])),
                            pack_bf16x2(__uint_as_float(gv[8 * m + 4]), __uint_as_float(gv[8 * m + 5])),
                            pack_bf16x2(__uint_as_float(gv[8 * m + 6]), __uint_as_float(gv[8 * m + 7])));
                    }
                }
                fence_async_smem();
                tc_fence_before();
                mbar_arrive(&sm.bar_goff);
                // the P ring reuses these TMEM columns: wait until every warp has read them
                ok = warp_wait(&sm.bar_goff, si & 1, abort);
                if (!ok) break;
                tc_fence_after();
            }
            const uint32_t J0 = J;   // first head of the segment
            const int snh = sg.nh;
            const int sh0 = sg.h0;
            const bool row_in = tau < sg.len;   // this thread's row exists in the chunk
            // output row tau of the segment's first head, this warp's 32 columns
            const int64_t yseg = ((sg.b * seqlen + sg.t0 + tau) * H + sh0) * (int64_t)kP + 32 * cq;
            for (int j = 0; ok && j <= snh; ++j) {
                if (j < snh) {
                    const uint32_t Jj = J0 + j;
                    const int vs = Jj % kScanVecStages;
                    if (!warp_wait(&sm.bar_vec_full[vs], (Jj / kScanVecStages) & 1, abort)) {
                        ok = false;
                        break;
                    }
                    const float *cs_s = sm.cs_v[vs];
                    const float *dt_s = sm.dt_v[vs];
                    if (offd) {
                        // x rows [0, 128) *= exp(cs_127 - cs_i) dt_i; h_in *= exp(cs_127)
                        const int xs = Jj % nst;
                        if (!warp_wait(&sm.bar_xh_full[xs], (Jj / nst) & 1, abort)) {
                            ok = false;
                            break;
                        }
                        uint8_t *stg = scan_stage(sm, xs, offd);
                        // reference row 127 (x rows * exp(cs_127 - cs_i) dt_i, h_in *
                        // exp(cs_127)), or, where the chunk decays by at most exp(kRef0Floor),
                        // reference "row -1" (x rows * exp(-cs_i) dt_i, h_in as it is): all
                        // factors then lie in [exp(kRef0Floor), exp(-kRef0Floor)], and the h_in
                        // pass is saved
                        const float ref = scan_ref0(cs_s[Q - 1]) ? 0.f : cs_s[127];
                        scale_pieces<1024 / kScanWorkers>(stg, wt, kScanWorkers, [&](int c) {
                            const int i = c >> 3;
                            return __expf(ref - cs_s[i]) * dt_s[i];
                        });
                        if (ref != 0.f) {
                            const float sh = __expf(ref);
                            scale_pieces<1024 / kScanWorkers>(stg + scan_hoff(offd), wt,
                                                              kScanWorkers,
                                                              [&](int) { return sh; });
                        }
                        fence_async_smem();
                        mbar_arrive(&sm.bar_xv_ready[xs]);
                    }
                    const float Dh = D[sh0 + j];
                    const float ct = cs_s[tau];
                    // Row and column factors: below the 32 x 32 diagonal sub-block relative to
                    // row r, both <= 1; inside it relative to m = r + 1, the slice's first row:
                    // exp(cs_m - cs_i) <= exp(32 max|dt A|) and exp(cs_t - cs_m) <= 1, so
                    // neither over- nor underflows, and no element needs an exponential of its
                    // own.
                    const float cm = cs_s[r + 1];
                    const float crf = cs_s[r < 0 ? 0 : r];
                    const float um = __expf(ct - cm);
                    const float uf = qd > 0 ? __expf(ct - crf) : 0.f;
#pragma unroll
                    for (int qb = 0; qb < 2; ++qb) {
                        // lane l: column 32 u + l of the diagonal block, u = 2 qb + cq
                        const int uu = 2 * qb + cq;
                        const int cl = uu < qd ? 0 : (uu == qd ? 1 : 2);
                        const int i = kTileRows * T + 32 * uu + lane;
                        const float ref = cl == 0 ? crf : cm;
                        const float v = __expf(ref - cs_s[i]) * dt_s[i];
                        vt[32 * qb + lane] = cl < 2 ? v : 0.f;
                    }
                    __syncwarp();
#pragma unroll
                    for (int qb = 0; qb < 2; ++qb) {
                        const uint32_t blk = 2 * Jj + qb;
                        const uint32_t slot = blk % kRing, su = blk / kRing;
                        const int cl = qb ? cls1 : cls0;
                        const float *vq = vt + 32 * qb;
                        // this warp's part of the diagonal block of C B^T: it stays in TMEM for
                        // the whole segment (the P ring and the accumulators use other
                        // columns), so it is read again per head instead of held in registers
                        uint32_t gv[32];
                        if (cl < 2) {
                            tmem_ld32(lane_base + gdiag + 32 * (qb ? u1 : u0), gv);
                            tmem_ld_wait();
                        }
                        uint32_t pk[16];
                        if (cl == 0) {
                            const float2 uu = make_float2(uf, uf);
#pragma unroll
                            for (int c = 0; c < 8; ++c) {
                                const float4 vv = *reinterpret_cast<const float4 *>(vq + 4 * c);
                                const float2 p0 = fmul2(
                                    fmul2(make_float2(__uint_as_float(gv[4 * c]),
                                                      __uint_as_float(gv[4 * c + 1])),
                                          make_float2(vv.x, vv.y)), uu);
                                const float2 p1 = fmul2(
                                    fmul2(make_float2(__uint_as_float(gv[4 * c + 2]),
                                                      __uint_as_float(gv[4 * c + 3])),
                                          make_float2(vv.z, vv.w)), uu);
                                pk[2 * c] = pack_bf16x2(p0.x, p0.y);
                                pk[2 * c + 1] = pack_bf16x2(p1.x, p1.y);
                            }
                        } else if (cl == 1) {
                            // the causal 32 x 32 sub-block: local column lc kept for lc <= lane,
                            // + D at lc = lane
                            const float2 uu = make_float2(um, um);
#pragma unroll
                            for (int c = 0; c < 16; ++c) {
                                const float2 ww = *reinterpret_cast<const float2 *>(vq + 2 * c);
                                float2 pp = fmul2(fmul2(make_float2(__uint_as_float(gv[2 * c]),
                                                                    __uint_as_float(gv[2 * c + 1])),
                                                        ww), uu);
                                const int lc = 2 * c;
                                pp.x = (lc <= lane) ? pp.x : 0.f;
                                pp.y = (lc + 1 <= lane) ? pp.y : 0.f;
                                pp.x += (lc == lane) ? Dh : 0.f;
                                pp.y += (lc + 1 == lane) ? Dh : 0.f;
                                pk[c] = pack_bf16x2(pp.x, pp.y);
                            }
                        } else {
#pragma unroll
                            for (int c = 0; c < 16; ++c) pk[c] = 0u;
                        }
                        if (su >= 1 &&
                            !warp_wait(&sm.bar_slot_free[slot], (su - 1) & 1, abort)) {
                            ok = false;
                            break;
                        }
                        // a slice above the diagonal is all zero; a slot always holds the same
                        // block qb and so the same slices, so once its zeros are written (by
                        // the segment's first two heads: C B^T of a tile with an off-diagonal
                        // block overwrites the ring at every segment) they stay
                        if (cl != 2 || j < 2) {
                            tmem_st16(lane_base + pcol + 32 * slot + 16 * cq, pk);
                            tmem_st_wait();
                        }
                        tc_fence_before();
                        mbar_arrive(&sm.bar_slot_full[slot]);
                    }
                    if (!ok) break;
                }
                if (j >= 1) {
                    // epilogue of head jj = j - 1 for output columns [32 cq, 32 cq + 32)
                    const uint32_t Jj = J0 + j - 1;
                    const int a = Jj & 1;
                    const int64_t yoff = yseg + (int64_t)(j - 1) * kP;
                    // gated output (z given): y * z * sigmoid(z), z as packed bf16 pairs, this
                    // thread's four 16-byte pieces of row t read from the z stage (swizzled)
                    // before the accumulator wait
                    const bool gz = kGate && row_in;
                    uint4 zq[4];
                    if (kGate) {
                        if (!warp_wait_each(&sm.bar_z_full, Jj & 1, abort)) {
                            ok = false;
                            break;
                        }
                        const uint8_t *zrow = zst + t * kRowBytes;
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            zq[q] = *reinterpret_cast<const uint4 *>(
                                zrow + (((4 * cq + q) ^ (t & 7)) << 4));
                        // the next head's rows arrive by TMA (the async proxy): order these
                        // reads before it
                        fence_async_smem();
                        mbar_arrive(&sm.bar_z_free);
                    } else {
#pragma unroll
                        for (int q = 0; q < 4; ++q) zq[q] = make_uint4(0u, 0u, 0u, 0u);
                    }
                    if (!warp_wait(&sm.bar_acc_full[a], (Jj >> 1) & 1, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t col = lane_base + kAccCol + 128 * a + 32 * cq;
                    uint32_t d0[32], a0[32];
                    tmem_ld32(col, d0);
                    tmem_ld32(col + 64, a0);
                    const int vs = Jj % kScanVecStages;
                    const float *cs_j = sm.cs_v[vs];
                    const float fct =
                        __expf(cs_j[tau] - (T && !scan_ref0(cs_j[Q - 1]) ? cs_j[127] : 0.f));
                    tmem_ld_wait();
                    tc_fence_before();
                    mbar_arrive(&sm.bar_acc_free[a]);
                    // done with this head's cs / dt rows, which the producer's next bulk copy
                    // (the async proxy) overwrites: order these reads before it
                    fence_async_smem();
                    mbar_arrive(&sm.bar_vec_free[vs]);
                    uint4 *yrow = reinterpret_cast<uint4 *>(y + yoff);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {   // 8 columns per 16-byte store
                        const uint32_t zw[4] = {zq[q].x, zq[q].y, zq[q].z, zq[q].w};
                        uint32_t pk[4];
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const int e = 8 * q + 2 * c;
                            float v0 = fmaf(fct, __uint_as_float(a0[e]), __uint_as_float(d0[e]));
                            float v1 = fmaf(fct, __uint_as_float(a0[e + 1]),
                                            __uint_as_float(d0[e + 1]));
                            if (gz) {
                                const float2 zf = __bfloat1622float2(
                                    *reinterpret_cast<const __nv_bfloat162 *>(&zw[c]));
                                v0 *= silu_approx(zf.x);
                                v1 *= silu_approx(zf.y);
                            }
                            pk[c] = pack_bf16x2(v0, v1);
                        }
                        if (row_in) yrow[q] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    }
                }
            }
            J = J0 + snh;
            ++si;
        }
    }
    __syncthreads();
    if (sm.abort) {
        if (warp == 1 && lane == 0) {
            mma_commit(&sm.bar_drain);
            mbar_wait_drain(&sm.bar_drain, 0);
        }
        if (threadIdx.x == 0) {
            drain_sleep();
            atomicOr(status, 2);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kScanTmemCols);
    }
}
#undef segment

// ============================================================ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// bf16 tensor map, 128-byte swizzle, box inner extent 64 elements (128 bytes).
bool make_map(CUtensorMap *m, const void *ptr, int rank, const cuuint64_t *dims,
              const cuuint64_t *strides_bytes, const cuuint32_t *box)
{
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void *>(ptr),
              dims, strides_bytes, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// (batch, seqlen, heads_or_groups, 64 * m) bf16 -> 4-D map {inner, heads, seqlen, batch} with
// a 64 x 1 x 128 x 1 box.
bool make_seq_map(CUtensorMap *m, const void *ptr, int64_t batch, int64_t seqlen, int64_t mid,
                  int64_t inner, int box_rows = kTileRows)
{
    const cuuint64_t dims[4] = {(cuuint64_t)inner, (cuuint64_t)mid, (cuuint64_t)seqlen,
                                (cuuint64_t)batch};
    const cuuint64_t strides[3] = {(cuuint64_t)(inner * 2), (cuuint64_t)(mid * inner * 2),
                                   (cuuint64_t)(seqlen * mid * inner * 2)};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
    return make_map(m, ptr, 4, dims, strides, box);
}

}  // namespace

bool tc_supported(bool is_bf16, int P, int N, int Q)
{
    return is_bf16 && P == kP && N == kN && (Q == 128 || Q == 256);
}

cudaError_t launch_chunk_state_tc(const bf16 *x, const float *dtc, const bf16 *B,
                                  const float *cs, float *states, int *status, int64_t batch,
                                  int64_t seqlen, int H, int G, int Q, int64_t nchunks,
                                  cudaStream_t st, const char **why, const int2 *tab, bool split,
                                  bool rev)
{
    if ((split && Q != 64) || (!split && Q != 128 && Q != 256) || (rev && (tab || !split))) {
        *why = "chunk state: unsupported chunk / split / reversal combination";
        return cudaErrorInvalidValue;
    }
    CUtensorMap mx, mb;   // boxes of a whole chunk (Q rows)
    if (!make_seq_map(&mx, x, batch, seqlen, H, kP, Q) ||
        !make_seq_map(&mb, B, batch, seqlen, G, kN, Q)) {
        *why = "chunk state: cuTensorMapEncodeTiled failed";
        return cudaErrorInvalidValue;
    }
    const int64_t nitems = batch * nchunks * H;   // (batch, chunk, group, head) items
    if (nitems == 0) return cudaSuccess;
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const size_t smem = sizeof(StateSmem) + 1024;
    auto kern = !split ? chunk_state_tc_kernel<false, false>
                       : (rev ? chunk_state_tc_kernel<true, true>
                              : chunk_state_tc_kernel<true, false>);
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) { *why = "chunk state: set smem attribute"; return e; }
    const unsigned grid = (unsigned)std::min<int64_t>(sms, nitems);
    *why = "chunk state (tcgen05) launch";
    return launch_pdl(kern, grid, kStateThreads, smem, st, mx, mb, dtc, cs,
                      states, status, H, G, Q, nchunks, nitems, seqlen, tab,
                      take_test_skip(kTestChunkState));
}

// The share (per 1024) of each second-tile run that a third group of CTAs takes (see scan_work).
// Measured at the 2.7B-layer shape (80 heads per group: the C and B tiles and C B^T computed
// once per 80 heads) and at b = 1, L = 65536, 32 heads in 8 groups (4 heads per group, where
// the second tile's per-segment work, C B^T over 256 columns and its bf16 copy, weighs more);
// the gated output (a longer epilogue in both tile classes) at the 2.7B-layer shape.
constexpr int kTailLongSeg = 64, kTailShortSeg = 128;
constexpr int kTailLongSegGated = 96;
static int scan_tail(int heads_per_group, bool gated)
{
    if (gated && heads_per_group >= 16) return kTailLongSegGated;
    return heads_per_group >= 16 ? kTailLongSeg : kTailShortSeg;
}

cudaError_t launch_chunk_scan_tc(const bf16 *x, const float *dtc, const bf16 *B, const bf16 *C,
                                 const float *cs, const bf16 *hin, const float *D, bf16 *y,
                                 int *status, int64_t batch, int64_t seqlen, int H, int G,
                                 int Q, int64_t nchunks, cudaStream_t st, const char **why,
                                 const int2 *tab, const bf16 *z)
{
    CUtensorMap mx, mx2, mb, mc, mz;
    if (z) {
        if (!make_seq_map(&mz, z, batch, seqlen, H, kP)) {
            *why = "chunk scan: cuTensorMapEncodeTiled failed (z)";
            return cudaErrorInvalidValue;
        }
    } else {
        mz = {};
    }
    if (!make_seq_map(&mx, x, batch, seqlen, H, kP) ||
        !make_seq_map(&mx2, x, batch, seqlen, H, kP, 2 * kTileRows) ||
        !make_seq_map(&mb, B, batch, seqlen, G, kN) ||
        !make_seq_map(&mc, C, batch, seqlen, G, kN)) {
        *why = "chunk scan: cuTensorMapEncodeTiled failed";
        return cudaErrorInvalidValue;
    }
    const int64_t nitems = batch * nchunks * H;   // (batch, chunk, group, head) items per class
    if (nitems == 0) return cudaSuccess;
    const int nT = Q / kTileRows;
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // Q = 256: half the SMs per tile class, with identical runs, and a third group of CTAs for
    // the tails of the second-tile runs (see scan_work)
    const int per = (int)std::min<int64_t>(nT == 2 ? sms / 2 : sms, nitems);
    const int grid = nT == 2 ? 3 * per : per;
    const int ncta1 = nT == 2 ? per : 0;
    const size_t smem = sizeof(ScanSmem) + 1024 + (z ? kZStageBytes : 0);
    auto kern = z ? chunk_scan_tc_kernel<true> : chunk_scan_tc_kernel<false>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) { *why = "chunk scan: set smem attribute"; return e; }
    *why = "chunk scan (tcgen05) launch";
    return launch_pdl(kern, (unsigned)grid, z ? kScanThreads + 32 : kScanThreads, smem, st, mx,
                      mb, mc, mx2, mz, hin,
                      dtc, cs, D, y, status, seqlen, H, G, Q, nchunks, nitems, ncta1, tab, z,
                      scan_tail(H / G, z != nullptr), take_test_skip(kTestChunkScan));
}

}  // namespace ssd
