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
//     One CTA per (batch, chunk, group, block of heads).  The chunk's B rows are loaded once and
//     shared by the heads of the block; per head, the x tile is TMA-loaded, scaled row by row
//     by w (CUDA cores, in shared memory), and one M=128 (n) x N=64 (p) x K=Q MMA chain
//     accumulates S^T in TMEM, double-buffered so that head j+1's MMAs run under head j's
//     TMEM -> global epilogue.
//
// chunk_scan_tc_kernel    y = (C B^T o L o dt + diag(D)) X  +  exp(cs) o (C h_in^T)
//     One CTA per (batch, chunk, 128-row tile of the chunk, group, block of heads).  G = C B^T
//     (128 x KI, KI = 128 * (tile + 1) causal columns) is computed once per CTA into TMEM and
//     shared by the heads (all heads of a group see the same B, C).  Per head the mask warps
//     read G from TMEM, apply the decay exp(cs_t - cs_i) dt_i (and D on the diagonal), round to
//     bf16 and write 64-column blocks of the K-major A operand into a 4-slot shared-memory ring
//     that the MMA thread consumes as it fills; the off-chunk term C h_in^T is a second TMEM
//     accumulator; the epilogue warps combine both as y = Y1 + exp(cs_t) Y2 and store bf16.
//     The decay is factorised to keep the exponentials off the inner loop: for columns i at or
//     before r (the row just above the warp's 32-row slice), exp(cs_t - cs_i) = exp(cs_t - cs_r)
//     * exp(cs_r - cs_i), both factors <= 1 (cs is non-increasing), so each element costs two
//     multiplies; only the 32 x 32 diagonal block evaluates exp per element.
//
// Roles (warp-specialised; every wait is on an mbarrier and bounded, see sm100.cuh):
//   state kernel: warp 0 TMA, warp 1 MMA, warp 2 TMEM owner, warps 4-7 scale + epilogue
//   scan  kernel: warp 0 TMA, warp 1 MMA, warp 2 TMEM owner, warps 4-7 mask, warps 8-11 epilogue
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "sm100.cuh"

namespace ssd {
namespace {

using namespace sm100;

constexpr int kP = 64;
constexpr int kN = 128;
constexpr int kHeadsPerCta = 8;
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

// ============================================================ chunk state
constexpr int kStateStages = 4;
struct alignas(1024) StateSmem {
    bf16 Bs[2][256 * 64];                 // MN-major A operand: [n atom][Q rows tau][64 n]
    bf16 Xs[kStateStages][256 * 64];      // MN-major B operand per stage: [Q rows tau][64 p]
    float cs_v[kStateStages][256];        // per stage: the head's chunk-local cumsum row
    float dt_v[kStateStages][256];        // per stage: the head's dt row (0 past the end)
    uint64_t bar_b;
    uint64_t bar_x_full[kStateStages], bar_x_ready[kStateStages], bar_x_free[kStateStages];
    uint64_t bar_acc_full[2], bar_acc_free[2];
    uint64_t bar_drain;
    uint32_t tmem_base;
    int abort;
};
// warp 0 TMA, warp 1 MMA, warp 2 TMEM owner, warp 3 idle, warps 4-11 scale x, warps 12-15 epilogue
constexpr int kStateThreads = 512;
constexpr int kStateScaleThreads = 256;
constexpr uint32_t kStateTmemCols = 128;

__global__ void __launch_bounds__(kStateThreads, 1)
chunk_state_tc_kernel(const __grid_constant__ CUtensorMap tm_x,
                      const __grid_constant__ CUtensorMap tm_b, const float *__restrict__ dtc,
                      const float *__restrict__ cs, float *__restrict__ states,
                      int *__restrict__ status, int H, int G, int Q, int64_t nchunks, int nhb)
{
    extern __shared__ uint8_t smem_raw[];
    StateSmem &sm = *reinterpret_cast<StateSmem *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    int64_t u = blockIdx.x;
    const int hb = (int)(u % nhb); u /= nhb;
    const int g = (int)(u % G); u /= G;
    const int64_t k = u % nchunks, b = u / nchunks;
    const int hpg = H / G;
    const int h0 = g * hpg + hb * kHeadsPerCta;
    const int nh = min(kHeadsPerCta, hpg - hb * kHeadsPerCta);
    const int64_t t0 = k * Q;
    const int nrb = Q / kTileRows;

    if (threadIdx.x == 0) {
        mbar_init(&sm.bar_b, 1);
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
    const uint32_t tmem = sm.tmem_base;
    volatile int *abort = &sm.abort;

    if (warp == 0) {
        // ---------------- TMA producer: B once, then per head its x tile and cs / dt rows
        if (lane == 0) {
            tma_prefetch_desc(&tm_x);
            tma_prefetch_desc(&tm_b);
            mbar_arrive_expect_tx(&sm.bar_b, 2u * Q * kRowBytes);
            for (int a = 0; a < 2; ++a)
                for (int r = 0; r < nrb; ++r)
                    tma_load_4d(&sm.Bs[a][r * kTileRows * 64], &tm_b, &sm.bar_b, 64 * a, g,
                                (int)(t0 + kTileRows * r), (int)b);
        }
        for (int j = 0; j < nh; ++j) {
            const int s = j % kStateStages;
            const uint32_t use = j / kStateStages;
            if (j >= kStateStages && !warp_wait(&sm.bar_x_free[s], (use - 1) & 1, abort)) break;
            if (lane == 0) {
                const int64_t vrow = ((b * nchunks + k) * H + h0 + j) * (int64_t)Q;
                mbar_arrive_expect_tx(&sm.bar_x_full[s], (uint32_t)Q * (kRowBytes + 8));
                for (int r = 0; r < nrb; ++r)
                    tma_load_4d(&sm.Xs[s][r * kTileRows * 64], &tm_x, &sm.bar_x_full[s], 0,
                                h0 + j, (int)(t0 + kTileRows * r), (int)b);
                bulk_load(sm.cs_v[s], cs + vrow, Q * 4, &sm.bar_x_full[s]);
                bulk_load(sm.dt_v[s], dtc + vrow, Q * 4, &sm.bar_x_full[s]);
            }
            __syncwarp();
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer: D[n][p] += sum_tau B[tau][n] * Xw[tau][p]
        const uint32_t idesc = idesc_bf16_f32(128, kP, true, true);
        const uint32_t atom_bytes = 256 * kRowBytes;  // distance between the two n atoms of Bs
        if (warp_wait(&sm.bar_b, 0, abort)) {
            for (int j = 0; j < nh; ++j) {
                const int s = j % kStateStages;
                const uint32_t use = j / kStateStages;
                const int a = j & 1;
                if (!warp_wait(&sm.bar_x_ready[s], use & 1, abort)) break;
                if (j >= 2 && !warp_wait(&sm.bar_acc_free[a], ((j >> 1) - 1) & 1, abort)) break;
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t d = tmem + a * kP;
                    const uint32_t a0 = smem_u32(&sm.Bs[0][0]), b0 = smem_u32(&sm.Xs[s][0]);
                    for (int kk = 0; kk < Q / 16; ++kk) {
                        const uint64_t ad = smem_desc_sw128(a0 + kk * 2048, atom_bytes, 1024);
                        const uint64_t bd = smem_desc_sw128(b0 + kk * 2048, atom_bytes, 1024);
                        mma_bf16(d, ad, bd, idesc, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&sm.bar_x_free[s]);
                    mma_commit(&sm.bar_acc_full[a]);
                }
                __syncwarp();
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
                const int tau = c >> 3;
                const float w = __expf(cs_last - sm.cs_v[s][tau]) * sm.dt_v[s][tau];
                uint4 *ptr = reinterpret_cast<uint4 *>(&sm.Xs[s][0]) + c;
                uint4 v = *ptr;
                uint32_t *wv = &v.x;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __bfloat1622float2(
                        *reinterpret_cast<const __nv_bfloat162 *>(&wv[e]));
                    const float2 sc = fmul2(f, make_float2(w, w));
                    wv[e] = pack_bf16x2(sc.x, sc.y);
                }
                *ptr = v;
            }
            fence_async_smem();
            mbar_arrive(&sm.bar_x_ready[s]);
        }
    } else if (warp >= 12) {
        // ---------------- epilogue: TMEM (lane n, column p) -> states[b][k][h][p][n]
        const int q = warp & 3;
        for (int j = 0; j < nh; ++j) {
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
            const int n = q * 32 + lane;
            float *out = states + ((b * nchunks + k) * H + h0 + j) * (int64_t)(kP * kN) + n;
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
constexpr int kXStages = 3;      // x / h_in stages; the third lives in the B tile's space
constexpr int kVecStages = 4;    // cs / dt row stages
constexpr int kRing = 4;         // 64-column blocks of P in TMEM
constexpr int kStageBytes = 256 * kRowBytes + 2 * kP * kRowBytes;  // x (<= 256 rows) + h_in
struct alignas(1024) ScanSmem {
    bf16 Cs[2][kTileRows * 64];     // K-major A (C tile): [n atom][128 rows t][64 n]
    uint8_t R[kStageBytes + 16384]; // B rows for C B^T (K-major [n atom][KI rows][64]); after
                                    // that, x / h_in stage 2
    uint8_t S01[2][kStageBytes];    // x / h_in stages 0 and 1: [KI rows i][64 p] then
                                    // [n atom][64 rows p][64 n]
    float cs_v[kVecStages][256];    // per stage: the head's chunk-local cumsum row
    float dt_v[kVecStages][256];    // per stage: the head's dt row (0 past the end)
    float vt[8][256];               // per mask warp: exp(cs_r - cs_i) dt_i
    float Dv[kHeadsPerCta];         // D of the CTA's heads
    uint64_t bar_cb, bar_g;
    uint64_t bar_xh_full[kXStages], bar_xh_free[kXStages];
    uint64_t bar_vec_full[kVecStages], bar_vec_free[kVecStages];
    uint64_t bar_slot_full[kRing], bar_slot_free[kRing];
    uint64_t bar_acc_full, bar_acc_free;
    uint64_t bar_drain;
    uint32_t tmem_base;
    int abort;
};
// warp 0 TMA, warp 1 MMA, warp 2 TMEM owner, warp 3 idle, warps 4-11 mask (two per TMEM lane
// quarter, splitting each 64-column block), warps 12-15 epilogue
constexpr int kScanThreads = 512;
constexpr uint32_t kScanTmemCols = 512;
constexpr uint32_t kPCol = 256;     // P ring: block slot s at columns [256 + 32 s, +32)
constexpr uint32_t kAccCol = 384;   // Y1 at [384, 448), Y2 at [448, 512)

static_assert(sizeof(StateSmem) + 1024 <= 232448, "chunk state smem exceeds 227 KB");
static_assert(sizeof(ScanSmem) + 1024 <= 232448, "chunk scan smem exceeds 227 KB");

__device__ __forceinline__ uint8_t *scan_stage(ScanSmem &sm, int s)
{
    return s < 2 ? sm.S01[s] : sm.R;
}

__global__ void __launch_bounds__(kScanThreads, 1)
chunk_scan_tc_kernel(const __grid_constant__ CUtensorMap tm_x,
                     const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_c,
                     const __grid_constant__ CUtensorMap tm_h, const float *__restrict__ dtc,
                     const float *__restrict__ cs, const float *__restrict__ D,
                     bf16 *__restrict__ y, int *__restrict__ status, int64_t seqlen, int H,
                     int G, int Q, int64_t nchunks, int nhb)
{
    extern __shared__ uint8_t smem_raw[];
    ScanSmem &sm = *reinterpret_cast<ScanSmem *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    const int nT = Q / kTileRows;
    int64_t u = blockIdx.x;
    const int T = nT - 1 - (int)(u % nT); u /= nT;       // heavier (later) tiles first
    const int hb = (int)(u % nhb); u /= nhb;
    const int g = (int)(u % G); u /= G;
    const int64_t k = u % nchunks, b = u / nchunks;
    const int hpg = H / G;
    const int h0 = g * hpg + hb * kHeadsPerCta;
    const int nh = min(kHeadsPerCta, hpg - hb * kHeadsPerCta);
    const int64_t t0 = k * Q;
    const int len = (int)min((int64_t)Q, seqlen - t0);
    if (T * kTileRows >= len) return;  // tile entirely past the end of the sequence
    const int KI = kTileRows * (T + 1);  // causal source columns of this tile
    const int nblk = KI / 64;

    if (threadIdx.x == 0) {
        mbar_init(&sm.bar_cb, 1);
        mbar_init(&sm.bar_g, 1);
        for (int s = 0; s < kXStages; ++s) {
            mbar_init(&sm.bar_xh_full[s], 1);
            mbar_init(&sm.bar_xh_free[s], 1);
        }
        for (int s = 0; s < kVecStages; ++s) {
            mbar_init(&sm.bar_vec_full[s], 1);
            mbar_init(&sm.bar_vec_free[s], 256 + 128);
        }
        for (int s = 0; s < kRing; ++s) {
            mbar_init(&sm.bar_slot_full[s], 256);
            mbar_init(&sm.bar_slot_free[s], 1);
        }
        mbar_init(&sm.bar_acc_full, 1);
        mbar_init(&sm.bar_acc_free, 128);
        mbar_init(&sm.bar_drain, 1);
        sm.abort = 0;
        fence_mbar_init();
    }
    if (threadIdx.x >= 32 && threadIdx.x < 32 + nh) sm.Dv[threadIdx.x - 32] = D[h0 + threadIdx.x - 32];
    if (warp == 2) {
        tmem_alloc(&sm.tmem_base, kScanTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    volatile int *abort = &sm.abort;

    if (warp == 0) {
        // ---------------- TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_x);
            tma_prefetch_desc(&tm_b);
            tma_prefetch_desc(&tm_c);
            tma_prefetch_desc(&tm_h);
            mbar_arrive_expect_tx(&sm.bar_cb, (uint32_t)(2 * kBoxBytes + 2 * KI * kRowBytes));
            for (int a = 0; a < 2; ++a)
                tma_load_4d(&sm.Cs[a][0], &tm_c, &sm.bar_cb, 64 * a, g,
                            (int)(t0 + kTileRows * T), (int)b);
            for (int a = 0; a < 2; ++a)
                for (int r = 0; r <= T; ++r)
                    tma_load_4d(sm.R + a * KI * kRowBytes + r * kBoxBytes, &tm_b, &sm.bar_cb,
                                64 * a, g, (int)(t0 + kTileRows * r), (int)b);
        }
        for (int j = 0; j < nh; ++j) {
            const int h = h0 + j;
            const int vs = j % kVecStages;
            const uint32_t vu = j / kVecStages;
            if (j >= kVecStages && !warp_wait(&sm.bar_vec_free[vs], (vu - 1) & 1, abort)) break;
            if (lane == 0) {
                const int64_t vrow = ((b * nchunks + k) * H + h) * (int64_t)Q;
                mbar_arrive_expect_tx(&sm.bar_vec_full[vs], (uint32_t)(8 * Q));
                bulk_load(sm.cs_v[vs], cs + vrow, Q * 4, &sm.bar_vec_full[vs]);
                bulk_load(sm.dt_v[vs], dtc + vrow, Q * 4, &sm.bar_vec_full[vs]);
            }
            const int xs = j % kXStages;
            const uint32_t xu = j / kXStages;
            if (j >= kXStages && !warp_wait(&sm.bar_xh_free[xs], (xu - 1) & 1, abort)) break;
            if (xs == 2 && xu == 0 && !warp_wait(&sm.bar_g, 0, abort)) break;  // B tile in use
            if (lane == 0) {
                uint8_t *stg = scan_stage(sm, xs);
                mbar_arrive_expect_tx(&sm.bar_xh_full[xs],
                                      (uint32_t)(KI * kRowBytes + 2 * kP * kRowBytes));
                for (int r = 0; r <= T; ++r)
                    tma_load_4d(stg + r * kBoxBytes, &tm_x, &sm.bar_xh_full[xs], 0, h,
                                (int)(t0 + kTileRows * r), (int)b);
                const int hrow = (int)(((b * nchunks + k) * H + h) * kP);
                for (int a = 0; a < 2; ++a)
                    tma_load_2d(stg + 256 * kRowBytes + a * kP * kRowBytes, &tm_h,
                                &sm.bar_xh_full[xs], 64 * a, hrow);
            }
            __syncwarp();
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        const uint32_t id_g = idesc_bf16_f32(128, KI, false, false);
        const uint32_t id_h = idesc_bf16_f32(128, kP, false, false);
        const uint32_t id_y = idesc_bf16_f32(128, kP, false, true);
        const uint32_t c0 = smem_u32(&sm.Cs[0][0]);
        const uint32_t rg = smem_u32(sm.R);
        bool ok = warp_wait(&sm.bar_cb, 0, abort);
        if (ok) {
            tc_fence_after();
            if (lane == 0) {
                // G = C B^T: M = 128 rows t, N = KI columns i, K = 128 (n)
                for (int kk = 0; kk < kN / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
                    const uint32_t boff = (kk >> 2) * KI * kRowBytes + (kk & 3) * 32;
                    mma_bf16(tmem, smem_desc_sw128(c0 + off, 16, 1024),
                             smem_desc_sw128(rg + boff, 16, 1024), id_g, kk > 0 ? 1u : 0u);
                }
                mma_commit(&sm.bar_g);
            }
            __syncwarp();
        }
        const uint32_t d1 = tmem + kAccCol, d2 = tmem + kAccCol + 64;
        uint32_t blk = 0;
        for (int j = 0; ok && j < nh; ++j) {
            const int xs = j % kXStages;
            const uint32_t xu = j / kXStages;
            if (!warp_wait(&sm.bar_xh_full[xs], xu & 1, abort)) break;
            if (j >= 1 && !warp_wait(&sm.bar_acc_free, (j - 1) & 1, abort)) break;
            tc_fence_after();
            const uint32_t stg = smem_u32(scan_stage(sm, xs));
            if (lane == 0) {
                // Y2 = C h_in^T: M = 128, N = 64 (p), K = 128 (n)
                for (int kk = 0; kk < kN / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
                    const uint32_t hoff = 256 * kRowBytes + (kk >> 2) * (kP * kRowBytes) +
                                          (kk & 3) * 32;
                    mma_bf16(d2, smem_desc_sw128(c0 + off, 16, 1024),
                             smem_desc_sw128(stg + hoff, 16, 1024), id_h, kk > 0 ? 1u : 0u);
                }
            }
            __syncwarp();
            for (int qb = 0; qb < nblk; ++qb, ++blk) {
                const uint32_t slot = blk % kRing, su = blk / kRing;
                if (!warp_wait(&sm.bar_slot_full[slot], su & 1, abort)) { ok = false; break; }
                tc_fence_after();
                if (lane == 0) {
                    // Y1 += P[:, 64qb : 64qb+64] X[64qb : 64qb+64, :], P read from TMEM
                    const uint32_t pa = tmem + kPCol + 32 * slot;
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t bd =
                            smem_desc_sw128(stg + (qb * 4 + kk) * 2048, 256 * kRowBytes, 1024);
                        mma_bf16_ts(d1, pa + 8 * kk, bd, id_y, (qb | kk) != 0 ? 1u : 0u);
                    }
                    mma_commit(&sm.bar_slot_free[slot]);
                }
                __syncwarp();
            }
            if (!ok) break;
            if (lane == 0) {
                mma_commit(&sm.bar_acc_full);
                mma_commit(&sm.bar_xh_free[xs]);
            }
            __syncwarp();
        }
    } else if (warp >= 4 && warp < 12) {
        // ---------------- mask: P[t][i] = G[t][i] exp(cs_t - cs_i) dt_i (i <= t), + D at i = t
        const int qd = warp & 3;
        const int half = (warp - 4) >> 2;          // which 32 columns of each 64-column block
        const int t = qd * 32 + lane;             // row within the tile = TMEM lane
        const int tau = kTileRows * T + t;        // row within the chunk
        const int r = kTileRows * T + qd * 32 - 1;  // reference row for the factorised decay
        const uint32_t lane_base = tmem + ((uint32_t)(qd * 32) << 16);
        float *vt = sm.vt[warp - 4];
        bool ok = warp_wait(&sm.bar_g, 0, abort);
        tc_fence_after();
        uint32_t blk = 0;
        for (int j = 0; ok && j < nh; ++j) {
            const int vs = j % kVecStages;
            if (!warp_wait(&sm.bar_vec_full[vs], (j / kVecStages) & 1, abort)) break;
            const float *cs_s = sm.cs_v[vs];
            const float *dt_s = sm.dt_v[vs];
            const float Dh = sm.Dv[j];
            const float ct = cs_s[tau];
            float uf = 0.f;
            __syncwarp();
            if (r >= 0) {
                const float cr = cs_s[r];
                // v for the columns of this warp's off-diagonal sub-blocks
                for (int qb = 0; qb < nblk; ++qb) {
                    const int i = qb * 64 + half * 32 + lane;
                    if (i <= r) vt[i] = __expf(cr - cs_s[i]) * dt_s[i];
                }
                uf = __expf(ct - cr);
            }
            __syncwarp();
            for (int qb = 0; qb < nblk; ++qb, ++blk) {
                const uint32_t slot = blk % kRing, su = blk / kRing;
                if (su >= 1 && !warp_wait(&sm.bar_slot_free[slot], (su - 1) & 1, abort)) {
                    ok = false;
                    break;
                }
                const int col0 = qb * 64 + half * 32;
                uint32_t pk[16];
                if (col0 + 32 <= r + 1) {
                    uint32_t gv[32];
                    tmem_ld32(lane_base + col0, gv);
                    tmem_ld_wait();
                    const float2 uu = make_float2(uf, uf);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const float4 vv = *reinterpret_cast<const float4 *>(vt + col0 + 4 * c);
                        const float2 p0 = fmul2(fmul2(make_float2(__uint_as_float(gv[4 * c]),
                                                                  __uint_as_float(gv[4 * c + 1])),
                                                      make_float2(vv.x, vv.y)), uu);
                        const float2 p1 = fmul2(fmul2(make_float2(__uint_as_float(gv[4 * c + 2]),
                                                                  __uint_as_float(gv[4 * c + 3])),
                                                      make_float2(vv.z, vv.w)), uu);
                        pk[2 * c] = pack_bf16x2(p0.x, p0.y);
                        pk[2 * c + 1] = pack_bf16x2(p1.x, p1.y);
                    }
                } else if (col0 == r + 1) {
                    uint32_t gv[32];
                    tmem_ld32(lane_base + col0, gv);
                    tmem_ld_wait();
                    float pv[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const int i = col0 + c;
                        float v = 0.f;
                        if (i <= tau)
                            v = __uint_as_float(gv[c]) * __expf(ct - cs_s[i]) * dt_s[i];
                        if (i == tau) v += Dh;
                        pv[c] = v;
                    }
#pragma unroll
                    for (int c = 0; c < 16; ++c) pk[c] = pack_bf16x2(pv[2 * c], pv[2 * c + 1]);
                } else {
#pragma unroll
                    for (int c = 0; c < 16; ++c) pk[c] = 0u;
                }
                tmem_st16(lane_base + kPCol + 32 * slot + 16 * half, pk);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&sm.bar_slot_full[slot]);
            }
            if (ok) mbar_arrive(&sm.bar_vec_free[vs]);   // done with this stage's cs / dt
        }
    } else if (warp >= 12) {
        // ---------------- epilogue: y = Y1 + exp(cs_t) Y2
        const int qd = warp & 3;
        const int t = qd * 32 + lane;
        const int tau = kTileRows * T + t;
        const uint32_t lane_base = tmem + ((uint32_t)(qd * 32) << 16);
        for (int j = 0; j < nh; ++j) {
            if (!warp_wait(&sm.bar_acc_full, j & 1, abort)) break;
            tc_fence_after();
            const int vs = j % kVecStages;
            if (!warp_wait(&sm.bar_vec_full[vs], (j / kVecStages) & 1, abort)) break;
            const float e = __expf(sm.cs_v[vs][tau]);
            mbar_arrive(&sm.bar_vec_free[vs]);              // done with this stage's cs
            uint32_t a0[32], c0[32], pk[32];
            tmem_ld32(lane_base + kAccCol, a0);
            tmem_ld32(lane_base + kAccCol + 64, c0);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 16; ++c)
                pk[c] = pack_bf16x2(fmaf(e, __uint_as_float(c0[2 * c]), __uint_as_float(a0[2 * c])),
                                    fmaf(e, __uint_as_float(c0[2 * c + 1]),
                                         __uint_as_float(a0[2 * c + 1])));
            tmem_ld32(lane_base + kAccCol + 32, a0);
            tmem_ld32(lane_base + kAccCol + 96, c0);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(&sm.bar_acc_free);
#pragma unroll
            for (int c = 0; c < 16; ++c)
                pk[16 + c] = pack_bf16x2(
                    fmaf(e, __uint_as_float(c0[2 * c]), __uint_as_float(a0[2 * c])),
                    fmaf(e, __uint_as_float(c0[2 * c + 1]), __uint_as_float(a0[2 * c + 1])));
            if (tau < len) {
                uint4 *yrow = reinterpret_cast<uint4 *>(
                    y + ((b * seqlen + t0 + tau) * H + h0 + j) * (int64_t)kP);
#pragma unroll
                for (int m = 0; m < 8; ++m)
                    yrow[m] = make_uint4(pk[4 * m], pk[4 * m + 1], pk[4 * m + 2], pk[4 * m + 3]);
            }
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
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, kScanTmemCols);
    }
}

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
                  int64_t inner)
{
    const cuuint64_t dims[4] = {(cuuint64_t)inner, (cuuint64_t)mid, (cuuint64_t)seqlen,
                                (cuuint64_t)batch};
    const cuuint64_t strides[3] = {(cuuint64_t)(inner * 2), (cuuint64_t)(mid * inner * 2),
                                   (cuuint64_t)(seqlen * mid * inner * 2)};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)kTileRows, 1};
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
                                  cudaStream_t st, const char **why)
{
    CUtensorMap mx, mb;
    if (!make_seq_map(&mx, x, batch, seqlen, H, kP) || !make_seq_map(&mb, B, batch, seqlen, G, kN)) {
        *why = "chunk state: cuTensorMapEncodeTiled failed";
        return cudaErrorInvalidValue;
    }
    const int hpg = H / G;
    const int nhb = (hpg + kHeadsPerCta - 1) / kHeadsPerCta;
    const size_t smem = sizeof(StateSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(chunk_state_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) { *why = "chunk state: set smem attribute"; return e; }
    const unsigned grid = (unsigned)(batch * nchunks * G * nhb);
    chunk_state_tc_kernel<<<grid, kStateThreads, smem, st>>>(mx, mb, dtc, cs, states, status,
                                                             H, G, Q, nchunks, nhb);
    *why = "chunk state (tcgen05) launch";
    return cudaGetLastError();
}

cudaError_t launch_chunk_scan_tc(const bf16 *x, const float *dtc, const bf16 *B, const bf16 *C,
                                 const float *cs, const bf16 *hin, const float *D, bf16 *y,
                                 int *status, int64_t batch, int64_t seqlen, int H, int G,
                                 int Q, int64_t nchunks, cudaStream_t st, const char **why)
{
    CUtensorMap mx, mb, mc, mh;
    const int64_t hrows = batch * nchunks * H * kP;
    const cuuint64_t hdims[2] = {(cuuint64_t)kN, (cuuint64_t)hrows};
    const cuuint64_t hstr[1] = {(cuuint64_t)(kN * 2)};
    const cuuint32_t hbox[2] = {64, (cuuint32_t)kP};
    if (hrows > 0x7fffffffLL || !make_seq_map(&mx, x, batch, seqlen, H, kP) ||
        !make_seq_map(&mb, B, batch, seqlen, G, kN) ||
        !make_seq_map(&mc, C, batch, seqlen, G, kN) || !make_map(&mh, hin, 2, hdims, hstr, hbox)) {
        *why = "chunk scan: cuTensorMapEncodeTiled failed";
        return cudaErrorInvalidValue;
    }
    const int hpg = H / G;
    const int nhb = (hpg + kHeadsPerCta - 1) / kHeadsPerCta;
    const size_t smem = sizeof(ScanSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(chunk_scan_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) { *why = "chunk scan: set smem attribute"; return e; }
    const unsigned grid = (unsigned)(batch * nchunks * G * nhb * (Q / kTileRows));
    chunk_scan_tc_kernel<<<grid, kScanThreads, smem, st>>>(mx, mb, mc, mh, dtc, cs, D, y, status,
                                                           seqlen, H, G, Q, nchunks, nhb);
    *why = "chunk scan (tcgen05) launch";
    return cudaGetLastError();
}

}  // namespace ssd
