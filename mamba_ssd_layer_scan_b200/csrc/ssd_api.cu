// C ABI entry points (include/ssd.h): argument validation, workspace carving, kernel dispatch.
//
// ssd_chunk_scan_fwd enqueues, on the caller's stream and in this order:
//   1. dA cumsum            chunk-local prefix sums of dt*A            (chunk_cumsum.cu)
//   2. chunk state          each chunk's own contribution to its end state (chunk_tc.cu /
//                           chunk_simt.cu)
//   3. state passing        the recurrence across chunks               (state_passing.cu)
//   4. chunk scan           within-chunk quadratic form + off-chunk term (chunk_tc.cu /
//                           chunk_simt.cu)
// following the block decomposition of mohakchugh.is-a.dev "Mamba-2" (Block Decomposition:
// quadratic form inside a chunk, linear recurrence across chunks).  Nothing is allocated and
// nothing synchronises; errors are reported through the returned status.
#include <cstdarg>
#include <cstdio>

#include <atomic>

#include "../../include/ssd.h"
#include "../../include/ssd_testing.h"
#include "common.cuh"

namespace {

thread_local char g_err[512] = "";

ssd_status fail(ssd_status s, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return s;
}

ssd_status cuda_fail(cudaError_t e, const char *what)
{
    return fail(SSD_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

cudaError_t record(void *const *events, int i, cudaStream_t st)
{
    return events ? cudaEventRecord(static_cast<cudaEvent_t>(events[i]), st) : cudaSuccess;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round256(size_t v) { return (v + 255) & ~size_t(255); }

ssd_status check_shape(const ssd_shape *s, bool need_seq)
{
    if (!s) return fail(SSD_ERR_INVALID_ARG, "shape is NULL");
    if (s->batch < 0 || (need_seq && s->seqlen < 0))
        return fail(SSD_ERR_INVALID_ARG, "batch and seqlen must be >= 0");
    if (s->nheads < 1 || s->ngroups < 1 || s->nheads % s->ngroups != 0)
        return fail(SSD_ERR_INVALID_ARG, "need nheads >= 1, ngroups >= 1, nheads %% ngroups == 0 "
                    "(got %lld, %lld)", (long long)s->nheads, (long long)s->ngroups);
    if (s->dtype != SSD_F32 && s->dtype != SSD_BF16)
        return fail(SSD_ERR_INVALID_ARG, "dtype must be SSD_F32 or SSD_BF16");
    if (s->headdim < 1 || s->headdim > 128)
        return fail(SSD_ERR_UNSUPPORTED, "headdim must be in 1..128 (got %lld)",
                    (long long)s->headdim);
    if (s->dstate < 32 || s->dstate > 256 || s->dstate % 32 != 0)
        return fail(SSD_ERR_UNSUPPORTED, "dstate must be a multiple of 32 in 32..256 (got %lld)",
                    (long long)s->dstate);
    if (s->headdim * s->dstate > 16384)
        return fail(SSD_ERR_UNSUPPORTED, "headdim * dstate must be <= 16384");
    if (s->nheads > 65535 || s->batch > 65535)
        return fail(SSD_ERR_UNSUPPORTED, "batch and nheads must be <= 65535");
    return SSD_OK;
}

bool valid_chunk(int q) { return q == 16 || q == 32 || q == 64 || q == 128 || q == 256; }

ssd::WsLayout layout(const ssd_shape *s, int Q)
{
    const int64_t nchunks = (s->seqlen + Q - 1) / Q;
    const size_t rows = (size_t)s->batch * nchunks * s->nheads;
    ssd::WsLayout w;
    w.status = 0;
    w.cs = 256;
    const bool tc = ssd::tc_supported(s->dtype == SSD_BF16, (int)s->headdim, (int)s->dstate, Q);
    w.dtc = w.cs + round256(rows * Q * sizeof(float));
    w.states = w.dtc + (tc ? round256(rows * Q * sizeof(float)) : 0);
    w.hin_bf16 = w.states + round256(rows * s->headdim * s->dstate * sizeof(float));
    w.total = w.hin_bf16 + (tc ? round256(rows * s->headdim * s->dstate * sizeof(uint16_t)) : 0);
    return w;
}

// Workspace of a variable-length call: the status word, the chunk table (one slot per possible
// chunk: L / Q + nseq bounds the chunks of any split of L tokens into nseq sequences), the
// first chunk of each sequence, then the tensor-core path's per-chunk regions.
struct VarlenLayout {
    size_t status, tab, cstart, cs, dtc, states, hin, total;
    int64_t slots;
};

VarlenLayout varlen_layout(const ssd_shape *s, int nseq, int Q)
{
    VarlenLayout w;
    w.slots = s->seqlen / Q + nseq;
    const size_t rows = (size_t)w.slots * s->nheads;
    const size_t pn = (size_t)s->headdim * s->dstate;
    w.status = 0;
    w.tab = 256;
    w.cstart = w.tab + round256((size_t)w.slots * 8);
    w.cs = w.cstart + round256((size_t)(nseq + 1) * 4);
    w.dtc = w.cs + round256(rows * Q * 4);
    w.states = w.dtc + round256(rows * Q * 4);
    w.hin = w.states + round256(rows * pn * 4);
    w.total = w.hin + round256(rows * pn * 2);
    return w;
}

ssd_status check_varlen(const ssd_shape *s, int nseq, int Q)
{
    ssd_status st = check_shape(s, true);
    if (st != SSD_OK) return st;
    if (s->batch != 1)
        return fail(SSD_ERR_INVALID_ARG, "variable-length input is packed: batch must be 1 (got %lld)",
                    (long long)s->batch);
    if (nseq < 1) return fail(SSD_ERR_INVALID_ARG, "nseq must be >= 1 (got %d)", nseq);
    if (s->seqlen > 0x7fffffffLL - 256)
        return fail(SSD_ERR_UNSUPPORTED, "packed token count must fit int32 cu_seqlens");
    if (!valid_chunk(Q))
        return fail(SSD_ERR_UNSUPPORTED, "chunk_size must be 16, 32, 64, 128 or 256 (got %d)", Q);
    if (!ssd::tc_supported(s->dtype == SSD_BF16, (int)s->headdim, (int)s->dstate, Q))
        return fail(SSD_ERR_UNSUPPORTED,
                    "variable-length scan runs on the tensor-core path only: bf16, headdim 64, "
                    "dstate 128, chunk_size 128 or 256");
    return SSD_OK;
}

}  // namespace

void ssd::set_last_error(const char *msg) { snprintf(g_err, sizeof(g_err), "%s", msg); }

namespace {
std::atomic<int> g_test_kernel{0};
std::atomic<int> g_test_cta{-1};
}  // namespace

int ssd::take_test_skip(int kernel)
{
    int k = kernel;
    if (!g_test_kernel.compare_exchange_strong(k, 0)) return -1;
    return g_test_cta.exchange(-1);
}

extern "C" {

const char *ssd_last_error(void) { return g_err; }

const char *ssd_version(void) { return "ssd-b200 0.1 (sm_100a)"; }

ssd_status ssd_testing_skip_stage(int kernel, int cta)
{
    if (kernel != SSD_TESTING_CHUNK_STATE && kernel != SSD_TESTING_CHUNK_SCAN)
        return fail(SSD_ERR_INVALID_ARG, "kernel must be SSD_TESTING_CHUNK_STATE or "
                                         "SSD_TESTING_CHUNK_SCAN (got %d)", kernel);
    if (cta < 0) return fail(SSD_ERR_INVALID_ARG, "cta must be >= 0 (got %d)", cta);
    g_test_cta.store(cta);
    g_test_kernel.store(kernel == SSD_TESTING_CHUNK_STATE ? ssd::kTestChunkState
                                                          : ssd::kTestChunkScan);
    return SSD_OK;
}

size_t ssd_chunk_scan_workspace_size(const ssd_shape *shape, int chunk_size)
{
    if (check_shape(shape, true) != SSD_OK) return 0;
    if (!valid_chunk(chunk_size)) {
        fail(SSD_ERR_UNSUPPORTED, "chunk_size must be 16, 32, 64, 128 or 256 (got %d)",
             chunk_size);
        return 0;
    }
    return layout(shape, chunk_size).total;
}

ssd_status ssd_chunk_scan_fwd(const ssd_shape *shape, const void *x, const float *dt,
                              const float *A, const void *B, const void *C, const float *D,
                              int chunk_size, const float *init_state, void *y,
                              float *final_state, void *workspace, size_t workspace_bytes,
                              void *stream)
{
    return ssd_chunk_scan_fwd_staged(shape, x, dt, A, B, C, D, chunk_size, init_state, y,
                                     final_state, workspace, workspace_bytes, stream, nullptr);
}

}  // extern "C"

namespace {

bool prologue_active(const ssd_fwd_options *o)
{
    return o && (o->dt_bias || o->dt_softplus || o->dt_max > 0.f);
}

// The whole chunked scan; stage_events and options are both nullable.
ssd_status scan_impl(const ssd_shape *shape, const void *x, const float *dt, const float *A,
                     const void *B, const void *C, const float *D, int chunk_size,
                     const float *init_state, void *y, float *final_state, void *workspace,
                     size_t workspace_bytes, void *stream, void *const *stage_events,
                     const ssd_fwd_options *opts)
{
    ssd_status st = check_shape(shape, true);
    if (st != SSD_OK) return st;
    if (!valid_chunk(chunk_size))
        return fail(SSD_ERR_UNSUPPORTED, "chunk_size must be 16, 32, 64, 128 or 256 (got %d)",
                    chunk_size);
    const ssd_shape s = *shape;
    const int H = (int)s.nheads, G = (int)s.ngroups, P = (int)s.headdim, N = (int)s.dstate;
    const int Q = chunk_size;
    const bool bf = s.dtype == SSD_BF16;
    cudaStream_t cs_stream = static_cast<cudaStream_t>(stream);
    const int64_t PNtot = s.batch * s.nheads * s.headdim * s.dstate;

    if (final_state && !aligned16(final_state))
        return fail(SSD_ERR_INVALID_ARG, "final_state must be 16-byte aligned");
    if (init_state && !aligned16(init_state))
        return fail(SSD_ERR_INVALID_ARG, "init_state must be 16-byte aligned");
    if (s.batch == 0) return SSD_OK;
    if (s.seqlen == 0) {
        if (final_state) {
            cudaError_t e = ssd::launch_fill_final(init_state, final_state, PNtot, cs_stream);
            if (e != cudaSuccess) return cuda_fail(e, "fill final state");
        }
        return SSD_OK;
    }
    if (!x || !dt || !A || !B || !C || !D || !y || !workspace)
        return fail(SSD_ERR_INVALID_ARG, "x, dt, A, B, C, D, y and workspace must be non-NULL");
    if (!aligned16(x) || !aligned16(B) || !aligned16(C) || !aligned16(y))
        return fail(SSD_ERR_INVALID_ARG, "x, B, C and y must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(SSD_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    const void *z = opts ? opts->z : nullptr;
    if (z && !aligned16(z)) return fail(SSD_ERR_INVALID_ARG, "z must be 16-byte aligned");
    const bool pro = prologue_active(opts);
    if (pro && opts->dt_max > 0.f && !(opts->dt_min <= opts->dt_max))
        return fail(SSD_ERR_INVALID_ARG, "dt_min must not exceed dt_max");
    const int64_t nchunks = (s.seqlen + Q - 1) / Q;
    if (s.batch * nchunks * s.nheads * ((Q + 31) / 32) > 0x7fffffffLL)
        return fail(SSD_ERR_UNSUPPORTED, "problem too large for one launch grid");
    const ssd::WsLayout wl = layout(&s, Q);
    const size_t need = wl.total + (pro ? round256((size_t)s.batch * s.seqlen * H * 4) : 0);
    if (workspace_bytes < need)
        return fail(SSD_ERR_INVALID_ARG, "workspace too small: need %zu bytes, got %zu", need,
                    workspace_bytes);

    char *ws = static_cast<char *>(workspace);
    int *status = reinterpret_cast<int *>(ws + wl.status);
    float *cs = reinterpret_cast<float *>(ws + wl.cs);
    float *states = reinterpret_cast<float *>(ws + wl.states);
    cudaError_t e = record(stage_events, 0, cs_stream);
    if (e != cudaSuccess) return cuda_fail(e, "record stage event");
    if (pro) {   // dt <- clamp(softplus(dt + dt_bias)) into the workspace; the scan reads that
        float *dt_eff = reinterpret_cast<float *>(ws + wl.total);
        e = ssd::launch_dt_prologue(dt, opts->dt_bias, dt_eff, s.batch * s.seqlen, H,
                                    opts->dt_softplus != 0, opts->dt_max > 0.f, opts->dt_min,
                                    opts->dt_max, cs_stream);
        if (e != cudaSuccess) return cuda_fail(e, "dt prologue launch");
        dt = dt_eff;
    }
    const bool tc = ssd::tc_supported(bf, P, N, Q);
    float *dtc = tc ? reinterpret_cast<float *>(ws + wl.dtc) : nullptr;
    e = ssd::launch_chunk_cumsum(dt, A, cs, dtc, status, s.batch, s.seqlen, H, Q, nchunks,
                                 cs_stream);
    if (e != cudaSuccess) return cuda_fail(e, "dA cumsum launch");
    if ((e = record(stage_events, 1, cs_stream)) != cudaSuccess)
        return cuda_fail(e, "record stage event");

    if (tc) {
        const char *why = "";
        ssd::bf16 *hin = reinterpret_cast<ssd::bf16 *>(ws + wl.hin_bf16);
        e = ssd::launch_chunk_state_tc((const ssd::bf16 *)x, dtc, (const ssd::bf16 *)B, cs,
                                       states, status, s.batch, s.seqlen, H, G, Q, nchunks,
                                       cs_stream, &why);
        if (e != cudaSuccess) return cuda_fail(e, why);
        if ((e = record(stage_events, 2, cs_stream)) != cudaSuccess)
            return cuda_fail(e, "record stage event");
        e = ssd::launch_state_passing(states, cs, init_state, final_state, hin, s.batch, H, P, N,
                                      Q, nchunks, cs_stream);
        if (e != cudaSuccess) return cuda_fail(e, "state passing launch");
        if ((e = record(stage_events, 3, cs_stream)) != cudaSuccess)
            return cuda_fail(e, "record stage event");
        e = ssd::launch_chunk_scan_tc((const ssd::bf16 *)x, dtc, (const ssd::bf16 *)B,
                                      (const ssd::bf16 *)C, cs, hin, D, (ssd::bf16 *)y, status,
                                      s.batch, s.seqlen, H, G, Q, nchunks, cs_stream, &why,
                                      nullptr, (const ssd::bf16 *)z);
        if (e != cudaSuccess) return cuda_fail(e, why);
        if ((e = record(stage_events, 4, cs_stream)) != cudaSuccess)
            return cuda_fail(e, "record stage event");
        return SSD_OK;
    }

    e = ssd::launch_chunk_state_simt(bf, x, dt, B, cs, states, s.batch, s.seqlen, H, G, P, N, Q,
                                     nchunks, cs_stream);
    if (e != cudaSuccess) return cuda_fail(e, "chunk state launch");
    if ((e = record(stage_events, 2, cs_stream)) != cudaSuccess)
        return cuda_fail(e, "record stage event");
    e = ssd::launch_state_passing(states, cs, init_state, final_state, nullptr, s.batch, H, P, N,
                                  Q, nchunks, cs_stream);
    if (e != cudaSuccess) return cuda_fail(e, "state passing launch");
    if ((e = record(stage_events, 3, cs_stream)) != cudaSuccess)
        return cuda_fail(e, "record stage event");
    e = ssd::launch_chunk_scan_simt(bf, x, dt, B, C, cs, states, D, y, s.batch, s.seqlen, H, G,
                                    P, N, Q, nchunks, cs_stream, z);
    if (e != cudaSuccess) return cuda_fail(e, "chunk scan launch");
    if ((e = record(stage_events, 4, cs_stream)) != cudaSuccess)
        return cuda_fail(e, "record stage event");
    return SSD_OK;
}

}  // namespace

extern "C" {

ssd_status ssd_chunk_scan_fwd_staged(const ssd_shape *shape, const void *x, const float *dt,
                                     const float *A, const void *B, const void *C,
                                     const float *D, int chunk_size, const float *init_state,
                                     void *y, float *final_state, void *workspace,
                                     size_t workspace_bytes, void *stream,
                                     void *const *stage_events)
{
    return scan_impl(shape, x, dt, A, B, C, D, chunk_size, init_state, y, final_state,
                     workspace, workspace_bytes, stream, stage_events, nullptr);
}

size_t ssd_chunk_scan_fwd_ex_workspace_size(const ssd_shape *shape, int chunk_size,
                                            const ssd_fwd_options *options)
{
    const size_t base = ssd_chunk_scan_workspace_size(shape, chunk_size);
    if (base == 0 || !prologue_active(options)) return base;
    return base + round256((size_t)shape->batch * shape->seqlen * shape->nheads * 4);
}

ssd_status ssd_chunk_scan_fwd_ex(const ssd_shape *shape, const void *x, const float *dt,
                                 const float *A, const void *B, const void *C, const float *D,
                                 int chunk_size, const float *init_state, void *y,
                                 float *final_state, void *workspace, size_t workspace_bytes,
                                 void *stream, const ssd_fwd_options *options)
{
    return scan_impl(shape, x, dt, A, B, C, D, chunk_size, init_state, y, final_state,
                     workspace, workspace_bytes, stream, nullptr, options);
}

size_t ssd_chunk_scan_varlen_workspace_size(const ssd_shape *shape, int nseq, int chunk_size)
{
    if (check_varlen(shape, nseq, chunk_size) != SSD_OK) return 0;
    return varlen_layout(shape, nseq, chunk_size).total;
}

ssd_status ssd_chunk_scan_varlen_fwd(const ssd_shape *shape, const void *x, const float *dt,
                                     const float *A, const void *B, const void *C,
                                     const float *D, int chunk_size, const int32_t *cu_seqlens,
                                     int nseq, const float *init_states, void *y,
                                     float *final_states, void *workspace,
                                     size_t workspace_bytes, void *stream)
{
    ssd_status st = check_varlen(shape, nseq, chunk_size);
    if (st != SSD_OK) return st;
    const ssd_shape s = *shape;
    const int H = (int)s.nheads, G = (int)s.ngroups, P = (int)s.headdim, N = (int)s.dstate;
    const int Q = chunk_size;
    cudaStream_t cst = static_cast<cudaStream_t>(stream);
    if (final_states && !aligned16(final_states))
        return fail(SSD_ERR_INVALID_ARG, "final_states must be 16-byte aligned");
    if (init_states && !aligned16(init_states))
        return fail(SSD_ERR_INVALID_ARG, "init_states must be 16-byte aligned");
    if (s.seqlen == 0) {   // every sequence is empty: final = init
        if (final_states) {
            cudaError_t e = ssd::launch_fill_final(init_states, final_states,
                                                   (int64_t)nseq * H * P * N, cst);
            if (e != cudaSuccess) return cuda_fail(e, "fill final states");
        }
        return SSD_OK;
    }
    if (!x || !dt || !A || !B || !C || !D || !y || !cu_seqlens || !workspace)
        return fail(SSD_ERR_INVALID_ARG,
                    "x, dt, A, B, C, D, y, cu_seqlens and workspace must be non-NULL");
    if (!aligned16(x) || !aligned16(B) || !aligned16(C) || !aligned16(y))
        return fail(SSD_ERR_INVALID_ARG, "x, B, C and y must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(SSD_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    const VarlenLayout wl = varlen_layout(&s, nseq, Q);
    if (workspace_bytes < wl.total)
        return fail(SSD_ERR_INVALID_ARG, "workspace too small: need %zu bytes, got %zu",
                    wl.total, workspace_bytes);
    if (wl.slots * H * ((Q + 31) / 32) > 0x7fffffffLL)
        return fail(SSD_ERR_UNSUPPORTED, "problem too large for one launch grid");

    char *ws = static_cast<char *>(workspace);
    int *status = reinterpret_cast<int *>(ws + wl.status);
    int2 *tab = reinterpret_cast<int2 *>(ws + wl.tab);
    int32_t *cstart = reinterpret_cast<int32_t *>(ws + wl.cstart);
    float *cs = reinterpret_cast<float *>(ws + wl.cs);
    float *dtc = reinterpret_cast<float *>(ws + wl.dtc);
    float *states = reinterpret_cast<float *>(ws + wl.states);
    ssd::bf16 *hin = reinterpret_cast<ssd::bf16 *>(ws + wl.hin);
    const char *why = "";
    cudaError_t e = ssd::launch_build_chunk_table(cu_seqlens, nseq, s.seqlen, Q, wl.slots, tab,
                                                  cstart, status, cst);
    if (e != cudaSuccess) return cuda_fail(e, "chunk table launch");
    e = ssd::launch_chunk_cumsum(dt, A, cs, dtc, nullptr, 1, s.seqlen, H, Q, wl.slots, cst, tab);
    if (e != cudaSuccess) return cuda_fail(e, "dA cumsum launch");
    e = ssd::launch_chunk_state_tc((const ssd::bf16 *)x, dtc, (const ssd::bf16 *)B, cs, states,
                                   status, 1, s.seqlen, H, G, Q, wl.slots, cst, &why, tab);
    if (e != cudaSuccess) return cuda_fail(e, why);
    e = ssd::launch_state_passing_varlen(states, cs, init_states, final_states, hin, cstart,
                                         nseq, H, P, N, Q, wl.slots, cst);
    if (e != cudaSuccess) return cuda_fail(e, "state passing launch");
    e = ssd::launch_chunk_scan_tc((const ssd::bf16 *)x, dtc, (const ssd::bf16 *)B,
                                  (const ssd::bf16 *)C, cs, hin, D, (ssd::bf16 *)y, status, 1,
                                  s.seqlen, H, G, Q, wl.slots, cst, &why, tab);
    if (e != cudaSuccess) return cuda_fail(e, why);
    return SSD_OK;
}

// ---- backward pass (the gradients of the chunked scan)
namespace {
constexpr int kBwdSimtChunk = 64;   // chunk of the two CUDA-core scans (head dim N, state P)

struct BwdLayout {
    size_t r_ws, s_ws;                          // the reversed scan's and the dB / dC scans'
    size_t dtc_s;                               // the dB / dC scans' per-chunk weight rows
    size_t dyr, Cr, Br, dtr, zerosD, gb, Fr;
    size_t ys, fin_s;                           // the dB / dC scans' output and final state
    size_t ydot, ddt_in, q, xdy, fdot, part, total;
    size_t r_bytes, s_bytes;
};

ssd_shape simt_shape(const ssd_shape &s)
{
    ssd_shape t = s;          // head dimension N, state dimension P, one group per head, f32
    t.headdim = s.dstate;
    t.dstate = s.headdim;
    t.ngroups = s.nheads;
    t.dtype = SSD_F32;
    return t;
}

BwdLayout bwd_layout(const ssd_shape *s, int Q)
{
    BwdLayout w;
    const size_t b = s->batch, L = s->seqlen, H = s->nheads, P = s->headdim, N = s->dstate,
                 G = s->ngroups;
    const ssd_shape t = simt_shape(*s);
    w.r_bytes = layout(s, Q).total;
    w.s_bytes = layout(&t, kBwdSimtChunk).total;
    size_t o = 0;
    auto take = [&](size_t bytes) { const size_t at = o; o += round256(bytes); return at; };
    w.r_ws = take(w.r_bytes);   // first: its status word is the workspace's
    w.s_ws = take(w.s_bytes);
    w.dtc_s = take(b * ((L + kBwdSimtChunk - 1) / kBwdSimtChunk) * H * kBwdSimtChunk * 4);
    w.dyr = take(b * L * H * P * 2);
    w.Cr = take(b * L * G * N * 2);
    w.Br = take(b * L * G * N * 2);
    w.dtr = take(b * L * H * 4);
    w.zerosD = take(H * 4);
    w.gb = take(b * L * H * P * 2);
    w.Fr = take(b * H * P * N * 4);
    w.ys = take(b * L * H * N * 4);
    w.fin_s = take(b * H * N * P * 4);
    w.ydot = take(b * L * H * 4);
    w.ddt_in = take(b * L * H * 4);
    w.q = take(b * L * H * 4);
    w.xdy = take(b * L * H * 4);
    w.fdot = take(b * H * 4);
    w.part = take(2 * b * H * 4);
    w.total = o;
    return w;
}

ssd_status check_bwd(const ssd_shape *s, int Q)
{
    ssd_status st = check_shape(s, true);
    if (st != SSD_OK) return st;
    if (!valid_chunk(Q) ||
        !ssd::tc_supported(s->dtype == SSD_BF16, (int)s->headdim, (int)s->dstate, Q) ||
        !ssd::bwd_scan_supported((int)s->headdim, (int)s->dstate))
        return fail(SSD_ERR_UNSUPPORTED,
                    "the backward pass runs for the tensor-core shapes: bf16, headdim 64, "
                    "dstate 128, chunk_size 128 or 256");
    return SSD_OK;
}
}  // namespace

size_t ssd_chunk_scan_bwd_workspace_size(const ssd_shape *shape, int chunk_size)
{
    if (check_bwd(shape, chunk_size) != SSD_OK) return 0;
    return bwd_layout(shape, chunk_size).total;
}

ssd_status ssd_chunk_scan_bwd(const ssd_shape *shape, const void *x, const float *dt,
                              const float *A, const void *B, const void *C, const float *D,
                              int chunk_size, const float *init_state, const void *dy,
                              const float *dfinal, float *dx, float *ddt, float *dA, float *dB,
                              float *dC, float *dD, float *dinit, void *workspace,
                              size_t workspace_bytes, void *stream)
{
    ssd_status st = check_bwd(shape, chunk_size);
    if (st != SSD_OK) return st;
    const ssd_shape s = *shape;
    const int H = (int)s.nheads, G = (int)s.ngroups, P = (int)s.headdim, N = (int)s.dstate;
    const int Q = chunk_size;
    const int64_t b = s.batch, L = s.seqlen;
    cudaStream_t cst = static_cast<cudaStream_t>(stream);
    if (!dA || !dD) return fail(SSD_ERR_INVALID_ARG, "dA and dD must be non-NULL");
    if (b == 0 || L == 0) {   // no token: only dinit (= dfinal) and the zero dA, dD
        cudaError_t e = cudaMemsetAsync(dA, 0, H * 4, cst);
        if (e == cudaSuccess) e = cudaMemsetAsync(dD, 0, H * 4, cst);
        if (e == cudaSuccess && dinit)
            e = ssd::launch_fill_final(dfinal, dinit, b * H * P * N, cst);
        return e == cudaSuccess ? SSD_OK : cuda_fail(e, "empty backward");
    }
    if (!x || !dt || !A || !B || !C || !D || !dy || !dx || !ddt || !dB || !dC || !workspace)
        return fail(SSD_ERR_INVALID_ARG, "inputs, dy and the gradient buffers must be non-NULL");
    if (!aligned16(x) || !aligned16(B) || !aligned16(C) || !aligned16(dy) || !aligned16(dx) ||
        (init_state && !aligned16(init_state)) || (dfinal && !aligned16(dfinal)) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(SSD_ERR_INVALID_ARG, "x, B, C, dy, dx and the states must be 16-byte, the "
                                         "workspace 256-byte aligned");
    const BwdLayout wl = bwd_layout(&s, Q);
    if (workspace_bytes < wl.total)
        return fail(SSD_ERR_INVALID_ARG, "workspace too small: need %zu bytes, got %zu",
                    wl.total, workspace_bytes);
    char *ws = static_cast<char *>(workspace);
    auto F = [&](size_t off) { return reinterpret_cast<float *>(ws + off); };
    auto Hh = [&](size_t off) { return reinterpret_cast<ssd::bf16 *>(ws + off); };
    float *zerosD = F(wl.zerosD);
    cudaError_t e = ssd::launch_fill(zerosD, 0.f, H, cst);
    if (e != cudaSuccess) return cuda_fail(e, "fill");

    // 1. g_t B_t: the forward scan of the reversed sequence (x' = dy, B' = C, C' = B), unit
    // input weights, decays shifted by one token, started from dfinal; its final state is g_0.
    // Its cumsum clears the workspace status word (offset 0) that the tensor-core kernels set.
    const int64_t nch = (L + Q - 1) / Q;
    const ssd::WsLayout rl = layout(&s, Q);
    char *rw = ws + wl.r_ws;
    int *status = reinterpret_cast<int *>(rw + rl.status);
    float *cs_r = reinterpret_cast<float *>(rw + rl.cs);
    float *dtc_r = reinterpret_cast<float *>(rw + rl.dtc);
    float *states_r = reinterpret_cast<float *>(rw + rl.states);
    ssd::bf16 *hin_r = reinterpret_cast<ssd::bf16 *>(rw + rl.hin_bf16);
    const char *why = "";
    using ssd::bf16;
    const bf16 *xb = static_cast<const bf16 *>(x), *dyb = static_cast<const bf16 *>(dy);
    const bf16 *Bb = static_cast<const bf16 *>(B), *Cb = static_cast<const bf16 *>(C);
    if ((e = ssd::launch_gather(dyb, Hh(wl.dyr), b, L, H, H, P, true, cst)) ||
        (e = ssd::launch_gather(Cb, Hh(wl.Cr), b, L, G, G, N, true, cst)) ||
        (e = ssd::launch_gather(Bb, Hh(wl.Br), b, L, G, G, N, true, cst)) ||
        (e = ssd::launch_reverse_shift_dt(dt, F(wl.dtr), b, L, H, cst)))
        return cuda_fail(e, "reverse inputs");
    e = ssd::launch_chunk_cumsum(F(wl.dtr), A, cs_r, dtc_r, status, b, L, H, Q, nch, cst,
                                 nullptr, true);
    if (e != cudaSuccess) return cuda_fail(e, "reversed cumsum");
    e = ssd::launch_chunk_state_tc(Hh(wl.dyr), dtc_r, Hh(wl.Cr), cs_r, states_r, status, b, L, H,
                                   G, Q, nch, cst, &why);
    if (e != cudaSuccess) return cuda_fail(e, why);
    e = ssd::launch_state_passing(states_r, cs_r, dfinal, F(wl.Fr), hin_r, b, H, P, N, Q, nch,
                                  cst);
    if (e != cudaSuccess) return cuda_fail(e, "reversed state passing");
    e = ssd::launch_chunk_scan_tc(Hh(wl.dyr), dtc_r, Hh(wl.Cr), Hh(wl.Br), cs_r, hin_r, zerosD,
                                  Hh(wl.gb), status, b, L, H, G, Q, nch, cst, &why);
    if (e != cudaSuccess) return cuda_fail(e, why);
    if (dinit && (e = ssd::launch_scale_init_grad(F(wl.Fr), dt, A, dinit, b, L, H, P * N, cst)))
        return cuda_fail(e, "dinit");

    // 2. dB and dC: scans with head dimension N and state dimension P, summed over the heads of
    // each group.  Their chunk states come from the tensor-core chunk-state kernel with its
    // operands swapped (x'' in the place of B, B'' in the place of x) and split into bf16 pairs
    // (float32-accurate states, stored [p][n] like the forward's); the chunk outputs from the
    // float32 CUDA-core kernel, which reads the bf16 operands in place.  Their per-head outputs
    // also give, contracted with B (resp. C), the two float32 dot products of the decay
    // gradient: <x_t, g_t B_t> and <dy_t, y_t - D x_t>.
    const ssd_shape t = simt_shape(s);
    const int Qs = kBwdSimtChunk;
    const int64_t nchs = (L + Qs - 1) / Qs;
    const ssd::WsLayout sl = layout(&t, Qs);
    char *sw = ws + wl.s_ws;
    float *cs_s = reinterpret_cast<float *>(sw + sl.cs);
    float *states_s = reinterpret_cast<float *>(sw + sl.states);
    float *dtc_s = F(wl.dtc_s);
    for (int pass = 0; pass < 2; ++pass) {   // 0: dB (reversed), 1: dC (forward)
        const bool rev = pass == 0;
        const float *init_s = rev ? dfinal : init_state;   // (p, n), as the states
        const float *w_s = rev ? nullptr : dt;
        // decays from the (reversed, shifted) dt; weights dt (dC) or 1 (dB) as the dt rows
        e = ssd::launch_chunk_cumsum(rev ? F(wl.dtr) : dt, A, cs_s, dtc_s, nullptr, b, L, H, Qs,
                                     nchs, cst, nullptr, rev);
        const char *why = "dB / dC chunk state";
        if (e == cudaSuccess)
            e = ssd::launch_chunk_state_tc(rev ? dyb : xb, dtc_s, rev ? Cb : Bb, cs_s, states_s,
                                           status, b, L, H, G, Qs, nchs, cst, &why, nullptr,
                                           true, rev);
        if (e == cudaSuccess)
            e = ssd::launch_state_passing(states_s, cs_s, init_s, rev ? nullptr : F(wl.fin_s),
                                          nullptr, b, H, P, N, Qs, nchs, cst);
        // the chunk outputs, summed over runs of heads (weighted by dt for dB), then the runs'
        // partial sums over each group
        const int hpc = ssd::bwd_scan_heads_per_cta(H, G);
        if (e == cudaSuccess)
            e = ssd::launch_bwd_chunk_scan(rev ? Cb : Bb, rev ? dyb : xb, rev ? xb : dyb, w_s,
                                           cs_s, states_s, rev ? Bb : Cb, rev ? dt : nullptr,
                                           F(wl.ys), F(rev ? wl.ddt_in : wl.ydot), b, L, H, G,
                                           nchs, rev, cst);
        if (e == cudaSuccess)
            e = ssd::launch_group_sum(F(wl.ys), nullptr, rev ? dB : dC, b, L, H / hpc, G, N,
                                      false, cst);
        if (e != cudaSuccess) return cuda_fail(e, rev ? "dB scan" : "dC scan");
    }

    // 3. dx, the decay-gradient terms and their reverse cumsum: ddt, dA, dD
    // <dfinal, final>, both transposed to (n, p): the final state's share of the decay gradient
    if (dfinal && (e = ssd::launch_state_dot(dfinal, F(wl.fin_s), F(wl.fdot), b * H, P * N,
                                             cst)))
        return cuda_fail(e, "final-state term");
    if ((e = ssd::launch_bwd_tokens(xb, dyb, dt, D, Hh(wl.gb), F(wl.ydot), F(wl.ddt_in),
                                    dfinal ? F(wl.fdot) : nullptr, dx, F(wl.q), F(wl.xdy), b, L,
                                    H, P, cst)) ||
        (e = ssd::launch_bwd_decay(F(wl.q), F(wl.ddt_in), dt, A, F(wl.xdy), ddt, dA, dD,
                                   F(wl.part), b, L, H, cst)))
        return cuda_fail(e, "token gradients");
    return SSD_OK;
}

// ---- sequence parallelism (one contiguous segment of the sequence per rank)
namespace {
ssd_status check_seqpar(const ssd_shape *s, int Q)
{
    ssd_status st = check_shape(s, true);
    if (st != SSD_OK) return st;
    if (!valid_chunk(Q))
        return fail(SSD_ERR_UNSUPPORTED, "chunk_size must be 16, 32, 64, 128 or 256 (got %d)", Q);
    if (!ssd::tc_supported(s->dtype == SSD_BF16, (int)s->headdim, (int)s->dstate, Q))
        return fail(SSD_ERR_UNSUPPORTED,
                    "sequence-parallel scan runs on the tensor-core path only: bf16, headdim 64, "
                    "dstate 128, chunk_size 128 or 256");
    return SSD_OK;
}
size_t seqpar_hseg_offset(const ssd_shape *s, int Q) { return layout(s, Q).total; }
}  // namespace

size_t ssd_seqpar_workspace_size(const ssd_shape *shape, int chunk_size)
{
    if (check_seqpar(shape, chunk_size) != SSD_OK) return 0;
    return seqpar_hseg_offset(shape, chunk_size) +
           round256((size_t)shape->batch * shape->nheads * shape->headdim * shape->dstate * 4);
}

ssd_status ssd_seqpar_local(const ssd_shape *shape, const void *x, const float *dt,
                            const float *A, const void *B, int chunk_size, float *h_loc,
                            float *log_decay, void *workspace, size_t workspace_bytes,
                            void *stream)
{
    ssd_status st = check_seqpar(shape, chunk_size);
    if (st != SSD_OK) return st;
    const ssd_shape s = *shape;
    const int H = (int)s.nheads, G = (int)s.ngroups, P = (int)s.headdim, N = (int)s.dstate;
    const int Q = chunk_size;
    cudaStream_t cst = static_cast<cudaStream_t>(stream);
    if (!h_loc || !log_decay || !aligned16(h_loc))
        return fail(SSD_ERR_INVALID_ARG, "h_loc (16-byte aligned) and log_decay must be non-NULL");
    if (s.batch == 0) return SSD_OK;
    cudaError_t e;
    if (s.seqlen == 0) {   // an empty segment: no state of its own, no decay
        e = cudaMemsetAsync(h_loc, 0, (size_t)s.batch * H * P * N * 4, cst);
        if (e == cudaSuccess) e = cudaMemsetAsync(log_decay, 0, (size_t)s.batch * H * 4, cst);
        return e == cudaSuccess ? SSD_OK : cuda_fail(e, "clear empty segment");
    }
    if (!x || !dt || !A || !B || !workspace)
        return fail(SSD_ERR_INVALID_ARG, "x, dt, A, B and workspace must be non-NULL");
    if (!aligned16(x) || !aligned16(B) || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(SSD_ERR_INVALID_ARG, "x, B must be 16-byte and workspace 256-byte aligned");
    if (workspace_bytes < ssd_seqpar_workspace_size(shape, Q))
        return fail(SSD_ERR_INVALID_ARG, "workspace too small");
    const int64_t nchunks = (s.seqlen + Q - 1) / Q;
    const ssd::WsLayout wl = layout(&s, Q);
    char *ws = static_cast<char *>(workspace);
    int *status = reinterpret_cast<int *>(ws + wl.status);
    float *cs = reinterpret_cast<float *>(ws + wl.cs);
    float *dtc = reinterpret_cast<float *>(ws + wl.dtc);
    float *states = reinterpret_cast<float *>(ws + wl.states);
    ssd::bf16 *hin = reinterpret_cast<ssd::bf16 *>(ws + wl.hin_bf16);
    const char *why = "";
    e = ssd::launch_chunk_cumsum(dt, A, cs, dtc, status, s.batch, s.seqlen, H, Q, nchunks, cst);
    if (e != cudaSuccess) return cuda_fail(e, "dA cumsum launch");
    e = ssd::launch_chunk_state_tc((const ssd::bf16 *)x, dtc, (const ssd::bf16 *)B, cs, states,
                                   status, s.batch, s.seqlen, H, G, Q, nchunks, cst, &why);
    if (e != cudaSuccess) return cuda_fail(e, why);
    // from a zero initial state: the final state is the segment's own contribution h_loc (the
    // entering states it also writes are replaced in the finish phase; chunk states are kept)
    e = ssd::launch_state_passing(states, cs, nullptr, h_loc, hin, s.batch, H, P, N, Q, nchunks,
                                  cst);
    if (e != cudaSuccess) return cuda_fail(e, "state passing launch");
    e = ssd::launch_segment_log_decay(cs, log_decay, s.batch, H, Q, nchunks, cst);
    if (e != cudaSuccess) return cuda_fail(e, "segment decay launch");
    return SSD_OK;
}

ssd_status ssd_seqpar_finish(const ssd_shape *shape, const void *x, const void *B, const void *C,
                             const float *D, int chunk_size, const float *h_loc_all,
                             const float *log_decay_all, int nranks, int rank,
                             const float *init_state, void *y, float *final_state,
                             void *workspace, size_t workspace_bytes, void *stream)
{
    ssd_status st = check_seqpar(shape, chunk_size);
    if (st != SSD_OK) return st;
    if (nranks < 1 || rank < 0 || rank >= nranks)
        return fail(SSD_ERR_INVALID_ARG, "rank %d out of range for %d ranks", rank, nranks);
    const ssd_shape s = *shape;
    const int H = (int)s.nheads, G = (int)s.ngroups, P = (int)s.headdim, N = (int)s.dstate;
    const int Q = chunk_size;
    cudaStream_t cst = static_cast<cudaStream_t>(stream);
    if ((rank > 0 && (!h_loc_all || !log_decay_all)) || !workspace)
        return fail(SSD_ERR_INVALID_ARG, "h_loc_all, log_decay_all and workspace must be non-NULL");
    if ((h_loc_all && !aligned16(h_loc_all)) || (init_state && !aligned16(init_state)) ||
        (final_state && !aligned16(final_state)) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(SSD_ERR_INVALID_ARG, "state pointers must be 16-byte aligned, workspace 256");
    if (workspace_bytes < ssd_seqpar_workspace_size(shape, Q))
        return fail(SSD_ERR_INVALID_ARG, "workspace too small");
    if (s.batch == 0) return SSD_OK;
    char *ws = static_cast<char *>(workspace);
    float *hseg = reinterpret_cast<float *>(ws + seqpar_hseg_offset(&s, Q));
    const int64_t BH = s.batch * H;
    cudaError_t e = ssd::launch_seqpar_combine(h_loc_all, log_decay_all, init_state, hseg, nranks,
                                               rank, BH, P * N, cst);
    if (e != cudaSuccess) return cuda_fail(e, "combine launch");
    if (s.seqlen == 0) {
        if (final_state) {
            e = ssd::launch_fill_final(hseg, final_state, BH * P * N, cst);
            if (e != cudaSuccess) return cuda_fail(e, "fill final state");
        }
        return SSD_OK;
    }
    if (!x || !B || !C || !D || !y) return fail(SSD_ERR_INVALID_ARG, "x, B, C, D, y must be non-NULL");
    if (!aligned16(x) || !aligned16(B) || !aligned16(C) || !aligned16(y))
        return fail(SSD_ERR_INVALID_ARG, "x, B, C and y must be 16-byte aligned");
    const int64_t nchunks = (s.seqlen + Q - 1) / Q;
    const ssd::WsLayout wl = layout(&s, Q);
    int *status = reinterpret_cast<int *>(ws + wl.status);
    float *cs = reinterpret_cast<float *>(ws + wl.cs);
    float *dtc = reinterpret_cast<float *>(ws + wl.dtc);
    float *states = reinterpret_cast<float *>(ws + wl.states);
    ssd::bf16 *hin = reinterpret_cast<ssd::bf16 *>(ws + wl.hin_bf16);
    const char *why = "";
    e = ssd::launch_state_passing(states, cs, hseg, final_state, hin, s.batch, H, P, N, Q,
                                  nchunks, cst);
    if (e != cudaSuccess) return cuda_fail(e, "state passing launch");
    e = ssd::launch_chunk_scan_tc((const ssd::bf16 *)x, dtc, (const ssd::bf16 *)B,
                                  (const ssd::bf16 *)C, cs, hin, D, (ssd::bf16 *)y, status,
                                  s.batch, s.seqlen, H, G, Q, nchunks, cst, &why);
    if (e != cudaSuccess) return cuda_fail(e, why);
    return SSD_OK;
}

ssd_status ssd_state_update_ex(const ssd_shape *shape, float *state, const void *x,
                               const float *dt, const float *A, const void *B, const void *C,
                               const float *D, void *y, void *stream,
                               const ssd_fwd_options *options)
{
    ssd_status st = check_shape(shape, false);
    if (st != SSD_OK) return st;
    const ssd_shape s = *shape;
    if (s.batch == 0) return SSD_OK;
    if (!state || !x || !dt || !A || !B || !C || !D || !y)
        return fail(SSD_ERR_INVALID_ARG, "state, x, dt, A, B, C, D and y must be non-NULL");
    if (!aligned16(state) || !aligned16(B) || !aligned16(C))
        return fail(SSD_ERR_INVALID_ARG, "state, B and C must be 16-byte aligned");
    ssd::DecodeOptions opt;
    if (options) {
        if (options->dt_max > 0.f && !(options->dt_min <= options->dt_max))
            return fail(SSD_ERR_INVALID_ARG, "dt_min must not exceed dt_max");
        opt.z = options->z;
        opt.dt_bias = options->dt_bias;
        opt.softplus = options->dt_softplus != 0;
        opt.clamp = options->dt_max > 0.f;
        opt.lo = options->dt_min;
        opt.hi = options->dt_max;
    }
    cudaError_t e = ssd::launch_state_update(s.dtype == SSD_BF16, state, x, dt, A, B, C, D, y,
                                             s.batch, (int)s.nheads, (int)s.ngroups,
                                             (int)s.headdim, (int)s.dstate,
                                             static_cast<cudaStream_t>(stream), opt);
    if (e != cudaSuccess) return cuda_fail(e, "state update launch");
    return SSD_OK;
}

ssd_status ssd_state_update(const ssd_shape *shape, float *state, const void *x,
                            const float *dt, const float *A, const void *B, const void *C,
                            const float *D, void *y, void *stream)
{
    return ssd_state_update_ex(shape, state, x, dt, A, B, C, D, y, stream, nullptr);
}

ssd_status ssd_workspace_status(const void *workspace, size_t workspace_bytes, void *stream)
{
    if (!workspace || workspace_bytes < sizeof(int))
        return fail(SSD_ERR_INVALID_ARG, "workspace is NULL or too small");
    int word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost,
                                    static_cast<cudaStream_t>(stream));
    if (e == cudaSuccess) e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "read workspace status");
    if (word & ssd::kStatusBadSeqlens)
        return fail(SSD_ERR_INVALID_ARG,
                    "cu_seqlens must start at 0, never decrease and end at the token count");
    if (word != 0)
        return fail(SSD_ERR_TIMEOUT, "an in-kernel barrier wait exceeded its bound (code %d)",
                    word);
    return SSD_OK;
}

}  // extern "C"
