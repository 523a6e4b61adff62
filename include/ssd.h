/*
 * ssd.h -- C ABI of the B200 (sm_100a) Mamba-2 SSD sequence mixer.
 *
 * The operation (per batch b, head h; g = h / (H/G) is the head's group of B/C):
 *
 *     a_t    = exp(dt_t * A_h)
 *     h_t    = a_t * h_{t-1} + dt_t * x_t (outer) B_t      state P x N, h_{-1} = init or 0
 *     y_t    = h_t C_t + D_h * x_t
 *
 * This is the selective SSM recurrence with a scalar-times-identity transition per head
 * (ql.gl "Why Does Mamba-2 Resemble the Transformer?", The Problem; chipfoundryservices.com
 * "hybrid attention-SSM", third paragraph), with A-bar = exp(dt A) and the D skip term
 * (mohakchugh.is-a.dev "Mamba-2", State Space Models: The Core Abstraction), and the input
 * scaled by dt as the same page's Multi-Head SSM block feeds it.
 *
 * Layouts (row-major, innermost last; all tensors dense and contiguous):
 *     x, y        (batch, seqlen, nheads, headdim)    element type `dtype`
 *     dt          (batch, seqlen, nheads)             float32, already positive (post-softplus)
 *     A, D        (nheads)                            float32
 *     B, C        (batch, seqlen, ngroups, dstate)    element type `dtype`
 *     state, init_state, final_state
 *                 (batch, nheads, headdim, dstate)    float32, dstate fastest
 *
 * Ownership: every pointer is a device pointer owned by the caller; the library allocates no
 * device or host memory in these calls and keeps no state across calls except a thread-local
 * error string.  Scratch space for the chunked scan is passed in by the caller (`workspace`).
 * All pointers to x, y, B, C, states and the workspace must be 16-byte aligned.
 *
 * Errors: functions return an ssd_status and never abort or throw.  Calls are asynchronous on
 * `stream` (a cudaStream_t passed as void*; NULL is the legacy default stream): the status
 * covers argument validation and launch errors only; faults inside a kernel surface at the
 * caller's next synchronisation.  ssd_last_error() describes the last non-OK status of the
 * calling thread.
 */
#ifndef SSD_B200_SSD_H
#define SSD_B200_SSD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SSD_OK = 0,
    SSD_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer, short workspace */
    SSD_ERR_UNSUPPORTED = 2,   /* a size outside the ranges listed below */
    SSD_ERR_CUDA = 3,          /* a CUDA call or kernel launch failed */
    SSD_ERR_TIMEOUT = 4        /* a bounded in-kernel wait gave up (see ssd_workspace_status) */
} ssd_status;

typedef enum { SSD_F32 = 0, SSD_BF16 = 1 } ssd_dtype;

/* Problem sizes.  seqlen is ignored by ssd_state_update (one token per call). */
typedef struct {
    int64_t batch;     /* >= 0 */
    int64_t seqlen;    /* >= 0 */
    int64_t nheads;    /* H >= 1 */
    int64_t headdim;   /* P: 1..128 */
    int64_t dstate;    /* N: multiple of 32 in 32..256, headdim * dstate <= 16384 */
    int64_t ngroups;   /* G >= 1, nheads % ngroups == 0 */
    int32_t dtype;     /* ssd_dtype of x, B, C and y */
} ssd_shape;

/*
 * Bytes of workspace ssd_chunk_scan_fwd needs for this shape and chunk size (0 when the
 * arguments are invalid; the call then also fails with the reason).  The workspace holds the
 * per-chunk cumulative log-decays, the per-chunk states and a device status word.
 */
size_t ssd_chunk_scan_workspace_size(const ssd_shape *shape, int chunk_size);

/*
 * Chunked (block-decomposed) SSD scan over a whole sequence: y for every token and, when
 * final_state is non-NULL, the state after the last token.
 *
 * The sequence is cut into chunks of chunk_size tokens (the last one may be partial); within a
 * chunk the output is the masked quadratic form (C B^T o L) (dt x) computed as dense matrix
 * products on tensor cores, and across chunks a P x N state is carried by the linear
 * recurrence (mohakchugh.is-a.dev "Mamba-2", Block Decomposition and The Tensor Core
 * Connection; ql.gl, The Core of SSD).  The result equals the token-by-token recurrence above
 * up to rounding, for any chunk_size.
 *
 *   chunk_size     Q in {16, 32, 64, 128, 256}.  bf16 with headdim 64, dstate 128 and
 *                  Q in {128, 256} runs the tensor-core (tcgen05) kernels; every other
 *                  supported shape runs the CUDA-core kernels in float32.
 *   init_state     nullable: NULL means a zero initial state.
 *   final_state    nullable: NULL means not written.  May alias init_state.
 *   y              must not alias any input.
 *   workspace      at least ssd_chunk_scan_workspace_size() bytes, 256-byte aligned; its
 *                  contents on entry do not matter and on exit are unspecified.
 *
 * Concurrent calls must use distinct workspaces.  batch == 0 or seqlen == 0 is valid: y is
 * empty and final_state is set to init_state (or zeros).
 */
ssd_status ssd_chunk_scan_fwd(const ssd_shape *shape, const void *x, const float *dt,
                              const float *A, const void *B, const void *C, const float *D,
                              int chunk_size, const float *init_state, void *y,
                              float *final_state, void *workspace, size_t workspace_bytes,
                              void *stream);

/*
 * Same as ssd_chunk_scan_fwd, and additionally records caller-created CUDA events on `stream`
 * around its kernels so that each stage can be timed on the device:
 *     stage_events[0]  before the dA cumsum kernel
 *     stage_events[1]  after it (before the chunk-state kernel)
 *     stage_events[2]  after the chunk-state kernel (before state passing)
 *     stage_events[3]  after state passing (before the chunk-scan kernel)
 *     stage_events[4]  after the chunk-scan kernel
 * stage_events points to 5 cudaEvent_t values (passed as void*); NULL behaves exactly like
 * ssd_chunk_scan_fwd.  The events are only recorded, never created, waited on or destroyed.
 */
ssd_status ssd_chunk_scan_fwd_staged(const ssd_shape *shape, const void *x, const float *dt,
                                     const float *A, const void *B, const void *C,
                                     const float *D, int chunk_size, const float *init_state,
                                     void *y, float *final_state, void *workspace,
                                     size_t workspace_bytes, void *stream,
                                     void *const *stage_events);

/*
 * Options of ssd_chunk_scan_fwd_ex: the Mamba-2 block's elementwise steps around the scan, fused
 * into it (mohakchugh.is-a.dev "Mamba-2", Architecture: the SSM output is gated by SiLU of a
 * second projection z; the discretisation step dt is the softplus of a projection plus a
 * per-head bias).  Every field is optional; a zeroed struct (or NULL options) is the plain scan.
 *
 *   z            nullable; (batch, seqlen, nheads, headdim), element type `dtype`, 16-byte
 *                aligned.  The output becomes y * z * sigmoid(z) (y as defined above).
 *   dt_bias      nullable; (nheads,) float32, added to dt before the softplus.
 *   dt_softplus  nonzero: the dt actually used is softplus(dt + dt_bias) = log(1 + exp(.)).
 *   dt_min, dt_max
 *                when dt_max > 0, that dt is then clamped to [dt_min, dt_max].
 * With any of dt_bias, dt_softplus or the clamp active, `dt` is the raw projection (any sign).
 */
typedef struct {
    const void *z;
    const float *dt_bias;
    int32_t dt_softplus;
    float dt_min;
    float dt_max;
} ssd_fwd_options;

/* Workspace bytes of ssd_chunk_scan_fwd_ex (0 when the arguments are invalid). */
size_t ssd_chunk_scan_fwd_ex_workspace_size(const ssd_shape *shape, int chunk_size,
                                            const ssd_fwd_options *options);

/* ssd_chunk_scan_fwd with the fused prologue / epilogue of `options` (nullable). */
ssd_status ssd_chunk_scan_fwd_ex(const ssd_shape *shape, const void *x, const float *dt,
                                 const float *A, const void *B, const void *C, const float *D,
                                 int chunk_size, const float *init_state, void *y,
                                 float *final_state, void *workspace, size_t workspace_bytes,
                                 void *stream, const ssd_fwd_options *options);

/*
 * Variable-length packed sequences: nseq sequences stored back to back along the token axis of
 * a batch-1 tensor, each with its own state.  Sequence s covers tokens
 * [cu_seqlens[s], cu_seqlens[s + 1]); its recurrence starts from init_states[s] (or zeros) at
 * its first token and ends in final_states[s]; no state crosses a boundary, so the result for
 * every sequence equals ssd_chunk_scan_fwd on that sequence alone (the state is carried between
 * blocks of one sequence only: mohakchugh.is-a.dev "Mamba-2", Block Decomposition; packed
 * sequences need no padding).  Sequences of any length, including 0, are allowed; a chunk never
 * spans two sequences (each sequence's last chunk may be partial).
 *
 *   shape          batch must be 1; seqlen = total tokens = cu_seqlens[nseq].
 *   x, y, dt, B, C (1, seqlen, ...) as for ssd_chunk_scan_fwd.
 *   cu_seqlens     device int32[nseq + 1], cu_seqlens[0] = 0, non-decreasing, last = seqlen.
 *                  Checked on the device: if inconsistent nothing is computed and
 *                  ssd_workspace_status() returns SSD_ERR_INVALID_ARG.
 *   init_states    nullable, float32 (nseq, nheads, headdim, dstate).
 *   final_states   nullable, float32 (nseq, nheads, headdim, dstate).
 *   workspace      ssd_chunk_scan_varlen_workspace_size() bytes, 256-byte aligned.
 *
 * Runs on the tensor-core path only (bf16, headdim 64, dstate 128, chunk_size 128 or 256);
 * other shapes return SSD_ERR_UNSUPPORTED.  Returns 0 from the size query when the arguments
 * are invalid.
 */
size_t ssd_chunk_scan_varlen_workspace_size(const ssd_shape *shape, int nseq, int chunk_size);
ssd_status ssd_chunk_scan_varlen_fwd(const ssd_shape *shape, const void *x, const float *dt,
                                     const float *A, const void *B, const void *C,
                                     const float *D, int chunk_size, const int32_t *cu_seqlens,
                                     int nseq, const float *init_states, void *y,
                                     float *final_states, void *workspace,
                                     size_t workspace_bytes, void *stream);

/*
 * Sequence parallelism: one long sequence split into contiguous segments, one per rank (GPU),
 * with one exchange of states between the two phases (the state is carried across segments
 * exactly as across chunks: mohakchugh.is-a.dev "Mamba-2", Block Decomposition).  Every rank r
 * holds its segment's x, dt, B, C as a (batch, seqlen_r, ...) tensor and calls
 *
 *   1. ssd_seqpar_local: chunk states of the segment and, from a zero initial state, its local
 *      final state h_loc (batch, nheads, headdim, dstate) float32 and its total log-decay
 *      log_decay (batch, nheads) float32 = sum of dt * A_h over the segment's tokens;
 *   2. (the caller) all-gathers h_loc and log_decay of all ranks in rank order, e.g. with
 *      torch.distributed.all_gather_into_tensor over NCCL: h_loc_all [nranks][batch][H][P][N],
 *      log_decay_all [nranks][batch][H];
 *   3. ssd_seqpar_finish: the segment's initial state
 *          h_in(r) = sum_{q<r} exp(sum_{q<s<r} log_decay_s) h_loc(q)
 *                    + exp(sum_{s<r} log_decay_s) init_state
 *      (init_state: the whole sequence's initial state, nullable; every rank passes the same),
 *      then y of the segment and, in final_state (nullable), the state after the segment's
 *      last token -- the sequence's final state on the last rank.
 *
 * Both phases take the same workspace (ssd_seqpar_workspace_size bytes, 256-byte aligned),
 * which carries the chunk states from phase 1 to phase 3.  On one rank (nranks = 1) the result
 * equals ssd_chunk_scan_fwd.  Tensor-core path only (bf16, headdim 64, dstate 128, chunk_size
 * 128 or 256); other shapes return SSD_ERR_UNSUPPORTED.  log_decay_all and h_loc_all may be
 * NULL on rank 0 (nothing precedes it).
 */
size_t ssd_seqpar_workspace_size(const ssd_shape *shape, int chunk_size);
ssd_status ssd_seqpar_local(const ssd_shape *shape, const void *x, const float *dt,
                            const float *A, const void *B, int chunk_size, float *h_loc,
                            float *log_decay, void *workspace, size_t workspace_bytes,
                            void *stream);
ssd_status ssd_seqpar_finish(const ssd_shape *shape, const void *x, const void *B, const void *C,
                             const float *D, int chunk_size, const float *h_loc_all,
                             const float *log_decay_all, int nranks, int rank,
                             const float *init_state, void *y, float *final_state,
                             void *workspace, size_t workspace_bytes, void *stream);

/*
 * Backward pass of the chunked scan: the gradients of a scalar loss with respect to every input,
 * given its gradients dy (with respect to y) and dfinal (with respect to the final state).
 * The pages give no backward; it is the reverse-mode derivative of the forward definition.  The
 * scan is a multiplication by a semiseparable matrix (mohakchugh.is-a.dev "Mamba-2", The
 * Duality), whose transpose is semiseparable too, so the adjoint state g_t = dL/dh_t obeys a
 * recurrence of the same form run backwards in time, g_t = exp(dt_{t+1} A_h) g_{t+1} + dy_t C_t^T with g_{L-1} = dy_{L-1} C_{L-1}^T + dfinal,
 * and the three contractions of the backward are scans of the forward's kind:
 *     dx_t = D_h dy_t + dt_t g_t B_t                  (tensor cores, time-reversed scan)
 *     dB_t = sum over the group's heads of dt_t g_t^T x_t     (CUDA cores, float32)
 *     dC_t = sum over the group's heads of h_t^T dy_t         (CUDA cores, float32)
 *     ddt_t = <x_t, g_t B_t> + A_h sum_{k>=t} q_k,
 *         q_k = <dy_k, y_k - D_h x_k> - dt_k <x_k, g_k B_k> (+ <dfinal, h_{L-1}> at k = L-1)
 *     dA_h = sum_{b,t} dt_t sum_{k>=t} q_k,   dD_h = sum_{b,t} <dy_t, x_t>,
 *     dinit = exp(dt_0 A_h) g_0.
 * Nothing needs to be kept from the forward call: the dC scan runs the forward recurrence
 * again (float32).  The decay gradient is a reverse cumulative sum that telescopes, so its two
 * dot products are taken from the float32 scans (<dy_k, y_k - D x_k> = <h_k^T dy_k, C_k>,
 * <x_k, g_k B_k> = <g_k^T x_k, B_k>), not from bf16 intermediates.
 *
 *   x, B, C, dy, dt, A, D, init_state: as for ssd_chunk_scan_fwd (dy has y's layout and dtype).
 *   dfinal   (batch, nheads, headdim, dstate) float32, nullable (= zero).
 *   dx (batch, seqlen, nheads, headdim), ddt (batch, seqlen, nheads), dA (nheads),
 *   dB, dC (batch, seqlen, ngroups, dstate), dD (nheads): float32 outputs, all required;
 *   dinit (batch, nheads, headdim, dstate) float32, nullable (skipped).  dA and dD are summed
 *   over the batch.  No output may alias an input.  x, B, C, dy, dx and the states must be
 *   16-byte aligned.
 *   workspace: ssd_chunk_scan_bwd_workspace_size bytes, 256-byte aligned, caller-owned; its
 *   status word (ssd_workspace_status) reports an in-kernel timeout as for the forward.
 * Tensor-core shapes only (bf16, headdim 64, dstate 128, chunk_size 128 or 256); others return
 * SSD_ERR_UNSUPPORTED, and the size query returns 0 for them.  Launches only on `stream`.
 */
size_t ssd_chunk_scan_bwd_workspace_size(const ssd_shape *shape, int chunk_size);
ssd_status ssd_chunk_scan_bwd(const ssd_shape *shape, const void *x, const float *dt,
                              const float *A, const void *B, const void *C, const float *D,
                              int chunk_size, const float *init_state, const void *dy,
                              const float *dfinal, float *dx, float *ddt, float *dA, float *dB,
                              float *dC, float *dD, float *dinit, void *workspace,
                              size_t workspace_bytes, void *stream);

/*
 * One recurrent (decode) step for one new token per sequence, O(1) in the length of the past
 * (crackai.dev "Transformers are SSMs", Why It Matters; mohakchugh.is-a.dev "Mamba-2", Why
 * This Matters for Hardware, linear mode):
 *     state <- exp(dt A) * state + dt * x (outer) B,     y = state C + D x
 *
 *   state  (batch, nheads, headdim, dstate) float32, updated in place.
 *   x, y   (batch, nheads, headdim)         element type `dtype`
 *   dt     (batch, nheads) float32;  B, C (batch, ngroups, dstate) element type `dtype`.
 *   y must not alias state or the inputs.
 */
ssd_status ssd_state_update(const ssd_shape *shape, float *state, const void *x,
                            const float *dt, const float *A, const void *B, const void *C,
                            const float *D, void *y, void *stream);

/*
 * ssd_state_update with the block's fused steps of `options` (nullable; see ssd_fwd_options):
 * z (batch, nheads, headdim) gates the output, y * z * sigmoid(z); dt_bias, dt_softplus and the
 * clamp turn the raw dt projection into the step used, as for ssd_chunk_scan_fwd_ex.
 */
ssd_status ssd_state_update_ex(const ssd_shape *shape, float *state, const void *x,
                               const float *dt, const float *A, const void *B, const void *C,
                               const float *D, void *y, void *stream,
                               const ssd_fwd_options *options);

/*
 * Synchronises `stream` and reads the device status word the last ssd_chunk_scan_fwd (or
 * ssd_chunk_scan_varlen_fwd) call on this workspace left behind: SSD_OK; SSD_ERR_TIMEOUT when
 * an in-kernel wait on a shared-memory barrier exceeded its bound and the kernel returned early
 * (its outputs are then incomplete); SSD_ERR_INVALID_ARG when a variable-length call's
 * cu_seqlens was inconsistent (nothing was computed).  Returns SSD_ERR_CUDA if the
 * synchronisation itself reports an error.
 */
ssd_status ssd_workspace_status(const void *workspace, size_t workspace_bytes, void *stream);

/*
 * The chunked scan for callers that cannot allocate device memory.  (No counterpart in the
 * paper or on its pages: this is a deployment convenience of this library.)
 *
 * Some callers cannot call cudaMalloc -- or any allocator -- where they run the scan: code inside
 * a framework's memory-planning or capture phase where the allocator is locked, a runtime that
 * owns all device memory and hands out only the tensors it planned, or a host that forbids
 * allocation after start-up.  They pass inputs and outputs exactly as for ssd_chunk_scan_fwd,
 * but no workspace: the scan uses a fixed 32 MiB scratch array built into this library
 * (resident on every GPU that loads the library until the process exits).
 *
 *   - Problems whose ssd_chunk_scan_workspace_size() exceeds 32 MiB (33554432 bytes) are
 *     rejected with SSD_ERR_UNSUPPORTED and a message naming both sizes; e.g. batch 2 x 2048
 *     tokens x 24 heads (headdim 64, dstate 128, chunk 256) needs about 19.3 MB and fits.
 *   - The first call on each device, with that device current, looks up the array's device
 *     address (cudaGetSymbolAddress) and caches it; make that first call before any stream
 *     capture.  The array of the calling thread's current device is used, so `stream` must
 *     belong to that device.
 *   - No memory is allocated or freed.  The array keeps the last call's contents; nothing in it
 *     needs to start at zero (the scan clears its own status word).
 *   - All calls on a device share the one array: calls whose kernels overlap on the GPU (other
 *     streams, other host threads) race and corrupt each other's results.  Issue them one after
 *     another on a single stream.
 *   - The address is cached per device for the device's primary context (the CUDA runtime's);
 *     running the scan in another context, or after a device reset, is not supported.
 *   - Results are bit-identical to ssd_chunk_scan_fwd's for the same arguments.
 *   - An in-kernel timeout is recorded in the array's status word, which
 *     ssd_chunk_scan_fwd_static_status() reads.
 */
ssd_status ssd_chunk_scan_fwd_static(const ssd_shape *shape, const void *x, const float *dt,
                                     const float *A, const void *B, const void *C,
                                     const float *D, int chunk_size, const float *init_state,
                                     void *y, float *final_state, void *stream);

/*
 * The status word that the last ssd_chunk_scan_fwd_static call on the current device left in
 * the built-in scratch array, as ssd_workspace_status() reports it for a caller workspace:
 * synchronises `stream`, then SSD_OK, or SSD_ERR_TIMEOUT when a bounded in-kernel wait gave up
 * (the outputs of that call are then incomplete).  SSD_ERR_CUDA if the array's address cannot
 * be looked up or the synchronisation reports an error.  Allocates nothing.
 */
ssd_status ssd_chunk_scan_fwd_static_status(void *stream);

/* Message for the calling thread's last non-OK status ("" if none). */
const char *ssd_last_error(void);

/* Library version string. */
const char *ssd_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SSD_B200_SSD_H */
