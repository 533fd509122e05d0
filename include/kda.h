/*
 * libkda: Kimi Delta Attention (KDA) prefill and decode on NVIDIA B200 (sm_100a).
 *
 * The operation (per sequence n and head h, tokens t in order):
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(exp g_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t,          log-decay g bounded below at -5
 *
 * i.e. linear attention with a fixed-size per-head state S (dk x dv) updated
 * by the delta rule with per-channel retention.  The pages that describe it:
 *   - neurohive.io, "Kimi K3 ... overview", section "Sequence length: hybrid
 *     KDA and Gated MLA attention": delta rule (forget old content, write new
 *     content), fixed-size recurrent state, log-decay bounded from below at
 *     -5 so that every tile can run as a dense tensor-core product.
 *   - best.xiaohu.ai, "Kimi K3 tech report", section "Sequence length:
 *     replacing most attention layers with fixed-size memory": the state
 *     decays gradually across channels; memory stays constant in length.
 *   - neurohive.io, same article, section "Training and inference
 *     infrastructure": the KDA recurrent state is fixed in size with a single
 *     copy per request (the decode step updates it in place).
 *
 * Conventions shared by every call
 * --------------------------------
 *  - All tensor arguments are DEVICE pointers owned by the caller, dense and
 *    row-major in the shapes given; the library never frees or keeps them.
 *    (kda_chunk_prefill_host alone takes host pointers for its tensors.)
 *  - q, k, g share the shape [rows, H, dk]; v and o are [rows, H, dv];
 *    beta is [rows, H].  Element type is `dtype` for q, k, v, g and beta.
 *  - o is always fp32, and so is the state [N, H, dk, dv]: row c = key
 *    channel, column j = value channel, so o_t[j] = sum_c S_t[c][j] q_t[c].
 *    (Both accumulate in fp32; rounding o to bf16 alone would cost up to
 *    ~4e-2 of max|error|/rms(o) on heavy-tailed outputs.)
 *  - g is the per-step log-decay; the contract is g in [-5, 0].  Values
 *    below -5 are treated as -5 (max(g, -5)); values above 0 are used as
 *    given.  q and k are expected L2-normalised by the caller; the library
 *    does not normalise and applies no 1/sqrt(dk) scale.
 *  - Supported sizes: dk == dv, both 64 or 128.  Anything else returns
 *    KDA_ERR_UNSUPPORTED with nothing launched.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream).  Argument errors are returned synchronously, before
 *    anything is launched.  Launch failures return KDA_ERR_CUDA.
 *  - Device-side waits are bounded: a kernel that gives up waiting records
 *    it in a per-library error word and exits; kda_check_device_error()
 *    reports it as KDA_ERR_TIMEOUT.  Kernels never trap.
 *  - Thread safety: calls on different streams may run concurrently, except
 *    that the error word is shared by every call in the process.  A wait that
 *    gives up ends only the launch it belongs to: a timeout recorded by an
 *    earlier or a concurrent launch never cuts short another launch's work.
 *  - Debug input scan: with the environment variable KDA_DEBUG_CHECKS=1 (read
 *    at every call), each prefill and decode call first scans g and records
 *    any value outside [-5, 0] (or NaN) in the error word, which the next
 *    kda_check_device_error() reports as KDA_ERR_INPUT_RANGE.  The contract
 *    on g is a property of the model's gate (the lower bound of neurohive.io
 *    "Kimi K3 ... overview", section "Sequence length: hybrid KDA and Gated
 *    MLA attention"); the scan reports a caller's inputs leaving it and
 *    changes no result.  It is skipped when g holds gate logits
 *    (KDA_PREP_GATE_LOGIT); for packed sequences it covers the rows
 *    [cu_seqlens[0], cu_seqlens[N]).
 */
#ifndef KDA_H
#define KDA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KDA_API __attribute__((visibility("default")))
#else
#define KDA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,   /* NULL required pointer, negative size, bad cu_seqlens shape, short workspace */
    KDA_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. dk != dv, d not 64/128) */
    KDA_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
    KDA_ERR_TIMEOUT = 4,       /* a device-side bounded wait gave up (see kda_check_device_error) */
    KDA_ERR_INPUT_RANGE = 5    /* debug scan only: a log-decay outside [-5, 0] or NaN (KDA_DEBUG_CHECKS) */
} kda_status;

typedef enum {
    KDA_F32 = 0,   /* fp32 q, k, v, g, beta; fp32 arithmetic throughout (reference precision) */
    KDA_BF16 = 1   /* bf16 q, k, v, g, beta; tensor-core products (tf32 for the decay-rescaled
                      intra-chunk products, fp16 elsewhere) with fp32 accumulation; fp32 state
                      and o.  |v| and |state| must stay below 65504 (fp16 operand range). */
} kda_dtype;

/*
 * Bytes of device workspace kda_chunk_prefill needs for a call with
 * `rows` = B*T packed tokens, N sequences and H heads.  The value is an
 * upper bound valid for every cu_seqlens with that many rows and sequences.
 * Returns 0 when the call needs no workspace (the fp32 path).
 */
KDA_API size_t kda_chunk_prefill_workspace_bytes(int64_t rows, int N, int H, int dk, int dv,
                                         kda_dtype dtype);

/*
 * Chunked prefill: runs the recurrence above over whole sequences.
 *
 * Chunked form (chunk C = 64 tokens; exact arithmetic does not depend on C):
 * chunk-local log-space cumulative decay G, decay-rescaled intra-chunk
 * products Akk/Aqk, the unit-lower-triangular (UT/WY) solve that turns the
 * sequential delta rule into matrix products, then the inter-chunk pass of
 * the fp32 state with the outputs.
 *
 *  q, k, g     [B, T, H, dk]  (B == 1 when cu_seqlens is given)
 *  v           [B, T, H, dv]
 *  beta        [B, T, H]
 *  state_in    [N, H, dk, dv] fp32, or NULL for a zero initial state
 *  cu_seqlens  device int32 [N+1], offsets of the N packed sequences into the
 *              T rows (cu_seqlens[0] == 0, non-decreasing, cu_seqlens[N] <= T),
 *              or NULL: then N must equal B and sequence b owns batch row b.
 *              Values are read on the device.  Offsets that break these rules
 *              never make the library read or write outside the buffers
 *              (offsets are clamped to [0, T] and raised to the previous
 *              offset), but the results for such sequences are unspecified.
 *  o           [B, T, H, dv] fp32, written for every token that belongs to a sequence
 *  state_out   [N, H, dk, dv] fp32, final state per sequence, or NULL (not
 *              written).  May alias state_in exactly (in-place update).
 *              A zero-length sequence gets state_out = state_in (or zeros).
 *  With dtype KDA_BF16 and d = 128 (the tensor-core path) q, k, g and v are
 *  read as TMA tiles: their base addresses must be 16-byte aligned (else
 *  KDA_ERR_INVALID_ARG) and B*T must stay below 2^31 (else KDA_ERR_UNSUPPORTED).
 *  workspace   device scratch of at least kda_chunk_prefill_workspace_bytes()
 *              bytes, 256-byte aligned, or NULL when that size is 0.  Its
 *              contents on return are the per-chunk intermediates of the
 *              bf16 path (laid out for the state pass); callers may ignore them.
 *
 * bf16 at d = 128 with at most 37 (sequence, head) units runs both phases in
 * one launch (the state pass beside the intra-chunk work, handed each chunk's
 * intermediates through ready words in the workspace, every wait bounded);
 * more units run the intra-chunk kernel, then the state pass.  The choice
 * depends on the shapes only.
 */
KDA_API kda_status kda_chunk_prefill(const void *q, const void *k, const void *v,
                             const void *g, const void *beta,
                             const float *state_in, const int32_t *cu_seqlens,
                             int B, int64_t T, int N, int H, int dk, int dv,
                             kda_dtype dtype, void *o, float *state_out,
                             void *workspace, size_t workspace_bytes,
                             void *stream);

/*
 * Prefill that also stores intermediate states, for prefix caching: for each
 * sequence, the state after its first m * interval tokens for every m >= 1
 * with m * interval < its length (the state after all of its tokens is
 * state_out).  Serving layers keep such snapshots so that a later request
 * sharing a prefix resumes from one instead of recomputing it; the pages give
 * no interface for it.  Everything else is exactly kda_chunk_prefill.
 *  interval       tokens between snapshots: a positive multiple of 64 (the
 *                 chunk length), else KDA_ERR_UNSUPPORTED (also for KDA_F32
 *                 and for d = 64: snapshots come from the d = 128 bf16 path)
 *  ckpt           fp32 [ckpt_capacity, H, dk, dv], 16-byte aligned.  Entry
 *                 e = (number of snapshots of sequences 0..n-1) + m - 1 holds
 *                 sequence n's m-th snapshot; kda_prefill_checkpoint_count()
 *                 gives the total.  Snapshots past ckpt_capacity are not
 *                 written and the next kda_check_device_error() returns
 *                 KDA_ERR_INVALID_ARG.
 */
KDA_API kda_status kda_chunk_prefill_checkpointed(const void *q, const void *k, const void *v,
                                          const void *g, const void *beta,
                                          const float *state_in, const int32_t *cu_seqlens,
                                          int B, int64_t T, int N, int H, int dk, int dv,
                                          kda_dtype dtype, void *o, float *state_out,
                                          int64_t interval, float *ckpt, int64_t ckpt_capacity,
                                          void *workspace, size_t workspace_bytes,
                                          void *stream);

/*
 * Input preprocessing done inside the prefill (flags of kda_chunk_prefill_ex):
 *  KDA_PREP_GATE_LOGIT   g holds gate logits x; the log-decay used is
 *                        g = -5 sigmoid(x), which lies in (-5, 0) by
 *                        construction (the lower bound of neurohive.io "Kimi
 *                        K3 ... overview", section "Sequence length: hybrid KDA
 *                        and Gated MLA attention", written as a parametrisation)
 *  KDA_PREP_L2NORM_QK    q and k are normalised to unit L2 norm over dk per
 *                        (token, head) before use; an all-zero vector stays zero
 * The pages do not give the layer's gate form; this is the parametrisation the
 * synthetic inputs use, moved into the kernel so that callers pass raw
 * projections.
 */
enum { KDA_PREP_GATE_LOGIT = 1u, KDA_PREP_L2NORM_QK = 2u };

/*
 * The general prefill: kda_chunk_prefill with input preprocessing `flags`
 * (KDA_PREP_*; 0 = none) and, when ckpt_interval > 0, the intermediate states
 * of kda_chunk_prefill_checkpointed.  flags != 0 needs KDA_BF16 and d = 128
 * (else KDA_ERR_UNSUPPORTED); unknown flag bits are KDA_ERR_INVALID_ARG.  With
 * flags = 0 and ckpt_interval = 0 it is exactly kda_chunk_prefill.
 */
KDA_API kda_status kda_chunk_prefill_ex(const void *q, const void *k, const void *v,
                                const void *g, const void *beta,
                                const float *state_in, const int32_t *cu_seqlens,
                                int B, int64_t T, int N, int H, int dk, int dv,
                                kda_dtype dtype, uint32_t flags, void *o, float *state_out,
                                int64_t ckpt_interval, float *ckpt, int64_t ckpt_capacity,
                                void *workspace, size_t workspace_bytes, void *stream);

/*
 * Number of snapshots kda_chunk_prefill_checkpointed() writes, from the
 * host's copy of cu_seqlens (same clamping as the device) or, with
 * cu_seqlens_host NULL, for N = B sequences of T tokens.  -1 for invalid
 * arguments.
 */
KDA_API int64_t kda_prefill_checkpoint_count(const int32_t *cu_seqlens_host, int B, int64_t T,
                                             int N, int64_t interval);

/*
 * Single-token decode step, state updated in place (one read and one write
 * of each (n, h) state):
 *     S' = Diag(exp g) S;  delta = beta (v - S'^T k);  S = S' + k delta^T;
 *     o = S^T q
 *  q, k, g [N, H, dk];  v [N, H, dv];  beta [N, H];  o [N, H, dv] fp32
 *  state   [N, H, dk, dv] fp32, read and overwritten.
 */
KDA_API kda_status kda_decode_step(const void *q, const void *k, const void *v,
                           const void *g, const void *beta, float *state,
                           int N, int H, int dk, int dv, kda_dtype dtype,
                           void *o, void *stream);

/*
 * The same decode step on a pooled state (continuous batching): request n's
 * state is entry slots[n] of a pool of P, and only those entries are read and
 * overwritten.  This keeps the per-request state a single copy wherever the
 * serving layer keeps it (the "fixed-size state, single copy per request" of
 * neurohive.io "Kimi K3 ... overview", section "Training and inference
 * infrastructure"); the pages give no interface for it.
 *  q, k, g [N, H, dk];  v [N, H, dv];  beta [N, H];  o [N, H, dv] fp32
 *  state_pool  [P, H, dk, dv] fp32, 16-byte aligned, entries slots[n] updated in place
 *  slots       device int32 [N].  Must be distinct (two requests on one entry
 *              race).  Values are read on the device: an entry outside [0, P)
 *              is skipped (its o is not written, no memory outside the pool is
 *              touched) and the next kda_check_device_error() returns
 *              KDA_ERR_INVALID_ARG.
 */
KDA_API kda_status kda_decode_step_indexed(const void *q, const void *k, const void *v,
                                   const void *g, const void *beta, float *state_pool,
                                   const int32_t *slots, int N, int P, int H, int dk, int dv,
                                   kda_dtype dtype, void *o, void *stream);

/*
 * Backward of the recurrence (training): given do = dL/do [B, T, H, dv] fp32
 * and dL/dS_final (dstate_out [N, H, dk, dv] fp32, or NULL for zero), writes
 * dq, dk, dg [B, T, H, dk], dv [B, T, H, dv], dbeta [B, T, H] (all fp32, for
 * every token that belongs to a sequence) and dL/dS_0 (dstate_in, or NULL).
 * The inputs are those of the forward call (q, k, v, g, beta in `dtype`,
 * state_in fp32 or NULL, the same cu_seqlens convention).  g's clamp at -5
 * passes no gradient below the bound.  The pages give no formulas for the
 * backward; it is the exact derivative of the recurrence (fp32, recomputing
 * states from stored chunk starts; with few (sequence, head) units the value
 * columns are split over several CTAs whose partial sums are added in a fixed
 * order, so results are the same on every run).
 *  For bf16 with dk = 128 (the chunked form) q, k, v, g, do and dv must be
 *  16-byte aligned, else KDA_ERR_INVALID_ARG; state_in, dstate_out and
 *  dstate_in always must.
 *  workspace  at least kda_backward_workspace_bytes() bytes, 16-byte aligned
 *             (chunk-start states, per-token states of one chunk per unit, and
 *             the partial sums when the columns are split)
 * Supported sizes as for the prefill (dk == dv in {64, 128}).
 */
KDA_API size_t kda_backward_workspace_bytes(int64_t rows, int N, int H, int dk, int dv);
KDA_API kda_status kda_backward(const void *q, const void *k, const void *v, const void *g,
                                const void *beta, const float *state_in,
                                const int32_t *cu_seqlens, int B, int64_t T, int N, int H,
                                int dk, int dv, kda_dtype dtype, const float *dout,
                                const float *dstate_out, float *dq, float *dk_out, float *dv_out,
                                float *dg, float *dbeta, float *dstate_in, void *workspace,
                                size_t workspace_bytes, void *stream);

/*
 * Synchronises `stream`, then reads the device error word and reports ONE
 * recorded condition, clearing only that one, most severe first:
 *   KDA_ERR_TIMEOUT      a kernel gave up a bounded wait since it was last reported
 *   KDA_ERR_INVALID_ARG  a kernel skipped work because of an out-of-range index
 *                        read on the device (kda_decode_step_indexed slots, a
 *                        snapshot array too small for kda_chunk_prefill_checkpointed)
 *   KDA_ERR_INPUT_RANGE  the debug input scan (KDA_DEBUG_CHECKS=1) saw a
 *                        log-decay outside [-5, 0]
 * so calling it until it returns KDA_OK drains every condition.  Returns
 * KDA_ERR_CUDA if the stream reported an error, KDA_OK if nothing is recorded.
 */
KDA_API kda_status kda_check_device_error(void *stream);

/*
 * Diagnostic: launches one tiny kernel that waits on an mbarrier no one will
 * ever complete, with the same bounded wait the production kernels use,
 * giving up after `timeout_us` microseconds.  It records the timeout in the
 * error word exactly as a production kernel would, so a following
 * kda_check_device_error() returns KDA_ERR_TIMEOUT and the context stays
 * usable.  timeout_us must be in [1, 10^7]; otherwise KDA_ERR_INVALID_ARG.
 */
KDA_API kda_status kda_selftest_bounded_wait(int64_t timeout_us, void *stream);

/*
 * Kernel timing.  kda_profile_enable(1) makes every following prefill/decode
 * call on this device record CUDA events on its stream around each kernel it
 * launches; kda_profile_enable(0) stops it (and is the default).  Each call
 * replaces the previous record.  kda_profile_last() waits for the last
 * recorded event and writes the device time of each kernel of the most
 * recent call, in launch order, to ms[0 .. *count-1] (at most `capacity`).
 * Prefill (bf16) launches the intra-chunk products and the state pass, after a
 * chunk-table kernel when cu_seqlens is given; prefill (fp32) and decode
 * launch one.
 */
KDA_API kda_status kda_profile_enable(int enable);
KDA_API kda_status kda_profile_last(float *ms, int capacity, int *count);

/*
 * Prefill without any device allocation, for callers that cannot allocate:
 * code running in a serving step whose device memory is fully reserved up
 * front (a cudaMalloc there can fail under memory pressure and synchronises
 * the device, stalling every stream), or a plugin hosted by a runtime that
 * owns all allocation and gives it no allocator.  The paper has no
 * counterpart to this call; it is a property of this library.
 *
 * Same arguments and results as kda_chunk_prefill, without the workspace:
 * the bf16 path's scratch is a fixed array of KDA_STATIC_SCRATCH_BYTES in the
 * library's own device memory (every GPU that loads libkda holds it until the
 * process exits).  The caller still passes every input and output.
 *  - A call whose scratch need, kda_chunk_prefill_workspace_bytes(B*T, N, H,
 *    dk, dv, dtype), exceeds KDA_STATIC_SCRATCH_BYTES returns
 *    KDA_ERR_UNSUPPORTED with nothing launched (with H = 32 and d = 128 that
 *    is about 3.9k packed tokens per call for one sequence).
 *  - The first call on a device looks up the array's device address (no
 *    allocation); make that first call before any stream capture.
 *  - Every call on a device shares the one array, and the array keeps the
 *    last call's contents (nothing in it needs to start at zero: each call
 *    writes all the scratch it reads).  Calls whose kernels overlap on the
 *    GPU (other streams, other threads) race on it: serialise them.
 *  - The fp32 path needs no scratch and behaves exactly as kda_chunk_prefill.
 */
#define KDA_STATIC_SCRATCH_BYTES ((size_t)128 << 20)
KDA_API kda_status kda_chunk_prefill_static_scratch(const void *q, const void *k, const void *v,
                                                    const void *g, const void *beta,
                                                    const float *state_in,
                                                    const int32_t *cu_seqlens, int B, int64_t T,
                                                    int N, int H, int dk, int dv,
                                                    kda_dtype dtype, void *o, float *state_out,
                                                    void *stream);

/*
 * Prefill from HOST buffers, for a caller whose inputs and outputs live in
 * host memory: the same recurrence and results as kda_chunk_prefill over B
 * sequences of T tokens (no cu_seqlens), with the host <-> device copies done
 * by the library and overlapped with the computation.
 *
 * The T axis is cut into segments of `segment` tokens (a positive multiple of
 * 64; 0 picks 4096).  Segment s's inputs are copied in on one stream while
 * segment s - 1 is computed on `stream` and segment s - 2's o is copied out on
 * a third, so PCIe traffic in both directions overlaps and the call runs at
 * about the rate of the slower copy direction.  Segment s starts from segment
 * s - 1's final fp32 state, so the result is that of one call over all T
 * tokens (the recurrence is sequential; segments end on chunk boundaries).
 *
 *  q, k, g, v, beta, o   HOST pointers in the layouts of kda_chunk_prefill
 *                        (o fp32).  Page-locked memory (cudaHostAlloc,
 *                        cudaHostRegister) gives the overlap; pageable memory
 *                        is correct but copies synchronously.
 *  state_in, state_out   HOST fp32 [B, H, dk, dv], or NULL (zero / not written)
 *  workspace             DEVICE scratch of at least
 *                        kda_prefill_host_workspace_bytes() bytes, 256-byte
 *                        aligned: two segments of inputs and outputs, two
 *                        states and the prefill workspace of one segment.
 * The call is asynchronous on `stream` like every other: the host buffers
 * must stay valid, and o / state_out are complete, once `stream` has reached
 * the point after the call.  Returns KDA_ERR_UNSUPPORTED for sizes
 * kda_chunk_prefill does not support or a segment that is not a multiple of
 * 64, KDA_ERR_INVALID_ARG for NULL inputs or a short workspace.
 */
KDA_API size_t kda_prefill_host_workspace_bytes(int B, int64_t T, int H, int dk, int dv,
                                                kda_dtype dtype, int64_t segment);
KDA_API kda_status kda_chunk_prefill_host(const void *q, const void *k, const void *v,
                                          const void *g, const void *beta,
                                          const float *state_in, int B, int64_t T, int H,
                                          int dk, int dv, kda_dtype dtype, float *o,
                                          float *state_out, int64_t segment, void *workspace,
                                          size_t workspace_bytes, void *stream);

/* Static, human-readable name of a status code. */
KDA_API const char *kda_status_string(kda_status s);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H */
