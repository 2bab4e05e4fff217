/*
 * kda_decode.h -- C ABI of the B200 (sm_100a) recurrent Kimi Delta Attention
 * (KDA) decode step.
 *
 * The operation.  For every sequence n in [0, N), value head h in [0, HV) and
 * token t in [0, T), applied in token order to the fp32 state S[K][V] that the
 * sequence keeps in slot slot_idx[n] of a caller-owned state pool:
 *
 *     S   <- Diag(exp(g[n,t,h,:])) S                 per-key-channel decay
 *     u   <- beta[n,t,h] * (v[n,t,h,:] - S^T k[n,t,h,:])   delta-rule correction
 *     S   <- S + k[n,t,h,:] u^T                       rank-1 write
 *     o   <- scale * S^T q[n,t,h,:]                   readout of the updated state
 *     out[n,t,h,:] <- bf16(o)                          (kda_decode)
 *     out[n,t,h,:] <- bf16(o / sqrt(mean(o^2) + eps) * w * sigmoid(z[n,t,h,:]))
 *                                                     (kda_decode_gated_rmsnorm)
 *
 * Where it comes from (pages by title):
 *   - vLLM #57585 "Tune recurrent KDA launch configuration on SM90",
 *     "Microbenchmark and earlier serving limits": BF16 q/k/v, FP32 recurrent
 *     state, K = V = 128; "Retained baseline trace attribution": one recurrent
 *     KDA call per KDA layer per decode step, 8 local heads, head dim 128.
 *   - FlashInfer #4562 "feat(cake_kda): add optimized H12 packed decode across
 *     SM100 family": the kernel updates the state and writes the output
 *     (sequence diagram); the slot table `state_indices` and the scale
 *     0.08838834764831845 = 1/sqrt(128) are kernel arguments (binding launch);
 *     caller-stream execution, caller-owned output, indexed recurrent state,
 *     inactive graph-padding rows, CUDA graph replay (PR description).
 *   - b12x #249 "feat(gdn): add direct single-token KDA decode": decode, then
 *     a gated RMS norm of the decoded output with z (sequence diagram);
 *     output must not overlap the read-only inputs (review of `_overlaps`).
 *   None of the pages prints the recurrence as a formula: the step order
 *   above (decay, correction on the decayed state, write, readout after the
 *   write) is the plainest reading that all of them support.
 *
 * Layouts.  Every tensor is dense, row-major (last index fastest), in memory
 * the current CUDA device reads at the given address: its own device memory,
 * or page-locked host memory mapped into its address space at the same
 * address (see kda_host_memory_is_mapped; the kernel then reads and writes that
 * memory across PCIe, so no separate copy is needed):
 *     q, k        bf16  [N, T, HV, K]     (one q/k head per value head)
 *     v           bf16  [N, T, HV, V]
 *     g           fp32  [N, T, HV, K]     log-decay, decay = exp(g)
 *     beta        fp32  [N, T, HV]
 *     state_pool  fp32  [num_slots, HV, K, V], read and written in place
 *                 (bf16 for the *_bf16_state entry points; kda_decode_ex
 *                 also takes [num_slots, HV, V, K] blocks, see below)
 *     slot_idx    int32 [N]               slot of each row; < 0 = inactive row
 *     out         bf16  [N, T, HV, V]
 *     gate (z)    bf16  [N, T, HV, V]     gated variant only
 *     norm_weight bf16  [V]               gated variant only, shared by heads
 *
 * Supported sizes: K in {64, 128, 256}; V a multiple of 32; V <= 256 for the
 * gated variant (its V tiles form one thread-block cluster); HV >= 1;
 * N, T >= 0 (N == 0 or T == 0 is a no-op that touches no pointer).
 * Alignment: q, k, v, g, state_pool, out, gate, norm_weight on 16 bytes;
 * beta and slot_idx on 4 bytes.
 *
 * Ownership and execution.  The caller owns every buffer.  A call allocates
 * nothing, never synchronises the host, and enqueues exactly one kernel on
 * `stream` (NULL = the legacy default stream); it can be captured in a CUDA
 * graph.  The first call on a device reads that device's compute capability
 * once and caches it.
 *
 * Caller contract (checked only where noted):
 *   - active slots in slot_idx are distinct and < num_slots (the fixed entry
 *     points take no pool size and do not check the upper bound;
 *     kda_decode_ex checks it when kda_decode_args.num_slots is set);
 *   - rows with slot_idx[n] < 0 get an all-zero output and do not touch the
 *     pool (CUDA-graph padding rows);
 *   - out overlaps no input and no part of the pool; the library rejects an
 *     out/input overlap, and any buffer that starts inside the pool's slot-0
 *     block or that contains the pool base (KDA_ERR_ALIAS).
 *
 * Errors.  Every entry point validates on the host and returns a status; it
 * never aborts, throws or prints.  Nothing is enqueued unless it returns
 * KDA_OK.  KDA_ERR_CUDA reports a failed launch (cudaGetLastError is not
 * consumed for unrelated earlier errors).
 */
#ifndef KDA_DECODE_H
#define KDA_DECODE_H

#include <stdint.h>

#if defined(__GNUC__)
#define KDA_API __attribute__((visibility("default")))
#else
#define KDA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
struct CUstream_st;
typedef struct CUstream_st *kda_stream_t;
/* Same type as cudaEvent_t. */
struct CUevent_st;
typedef struct CUevent_st *kda_event_t;

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1, /* null pointer with work to do, negative size, bad eps */
    KDA_ERR_UNSUPPORTED = 2, /* K, V or HV outside the supported set */
    KDA_ERR_ALIAS = 3,       /* out overlaps an input or the pool */
    KDA_ERR_MISALIGNED = 4,  /* a pointer breaks the alignment rule above */
    KDA_ERR_DEVICE = 5,      /* current device is not compute capability 10.0 */
    KDA_ERR_CUDA = 6,        /* the CUDA runtime refused the launch */
    KDA_ERR_SCRATCH_LIMIT = 7 /* kda_prefill_no_alloc: the sizes need more than its fixed scratch */
} kda_status;

/*
 * Plain decode step (see the top of this file).  Writes bf16(o) to out and the
 * updated state back to each active row's slot.  scale is usually 1/sqrt(K).
 */
KDA_API kda_status kda_decode(const void *q, const void *k, const void *v, const float *g,
                      const float *beta, float *state_pool, const int32_t *slot_idx,
                      void *out, int64_t N, int64_t T, int64_t HV, int64_t K, int64_t V,
                      float scale, kda_stream_t stream);

/*
 * Decode step followed, in the same kernel, by the gated RMS norm over V of
 * each (n, t, h) output row: y = o / sqrt(mean_V(o^2) + eps) * norm_weight *
 * sigmoid(gate), computed in fp32 from the unrounded o, then rounded to bf16
 * into out.  eps must be finite and >= 0.  The state update is identical to
 * kda_decode's.
 */
KDA_API kda_status kda_decode_gated_rmsnorm(const void *q, const void *k, const void *v, const float *g,
                                    const float *beta, float *state_pool,
                                    const int32_t *slot_idx, const void *gate,
                                    const void *norm_weight, float eps, void *out, int64_t N,
                                    int64_t T, int64_t HV, int64_t K, int64_t V, float scale,
                                    kda_stream_t stream);

/*
 * The same two operations on a bf16 state pool (state_pool: bf16 bits,
 * [num_slots, HV, K, V]).  The state is widened exactly, every step runs in
 * fp32 exactly as in the fp32-pool entry points, and the state is rounded to
 * the nearest bf16 (ties to even) once, when it is written back after the
 * call's last token.  The pool's traffic halves.  Source: FlashInfer #4562
 * "feat(cake_kda): add optimized H12 packed decode across SM100 family"
 * keeps the recurrent state in bf16 (the binding's kernel launch passes the
 * state as `__nv_bfloat16*`).  Arguments, layouts, alignment, errors and the
 * caller contract are those of kda_decode / kda_decode_gated_rmsnorm.
 */
KDA_API kda_status kda_decode_bf16_state(const void *q, const void *k, const void *v, const float *g,
                                         const float *beta, void *state_pool, const int32_t *slot_idx,
                                         void *out, int64_t N, int64_t T, int64_t HV, int64_t K,
                                         int64_t V, float scale, kda_stream_t stream);

KDA_API kda_status kda_decode_gated_rmsnorm_bf16_state(const void *q, const void *k, const void *v,
                                                       const float *g, const float *beta,
                                                       void *state_pool, const int32_t *slot_idx,
                                                       const void *gate, const void *norm_weight,
                                                       float eps, void *out, int64_t N, int64_t T,
                                                       int64_t HV, int64_t K, int64_t V, float scale,
                                                       kda_stream_t stream);

/* Element type of the state pool (kda_decode_args.state_dtype). */
enum { KDA_STATE_FP32 = 0, KDA_STATE_BF16 = 1 };

/*
 * Layout of each (slot, head) state block (kda_decode_args.state_layout):
 * KDA_LAYOUT_KV = [K][V] (value index fastest; the layout of the fixed entry
 * points), KDA_LAYOUT_VK = [V][K] (key index fastest: each value column's K
 * entries are contiguous, the layout FlashInfer #4562's kernels keep their
 * recurrent state in).  The pool is [num_slots, HV, K, V] or
 * [num_slots, HV, V, K] respectively; the operation is the same.
 */
enum { KDA_LAYOUT_KV = 0, KDA_LAYOUT_VK = 1 };

/*
 * Arguments of kda_decode_ex: every operation above in one call, with row
 * strides and the serving input form.
 *
 * Row strides.  Each input is a sequence of N*T rows, row (n, t) starting
 * (n*T + t) * <x>_row_stride elements after the pointer; inside a row, head h
 * of q, k, g and raw_gate occupies elements [h*K, (h+1)*K), of v and gate
 * [h*V, (h+1)*V), of beta and raw_beta element h.  A stride must be at least
 * the row's width; q, k, v, gate strides must be multiples of 8 elements, the
 * g stride of 4, the raw_gate stride of 8.  This lets q, k and v be slices of
 * one packed row [q | k | v] ("mixed_qkv", FlashInfer #4562's launch passes
 * mixed_qkv.stride(0) for all three) and beta a strided column.  The
 * dense layouts of the fixed entry points are the strides HV*K, HV*V and HV.
 * out is always dense [N, T, HV, V].
 *
 * Decay and beta.  Either g (fp32 log-decay) and beta (fp32), or the serving
 * form raw_gate (bf16) with A_log (fp32 [HV]) and dt_bias (fp32 [HV, K]), and
 * raw_beta (bf16), activated in the kernel as
 *     g = -exp(A_log[h]) * softplus(raw_gate + dt_bias[h, :]),  beta = sigmoid(raw_beta).
 * FlashInfer #4562 (kernel launch) and b12x #249 (run_kda_single_token) take
 * these raw inputs, but neither prints the activation: this formula is the
 * usual KDA gate, taken as a reading.  g/beta and the raw inputs are
 * exclusive (KDA_ERR_INVALID_ARG otherwise).
 *
 * gate and norm_weight both NULL selects the plain step, both set the gated
 * RMS norm.  state_dtype selects an fp32 or bf16 pool, state_layout its
 * block layout (KDA_LAYOUT_KV or KDA_LAYOUT_VK; anything else is
 * KDA_ERR_INVALID_ARG).  Pointers without a
 * use in the selected form must be NULL.  Alignment: q, k, v, g, raw_gate,
 * dt_bias, state_pool, out, gate, norm_weight 16 bytes; beta, A_log,
 * slot_idx 4 bytes; raw_beta 2 bytes.
 */
typedef struct {
    const void *q;        int64_t q_row_stride;
    const void *k;        int64_t k_row_stride;
    const void *v;        int64_t v_row_stride;
    const float *g;       int64_t g_row_stride;       /* also the raw_gate row stride */
    const float *beta;    int64_t beta_row_stride;    /* also the raw_beta row stride */
    const void *raw_gate;
    const float *A_log;
    const float *dt_bias;
    const void *raw_beta;
    void *state_pool;     int32_t state_dtype;        int32_t state_layout;
    const int32_t *slot_idx;
    const void *gate;     int64_t gate_row_stride;
    const void *norm_weight;
    float eps;
    void *out;
    int64_t N, T, HV, K, V;
    float scale;
    /*
     * Checked slots.  num_slots = 0 leaves slot_idx unchecked (the caller
     * contract above).  num_slots > 0 declares the pool's size: an active row
     * whose slot_idx[n] >= num_slots is then treated as an inactive row (all-zero
     * output, no pool access) and, when status is not NULL, the kernel stores 1
     * to *status (device int32, 4-byte aligned, caller-owned; the library never
     * clears it, so the caller zeroes it before the calls it wants to watch).
     * FlashInfer #4562 (PR description) runs the step on an indexed, non-compact
     * recurrent state: the slot table is data on the device that the host cannot
     * validate before the launch, so the check is made by the kernel.  A checked
     * call also lets the library see the pool's whole extent for its aliasing
     * check.  Checked calls run the row-strided kernels (one integer compare per
     * CTA); the fixed entry points are unchecked.
     */
    int64_t num_slots;
    int32_t *status;
} kda_decode_args;

/*
 * The general entry point (see kda_decode_args).  The operation, the caller
 * contract, ownership and errors are those of kda_decode and
 * kda_decode_gated_rmsnorm.  args is read during the call only.
 */
KDA_API kda_status kda_decode_ex(const kda_decode_args *args, kda_stream_t stream);

/*
 * The step fed from and returning to host memory, in one call.  It enqueues on
 * `stream`, in order: a host-to-device copy of in_bytes bytes from host_in to
 * dev_in; the step that kda_decode_ex(args) enqueues; a device-to-host copy of
 * the output (N*T*HV*V bf16 from args->out) to host_out.  The caller stages a
 * step's inputs in host_in so that, once copied, args' input pointers (q, k,
 * v, g/beta or the raw inputs, slot_idx, gate, norm_weight) point at them
 * inside dev_in; the state pool stays on the device.  For the copies to run
 * asynchronously host_in and host_out must be page-locked; host_out holds the
 * output once the stream has reached the end of the call.  The library
 * allocates nothing: dev_in is caller-owned device memory.  None of the pages
 * describes such an entry point: it is this library's own, for callers that
 * measure or run the step end to end from host memory.
 *
 * Errors: those of kda_decode_ex; KDA_ERR_INVALID_ARG also for in_bytes < 0,
 * a NULL host_in or dev_in with in_bytes > 0, or a NULL host_out;
 * KDA_ERR_ALIAS if dev_in overlaps the state pool's visible extent.  Nothing
 * is enqueued unless validation passes; N == 0 or T == 0 enqueues nothing.
 */
KDA_API kda_status kda_decode_host(const kda_decode_args *args, const void *host_in, void *dev_in,
                                   int64_t in_bytes, void *host_out, kda_stream_t stream);

/*
 * kda_decode_host with the copy in on a second stream, so that consecutive
 * steps overlap: one step's copy in runs while the previous step computes and
 * copies its output out.  Like kda_decode_host, none of the pages describes
 * such an entry point: it is this library's own, for callers that feed the
 * step from host memory step after step (FlashInfer #4562's PR description
 * names caller-stream execution and caller-owned buffers, which this keeps).
 *
 * It enqueues, in order:
 *   on copy_stream: a wait for staging_free, the copy of in_bytes bytes from
 *                   host_in to dev_in, a record of staging_ready;
 *   on stream:      a wait for staging_ready, the step of kda_decode_ex(args),
 *                   a record of staging_free, the copy of the output
 *                   (N*T*HV*V bf16 from args->out) to host_out.
 * A "staging set" is (host_in, dev_in, host_out, staging_ready, staging_free)
 * with args pointing into dev_in.  The caller cycles two (or more) sets: the
 * wait on staging_free keeps a copy in from overwriting dev_in while the step
 * that reads it may still run (an event never recorded counts as complete).
 * Steps run in the order of the calls on `stream`, so the state pool is
 * updated step after step exactly as with kda_decode_host.  The caller owns
 * both streams (distinct, on the current device) and both events (created
 * once, e.g. cudaEventCreateWithFlags(..., cudaEventDisableTiming)); host_in
 * and host_out must be page-locked, and host_out holds the step's output once
 * `stream` has passed it.  The library allocates nothing.
 *
 * Errors: those of kda_decode_host; KDA_ERR_INVALID_ARG also for a NULL
 * stream, copy_stream, staging_ready or staging_free, or stream ==
 * copy_stream.  Nothing is enqueued unless validation passes.
 */
KDA_API kda_status kda_decode_host_pipelined(const kda_decode_args *args, const void *host_in, void *dev_in,
                                             int64_t in_bytes, void *host_out, kda_stream_t stream,
                                             kda_stream_t copy_stream, kda_event_t staging_ready,
                                             kda_event_t staging_free);

/*
 * 1 if [p, p + bytes) lies in one page-locked host allocation that the current
 * device reads and writes at the same address (cudaHostAlloc / cudaMallocHost
 * memory under unified addressing, or cudaHostRegister'd memory mapped at its
 * host address), else 0; also 0 without a device.  Such memory may be passed
 * to every entry point as inputs or output: the kernels then read the step's
 * inputs from host memory and write its output back to host memory across
 * PCIe in the one launch, with no separate copies.  Check each buffer once
 * before first use: a host pointer the device cannot reach would be an
 * illegal access.  This library's own helper; none of the pages describes it.
 */
KDA_API int32_t kda_host_memory_is_mapped(const void *p, int64_t bytes);

/*
 * Device-side error word of the decode kernels on the current device.  The
 * one-token gated kernels hand each value tile's outputs to the tile-0 CTA of
 * the row's cluster, which waits for them with a bounded poll (seconds,
 * against microseconds for the hand-over); if that wait ever gives up, the
 * row's output is left unwritten (its state is stored) and this word is set
 * to 1.
 * Writes the word (0: no kernel gave up since the last clear) to *word;
 * clear != 0 then resets it.  Synchronous: it waits for the device's work in
 * flight.  Errors: KDA_ERR_INVALID_ARG for a NULL word, KDA_ERR_CUDA if the
 * runtime refuses the read.  The library's own diagnostic; the pages describe
 * none.
 */
KDA_API kda_status kda_decode_device_error(int32_t *word, int32_t clear);

/* Static, NUL-terminated description of a status code. */
KDA_API const char *kda_status_string(kda_status status);

/* Library ABI version: (major << 16) | minor. */
KDA_API int32_t kda_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_DECODE_H */
