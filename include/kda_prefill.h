/*
 * kda_prefill.h -- C ABI of the chunked KDA prefill on B200 (sm_100a).
 *
 * The operation is the decode step of kda_decode.h taken over a long token
 * run: for every sequence n in [0, N), value head h in [0, HV) and token t in
 * [0, T), in token order, on the fp32 state S[K][V] held in slot slot_idx[n]:
 *
 *     S   <- Diag(exp(g[n,t,h,:])) S
 *     u   <- beta[n,t,h] * (v[n,t,h,:] - S^T k[n,t,h,:])
 *     S   <- S + k[n,t,h,:] u^T
 *     out[n,t,h,:] <- bf16(scale * S^T q[n,t,h,:])
 *
 * with the final state written back to the slot.  The result equals T calls of
 * the decode step up to fp32 rounding; what differs is how it is computed: the
 * tokens are taken in chunks of 64 in the WY / UT chunk form (a triangular
 * solve inside each chunk, a short state recurrence across chunks and the
 * chunk outputs as dense products on the tensor cores), which turns the work
 * of a long run into parallel per-chunk products instead of a token-by-token
 * chain.
 *
 * Source: vLLM #57585 "Tune recurrent KDA launch configuration on SM90",
 * Details: the related work it names (FlashInfer's fused KDA on Blackwell)
 * adds a prefill path for the SM100 family next to its decode kernels.  The
 * page prints no prefill algorithm; the chunk form used here is the delta rule
 * regrouped exactly (see kda_prefill_kernel.cuh for the formulas).
 *
 * Layouts: as kda_decode (dense, row-major, current device): q, k bf16
 * [N, T, HV, K]; v bf16 [N, T, HV, V]; g fp32 [N, T, HV, K] (log-decay);
 * beta fp32 [N, T, HV]; state_pool fp32 [num_slots, HV, K, V] (in place);
 * slot_idx int32 [N] (< 0 = inactive row: zero output, pool untouched);
 * out bf16 [N, T, HV, V].
 *
 * Supported sizes: K = V = 128; HV >= 1; N, T >= 0 (N == 0 or T == 0 is a
 * no-op that touches no pointer).  Other K or V: KDA_ERR_UNSUPPORTED.
 *
 * Workspace: the caller passes device memory of at least
 * kda_prefill_workspace_bytes(N, T, HV, K, V) bytes (16-byte aligned); the
 * library allocates nothing.  Per (sequence, head, chunk of 64 tokens) it holds
 * about 240 KB of fp32 intermediates (the chunk's solve results, decayed keys
 * and queries, its start state and corrections), after a 256-byte header.
 * Its contents are not meaningful between calls; calls that share a workspace
 * must not overlap on the device (stream order is enough).  The header's first
 * int32 is an error word: the output kernel waits for its tensor-core results
 * with a bounded poll, and if that wait ever gives up (it takes seconds; the
 * products take microseconds) it leaves that chunk's outputs unwritten and
 * stores 1 there.  The library never clears it: a caller that wants to watch
 * it zeroes it before the call.
 *
 * Execution: three kernels enqueued on `stream` in order (chunk preparation,
 * the state recurrence across chunks, the chunk outputs); no host sync; can be
 * captured in a CUDA graph.  Alignment: q, k, v, g, state_pool, out, workspace
 * on 16 bytes; beta, slot_idx on 4 bytes.
 *
 * Errors: the host-side validation of kda_decode (KDA_ERR_INVALID_ARG for a
 * null pointer with work to do, a negative size or a workspace smaller than
 * required; KDA_ERR_ALIAS if out, or the workspace, overlaps an input, the
 * pool's slot-0 block or each other; KDA_ERR_MISALIGNED; KDA_ERR_DEVICE;
 * KDA_ERR_CUDA if the runtime refuses a launch).  Nothing is enqueued unless
 * validation passes; the three launches are configured before the first is
 * enqueued.
 */
#ifndef KDA_PREFILL_H
#define KDA_PREFILL_H

#include "kda_decode.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Bytes of workspace kda_prefill needs for these sizes (0 when N, T or HV is
 * 0; -1 for sizes it does not support or negative sizes). */
KDA_API int64_t kda_prefill_workspace_bytes(int64_t N, int64_t T, int64_t HV, int64_t K, int64_t V);

/* Chunked prefill (see the top of this file).  Writes bf16 outputs for every
 * token and the final state of each active row back to its slot. */
KDA_API kda_status kda_prefill(const void *q, const void *k, const void *v, const float *g,
                               const float *beta, float *state_pool, const int32_t *slot_idx,
                               void *out, void *workspace, int64_t workspace_bytes, int64_t N,
                               int64_t T, int64_t HV, int64_t K, int64_t V, float scale,
                               kda_stream_t stream);

/*
 * One of kda_prefill's three kernels: stage 0 prepares every chunk (its solve
 * and decayed factors into the workspace), stage 1 runs the state recurrence
 * across the chunks (the final state into each active row's slot, each
 * chunk's start state and corrections into the workspace), stage 2 writes the
 * chunk outputs.  kda_prefill is stages 0, 1 and 2 in that order on one
 * stream.  Same arguments, validation and errors as kda_prefill, plus
 * KDA_ERR_INVALID_ARG for a stage outside 0..2; each stage reads what the
 * previous one left in the workspace, so a caller keeps their order on the
 * stream (stage 1 starts from the slot's state: run it once per prefill).
 * For callers that time the stages or put other work between them; the pages
 * name the chunk form's parts but no such entry point.
 */
KDA_API kda_status kda_prefill_stage(int32_t stage, const void *q, const void *k, const void *v,
                                     const float *g, const float *beta, float *state_pool,
                                     const int32_t *slot_idx, void *out, void *workspace,
                                     int64_t workspace_bytes, int64_t N, int64_t T, int64_t HV, int64_t K,
                                     int64_t V, float scale, kda_stream_t stream);

/*
 * The same chunked prefill for callers that cannot allocate device memory.
 * The pages have no counterpart to this entry point; it is this library's own.
 *
 * Some callers of an attention library may not call cudaMalloc at all: an
 * inference server that hands nearly all of the GPU's memory to its own
 * caching allocator at start-up (a later cudaMalloc then fails or fragments
 * that pool), a framework plugin whose host forbids allocations outside the
 * framework's allocator, or a runtime that records its work into CUDA graphs
 * and has no allocation step between captures.  kda_prefill needs a workspace
 * those callers cannot provide; this entry point takes none.  Instead it uses
 * a fixed scratch array of KDA_PREFILL_NO_ALLOC_SCRATCH_BYTES (32 MiB) that
 * the library declares in device memory: every GPU that loads the library
 * holds those 32 MiB until the process exits, whether or not it calls this.
 *
 * Arguments, layouts, results and errors are those of kda_prefill without the
 * workspace.  Sizes whose workspace (kda_prefill_workspace_bytes) exceeds the
 * scratch return KDA_ERR_SCRATCH_LIMIT before anything is enqueued: with
 * K = V = 128 that is N * HV * ceil(T / 64) <= 136 chunks (for example one
 * sequence of up to 1088 tokens at HV = 8).
 *
 * The first call on each device looks the scratch array's device address up
 * (cudaGetSymbolAddress, with that device current) and keeps it; make that
 * first call before capturing any stream into a CUDA graph.  Every call on a
 * device uses the same array, and the array keeps whatever the last call left
 * in it (nothing in it needs to start at zero: each call writes every part it
 * reads), so two calls whose kernels overlap on the GPU -- on different
 * streams without an ordering between them -- race on it and give wrong
 * results.  Calls in one stream, or otherwise ordered, are safe.
 */
#define KDA_PREFILL_NO_ALLOC_SCRATCH_BYTES (32LL << 20)

KDA_API kda_status kda_prefill_no_alloc(const void *q, const void *k, const void *v, const float *g,
                                        const float *beta, float *state_pool, const int32_t *slot_idx,
                                        void *out, int64_t N, int64_t T, int64_t HV, int64_t K, int64_t V,
                                        float scale, kda_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* KDA_PREFILL_H */
